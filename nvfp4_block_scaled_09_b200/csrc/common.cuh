// common.cuh -- shared host/device helpers of the NVFP4 MoE library (sm_100a).
//
// Device side: thin inline-PTX wrappers for the Blackwell data movers and
// tensor cores used by the kernels (mbarriers, TMA tensor and bulk copies,
// cp.async, tcgen05 tensor-memory allocation / copies / MMA / loads) and the
// bounded pipeline wait every kernel uses instead of an unbounded spin.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda.h>
#include <cuda_bf16.h>

#include "../../include/nvfp4moe.h"

namespace nvfp4 {

// Bits of the device status word.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadInput = 2u;

// Test-only behaviour flags (nvfp4_debug_set_flags); 0 on every normal launch.
constexpr uint32_t kCtlStallProducer = 1u;   // GEMM producer issues no loads: every consumer wait runs out

struct DeviceCtl {
    uint32_t* status;      // device status word (global memory)
    uint64_t timeout_ns;   // bound on one pipeline wait
    uint32_t flags;        // kCtl* test flags
};

// Epilogue modes of the grouped GEMM kernels (template argument): each instantiation carries only its own
// epilogue code.
constexpr int kEpiPlain = 0;      // BF16 output (NONE or SWIGLU)
constexpr int kEpiFinalize = 1;   // NONE + the fused top-k combine
constexpr int kEpiQuant = 2;      // SWIGLU with h written as NVFP4

// The gate/up GEMM's quantised h (moe_grouped_gemm_nvfp4_quant): the SwiGLU epilogue writes h as NVFP4
// with a static global scale instead of BF16 h; off when q == nullptr.
struct QuantOut {
    const float* gdec;     // device scalar: the static global scale of h (dequantisation multiplier g_dec)
    uint8_t* q;            // [rows, N/4] E2M1 codes of h [rows, N/2]
    uint8_t* sf;           // h's block scales in the K-stage layout, rows_per_slab rows per slab
    int64_t rows_per_slab;
};

// The grouped GEMM's fused top-k combine (moe_grouped_gemm_nvfp4_finalize); off when out == nullptr.
struct Finalize {
    const int32_t* src;    // [rows] token of each activation row (moe_permute's perm_src)
    const int32_t* inv;    // [T * k] row of each (token, slot) (moe_permute's inv_perm)
    const float* w;        // [T, k] combine weights
    uint32_t* counters;    // [T, col_blocks] arrivals per (token, 128-column block); zero on entry, left zero
    uint16_t* out;         // [T, N] combined BF16 output
    int32_t T, k, col_blocks;
};

// Host-side registry (api.cu).
uint32_t* status_word_ptr();          // nullptr on failure
uint32_t* sched_counter_slot();       // two zeroed words for one GEMM launch's dynamic schedule (nullptr on failure)
uint64_t wait_timeout_ns();
uint32_t debug_flags();
void count_launch(int n = 1);
int device_sm_count();
int device_smem_optin();
nvfp4_status check_launch();          // maps cudaGetLastError to a status
// The CTA-pair grouped GEMM (grouped_gemm_pair.cu).
size_t pair_gemm_smem_bytes();
int pair_gemm_tokens_max();
int pair_gemm_store_cols(int swiglu);   // output columns of one epilogue warp's tensor-store box
nvfp4_status launch_grouped_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_a_full,
                                      const CUtensorMap& tm_out, const CUtensorMap& tm_wsw,
                                      const CUtensorMap& tm_wsf, const uint8_t* a_sf,
                                      const float* a_gscale, const uint8_t* w_packed, const float* w_gscale,
                                      const int32_t* offsets, int32_t E, int64_t max_rows, int64_t N, int64_t K,
                                      int swiglu, uint16_t* out, uint32_t* out_amax, const Finalize& fin,
                                      const QuantOut& qo, cudaStream_t s, uint32_t* status);

#ifdef __CUDACC__
// Launch `kernel` on `s` with programmatic stream serialization (see pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
#endif

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, at most ctl.timeout_ns. On
// expiry (or when another role already gave up, *abort != 0) it latches the
// timeout bit, raises the CTA's abort flag and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  const DeviceCtl& ctl) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++spins & 15u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > ctl.timeout_ns) {
                *abort = 1;
                atomicOr(ctl.status, kStatusTimeout);
                return false;
            }
        }
    }
}

// mbar_wait_bounded for a wait known to be long: a pause of `pause_ns` between polls.
__device__ __forceinline__ bool mbar_wait_bounded_pause(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                        const DeviceCtl& ctl, uint32_t pause_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        __nanosleep(pause_ns);
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > ctl.timeout_ns) {
            *abort = 1;
            atomicOr(ctl.status, kStatusTimeout);
            return false;
        }
    }
}

// Drain wait used only on the abort path: bounded, never raises flags.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t budget_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > budget_ns) return false;
    }
    return true;
}

// Programmatic dependent launch. Kernels of the layer are launched with launch_pdl(), so a kernel
// may become resident while the previous one in the stream is still running. pdl_wait() blocks
// until that kernel -- and, since it waited in turn, every earlier one -- has completed and its
// writes are visible; every kernel calls it before its first global-memory access (and before any
// early return, so that no grid can complete ahead of its predecessor). pdl_launch_dependents()
// lets the next kernel start its prologue; it carries no memory ordering.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// L2 prefetch of [base, base + bytes), split over the CTAs of the grid: worker = cta * blockDim.x + thread of
// nworkers = ctas * blockDim.x, and the first thread of each CTA issues bulk prefetches (64 KB each) of its
// CTA's 16-byte-aligned slice. Used to start the next kernel's constant operand (expert weights) streaming
// into L2 while a short, latency-bound kernel runs (measured on B200, decode layer: 6-11 us less per layer
// call; one prefetch per 128-byte line from every thread gained 5-8 us).
__device__ __forceinline__ void l2_prefetch_slice(const uint8_t* base, int64_t bytes, int64_t worker, int64_t nworkers) {
    if (base == nullptr || bytes <= 0 || threadIdx.x != 0) return;
    const int64_t ctas = nworkers / blockDim.x, cta = worker / blockDim.x;
    const int64_t slice = ((bytes + ctas - 1) / ctas + 15) & ~int64_t(15);
    const int64_t lo = cta * slice, hi = lo + slice < bytes ? lo + slice : bytes;
    for (int64_t off = lo; off < hi; off += 65536) {
        const int64_t n = (hi - off < 65536 ? hi - off : 65536) & ~int64_t(15);
        if (n > 0) asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + off), "r"((uint32_t)n) : "memory");
    }
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// TMA: 2-D tiled tensor load into shared memory, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// TMA: 5-D tiled tensor load into shared memory (box written densely, dimension 0 fastest).
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2,
                                            int32_t c3, int32_t c4, uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}

// Contiguous bulk copy global -> shared (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// TMA: 2-D tiled tensor store shared -> global (box at coordinates {c0, c1}, both >= 0), tracked
// by this thread's bulk async-group.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(smem_u32(src))
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of this thread's bulk stores have been read.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 4-byte asynchronous copy with zero fill when src_bytes == 0.
__device__ __forceinline__ void cp_async_4(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05 (5th-generation tensor cores, tensor memory) -------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Copy 32 rows x 16 bytes of shared memory (described by `desc`) into tensor
// memory columns [taddr, taddr+4), replicated into all four 32-lane quadrants.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T with E2M1 operands and UE4M3 scales per 16 K.
__device__ __forceinline__ void mma_mxf4nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}
// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
        "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}
// Each thread of the warp writes 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
// Each thread of the warp writes one 32-bit column of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x1(uint32_t taddr, uint32_t v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05 format): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, swizzle mode in bits 61-63.
__device__ __forceinline__ uint64_t make_smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                                   uint32_t swizzle_mode) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;                       // version
    d |= (uint64_t)(swizzle_mode & 7u) << 61;      // 0: none, 2: 128-byte swizzle
    return d;
}

// Two FP32 values in one 64-bit register, for the packed FP32 multiply of sm_100 (mul.rn.f32x2: both
// halves rounded as two scalar multiplies would be)
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// Both halves rounded to BF16 (nearest even), the low half into the low 16 bits
__device__ __forceinline__ uint32_t f32x2_to_bf16x2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// SwiGLU of one output element: silu(g) * u with silu(g) = g / (1 + e^-g), in single precision
// without branches: e^-g as 2^(-g log2 e) on the ISA's base-2 exponential (ex2.approx), and the
// quotient as g times the ISA's approximate reciprocal (rcp.approx) of 1 + e^-g. Both are within a few
// FP32 ulp, far below the BF16 output's resolution. For g below about -88 the exponential overflows,
// the reciprocal is 0 and the result is -0 * u. (Measured on the prefill gate/up GEMM: 0.6% faster than
// the same formula through the fast-math exponential and division intrinsics, with the same bits.)
__device__ __forceinline__ float swiglu_f32(float g, float u) {
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(g * -1.4426950408889634f));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
    return (g * r) * u;
}

// FP32 -> E4M3, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3_satfinite(float s) {
    uint16_t pair;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pair) : "f"(0.0f), "f"(s));
    return pair & 0xFFu;
}

// Non-negative finite E4M3 byte -> FP32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return (float)m * 0.001953125f;  // m * 2^-9, exact
    return __uint_as_float(((e + 120u) << 23) | (m << 20));  // (1 + m/8) * 2^(e-7)
}

// FP32 -> E2M1 code (low 4 bits), round to nearest even, saturating to +-6, the sign kept on zero.
__device__ __forceinline__ uint32_t f32_to_e2m1(float y) {
    uint32_t w;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b32 %0, {t, t, t, t};\n\t}"
        : "=r"(w) : "f"(0.0f), "f"(y));
    return w & 15u;
}

// Block quantisation step shared by every quantiser (nvfp4_quantize and the GEMM epilogue that writes
// quantised h): the E4M3 scale of a 16-element block from its amax, and the FP32 factor that takes the
// block's values onto the E2M1 grid (0 when the scale is 0: the block's codes are +0).
__device__ __forceinline__ uint32_t block_scale(float amax_b, float g_enc, float& f) {
    const float s = __fmul_rn(__fdiv_rn(amax_b, 6.0f), g_enc);
    const uint32_t S = f32_to_e4m3_satfinite(s);
    const float sfv = e4m3_to_f32(S);
    f = sfv != 0.0f ? __fdiv_rn(g_enc, sfv) : 0.0f;
    return S;
}

// One E2M1 code per lane of a half-warp whose 16 lanes hold one 16-element block of a row (BF16 bits
// hb; valid = the lane's element exists): the block's scale byte (returned) and the lane's code, by the
// quantiser's steps with the given g_enc. Every lane of the warp must call it.
__device__ __forceinline__ uint32_t quantize_half_warp_block(uint32_t hb, bool valid, float g_enc, uint32_t& code) {
    uint32_t a = valid ? (hb & 0x7FFFu) : 0u;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) a = max(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    float f;
    const uint32_t S = block_scale(__uint_as_float(a << 16), g_enc, f);
    code = (S != 0u && valid) ? f32_to_e2m1(__fmul_rn(__uint_as_float(hb << 16), f)) : 0u;
    return S;
}

// FP64 -> BF16, round to nearest even, in effect a single rounding: truncate to FP32, mark inexactness
// in the last bit (round-to-odd), then round to BF16. (The combine's final rounding, shared by the
// separate combine kernel and the GEMM's fused combine so the two agree bit for bit.)
__device__ __forceinline__ uint32_t f64_to_bf16_bits(double d) {
    float f = __double2float_rz(d);
    if ((double)f != d) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Eight adjacent output columns [col, col + 8) of the top-k weighted combine for token t: the sum over the
// token's slots j ascending of w[t, j] * y[inv_perm[t*k + j], col..] in FP64 (each product of an FP32 weight and
// a BF16 value is exact), negative rows skipped, rounded once to BF16 and stored as one 16-byte piece. The
// slots are read in groups of kGroup so their loads overlap; y is read past L1 (other SMs wrote it).
template <int kGroup = 4>
__device__ __forceinline__ void combine_vec8(const uint16_t* y, int64_t ldy, const int32_t* inv_perm, const float* w,
                                             int32_t t, int32_t k, int64_t col, uint16_t* out, int64_t ldo) {
    double a[8];
#pragma unroll
    for (int i = 0; i < 8; i++) a[i] = 0.0;
    for (int32_t j0 = 0; j0 < k; j0 += kGroup) {
        int32_t p[kGroup];
        float s[kGroup];
#pragma unroll
        for (int u = 0; u < kGroup; u++) {
            p[u] = j0 + u < k ? __ldg(inv_perm + (int64_t)t * k + j0 + u) : -1;
            s[u] = j0 + u < k ? __ldg(w + (int64_t)t * k + j0 + u) : 0.0f;
        }
        uint4 v[kGroup];
#pragma unroll
        for (int u = 0; u < kGroup; u++)
            v[u] = p[u] >= 0 ? __ldcg(reinterpret_cast<const uint4*>(y + (int64_t)p[u] * ldy + col)) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kGroup; u++) {
            if (p[u] < 0) continue;
            const double sd = (double)s[u];
            const uint32_t x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                a[2 * i] = fma(sd, (double)__uint_as_float(x[i] << 16), a[2 * i]);
                a[2 * i + 1] = fma(sd, (double)__uint_as_float(x[i] & 0xFFFF0000u), a[2 * i + 1]);
            }
        }
    }
    uint4 o;
    o.x = f64_to_bf16_bits(a[0]) | (f64_to_bf16_bits(a[1]) << 16);
    o.y = f64_to_bf16_bits(a[2]) | (f64_to_bf16_bits(a[3]) << 16);
    o.z = f64_to_bf16_bits(a[4]) | (f64_to_bf16_bits(a[5]) << 16);
    o.w = f64_to_bf16_bits(a[6]) | (f64_to_bf16_bits(a[7]) << 16);
    *reinterpret_cast<uint4*>(out + (int64_t)t * ldo + col) = o;
}

// ---- thread-block clusters and CTA pairs (cta_group::2) ---------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t num_clusters_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_smem_addr(const void* local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
    return r;
}
// Arrive on a barrier of this or the peer CTA (release at CTA scope: the peer only learns that a
// TMEM slot was written or drained; the tcgen05 fences order the tensor-memory accesses).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Cluster-scope variants for barriers that carry data written by the other CTA of a pair through
// distributed shared memory (the work-item ring of the CTA-pair GEMM).
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// mbar_wait_bounded with cluster-scope acquire.
__device__ __forceinline__ bool mbar_wait_bounded_acq_cluster(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                              const DeviceCtl& ctl) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait_acq_cluster(bar, parity)) return true;
        if ((++spins & 15u) == 0u) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > ctl.timeout_ns) {
                *abort = 1;
                atomicOr(ctl.status, kStatusTimeout);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair MMA (issued by the even CTA): A rows [0,128) from this CTA's shared memory and [128,256)
// from the peer's at the same offset; B rows split the same way; D rows in each CTA's TMEM.
__device__ __forceinline__ void mma_mxf4nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}
// Arrive on the barrier at `bar`'s offset in both CTAs of the pair once every pair MMA issued so far
// completed (one commit signals both: each commit costs the issuing thread about as much as an MMA).
__device__ __forceinline__ void tc_commit_pair_both(const uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}
// Arrive on the barrier at `cluster_addr` (this or the peer CTA) once every pair MMA issued so far completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t cluster_addr) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// Each thread of the warp writes 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

#endif  // __CUDACC__

}  // namespace nvfp4

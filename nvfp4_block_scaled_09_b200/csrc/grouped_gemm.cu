// grouped_gemm.cu -- NVFP4 block-scaled MoE grouped GEMM on 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// What it computes: for every expert e and activation row m routed to it,
//   out[m, n] = epilogue( (g_A * g_W[e]) * sum_k A(m,k) W_e(n,k) )
// with E2M1 operands and one E4M3 scale per 16 K-elements on each side, the
// FP4 MoE grouped GEMM of "Peering into the CUTLASS Kernel Cache" (one launch
// over all experts, TMA warp-specialised) with the fused global-scale, SwiGLU
// and BF16 epilogue.
//
// Design (chosen for B200, not the SM120 tiles the pages analyse):
//  * Swap-AB orientation. Experts see 16-256 rows, so the 128-row MMA M side
//    holds weight rows and the activation rows ride on the MMA N side
//    (16..64 or 16..128, in steps of 16, picked per tile on the device). Every weight byte
//    is read once per (expert, row tile); decode is a pure weight stream.
//  * Tile = 2 x 128 weight rows x up to 64 activation rows, K stage = 256.
//    SWIGLU pairs gate rows [n0, n0+128) with up rows [N/2+n0, ...) so both
//    accumulators of one output column sit in the same TMEM lane; NONE covers
//    256 consecutive output columns.
//  * Weights arrive pre-packed (pack.cu): every 128-row x 256-K tile with its
//    scales is one contiguous 18 KB chunk already in the shared-memory image the
//    tensor core reads, so a weight stage is two contiguous bulk copies (the
//    weight stream is what decode is bound by, and contiguous pieces stream
//    ~15% faster from HBM than strided 2-D tiles).
//  * Warp roles ("Peering into the CUTLASS Kernel Scheduler", The Discovery:
//    explicit warp-specialised schedules that give A loads, B loads, MMA and
//    epilogue their own warps): warp 0 issues the weight bulk copies, the
//    TMA tiles of activations and one bulk copy of their scales; warps 8-11 (one
//    per TMEM lane quadrant) store every stage's
//    scales into a per-stage TMEM ring with tcgen05.st; warp 2 owns tensor
//    memory and issues only tcgen05.mma (scale copies issued on the MMA pipe
//    serialise with the MMAs; measured, this halved the decode stream rate);
//    warps 4-7 drain the FP32 accumulators from TMEM, apply the global scales /
//    SwiGLU and store BF16.
//  * Stage accounting: the expected transaction bytes of a stage are the A
//    tile bytes plus its scale bytes plus the B tile bytes ("Peering into the
//    CUTLASS SharedStorage", The Message: MK bytes + NK bytes per stage): two
//    packed weight tiles (codes + scales), the activation tile and its rows'
//    scales.
//  * Activation scales come in the K-stage layout (one [rows x 16 B] slab per
//    256-element K step), so a tile's scales for one stage are one contiguous
//    run, fetched with one bulk copy. A 16-byte-wide TMA box over row-major
//    scales costs one request per row: measured on B200 (loads alone, all SMs),
//    such a 256-row box took ~190 ns per stage and brought the CTA-pair
//    stage's loads from ~280 to ~440 ns.
//  * Shared memory: 4 stages x 46 KB (narrow) or 54 KB (wide) + scheduler
//    tables, checked against the
//    device's opt-in limit before launch (the same predicate
//    nvfp4_can_implement() reports, so a passing check never fails to launch).
//  * Persistent CTAs (one per SM) take (expert, column tile, row tile) work
//    items from a grid-wide counter (dynamic schedule: CTAs that run ahead take
//    the tail) and read expert offsets from device memory; no host
//    synchronisation. The producer passes each item to the other warp roles
//    through a small ring in shared memory. Two TMEM accumulator buffers let the
//    epilogue of one tile overlap the main loop of the next (narrow shape).
//  * Every wait is bounded (%globaltimer); on expiry the kernel latches
//    NVFP4_ERR_DEVICE_TIMEOUT, drains its in-flight copies and MMAs, frees
//    tensor memory and returns.
#include <mutex>

#include "common.cuh"

namespace nvfp4 {
namespace gg {

constexpr int kBM = 128;                         // weight rows per MMA (tcgen05 M)
constexpr int kNumA = 2;                         // weight row blocks per tile
constexpr int kBK = 256;                         // K elements per stage
constexpr int kRowBytes = kBK / 2;               // packed bytes per row per stage (one 128-byte swizzle row)
constexpr int kBNStep = 16;                      // N granularity = activation TMA box rows
constexpr int kMaxStages = 4;                    // barrier arrays are sized for the deepest shape
constexpr int kKSteps = kBK / 64;                // MMA K-steps per stage (K = 64 per MMA)
constexpr int kABlockBytes = kBM * kRowBytes;    // 16 KB
constexpr int kSFAtomBytes = 512;                // 128 rows x 4 scales
constexpr int kSFStageBytes = kKSteps * kSFAtomBytes;
constexpr int kPackedTileBytes = kABlockBytes + kSFStageBytes;  // one packed weight tile (codes + scales)
static_assert(kPackedTileBytes % 1024 == 0, "weight tiles keep the 128-byte swizzle's 1024-byte alignment");
// Stage layout: [A0 codes | A0 scales][A1 codes | A1 scales][B codes][B scales]
constexpr int kOffA0 = 0;
constexpr int kOffSFA0 = kABlockBytes;
constexpr int kOffA1 = kPackedTileBytes;
constexpr int kOffSFA1 = kOffA1 + kABlockBytes;
constexpr int kOffB = 2 * kPackedTileBytes;
constexpr int kMaxE = 1024;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemLimit = 232448;               // B200 opt-in shared memory per block

constexpr int kTileRing = 4;                     // work items the producer may publish ahead of the slowest role
constexpr int kTileConsumers = 9;                // MMA warp + 4 scale writers + 4 epilogue warps

struct Shared {
    uint64_t tq_full[kTileRing];                 // producer published tq[i]
    uint64_t tq_empty[kTileRing];                // every consumer role read tq[i]
    int32_t tq[kTileRing];                       // work item index (>= total: no more work)
    uint64_t full_tma[kMaxStages];
    uint64_t sf_ready[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int32_t total_tiles;
    int32_t off[kMaxE + 1];
    int32_t tile_start[kMaxE + 1];
    int32_t fin_tok[128];                        // fused combine: tokens of this tile whose last row it wrote
    uint64_t fin_bar;                            // fused combine: the 4 epilogue warps meet (bounded waits)
};

// Two tile shapes share one kernel body:
//  - narrow (decode): up to 64 activation rows per tile, two TMEM accumulator
//    buffers so the epilogue of one tile overlaps the main loop of the next;
//  - wide (prefill, dense): up to 128 activation rows per tile -- N = 128 MMAs
//    cost the same ~50 ns as N = 64 ones on B200, so the tensor rate doubles and
//    the activation re-reads from L2 halve -- with one accumulator buffer (two
//    128-column accumulators plus the scale ring fill the 512 TMEM columns).
template <int BN_MAX, int ACC_BUFS, int STAGES>
struct Cfg {
    static constexpr int kStages = STAGES;
    static constexpr int kBNMax = BN_MAX;
    static constexpr int kAccBufs = ACC_BUFS;
    static constexpr int kBBytes = BN_MAX * kRowBytes;
    static constexpr int kOffSFB = kOffB + kBBytes;
    static constexpr int kStageBytes = kOffSFB + kSFStageBytes;
    static constexpr uint32_t kAccCols = BN_MAX;
    // Scale factors live in a TMEM ring, one 48-column slot per pipeline stage:
    // [SFA block 0: 16][SFA block 1: 16][SFB: 16], after the accumulators.
    static constexpr uint32_t kTmemSFRing = ACC_BUFS * kNumA * kAccCols;
    static constexpr uint32_t kTmemSFSlot = (kNumA + 1) * 4 * kKSteps;
    static constexpr size_t kSmemBytes = 1024 /* alignment slack */ + (size_t)kStages * kStageBytes + sizeof(Shared);
    static_assert(BN_MAX % kBNStep == 0 && BN_MAX <= 128, "one scale atom covers at most 128 activation rows");
    static_assert(STAGES >= 2 && STAGES <= kMaxStages, "stage count");
    static_assert(kTmemSFRing + kStages * kTmemSFSlot <= kTmemCols, "TMEM budget");
    static_assert(kStageBytes % 1024 == 0, "stage buffers must keep 1024-byte swizzle alignment");
    static_assert(kSmemBytes + 256 <= (size_t)kSmemLimit, "shared memory budget (dynamic + static)");
};
using Narrow = Cfg<64, 2, 4>;
using Wide = Cfg<128, 1, 4>;

static_assert(kOffA1 % 1024 == 0 && kOffB % 1024 == 0, "swizzled operand tiles must start on 1024 bytes");

struct Params {
    const uint8_t* a_sf;
    const float* a_gscale;
    const uint8_t* w_packed;
    const float* w_gscale;
    const int32_t* offsets;
    uint16_t* out;
    int32_t E;
    int64_t max_rows;
    int64_t N;
    int64_t K;
    int32_t swiglu;
    uint32_t* amax_out;   // nullable: raised to max |out| (BF16 bits)
    uint32_t* sched;      // this launch's work counter [0] and finished-CTA counter [1]; zero at launch
    DeviceCtl ctl;
    Finalize fin;         // fused top-k combine (NONE epilogue), off when fin.out == nullptr
    QuantOut qo;          // quantised h (SWIGLU epilogue), off when qo.q == nullptr
};

struct Tile {
    int32_t e, nt, mt, row0, rows, bn;
};

template <int kBNMax>
__device__ __forceinline__ void decode_tile(const Shared& sh, int32_t E, int32_t n_col_tiles, int32_t w, Tile& t) {
    int32_t lo = 0, hi = E;  // tile_start[lo] <= w < tile_start[hi]
    while (hi - lo > 1) {
        const int32_t mid = (lo + hi) >> 1;
        if (sh.tile_start[mid] <= w) lo = mid;
        else hi = mid;
    }
    const int32_t M = sh.off[lo + 1] - sh.off[lo];
    const int32_t mtiles = (M + kBNMax - 1) / kBNMax;
    const int32_t local = w - sh.tile_start[lo];
    t.e = lo;
    t.nt = local / mtiles;
    t.mt = local - t.nt * mtiles;
    t.row0 = sh.off[lo] + t.mt * kBNMax;
    t.rows = min(kBNMax, M - t.mt * kBNMax);
    t.bn = (t.rows + kBNStep - 1) / kBNStep * kBNStep;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const DeviceCtl& ctl) {
    bool ok = mbar_wait_bounded(bar, parity, abort, ctl);
    return __all_sync(0xFFFFFFFFu, ok);
}

// The producer: take the next work item of the grid and publish it in the ring. False when a wait ran out.
__device__ __forceinline__ bool publish_tile(Shared& sh, const Params& p, int32_t total, uint32_t& qi,
                                             uint32_t& qphase, int32_t& w, volatile int* abort) {
    w = (int32_t)min(atomicAdd(p.sched, 1u), (uint32_t)total);
    if (!mbar_wait_bounded(&sh.tq_empty[qi], qphase ^ 1u, abort, p.ctl)) return false;
    *reinterpret_cast<volatile int32_t*>(&sh.tq[qi]) = w;
    mbar_arrive(&sh.tq_full[qi]);
    if (++qi == kTileRing) { qi = 0; qphase ^= 1u; }
    return true;
}

// Next work item of this CTA for one consumer role (a whole warp): the producer publishes the items it
// took from the launch's work counter in a ring of kTileRing entries. False when a wait ran out.
__device__ __forceinline__ bool next_tile(Shared& sh, uint32_t& qi, uint32_t& qphase, int32_t& w, int lane,
                                          volatile int* abort, const DeviceCtl& ctl) {
    if (!warp_wait(&sh.tq_full[qi], qphase, abort, ctl)) return false;
    w = *reinterpret_cast<volatile int32_t*>(&sh.tq[qi]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.tq_empty[qi]);
    if (++qi == kTileRing) { qi = 0; qphase ^= 1u; }
    return true;
}

template <class C, int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const Params p) {
    constexpr int kBNMax = C::kBNMax;
    constexpr int kOffSFB = C::kOffSFB;
    constexpr int kStageBytes = C::kStageBytes;
    constexpr uint32_t kAccCols = C::kAccCols;
    constexpr uint32_t kTmemSFRing = C::kTmemSFRing;
    constexpr uint32_t kTmemSFSlot = C::kTmemSFSlot;
    constexpr int kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    Shared& sh = *reinterpret_cast<Shared*>(smem + (size_t)kStages * kStageBytes);
    volatile int* abort = &sh.abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int32_t E = p.E;
    // NONE with N % 256 == 128: the last column tile holds one 128-row weight block ("half" tile)
    const int32_t n_col_tiles = (int32_t)(p.swiglu ? (p.N / 2) / kBM : (p.N + kNumA * kBM - 1) / (kNumA * kBM));
    const bool half_cols = !p.swiglu && (p.N % (kNumA * kBM)) != 0;

    if (tid == 0) {
        prefetch_tensormap(&tm_a);
        sh.abort = 0;
        for (int s = 0; s < kStages; s++) {
            mbar_init(&sh.full_tma[s], 1);
            mbar_init(&sh.sf_ready[s], 4);
            mbar_init(&sh.empty[s], 1);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&sh.acc_full[b], 1);
            mbar_init(&sh.acc_empty[b], 4);
        }
        mbar_init(&sh.drain, 1);
        mbar_init(&sh.fin_bar, 4);
        for (int i = 0; i < kTileRing; i++) {
            mbar_init(&sh.tq_full[i], 1);
            mbar_init(&sh.tq_empty[i], kTileConsumers);
        }
        fence_barrier_init();
    }
    // everything above overlaps the previous kernel; global memory only from here on
    pdl_launch_dependents();
    pdl_wait();
    // ---- scheduler tables: expert offsets and the first work item of each expert ----
    for (int i = tid; i <= E; i += kThreads) sh.off[i] = __ldg(p.offsets + i);
    __syncthreads();
    {
        // Each thread sums the tiles of 4 consecutive experts, then a block-wide exclusive scan.
        const int e0 = tid * 4;
        int32_t cnt[4];
        int32_t local = 0;
        bool bad = false;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = e0 + i;
            cnt[i] = 0;
            if (e < E) {
                const int32_t a = sh.off[e], b = sh.off[e + 1];
                if (a < 0 || b < a || (int64_t)b > p.max_rows) {
                    bad = true;  // inconsistent offsets: skip this expert
                } else {
                    cnt[i] = ((b - a + kBNMax - 1) / kBNMax) * n_col_tiles;
                }
            }
            local += cnt[i];
        }
        if (bad) atomicOr(p.ctl.status, kStatusBadInput);
        int32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        __shared__ int32_t warp_tot[kThreads / 32];
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int32_t before = 0;
        for (int w2 = 0; w2 < warp; w2++) before += warp_tot[w2];
        int32_t run = before + incl - local;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = e0 + i;
            if (e < E) sh.tile_start[e] = run;
            run += cnt[i];
        }
        if (tid == kThreads - 1) {
            sh.total_tiles = before + incl;
            sh.tile_start[E] = before + incl;
        }
    }
    // ---- tensor memory ----
    if (warp == 2) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int32_t total = sh.total_tiles;
    // K % 256 == 128: the last stage holds 128 K-elements (2 MMA K-steps); its weight tiles and activation
    // scales are zero-padded, and the activation tile's second half is outside the tensor (zero-filled)
    const int32_t ksteps_total = (int32_t)((p.K + kBK - 1) / kBK);
    const int last_ksteps = (p.K % kBK) ? (int)((p.K % kBK) / 64) : kKSteps;

    if (warp == 0) {
        // ================= TMA producer =================
        uint32_t issued_parity[kStages];
        bool issued[kStages];
#pragma unroll
        for (int s = 0; s < kStages; s++) issued[s] = false, issued_parity[s] = 0;
        if (lane == 0 && !(p.ctl.flags & kCtlStallProducer)) {
            // Weights read by one row tile only are streamed past L2; experts with
            // several row tiles re-read theirs from L2 (their tiles run back to back).
            const uint64_t pol_w_once = l2_policy_evict_first();
            const uint64_t pol_w_reuse = l2_policy_evict_normal();
            const uint64_t pol_a = l2_policy_evict_last();
            uint32_t stage = 0, phase = 0, qi = 0, qphase = 0;
            // dynamic schedule: work items of the whole grid in increasing order, so items that share a
            // weight tile (row tile fastest) still run side by side, and CTAs that run ahead take the
            // tail. The item after the current one is published before the current one's loads, so the
            // counter's round trip overlaps the MMAs.
            int32_t w = total, w_next = total;
            bool ok = publish_tile(sh, p, total, qi, qphase, w, abort);
            if (ok && w < total) ok = publish_tile(sh, p, total, qi, qphase, w_next, abort);
            while (ok && w < total) {
                Tile t;
                decode_tile<kBNMax>(sh, E, n_col_tiles, w, t);
                int64_t r0, r1;
                if (p.swiglu) {
                    r0 = (int64_t)t.nt * kBM;
                    r1 = p.N / 2 + (int64_t)t.nt * kBM;
                } else {
                    r0 = (int64_t)t.nt * (kNumA * kBM);
                    r1 = r0 + kBM;
                }
                const int64_t wr0 = (int64_t)t.e * p.N + r0, wr1 = (int64_t)t.e * p.N + r1;
                const uint8_t* wp0 = p.w_packed + (wr0 / kBM) * ksteps_total * (int64_t)kPackedTileBytes;
                const uint8_t* wp1 = p.w_packed + (wr1 / kBM) * ksteps_total * (int64_t)kPackedTileBytes;
                const bool reuse = (sh.off[t.e + 1] - sh.off[t.e]) > kBNMax;
                const uint64_t pol_w = reuse ? pol_w_reuse : pol_w_once;
                const int n_a = (half_cols && t.nt == n_col_tiles - 1) ? 1 : kNumA;   // weight blocks of this tile
                // MK part: the packed weight tiles (codes + scales); NK part: the activation
                // tile and the tile's rows of the K step's scale slab (16 bytes per row, one
                // contiguous run in the K-stage layout).
                const uint32_t tx = (uint32_t)(n_a * kPackedTileBytes + t.bn * kRowBytes + t.rows * 16);
                const uint8_t* sfb = p.a_sf + (int64_t)t.row0 * 16;
                for (int32_t kt = 0; kt < ksteps_total; kt++) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort, p.ctl)) { ok = false; break; }
                    uint8_t* sb = stages + (size_t)stage * kStageBytes;
                    uint64_t* bar = &sh.full_tma[stage];
                    mbar_arrive_expect_tx(bar, tx);
                    const int32_t kx = kt * kRowBytes;
                    bulk_load(sb + kOffA0, wp0 + (size_t)kt * kPackedTileBytes, kPackedTileBytes, bar, pol_w);
                    if (n_a == kNumA)
                        bulk_load(sb + kOffA1, wp1 + (size_t)kt * kPackedTileBytes, kPackedTileBytes, bar, pol_w);
                    for (int32_t i = 0; i < t.bn / kBNStep; i++)
                        tma_load_2d(sb + kOffB + i * kBNStep * kRowBytes, &tm_a, kx, t.row0 + i * kBNStep, bar, pol_a);
                    bulk_load(sb + kOffSFB, sfb + (int64_t)kt * p.max_rows * 16, (uint32_t)t.rows * 16u, bar, pol_a);
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                w = w_next;
                if (w < total) ok = publish_tile(sh, p, total, qi, qphase, w_next, abort);
            }
            if (!ok || *abort) {
                // Abort path: let every copy already issued land before the CTA can exit.
                for (int s = 0; s < kStages; s++)
                    if (issued[s]) mbar_wait_drain(&sh.full_tma[s], issued_parity[s], 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================= MMA issuer =================
        // Instruction descriptor: E2M1 x E2M1 (format 1), both K-major, UE4M3
        // scales, M = 128 (bits 24-28 hold M >> 4), N in bits 17-22 (N >> 3).
        const uint32_t idesc_base = (1u << 7) | (1u << 10) | ((uint32_t)(kBM >> 4) << 24);
        uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0, qi = 0, qphase = 0;
        bool ok = true;
        while (ok) {
            int32_t w;
            if (!next_tile(sh, qi, qphase, w, lane, abort, p.ctl)) { ok = false; break; }
            if (w >= total) break;
            Tile t;
            decode_tile<kBNMax>(sh, E, n_col_tiles, w, t);
            const uint32_t idesc = idesc_base | ((uint32_t)(t.bn >> 3) << 17);
            const int n_a = (half_cols && t.nt == n_col_tiles - 1) ? 1 : kNumA;
            if (!warp_wait(&sh.acc_empty[abuf], aphase ^ 1u, abort, p.ctl)) { ok = false; break; }
            tc_fence_after();
            for (int32_t kt = 0; kt < ksteps_total; kt++) {
                if (!warp_wait(&sh.full_tma[stage], phase, abort, p.ctl) ||
                    !warp_wait(&sh.sf_ready[stage], phase, abort, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sb = smem_u32(stages + (size_t)stage * kStageBytes);
                    const uint32_t sf = tmem + kTmemSFRing + stage * kTmemSFSlot;
                    // the stage's first descriptors; a K-step is 32 bytes on and a weight tile kPackedTileBytes on,
                    // added in the address field (bits 0-13 hold address / 16, below 2^14 in shared memory)
                    const uint64_t b0 = make_smem_desc(sb + kOffB, 16, 1024, 2);
                    const uint64_t a0 = make_smem_desc(sb, 16, 1024, 2);
                    const uint32_t acc0 = kt != 0 ? 1u : 0u;
                    auto mma_step = [&](int kc, int a) {
                        mma_mxf4nvf4(tmem + abuf * (kNumA * kAccCols) + a * kAccCols,
                                     a0 + (uint64_t)(a * (kPackedTileBytes >> 4) + 2 * kc), b0 + 2 * kc, idesc,
                                     sf + a * 4 * kKSteps + 4 * kc, sf + kNumA * 4 * kKSteps + 4 * kc, kc != 0 ? 1u : acc0);
                    };
                    if (n_a == kNumA && (kt != ksteps_total - 1 || last_ksteps == kKSteps)) {
#pragma unroll
                        for (int kc = 0; kc < kKSteps; kc++)
#pragma unroll
                            for (int a = 0; a < kNumA; a++) mma_step(kc, a);
                    } else {
                        // a half column tile (one weight block) and/or a last stage of 128 K-elements
                        const int n_kc = kt == ksteps_total - 1 ? last_ksteps : kKSteps;
                        for (int kc = 0; kc < n_kc; kc++)
                            for (int a = 0; a < n_a; a++) mma_step(kc, a);
                    }
                    tc_commit(&sh.empty[stage]);
                }
                __syncwarp();
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(&sh.acc_full[abuf]);
            __syncwarp();
            if (++abuf == (uint32_t)C::kAccBufs) { abuf = 0; aphase ^= 1u; }
        }
        if (!ok || *abort) {
            // Abort path: wait for every MMA issued so far before tensor memory is freed.
            if (lane == 0) {
                tc_commit(&sh.drain);
                mbar_wait_drain(&sh.drain, 0, 200000000ull);
            }
            __syncwarp();
        }
    } else if (warp >= 8) {
        // ================= scale writers =================
        // Warp 8 + q owns TMEM lane quadrant q. For each stage it reads the
        // scales from shared memory and stores them into that stage's TMEM ring
        // slot with tcgen05.st, so the MMA warp issues nothing but MMAs (a
        // tcgen05.cp on the MMA pipe serialises with the MMAs around it).
        // MMA reads: row m of a weight block at lane m, column base + 4 kc + m/32;
        // activation row n at lane n % 32 of every quadrant, column base + 4 kc + n/32.
        // Activation scales arrive as [rows][16 bytes] (the tile's rows of one K-stage slab).
        const int quad = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        uint32_t stage = 0, phase = 0, qi = 0, qphase = 0;
        bool ok = true;
        while (ok) {
            int32_t w;
            if (!next_tile(sh, qi, qphase, w, lane, abort, p.ctl)) break;
            if (w >= total) break;
            for (int32_t kt = 0; kt < ksteps_total; kt++) {
                if (!warp_wait(&sh.full_tma[stage], phase, abort, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* sb = stages + (size_t)stage * kStageBytes;
                const uint32_t slot = tmem + lane_addr + kTmemSFRing + stage * kTmemSFSlot;
                uint32_t word[kKSteps], v[16];
#pragma unroll
                for (int a = 0; a < kNumA; a++) {
                    const uint8_t* src = sb + (a ? kOffSFA1 : kOffSFA0) + lane * 16 + quad * 4;
#pragma unroll
                    for (int kc = 0; kc < kKSteps; kc++)
                        word[kc] = *reinterpret_cast<const uint32_t*>(src + kc * kSFAtomBytes);
                    // one column per K-step: the one this quadrant's rows are read from
#pragma unroll
                    for (int kc = 0; kc < kKSteps; kc++) tmem_st_32x32b_x1(slot + a * 4 * kKSteps + 4 * kc + quad, word[kc]);
                }
#pragma unroll
                for (int kc = 0; kc < kKSteps; kc++) {
#pragma unroll
                    for (int g = 0; g < 4; g++)   // activation row 32 g + lane: 16 scale bytes per row in smem
                        v[4 * kc + g] = g * 32 < kBNMax
                                            ? *reinterpret_cast<const uint32_t*>(sb + kOffSFB + (32 * g + lane) * 16 + 4 * kc)
                                            : 0u;
                }
                tmem_st_32x32b_x16(slot + kNumA * 4 * kKSteps, v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.sf_ready[stage]);
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
        }
    } else if (warp >= 4) {
        // ================= epilogue =================
        const int quad = warp & 3;              // TMEM lane quadrant this warp may access
        const int r = quad * 32 + lane;         // accumulator row = weight row within a block
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const float a_g = __ldg(p.a_gscale);
        const float h_genc = kEpi == kEpiQuant ? __fdiv_rn(1.0f, __ldg(p.qo.gdec)) : 0.0f;   // static scale of h
        uint32_t amax = 0;  // max |stored BF16| of this thread, as BF16 bits
        uint32_t abuf = 0, aphase = 0, qi = 0, qphase = 0, fphase = 0;
        // the 4 epilogue warps meet here (fused combine only); false when a wait ran out
        auto epi_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.fin_bar);
            const bool ok = warp_wait(&sh.fin_bar, fphase, abort, p.ctl);
            fphase ^= 1u;
            return ok;
        };
        while (true) {
            int32_t w;
            if (!next_tile(sh, qi, qphase, w, lane, abort, p.ctl)) break;
            if (w >= total) break;
            Tile t;
            decode_tile<kBNMax>(sh, E, n_col_tiles, w, t);
            if (!warp_wait(&sh.acc_full[abuf], aphase, abort, p.ctl)) break;
            tc_fence_after();
            const uint32_t cbase = tmem + lane_base + abuf * (kNumA * kAccCols);
            const float alpha = a_g * __ldg(p.w_gscale + t.e);
            const bool second = !(half_cols && t.nt == n_col_tiles - 1);   // NONE: the second weight block exists
            for (int c = 0; c * 16 < t.bn; c++) {
                float v0[16], v1[16];
                tmem_ld_32x32b_x16(cbase + c * 16, v0);
                tmem_ld_32x32b_x16(cbase + kAccCols + c * 16, v1);
                tmem_ld_wait();
                const int nrows = min(16, t.rows - c * 16);
                if (p.swiglu && kEpi == kEpiQuant) {
                    // h as NVFP4: lanes 16h..16h+15 of this warp hold one 16-column block of each token row
                    const int64_t hcols = p.N / 2;
                    const int64_t n = (int64_t)t.nt * kBM + r;               // this lane's column of h
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const bool valid = i < nrows;
                        const float g = alpha * v0[i], u = alpha * v1[i];
                        const uint32_t hb = __bfloat16_as_ushort(__float2bfloat16_rn(swiglu_f32(g, u)));
                        if (valid) amax = max(amax, (uint32_t)(hb & 0x7FFFu));
                        uint32_t code;
                        const uint32_t S = quantize_half_warp_block(hb, valid, h_genc, code);
                        const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, code, 1);
                        const int64_t row = (int64_t)t.row0 + c * 16 + i;
                        if (valid && (lane & 1) == 0) p.qo.q[row * (hcols / 2) + n / 2] = (uint8_t)(code | (hi << 4));
                        if (valid && (lane & 15) == 0) {
                            const int64_t b = n >> 4;
                            uint8_t* piece = p.qo.sf + ((b >> 4) * p.qo.rows_per_slab + row) * 16;
                            piece[b & 15] = (uint8_t)S;
                            if ((hcols & 255) == 128 && b == (hcols >> 4) - 1)   // the last slab's padding
                                *reinterpret_cast<uint2*>(piece + 8) = make_uint2(0u, 0u);
                        }
                    }
                } else {
                    // Lane r holds column r of the block for 16 tokens. Each lane rounds its tokens in pairs
                    // (one BF16x2 conversion per pair), then lanes 2m and 2m + 1 swap halves so that each stores
                    // 32-bit words holding columns (2m, 2m + 1) of one token: the even lane the even tokens,
                    // the odd lane the odd ones (half the store instructions of 16-bit stores).
                    const bool odd = (lane & 1) != 0;
                    const int64_t ldo = p.swiglu ? p.N / 2 : p.N;
                    const int64_t col = p.swiglu ? (int64_t)t.nt * kBM : (int64_t)t.nt * (kNumA * kBM);
                    uint16_t* o = p.out + ((int64_t)t.row0 + c * 16) * ldo + col + (r & ~1);
                    const uint64_t a2 = f32x2_pack(alpha, alpha);
                    auto put = [&](uint32_t mine, int i, int64_t off) {   // mine: this lane's tokens i, i + 1
                        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, mine, 1);
                        const uint32_t word = odd ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
                        const int tok = i + (odd ? 1 : 0);
                        if (tok < nrows) {
                            amax = max(amax, max(word & 0x7FFFu, (word >> 16) & 0x7FFFu));
                            *reinterpret_cast<uint32_t*>(o + (int64_t)tok * ldo + off) = word;
                        }
                    };
                    if (p.swiglu) {
#pragma unroll
                        for (int i = 0; i < 16; i += 2) {
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(swiglu_f32(alpha * v0[i], alpha * v1[i]),
                                                                            swiglu_f32(alpha * v0[i + 1], alpha * v1[i + 1]));
                            put(*reinterpret_cast<const uint32_t*>(&b2), i, 0);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; i += 2)
                            put(f32x2_to_bf16x2(f32x2_mul(f32x2_pack(v0[i], v0[i + 1]), a2)), i, 0);
                        if (second) {
#pragma unroll
                            for (int i = 0; i < 16; i += 2)
                                put(f32x2_to_bf16x2(f32x2_mul(f32x2_pack(v1[i], v1[i + 1]), a2)), i, kBM);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[abuf]);
            if (++abuf == (uint32_t)C::kAccBufs) { abuf = 0; aphase ^= 1u; }
            if (kEpi == kEpiFinalize) {
                // Fused combine. Every row of this tile holds one (token, slot) product for the tile's output
                // columns; count the rows in per (token, column tile). The CTA that brings a token's count
                // to k writes that token's combined output for these columns, whichever CTA wrote the other
                // k - 1 rows, with the combine's arithmetic, so the result does not depend on the order.
                __threadfence();                            // this thread's y stores, device-wide, first
                if (!epi_sync()) break;
                const int i = (warp - 4) * 32 + lane;
                int32_t tok = -1;
                if (i < t.rows) {
                    const int32_t tk = __ldg(p.fin.src + t.row0 + i);
                    if (tk >= 0 && tk < p.fin.T) {
                        uint32_t* cnt = p.fin.counters + (int64_t)tk * p.fin.col_blocks + 2 * t.nt;
                        if (atomicAdd(cnt, 1u) == (uint32_t)(p.fin.k - 1)) {
                            atomicExch(cnt, 0u);            // left at zero for the next launch
                            tok = tk;
                        }
                    }
                }
                sh.fin_tok[i] = tok;
                __threadfence();                            // the other rows' stores are visible before the reads
                if (!epi_sync()) break;
                // one warp per token: lane l combines columns [8l, 8l + 8) of the tile's 256 (128 for a half tile)
                const int64_t col = (int64_t)t.nt * (kNumA * kBM) + lane * 8;
                const bool lane_on = second || lane * 8 < kBM;
                for (int j = warp - 4; j < t.rows; j += 4) {
                    const int32_t tk = sh.fin_tok[j];
                    if (tk >= 0 && lane_on) combine_vec8(p.out, p.N, p.fin.inv, p.fin.w, tk, p.fin.k, col, p.fin.out, p.N);
                }
                if (!epi_sync()) break;                     // fin_tok is rewritten by the next tile
            }
        }
        if (p.amax_out != nullptr) {
            amax = __reduce_max_sync(0xFFFFFFFFu, amax);
            if (lane == 0 && amax != 0u) atomicMax(p.amax_out, amax);
        }
    }

    // ---- teardown: every role has drained its own asynchronous work ----
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tmem, kTmemCols);
    // The last CTA to finish (every producer has taken its final item) leaves the counters at zero for
    // the next launch that draws this slot.
    if (tid == 0 && atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.sched, 0u);
        atomicExch(p.sched + 1, 0u);
    }
}

}  // namespace gg
}  // namespace nvfp4

using namespace nvfp4;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D byte tensor [rows, row_bytes] loaded in boxes of box_rows x box_bytes (128-byte swizzle when
// box_bytes is 128, none otherwise); rows past the end read as zeros.
static bool encode_rows_map(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, uint32_t box_rows,
                            uint32_t box_bytes) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_bytes, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D BF16 output [rows, cols] stored in boxes of 32 rows x box_cols columns (no swizzle).
static bool encode_out_map(CUtensorMap* m, void* base, int64_t rows, int64_t cols, uint32_t box_cols) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {box_cols, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed SwiGLU weights [E, N, K] viewed as 5-D bytes for the CTA-pair kernel: {128 bytes of a row,
// 16 rows of a slab, gate/up (the up tile of the same columns lies N/2 rows further), 8 slabs of a
// packed tile, packed tile index}. A box {128, 16, 2, 4, 1} gathers one CTA's 64 gate rows and the
// matching 64 up rows, interleaved 16 at a time. Tiles run only over gate tiles plus the ones whose
// up tile still lies inside the tensor, so no box can leave the allocation.
// The same view with a ninth slab (the tile's 2 KB of scales, right after its 16 KB of codes) and a
// box of one slab: {128, 16, 2, 1, 1} at slab 8 brings the gate and the up tile's scales in one load.
static bool encode_swiglu_weights_map(CUtensorMap* m, const void* w_packed, int32_t E, int64_t N, int64_t K,
                                      uint32_t box_slabs) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const int64_t ksteps = (K + 255) / 256;
    const int64_t tile_bytes = 18432;
    const int64_t up_stride = (N / 2 / 128) * ksteps * tile_bytes;
    const int64_t tiles = ((int64_t)E * N - N / 2) / 128 * ksteps;
    cuuint64_t dims[5] = {128u, 16u, 2u, 9u, (cuuint64_t)tiles};
    cuuint64_t strides[4] = {128u, (cuuint64_t)up_stride, 2048u, (cuuint64_t)tile_bytes};
    cuuint32_t box[5] = {128u, 16u, 2u, box_slabs, 1u};
    cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(w_packed), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Experts averaging at least this many rows use the wide tile shape, at least
// kPairMinAvgRows the CTA-pair kernel (grouped_gemm_pair.cu). Measured on B200:
// at 32 rows per expert on average with Zipf skew (the big experts span many
// row tiles) the wide shape is faster (gate/up 0.573 vs 0.594 ms, down 0.326 vs
// 0.333 ms, same box), at 16 the narrow one ~0.7%.
static constexpr int64_t kWideMinAvgRows = 32;
static constexpr int64_t kPairMinAvgRows = 192;

extern "C" nvfp4_status nvfp4_gemm_get_plan(nvfp4_gemm_plan* plan) {
    if (!plan) return NVFP4_ERR_INVALID_ARG;
    plan->tile_weight_rows = gg::kNumA * gg::kBM;
    plan->tile_tokens_max = gg::Narrow::kBNMax;
    plan->stage_k = gg::kBK;
    plan->stages = gg::Narrow::kStages;
    plan->stage_bytes_weights = gg::kNumA * gg::kABlockBytes;   // arrives with its scales in one packed tile
    plan->stage_bytes_weight_sf = gg::kNumA * gg::kSFStageBytes;
    plan->stage_bytes_act_max = gg::Narrow::kBBytes;
    plan->stage_bytes_act_sf = gg::kSFStageBytes;
    plan->smem_bytes = (int32_t)gg::Narrow::kSmemBytes;
    plan->tmem_columns = (int32_t)gg::kTmemCols;
    plan->threads = gg::kThreads;
    plan->wide_tile_tokens_max = gg::Wide::kBNMax;
    plan->wide_stage_bytes_act_max = gg::Wide::kBBytes;
    plan->wide_smem_bytes = (int32_t)gg::Wide::kSmemBytes;
    plan->wide_min_avg_rows = (int32_t)kWideMinAvgRows;
    plan->pair_tile_tokens_max = pair_gemm_tokens_max();
    plan->pair_smem_bytes = (int32_t)pair_gemm_smem_bytes();
    plan->pair_min_avg_rows = (int32_t)kPairMinAvgRows;
    return NVFP4_OK;
}

extern "C" int64_t nvfp4_gemm_stage_tx_bytes(int32_t tokens, int32_t wide) {
    const int64_t bn_max = wide ? gg::Wide::kBNMax : gg::Narrow::kBNMax;
    if (tokens <= 0 || tokens > bn_max) return -1;
    const int64_t bn = (tokens + gg::kBNStep - 1) / gg::kBNStep * gg::kBNStep;
    // MK part: the two weight tiles with their scales (packed together); NK part: the activation
    // tile plus its rows' 16 scale bytes of the K step (one bulk copy from the K-stage slab).
    return (int64_t)gg::kNumA * gg::kPackedTileBytes + bn * gg::kRowBytes + (int64_t)tokens * 16;
}

extern "C" nvfp4_status nvfp4_can_implement_with_budget(int64_t N, int64_t K, int32_t E, nvfp4_epilogue epi,
                                                        int64_t smem_optin_bytes) {
    if (epi != NVFP4_EPI_NONE && epi != NVFP4_EPI_SWIGLU) return NVFP4_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || E <= 0) return NVFP4_ERR_INVALID_ARG;
    if (E > gg::kMaxE || K % (gg::kBK / 2) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // NONE: 128-row weight blocks; SWIGLU: gate and up halves of 128-row blocks each (N / 2 % 128 == 0)
    if (N % (epi == NVFP4_EPI_SWIGLU ? gg::kNumA * gg::kBM : gg::kBM) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)E * N > INT32_MAX || K / 2 > INT32_MAX) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    // both tile shapes must fit: the launcher picks one from the rows per expert
    int64_t need = (int64_t)(gg::Wide::kSmemBytes > gg::Narrow::kSmemBytes ? gg::Wide::kSmemBytes
                                                                            : gg::Narrow::kSmemBytes);
    if ((int64_t)pair_gemm_smem_bytes() > need) need = (int64_t)pair_gemm_smem_bytes();
    if (smem_optin_bytes < need) return NVFP4_ERR_SMEM_BUDGET;
    return NVFP4_OK;
}

extern "C" nvfp4_status nvfp4_can_implement(int64_t N, int64_t K, int32_t E, nvfp4_epilogue epi) {
    const int optin = device_smem_optin();
    if (optin < 0) return NVFP4_ERR_CUDA;
    return nvfp4_can_implement_with_budget(N, K, E, epi, optin);
}

template <class C, int kEpi>
static nvfp4_status launch_variant(const CUtensorMap& tm_a, gg::Params prm, cudaStream_t s) {
    // the kernel's shared-memory opt-in, once per device (thread-safe)
    static std::once_flag once[64];
    static cudaError_t set_result[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
    std::call_once(once[dev], [&] {
        set_result[dev] = cudaFuncSetAttribute(gg::grouped_gemm_kernel<C, kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)C::kSmemBytes);
    });
    if (set_result[dev] != cudaSuccess) return NVFP4_ERR_CUDA;
    prm.sched = sched_counter_slot();
    if (!prm.sched) return NVFP4_ERR_CUDA;
    launch_pdl(gg::grouped_gemm_kernel<C, kEpi>, dim3(device_sm_count()), dim3(gg::kThreads), C::kSmemBytes, s, tm_a,
               prm);
    return NVFP4_OK;
}

extern "C" nvfp4_status moe_grouped_gemm_nvfp4(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                               const uint8_t* w_packed, const float* w_gscale,
                                               const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                               int64_t N, int64_t K, nvfp4_epilogue epi, uint16_t* out,
                                               nvfp4_stream_t stream) {
    return moe_grouped_gemm_nvfp4_amax(a_q, a_sf, a_gscale, w_packed, w_gscale, expert_offsets, E, max_rows, N, K,
                                       epi, out, nullptr, stream);
}

// Validates, encodes the tensor maps and launches one of the three kernels.
static nvfp4_status grouped_gemm(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                 const uint8_t* w_packed, const float* w_gscale, const int32_t* expert_offsets,
                                 int32_t E, int64_t max_rows, int64_t N, int64_t K, nvfp4_epilogue epi, uint16_t* out,
                                 uint32_t* out_amax, const Finalize& fin, const QuantOut& qo, nvfp4_stream_t stream) {
    // quantised h replaces the BF16 output: `out` then only anchors the (unused) output tensor map
    if (qo.q != nullptr) out = reinterpret_cast<uint16_t*>(qo.q);
    if (!a_q || !a_sf || !a_gscale || !w_packed || !w_gscale || !expert_offsets || !out)
        return NVFP4_ERR_INVALID_ARG;
    if ((uintptr_t)out_amax & 3u) return NVFP4_ERR_MISALIGNED;
    if (max_rows < 0 || max_rows > INT32_MAX) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_q) || !aligned16(a_sf) || !aligned16(w_packed) || !aligned16(out) ||
        ((uintptr_t)a_gscale & 3u) || ((uintptr_t)w_gscale & 3u) || ((uintptr_t)expert_offsets & 3u))
        return NVFP4_ERR_MISALIGNED;
    const int optin = device_smem_optin();
    if (optin < 0) return NVFP4_ERR_CUDA;
    nvfp4_status st = nvfp4_can_implement_with_budget(N, K, E, epi, optin);
    if (st != NVFP4_OK) return st;
    if (max_rows == 0) return NVFP4_OK;
    uint32_t* status = status_word_ptr();
    if (!status) return NVFP4_ERR_CUDA;

    CUtensorMap tm_a;
    if (!encode_rows_map(&tm_a, a_q, max_rows, K / 2, gg::kBNStep, 128)) return NVFP4_ERR_CUDA;

    gg::Params prm;
    prm.a_sf = a_sf;
    prm.a_gscale = a_gscale;
    prm.w_packed = w_packed;
    prm.w_gscale = w_gscale;
    prm.offsets = expert_offsets;
    prm.out = out;
    prm.E = E;
    prm.max_rows = max_rows;
    prm.N = N;
    prm.K = K;
    prm.swiglu = epi == NVFP4_EPI_SWIGLU ? 1 : 0;
    prm.amax_out = out_amax;
    prm.fin = fin;
    prm.qo = qo;
    prm.sched = nullptr;   // drawn by the launcher that runs (one slot per launch)
    prm.ctl.status = status;
    prm.ctl.timeout_ns = wait_timeout_ns();
    prm.ctl.flags = debug_flags();
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the CTA-pair tile covers 256 weight rows per column tile: NONE with N % 256 == 128 stays on one SM
    if (max_rows >= kPairMinAvgRows * (int64_t)E && N % (2 * gg::kBM) == 0) {
        CUtensorMap tm_a_full;  // one CTA's half of a full pair tile: 128 rows x 128 bytes
        if (!encode_rows_map(&tm_a_full, a_q, max_rows, K / 2, (uint32_t)pair_gemm_tokens_max() / 2, 128))
            return NVFP4_ERR_CUDA;
        CUtensorMap tm_out;  // one epilogue warp's 32-token block of the output
        // (with quantised h the map spans the codes buffer, [max_rows, N/4] bytes, and is never used)
        const int64_t out_cols = qo.q != nullptr ? N / 8 : prm.swiglu ? N / 2 : N;
        if (!encode_out_map(&tm_out, out, max_rows, out_cols, (uint32_t)pair_gemm_store_cols(prm.swiglu)))
            return NVFP4_ERR_CUDA;
        CUtensorMap tm_wsw = tm_a;  // SWIGLU: interleaved gate/up weight slabs (unused otherwise)
        CUtensorMap tm_wsf = tm_a;  // SWIGLU: the gate and up tiles' scales (unused otherwise)
        if (prm.swiglu && (!encode_swiglu_weights_map(&tm_wsw, w_packed, E, N, K, 4) ||
                           !encode_swiglu_weights_map(&tm_wsf, w_packed, E, N, K, 1)))
            return NVFP4_ERR_CUDA;
        return launch_grouped_gemm_pair(tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, a_sf, a_gscale, w_packed, w_gscale,
                                        expert_offsets, E, max_rows, N, K, prm.swiglu, out, out_amax, fin, qo, s,
                                        status);
    }
    const bool wide = max_rows >= kWideMinAvgRows * (int64_t)E;
    nvfp4_status ls;
    if (qo.q != nullptr)
        ls = wide ? launch_variant<gg::Wide, kEpiQuant>(tm_a, prm, s) : launch_variant<gg::Narrow, kEpiQuant>(tm_a, prm, s);
    else if (fin.out != nullptr)
        ls = wide ? launch_variant<gg::Wide, kEpiFinalize>(tm_a, prm, s)
                  : launch_variant<gg::Narrow, kEpiFinalize>(tm_a, prm, s);
    else
        ls = wide ? launch_variant<gg::Wide, kEpiPlain>(tm_a, prm, s) : launch_variant<gg::Narrow, kEpiPlain>(tm_a, prm, s);
    if (ls != NVFP4_OK) return ls;
    count_launch();
    return check_launch();
}

extern "C" nvfp4_status moe_grouped_gemm_nvfp4_amax(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                                    const uint8_t* w_packed, const float* w_gscale,
                                                    const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                                    int64_t N, int64_t K, nvfp4_epilogue epi, uint16_t* out,
                                                    uint32_t* out_amax, nvfp4_stream_t stream) {
    const Finalize none = {};
    const QuantOut bf16_out = {};
    return grouped_gemm(a_q, a_sf, a_gscale, w_packed, w_gscale, expert_offsets, E, max_rows, N, K, epi, out, out_amax,
                        none, bf16_out, stream);
}

extern "C" nvfp4_status moe_grouped_gemm_nvfp4_quant(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                                     const uint8_t* w_packed, const float* w_gscale,
                                                     const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                                     int64_t N, int64_t K, const float* h_gscale, uint8_t* q_h,
                                                     uint8_t* sf_h, uint32_t* h_amax, nvfp4_stream_t stream) {
    if (!h_gscale || !q_h || !sf_h) return NVFP4_ERR_INVALID_ARG;
    if (((uintptr_t)h_gscale & 3u) || !aligned16(q_h) || !aligned16(sf_h)) return NVFP4_ERR_MISALIGNED;
    QuantOut qo;
    qo.gdec = h_gscale;
    qo.q = q_h;
    qo.sf = sf_h;
    qo.rows_per_slab = max_rows;
    const Finalize none = {};
    return grouped_gemm(a_q, a_sf, a_gscale, w_packed, w_gscale, expert_offsets, E, max_rows, N, K, NVFP4_EPI_SWIGLU,
                        nullptr, h_amax, none, qo, stream);
}

extern "C" size_t moe_finalize_counters_size(int32_t T, int64_t N) {
    if (T <= 0 || N <= 0) return 0;
    return (size_t)T * (size_t)((N + 127) / 128) * sizeof(uint32_t);
}

extern "C" nvfp4_status moe_grouped_gemm_nvfp4_finalize(const uint8_t* a_q, const uint8_t* a_sf,
                                                        const float* a_gscale, const uint8_t* w_packed,
                                                        const float* w_gscale, const int32_t* expert_offsets,
                                                        int32_t E, int64_t max_rows, int64_t N, int64_t K,
                                                        uint16_t* y, const int32_t* perm_src,
                                                        const int32_t* inv_perm, const float* topk_w, int32_t T,
                                                        int32_t k, uint32_t* counters, uint16_t* out,
                                                        nvfp4_stream_t stream) {
    if (!perm_src || !inv_perm || !topk_w || !counters || !out || !y) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (k > 32 || (int64_t)T * k > max_rows) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (((uintptr_t)perm_src & 3u) || ((uintptr_t)inv_perm & 3u) || ((uintptr_t)topk_w & 3u) ||
        ((uintptr_t)counters & 3u) || ((uintptr_t)out & 1u))
        return NVFP4_ERR_MISALIGNED;
    Finalize fin;
    fin.src = perm_src;
    fin.inv = inv_perm;
    fin.w = topk_w;
    fin.counters = counters;
    fin.out = out;
    fin.T = T;
    fin.k = k;
    fin.col_blocks = (int32_t)((N + 127) / 128);
    const QuantOut bf16_out = {};
    return grouped_gemm(a_q, a_sf, a_gscale, w_packed, w_gscale, expert_offsets, E, max_rows, N, K, NVFP4_EPI_NONE, y,
                        nullptr, fin, bf16_out, stream);
}

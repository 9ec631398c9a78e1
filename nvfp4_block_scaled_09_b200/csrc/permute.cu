// permute.cu -- routing gather: group (token, slot) pairs by expert, stable in
// (t ascending, j ascending), and copy the quantised activation rows into
// expert order ("Peering into the CUTLASS Kernel Cache", Knowledge Required:
// each expert's weights multiply only the subset of tokens routed to it).
//
// Deterministic counting sort, no atomics on the output order:
//   1. count:  CTA c counts, per expert, the pairs of its 256 tokens.
//   2. scan:   one CTA turns the per-chunk counts into expert offsets and into
//              the first output row of every (chunk, expert) pair.
//   3. rank:   CTA c marks, per expert, which of its tokens route there (one
//              bit per token); a pair's rank inside its expert is the number of
//              marked earlier tokens (popcount), so positions follow token
//              order. A token lists each expert at most once, so slot order
//              inside a token never decides a rank.
//   4. gather: one warp per output row copies K/2 code bytes and K/16 scale
//              bytes with 16-byte vector loads and stores. The scales go out
//              row-major or in the K-stage layout (the 16 bytes of each
//              256-element K step into that step's [R x 16 B] slab; the 8
//              warps of a CTA write 8 adjacent rows, so each slab receives
//              128 contiguous bytes per CTA).
#include <mutex>

#include "common.cuh"
#include "quant_math.cuh"

namespace nvfp4 {
namespace {

constexpr int kTok = 256;           // tokens per chunk (one thread each)
constexpr int kMaxE = 1024;
constexpr int kWordsPerExpert = kTok / 32;

__global__ void __launch_bounds__(kTok) permute_count_kernel(const int32_t* __restrict__ ids, int32_t T, int32_t k,
                                                               int32_t E, int32_t* __restrict__ counts,
                                                               uint32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int32_t hist[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int32_t t = blockIdx.x * kTok + threadIdx.x;
    if (t < T) {
        for (int j = 0; j < k; j++) {
            const int32_t e = ids[(int64_t)t * k + j];
            if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
            else atomicOr(status, kStatusBadInput);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One CTA of kMaxE threads: thread e owns expert e.
__global__ void __launch_bounds__(kMaxE) permute_scan_kernel(int32_t* __restrict__ counts, int32_t nchunks,
                                                               int32_t E, int32_t* __restrict__ offsets) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int32_t warp_sums[kMaxE / 32];
    const int e = threadIdx.x;
    int32_t total = 0;
    if (e < E)
        for (int c = 0; c < nchunks; c++) total += counts[(int64_t)c * E + e];
    // exclusive scan of `total` over e
    const int lane = e & 31, warp = e >> 5;
    int32_t incl = total;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t s = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xFFFFFFFFu, s, o);
            if (lane >= o) s += v;
        }
        warp_sums[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int32_t excl = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + total;
        int32_t run = excl;  // first output row of (chunk c, expert e)
        for (int c = 0; c < nchunks; c++) {
            const int32_t n = counts[(int64_t)c * E + e];
            counts[(int64_t)c * E + e] = run;
            run += n;
        }
    }
}

__global__ void __launch_bounds__(kTok) permute_rank_kernel(const int32_t* __restrict__ ids, int32_t T, int32_t k,
                                                              int32_t E, const int32_t* __restrict__ base,
                                                              int32_t* __restrict__ perm_src,
                                                              int32_t* __restrict__ inv_perm, uint32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ uint32_t bits[];  // [E][kWordsPerExpert]
    for (int i = threadIdx.x; i < E * kWordsPerExpert; i += blockDim.x) bits[i] = 0u;
    __syncthreads();
    const int tl = threadIdx.x;
    const int32_t t = blockIdx.x * kTok + tl;
    const uint32_t my_bit = 1u << (tl & 31);
    const int my_word = tl >> 5;
    if (t < T) {
        for (int j = 0; j < k; j++) {
            const int32_t e = ids[(int64_t)t * k + j];
            if (e >= 0 && e < E) {
                const uint32_t old = atomicOr(&bits[e * kWordsPerExpert + my_word], my_bit);
                if (old & my_bit) atomicOr(status, kStatusBadInput);  // expert listed twice by one token
            }
        }
    }
    __syncthreads();
    if (t < T) {
        for (int j = 0; j < k; j++) {
            const int32_t e = ids[(int64_t)t * k + j];
            int32_t pos = -1;
            if (e >= 0 && e < E) {
                const uint32_t* row = bits + e * kWordsPerExpert;
                int32_t rank = 0;
                for (int w = 0; w < my_word; w++) rank += __popc(row[w]);
                rank += __popc(row[my_word] & (my_bit - 1u));
                pos = base[(int64_t)blockIdx.x * E + e] + rank;
                perm_src[pos] = t;
            }
            inv_perm[(int64_t)t * k + j] = pos;
        }
    }
}

// Small batches in one CTA (1024 threads) and one launch: count, scan and stable rank. Shared memory holds
// one bit per (expert, token) and, per 32-token word, the number of the expert's pairs before that word
// (the expert's offset included), so a pair's position is that prefix plus the popcount of the earlier
// tokens in its word: token order inside each expert, as the multi-kernel path produces. Both tables are
// word-major ([W][E]), so the per-expert passes read consecutive words across a warp; a thread keeps the
// expert ids of its first kIdsCached pairs in registers for the second pass.
constexpr int kIdsCached = 8;
// The ranking of one CTA of kMaxE threads; small_sm: 2 * E * ceil(T/32) words of shared memory.
__device__ __forceinline__ void rank_small(const int32_t* __restrict__ ids, int32_t T, int32_t k, int32_t E,
                                           int32_t* __restrict__ offsets, int32_t* __restrict__ perm_src,
                                           int32_t* __restrict__ inv_perm, uint32_t* status, uint32_t* small_sm) {
    __shared__ int32_t warp_sums[kMaxE / 32];
    const int W = (T + 31) / 32;                  // 32-token words per expert
    uint32_t* bits = small_sm;                    // [W][E]
    int32_t* pre = reinterpret_cast<int32_t*>(small_sm + (size_t)E * W);   // [W][E]
    const int tid = threadIdx.x;
    for (int i = tid; i < E * W; i += kMaxE) bits[i] = 0u;
    __syncthreads();
    const int64_t R = (int64_t)T * k;
    int32_t my_e[kIdsCached];
#pragma unroll
    for (int c = 0; c < kIdsCached; c++) {
        const int64_t i = tid + (int64_t)c * kMaxE;
        my_e[c] = i < R ? __ldg(ids + i) : -1;
    }
    bool bad = false;
    auto mark = [&](int64_t i, int32_t e) {
        const int32_t t = (int32_t)(i / k);
        if (e >= 0 && e < E) {
            const uint32_t bit = 1u << (t & 31);
            if (atomicOr(&bits[(t >> 5) * E + e], bit) & bit) bad = true;   // expert listed twice by one token
        } else {
            bad = true;
        }
    };
#pragma unroll
    for (int c = 0; c < kIdsCached; c++)
        if (tid + (int64_t)c * kMaxE < R) mark(tid + (int64_t)c * kMaxE, my_e[c]);
    for (int64_t i = tid + (int64_t)kIdsCached * kMaxE; i < R; i += kMaxE) mark(i, __ldg(ids + i));
    if (bad) atomicOr(status, kStatusBadInput);
    __syncthreads();
    int32_t total = 0;
    if (tid < E)
        for (int w = 0; w < W; w++) total += __popc(bits[w * E + tid]);
    // exclusive scan of the experts' totals
    const int lane = tid & 31, warp = tid >> 5;
    int32_t incl = total;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int32_t sacc = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xFFFFFFFFu, sacc, o);
            if (lane >= o) sacc += v;
        }
        warp_sums[lane] = sacc;
    }
    __syncthreads();
    if (tid < E) {
        const int32_t excl = incl - total + (warp > 0 ? warp_sums[warp - 1] : 0);
        offsets[tid] = excl;
        if (tid == E - 1) offsets[E] = excl + total;
        int32_t run = excl;
        for (int w = 0; w < W; w++) {
            pre[w * E + tid] = run;
            run += __popc(bits[w * E + tid]);
        }
    }
    __syncthreads();
    auto place = [&](int64_t i, int32_t e) {
        const int32_t t = (int32_t)(i / k);
        int32_t pos = -1;
        if (e >= 0 && e < E) {
            const int w = t >> 5;
            pos = pre[w * E + e] + __popc(bits[w * E + e] & ((1u << (t & 31)) - 1u));
            perm_src[pos] = t;
        }
        inv_perm[i] = pos;
    };
#pragma unroll
    for (int c = 0; c < kIdsCached; c++)
        if (tid + (int64_t)c * kMaxE < R) place(tid + (int64_t)c * kMaxE, my_e[c]);
    for (int64_t i = tid + (int64_t)kIdsCached * kMaxE; i < R; i += kMaxE) place(i, __ldg(ids + i));
}

__global__ void __launch_bounds__(kMaxE) permute_small_kernel(const int32_t* __restrict__ ids, int32_t T, int32_t k,
                                                                int32_t E, int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ perm_src,
                                                                int32_t* __restrict__ inv_perm, uint32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ uint32_t small_sm[];
    rank_small(ids, T, k, E, offsets, perm_src, inv_perm, status, small_sm);
}

// ---- quantise while permuting (small batches): moe_quantize_permute ----------------------------------
// Front: CTA 0 ranks every pair (rank_small); CTAs 1..G take the packed |x| maximum of a slice of x into
// partial[blockIdx.x - 1]. The two steps need nothing from each other, so they run side by side.
__global__ void __launch_bounds__(kMaxE) quantize_permute_front_kernel(
    const int32_t* __restrict__ ids, int32_t T, int32_t k, int32_t E, int32_t* __restrict__ offsets,
    int32_t* __restrict__ perm_src, int32_t* __restrict__ inv_perm, uint32_t* status, const uint4* __restrict__ x,
    int64_t nvec, uint32_t* __restrict__ partial, const uint8_t* __restrict__ pf, int64_t pf_bytes) {
    pdl_launch_dependents();
    // the next GEMM's first weight tiles (constant: no wait needed) start streaming into L2 while CTA 0 ranks
    if (blockIdx.x > 0)
        l2_prefetch_slice(pf, pf_bytes, (int64_t)(blockIdx.x - 1) * blockDim.x + threadIdx.x,
                          (int64_t)(gridDim.x - 1) * blockDim.x);
    pdl_wait();
    extern __shared__ uint32_t small_sm[];
    if (blockIdx.x == 0) {
        rank_small(ids, T, k, E, offsets, perm_src, inv_perm, status, small_sm);
        return;
    }
    uint32_t m = 0;
    const int64_t stride = (int64_t)(gridDim.x - 1) * blockDim.x;
    for (int64_t i = (int64_t)(blockIdx.x - 1) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        const uint4 v = __ldg(x + i);
        m = absmax_pair(m, v.x);
        m = absmax_pair(m, v.y);
        m = absmax_pair(m, v.z);
        m = absmax_pair(m, v.w);
    }
    m = warp_max_u32(fold_pair(m));
    __shared__ uint32_t s_warp[kMaxE / 32];
    if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        const uint32_t v = warp_max_u32(s_warp[threadIdx.x]);
        if (threadIdx.x == 0) partial[blockIdx.x - 1] = v;
    }
}

// Quantise and scatter: one warp per 32-block piece of token t's BF16 row quantises it once (quantize_block: the quantiser's
// own steps, with the global scale folded from the front's partials) and writes the codes and scales of
// every 16-element block to the permuted rows of its k pairs (inv_perm, from the front's ranking). A pair
// without a row (an invalid expert id, inv_perm -1) is skipped. kKStage: scales in the K-stage layout,
// else row-major.
template <bool kKStage>
__global__ void __launch_bounds__(256) quantize_scatter_kernel(const uint4* __restrict__ x, int32_t T, int64_t K,
                                                               int32_t k, const uint32_t* __restrict__ partial,
                                                               int npartial, const int32_t* __restrict__ inv_perm,
                                                               int64_t R, uint2* __restrict__ q_perm,
                                                               uint8_t* __restrict__ sf_perm, float* __restrict__ gdec_out) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ float s_genc;
    if (threadIdx.x < 32) {
        uint32_t m = 0;
        for (int i = threadIdx.x; i < npartial; i += 32) m = max(m, partial[i]);
        m = warp_max_u32(m);
        const GlobalScale g = global_scale(bf16_bits_to_f32(m), nullptr);
        if (threadIdx.x == 0) {
            s_genc = g.enc;
            if (blockIdx.x == 0) *gdec_out = g.dec;
        }
    }
    __syncthreads();
    const float g_enc = s_genc;
    const int64_t nb = K >> 4;                         // 16-element blocks per row
    const int64_t nchunk = (nb + 31) / 32;             // 32-block pieces of a row, one warp each
    const int64_t wi = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int64_t t = wi / nchunk;
    if (t >= T) return;
    const int lane = threadIdx.x & 31;
    const int32_t my_dst = lane < k ? __ldg(inv_perm + t * k + lane) : -1;   // lane j: the row of pair (t, j)
    const uint4* xs = x + t * (K >> 3);
    {   // every lane takes part in the shuffles below, active or not
        const int64_t b = (wi - t * nchunk) * 32 + lane;
        const bool active = b < nb;
        uint2 packed = make_uint2(0u, 0u);
        uint32_t S = 0u;
        if (active) S = quantize_block(__ldg(xs + 2 * b), __ldg(xs + 2 * b + 1), g_enc, packed);
        for (int j = 0; j < k; j++) {
            const int32_t d = __shfl_sync(0xFFFFFFFFu, my_dst, j);
            if (d < 0 || !active) continue;
            q_perm[(int64_t)d * nb + b] = packed;
            if (kKStage) {
                // slab of the 256-element K step b / 16, row d's 16-byte piece, byte b % 16
                const int64_t off = ((b >> 4) * R + d) * 16 + (b & 15);
                sf_perm[off] = (uint8_t)S;
                // K % 256 == 128: the last slab's piece holds 8 scales; its other 8 bytes are zero scales
                if ((nb & 15) == 8 && b == nb - 1) *reinterpret_cast<uint2*>(sf_perm + off + 1) = make_uint2(0u, 0u);
            } else {
                sf_perm[(int64_t)d * nb + b] = (uint8_t)S;
            }
        }
    }
}

// One warp per output row; rows whose source index is invalid become zeros.
// kHalf: K % 256 == 128. A row-major scale row is then 8 bytes past a multiple of 16, so the scales
// move in 8-byte units, and the last K-stage slab gets the row's last 8 scales plus 8 zero bytes.
template <bool kKStage, bool kHalf>
__global__ void __launch_bounds__(256) permute_gather_kernel(const uint4* __restrict__ q, const uint4* __restrict__ sf,
                                                             int64_t qvec, int64_t sfvec,
                                                             const int32_t* __restrict__ perm_src, int32_t T,
                                                             int64_t R, uint4* __restrict__ q_perm,
                                                             uint4* __restrict__ sf_perm) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t p = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (p >= R) return;
    const int lane = threadIdx.x & 31;
    const int32_t src = perm_src[p];
    const bool ok = src >= 0 && src < T;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const uint4* qs = q + (int64_t)(ok ? src : 0) * qvec;
    uint4* qd = q_perm + p * qvec;
    // four 16-byte pieces per lane in flight before their stores
    for (int64_t i0 = lane; i0 < qvec; i0 += 4 * 32) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; u++) v[u] = (ok && i0 + 32 * u < qvec) ? __ldg(qs + i0 + 32 * u) : zero;
#pragma unroll
        for (int u = 0; u < 4; u++)
            if (i0 + 32 * u < qvec) qd[i0 + 32 * u] = v[u];
    }
    if (!kHalf) {
        const uint4* ss = sf + (int64_t)(ok ? src : 0) * sfvec;
        for (int64_t i = lane; i < sfvec; i += 32) {
            const uint4 v = ok ? __ldg(ss + i) : zero;
            if (kKStage) sf_perm[i * R + p] = v;   // K step i's slab, row p
            else sf_perm[p * sfvec + i] = v;
        }
    } else {
        // sfvec counts 8-byte units here (K / 128 per row)
        const uint2* ss = reinterpret_cast<const uint2*>(sf) + (int64_t)(ok ? src : 0) * sfvec;
        const uint2 z2 = make_uint2(0u, 0u);
        if (kKStage) {
            for (int64_t i = lane; i < (sfvec + 1) / 2; i += 32) {
                const uint2 lo = ok ? __ldg(ss + 2 * i) : z2;
                const uint2 hi = (ok && 2 * i + 1 < sfvec) ? __ldg(ss + 2 * i + 1) : z2;
                sf_perm[i * R + p] = make_uint4(lo.x, lo.y, hi.x, hi.y);
            }
        } else {
            uint2* sd = reinterpret_cast<uint2*>(sf_perm) + p * sfvec;
            for (int64_t i = lane; i < sfvec; i += 32) sd[i] = ok ? __ldg(ss + i) : z2;
        }
    }
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

static inline int32_t permute_chunks(int32_t T) { return (T + kTok - 1) / kTok; }

// The one-CTA path takes up to this many pairs and this much shared memory (2 * E * ceil(T/32) words).
constexpr int64_t kSmallMaxPairs = 32768;
constexpr size_t kSmallMaxSmem = 160 * 1024;

// Opt the one-CTA kernel into the shared memory it may need, once per device.
static bool small_kernel_ready() {
    static std::once_flag once[64];
    static bool ok[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(permute_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmallMaxSmem) == cudaSuccess;
    });
    return ok[dev];
}

static void launch_gather(const uint8_t* q, const uint8_t* sf, int64_t K, const int32_t* perm_src, int32_t T,
                          int64_t R, uint8_t* q_perm, uint8_t* sf_perm, nvfp4_sf_layout layout, cudaStream_t s) {
    const bool kstage = layout == NVFP4_SF_KSTAGE, half = K % 256 != 0;
    auto kernel = kstage ? (half ? permute_gather_kernel<true, true> : permute_gather_kernel<true, false>)
                         : (half ? permute_gather_kernel<false, true> : permute_gather_kernel<false, false>);
    launch_pdl(kernel, dim3((unsigned)((R + 7) / 8)), dim3(256), 0, s, reinterpret_cast<const uint4*>(q),
               reinterpret_cast<const uint4*>(sf), K / 32, half ? K / 128 : K / 256, perm_src, T, R,
               reinterpret_cast<uint4*>(q_perm), reinterpret_cast<uint4*>(sf_perm));
}

extern "C" size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E) {
    (void)k;
    if (T <= 0 || E <= 0) return 0;
    return (size_t)permute_chunks(T) * (size_t)E * sizeof(int32_t);
}

extern "C" nvfp4_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, const uint8_t* q,
                                    const uint8_t* sf, int64_t K, uint8_t* q_perm, uint8_t* sf_perm,
                                    nvfp4_sf_layout sf_perm_layout, int32_t* expert_offsets, int32_t* perm_src,
                                    int32_t* inv_perm, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!topk_ids || !q || !sf || !q_perm || !sf_perm || !expert_offsets || !perm_src || !inv_perm)
        return NVFP4_ERR_INVALID_ARG;
    if (sf_perm_layout != NVFP4_SF_ROWMAJOR && sf_perm_layout != NVFP4_SF_KSTAGE) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || E <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (k > 32 || E > kMaxE || (int64_t)T * k >= (int64_t)1 << 31 || K % 128 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(topk_ids) || !aligned16(q) || !aligned16(sf) || !aligned16(q_perm) || !aligned16(sf_perm) ||
        !aligned16(expert_offsets) || !aligned16(perm_src) || !aligned16(inv_perm))
        return NVFP4_ERR_MISALIGNED;
    const size_t need = moe_permute_workspace_size(T, k, E);
    if (!ws || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_MISALIGNED;
    uint32_t* status = status_word_ptr();
    if (!status) return NVFP4_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int32_t nchunks = permute_chunks(T);
    int32_t* counts = static_cast<int32_t*>(ws);
    const int64_t R = (int64_t)T * k;

    // small batches (decode): one CTA ranks every pair, then the gather -- two launches
    const size_t small_smem = 2 * (size_t)E * (size_t)((T + 31) / 32) * sizeof(uint32_t);
    if (R <= kSmallMaxPairs && small_smem <= kSmallMaxSmem && small_kernel_ready()) {
        launch_pdl(permute_small_kernel, dim3(1), dim3(kMaxE), small_smem, s, topk_ids, T, k, E, expert_offsets,
                   perm_src, inv_perm, status);
        launch_gather(q, sf, K, perm_src, T, R, q_perm, sf_perm, sf_perm_layout, s);
        count_launch(2);
        return check_launch();
    }
    launch_pdl(permute_count_kernel, dim3(nchunks), dim3(kTok), 0, s, topk_ids, T, k, E, counts, status);
    launch_pdl(permute_scan_kernel, dim3(1), dim3(kMaxE), 0, s, counts, nchunks, E, expert_offsets);
    const size_t rank_smem = (size_t)E * kWordsPerExpert * sizeof(uint32_t);
    launch_pdl(permute_rank_kernel, dim3(nchunks), dim3(kTok), rank_smem, s, topk_ids, T, k, E, counts, perm_src, inv_perm, status);
    launch_gather(q, sf, K, perm_src, T, R, q_perm, sf_perm, sf_perm_layout, s);
    count_launch(4);
    return check_launch();
}

// ---------------------------------------------------------------------------
// moe_quantize_permute: x quantised straight into expert order.
//
// Small batches (the one-CTA ranking applies): two launches -- the front (ranking beside the amax
// partials of x) and the quantise-scatter (each token's row quantised once and written to its k permuted
// rows) -- and no token-order copy of the codes. Larger batches: nvfp4_quantize into the workspace, then
// moe_permute (the same bytes either way).

static constexpr int kFrontMaxPartials = 148;

static bool front_kernel_ready() {
    static std::once_flag once[64];
    static bool ok[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(quantize_permute_front_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmallMaxSmem) == cudaSuccess;
    });
    return ok[dev];
}

static size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

extern "C" size_t moe_quantize_permute_workspace_size(int32_t T, int32_t k, int32_t E, int64_t H) {
    if (T <= 0 || k <= 0 || E <= 0 || H <= 0 || H % 16 != 0) return 0;
    size_t scratch = moe_permute_workspace_size(T, k, E);
    const size_t qws = nvfp4_quantize_workspace_size(T, H);
    if (qws > scratch) scratch = qws;
    if ((size_t)kFrontMaxPartials * 4 > scratch) scratch = (size_t)kFrontMaxPartials * 4;
    return align256((size_t)T * (size_t)H / 2) + align256((size_t)T * (size_t)H / 16) + align256(scratch);
}

namespace nvfp4 {
nvfp4_status quantize_permute(const uint16_t* x, int32_t T, int64_t H, const int32_t* topk_ids, int32_t k, int32_t E,
                              uint8_t* q_perm, uint8_t* sf_perm, nvfp4_sf_layout layout, float* g_x,
                              int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm, uint8_t* q_x,
                              uint8_t* sf_x, void* scratch, size_t scratch_bytes, cudaStream_t s,
                              const void* l2_next, size_t l2_next_bytes) {
    const int64_t R = (int64_t)T * k;
    const size_t small_smem = 2 * (size_t)E * (size_t)((T + 31) / 32) * sizeof(uint32_t);
    const int64_t nvec = (int64_t)T * H / 8;
    if (R <= kSmallMaxPairs && small_smem <= kSmallMaxSmem && front_kernel_ready()) {
        uint32_t* status = status_word_ptr();
        if (!status) return NVFP4_ERR_CUDA;
        if (scratch_bytes < (size_t)kFrontMaxPartials * 4) return NVFP4_ERR_WORKSPACE;
        int64_t parts = (nvec + (int64_t)kMaxE * 4 - 1) / ((int64_t)kMaxE * 4);   // ~4 vectors per thread
        if (parts > kFrontMaxPartials) parts = kFrontMaxPartials;
        if (parts < 1) parts = 1;
        uint32_t* partial = static_cast<uint32_t*>(scratch);
        launch_pdl(quantize_permute_front_kernel, dim3((unsigned)(1 + parts)), dim3(kMaxE), small_smem, s, topk_ids, T,
                   k, E, expert_offsets, perm_src, inv_perm, status, reinterpret_cast<const uint4*>(x), nvec, partial,
                   static_cast<const uint8_t*>(l2_next), (int64_t)l2_next_bytes);
        auto kernel = layout == NVFP4_SF_KSTAGE ? quantize_scatter_kernel<true> : quantize_scatter_kernel<false>;
        const int64_t warps = (int64_t)T * ((H / 16 + 31) / 32);
        launch_pdl(kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, reinterpret_cast<const uint4*>(x), T, H, k,
                   partial, (int)parts, inv_perm, R, reinterpret_cast<uint2*>(q_perm), sf_perm, g_x);
        count_launch(2);
        return check_launch();
    }
    nvfp4_status st = nvfp4_quantize(x, T, H, nullptr, q_x, sf_x, g_x, NVFP4_SF_ROWMAJOR, scratch, scratch_bytes, s);
    if (st != NVFP4_OK) return st;
    return moe_permute(topk_ids, T, k, E, q_x, sf_x, H, q_perm, sf_perm, layout, expert_offsets, perm_src, inv_perm,
                       scratch, scratch_bytes, s);
}
}  // namespace nvfp4

extern "C" nvfp4_status moe_quantize_permute_prefetch(const uint16_t* x, int32_t T, int64_t H,
                                                      const int32_t* topk_ids, int32_t k, int32_t E, uint8_t* q_perm,
                                                      uint8_t* sf_perm, nvfp4_sf_layout sf_perm_layout, float* g_x,
                                                      int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                                      void* ws, size_t ws_bytes, const void* l2_next,
                                                      size_t l2_next_bytes, nvfp4_stream_t stream) {
    if (!x || !topk_ids || !q_perm || !sf_perm || !g_x || !expert_offsets || !perm_src || !inv_perm)
        return NVFP4_ERR_INVALID_ARG;
    if (sf_perm_layout != NVFP4_SF_ROWMAJOR && sf_perm_layout != NVFP4_SF_KSTAGE) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || E <= 0 || H <= 0) return NVFP4_ERR_INVALID_ARG;
    if (k > 32 || E > kMaxE || (int64_t)T * k >= (int64_t)1 << 31 || H % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(topk_ids) || !aligned16(q_perm) || !aligned16(sf_perm) ||
        !aligned16(expert_offsets) || !aligned16(perm_src) || !aligned16(inv_perm) || ((uintptr_t)g_x & 3u))
        return NVFP4_ERR_MISALIGNED;
    if (l2_next == nullptr) l2_next_bytes = 0;
    if (l2_next_bytes != 0 && !aligned16(l2_next)) return NVFP4_ERR_MISALIGNED;   // bulk prefetches start on 16 B
    const size_t need = moe_quantize_permute_workspace_size(T, k, E, H);
    if (!ws || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_MISALIGNED;
    uint8_t* b = static_cast<uint8_t*>(ws);
    uint8_t* q_x = b;
    uint8_t* sf_x = q_x + align256((size_t)T * (size_t)H / 2);
    uint8_t* scratch = sf_x + align256((size_t)T * (size_t)H / 16);
    const size_t scratch_bytes = need - (size_t)(scratch - b);
    return quantize_permute(x, T, H, topk_ids, k, E, q_perm, sf_perm, sf_perm_layout, g_x, expert_offsets, perm_src,
                            inv_perm, q_x, sf_x, scratch, scratch_bytes, reinterpret_cast<cudaStream_t>(stream),
                            l2_next, l2_next_bytes);
}

extern "C" nvfp4_status moe_quantize_permute(const uint16_t* x, int32_t T, int64_t H, const int32_t* topk_ids,
                                             int32_t k, int32_t E, uint8_t* q_perm, uint8_t* sf_perm,
                                             nvfp4_sf_layout sf_perm_layout, float* g_x, int32_t* expert_offsets,
                                             int32_t* perm_src, int32_t* inv_perm, void* ws, size_t ws_bytes,
                                             nvfp4_stream_t stream) {
    return moe_quantize_permute_prefetch(x, T, H, topk_ids, k, E, q_perm, sf_perm, sf_perm_layout, g_x,
                                         expert_offsets, perm_src, inv_perm, ws, ws_bytes, nullptr, 0, stream);
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the same four kernels, with the count table in a fixed
// file-scope device array instead of a caller workspace (for callers that
// cannot allocate device memory). Host code must not pass the array's name to
// a kernel: on the host it is only a stand-in symbol, so its device address is
// looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------
static __device__ __align__(256) int32_t g_permute_noalloc_scratch[NVFP4_PERMUTE_NOALLOC_SCRATCH_ENTRIES];

namespace {
constexpr int kNoAllocMaxDevices = 64;
int32_t* g_noalloc_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device, or nullptr.
int32_t* noalloc_scratch_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        int32_t* p = nullptr;
        if (cudaGetSymbolAddress((void**)&p, g_permute_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" nvfp4_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                                            const uint8_t* q, const uint8_t* sf, int64_t K, uint8_t* q_perm,
                                            uint8_t* sf_perm, nvfp4_sf_layout sf_perm_layout,
                                            int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                            nvfp4_stream_t stream) {
    if (!topk_ids || !q || !sf || !q_perm || !sf_perm || !expert_offsets || !perm_src || !inv_perm)
        return NVFP4_ERR_INVALID_ARG;
    if (sf_perm_layout != NVFP4_SF_ROWMAJOR && sf_perm_layout != NVFP4_SF_KSTAGE) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || E <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (k > 32 || E > kMaxE || (int64_t)T * k >= (int64_t)1 << 31 || K % 128 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int32_t nchunks = permute_chunks(T);
    if ((int64_t)nchunks * E > NVFP4_PERMUTE_NOALLOC_SCRATCH_ENTRIES) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(topk_ids) || !aligned16(q) || !aligned16(sf) || !aligned16(q_perm) || !aligned16(sf_perm) ||
        !aligned16(expert_offsets) || !aligned16(perm_src) || !aligned16(inv_perm))
        return NVFP4_ERR_MISALIGNED;
    int32_t* counts = noalloc_scratch_ptr();
    uint32_t* status = status_word_ptr();
    if (!counts || !status) return NVFP4_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t R = (int64_t)T * k;
    launch_pdl(permute_count_kernel, dim3(nchunks), dim3(kTok), 0, s, topk_ids, T, k, E, counts, status);
    launch_pdl(permute_scan_kernel, dim3(1), dim3(kMaxE), 0, s, counts, nchunks, E, expert_offsets);
    const size_t rank_smem = (size_t)E * kWordsPerExpert * sizeof(uint32_t);
    launch_pdl(permute_rank_kernel, dim3(nchunks), dim3(kTok), rank_smem, s, topk_ids, T, k, E, counts, perm_src, inv_perm, status);
    launch_gather(q, sf, K, perm_src, T, R, q_perm, sf_perm, sf_perm_layout, s);
    count_launch(4);
    return check_launch();
}

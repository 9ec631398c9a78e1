// route.cu -- the MoE router: top-k experts of each token by logit and the
// softmax of the chosen logits, the routing that decides which tokens each
// expert's grouped GEMM sees ("Peering into the CUTLASS Kernel Cache",
// Knowledge Required: each expert's weights multiply the subset of tokens
// routed to it). The pages do not describe the router itself; the reading
// taken: the k largest logits by value, the lower expert index first among
// equal values, weights = softmax over the row restricted to those k and
// renormalised (= the softmax of the k chosen logits).
//
// One warp per token, no tensor cores, no shared memory:
//   - lane l holds logits e = l, l + 32, ... (coalesced 128-byte loads) as
//     64-bit keys: the float's order-preserving bit pattern above the bitwise
//     complement of e, so one integer max picks the larger value and, among
//     equal values, the lower index (-0 is turned into +0 first);
//   - k rounds of a lane-local max over the untaken keys and a 5-step shuffle
//     max across the warp; the owning lane marks its key taken;
//   - lane j < k computes exp(z_j - z_0) in FP64; lane 0 sums them in j order;
//     each lane rounds e_j / sum once to FP32. A token whose largest logit is
//     -inf gets 1/k per slot.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kWarps = 8;            // tokens per CTA
constexpr int kMaxPerLane = 32;      // E <= 1024
constexpr int kMaxE = 32 * kMaxPerLane;

__device__ __forceinline__ uint64_t route_key(float v, int e) {
    if (v == 0.0f) v = 0.0f;         // -0 and +0 are equal logits
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint32_t)(~(uint32_t)e);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

template <int kPerLane>
__global__ void __launch_bounds__(kWarps * 32) route_topk_kernel(const float* __restrict__ logits, int32_t T,
                                                                 int32_t E, int32_t k, int32_t* __restrict__ ids,
                                                                 float* __restrict__ w) {
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* z = logits + t * E;
    uint64_t key[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; i++) {
        const int e = lane + 32 * i;
        key[i] = e < E ? route_key(__ldg(z + e), e) : 0ull;   // 0 sorts below every logit's key
    }
    uint32_t taken = 0u;
    int32_t my_id = 0;      // lane j keeps the j-th choice
    float my_z = 0.0f;
    for (int j = 0; j < k; j++) {
        uint64_t best = 0ull;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < kPerLane; i++) {
            if (!((taken >> i) & 1u) && key[i] > best) {
                best = key[i];
                bi = i;
            }
        }
        const uint64_t win = warp_max_u64(best);
        if (best == win && best != 0ull) taken |= 1u << bi;   // keys are distinct: one lane owns the winner
        const int32_t e = (int32_t)(~(uint32_t)win);
        if (lane == j) {
            my_id = e;
            my_z = __ldg(z + e);
        }
    }
    // softmax of the chosen logits in FP64, summed in choice order, one rounding to FP32
    const float z0 = __shfl_sync(0xFFFFFFFFu, my_z, 0);
    const bool all_neg_inf = isinf(z0) && z0 < 0.0f;
    const double ex = lane < k ? exp((double)my_z - (double)z0) : 0.0;
    double sum = 0.0;
    for (int j = 0; j < k; j++) sum += __shfl_sync(0xFFFFFFFFu, ex, j);   // every lane adds in the same order
    if (lane < k) {
        ids[t * k + lane] = my_id;
        w[t * k + lane] = all_neg_inf ? (float)(1.0 / (double)k) : (float)(ex / sum);
    }
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* topk_ids,
                                       float* topk_w, nvfp4_stream_t stream) {
    if (!logits || !topk_ids || !topk_w) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || E <= 0 || k <= 0) return NVFP4_ERR_INVALID_ARG;
    if (E > kMaxE || k > 32 || k > E) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (((uintptr_t)logits & 3u) || ((uintptr_t)topk_ids & 3u) || ((uintptr_t)topk_w & 3u))
        return NVFP4_ERR_MISALIGNED;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)((T + kWarps - 1) / kWarps)), block(kWarps * 32);
    const int per_lane = (E + 31) / 32;
    if (per_lane <= 8)
        launch_pdl(route_topk_kernel<8>, grid, block, 0, s, logits, T, E, k, topk_ids, topk_w);
    else
        launch_pdl(route_topk_kernel<kMaxPerLane>, grid, block, 0, s, logits, T, E, k, topk_ids, topk_w);
    count_launch();
    return check_launch();
}

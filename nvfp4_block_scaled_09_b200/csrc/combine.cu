// combine.cu -- top-k weighted combine of the expert outputs back into token
// order: the final MoE output write that the FINALIZE epilogue performs
// ("Peering into the CUTLASS Kernel", Input Knowledge Required, item 5).
//
//   out[t, :] = BF16( sum_{j ascending} w[t, j] * y[inv_perm[t*k + j], :] )
//
// Memory bound (reads k rows of y per token, writes one row): each thread owns
// 8 consecutive columns (16-byte loads and stores; combine_vec8). The sum is accumulated in
// FP64: a product of an FP32 weight and a BF16 value has at most 32
// significant bits, so every product is exact and the only roundings are the
// FP64 additions and one final rounding to BF16 (through round-to-odd FP32,
// which keeps that single rounding correct). FP64 costs nothing here: the
// kernel moves 2 bytes per FMA.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;
constexpr int kColsPerThread = 8;

// One thread per (token, 16-byte column group): all of a token's k <= 8 slots are loaded before any is
// accumulated, so the k row reads are in flight together (the combine is latency-bound at decode sizes).
__global__ void __launch_bounds__(kThreads) combine_kernel(const uint16_t* __restrict__ y,
                                                           const int32_t* __restrict__ inv_perm,
                                                           const float* __restrict__ w, int64_t T, int32_t k,
                                                           int64_t H, uint16_t* __restrict__ out) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x;  // 16-byte column group
    if (c * kColsPerThread >= H) return;
    for (int64_t t = blockIdx.y; t < T; t += gridDim.y)
        combine_vec8<8>(y, H, inv_perm, w, (int32_t)t, k, c * kColsPerThread, out, H);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status moe_unpermute_combine(const uint16_t* y, const int32_t* inv_perm, const float* topk_w,
                                              int32_t T, int32_t k, int64_t H, uint16_t* out,
                                              nvfp4_stream_t stream) {
    if (!y || !inv_perm || !topk_w || !out) return NVFP4_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || H <= 0) return NVFP4_ERR_INVALID_ARG;
    if (k > 32 || H % kColsPerThread != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(y) || !aligned16(out) || ((uintptr_t)inv_perm & 3u) || ((uintptr_t)topk_w & 3u))
        return NVFP4_ERR_MISALIGNED;
    const int64_t hvec = H / kColsPerThread;
    dim3 grid((unsigned)((hvec + kThreads - 1) / kThreads), (unsigned)(T < 65535 ? T : 65535));  // tokens loop
    launch_pdl(combine_kernel, dim3(grid), dim3(kThreads), 0, reinterpret_cast<cudaStream_t>(stream), y, inv_perm,
               topk_w, (int64_t)T, k, H, out);
    count_launch();
    return check_launch();
}

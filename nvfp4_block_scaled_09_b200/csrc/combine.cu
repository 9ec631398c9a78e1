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
// Grid size in CTAs per SM. 4 CTAs fit on an SM at once (the launch bound keeps a thread at 64 registers:
// without it ptxas took 86-108 and 2 CTAs fit; measured 204 -> 170 us at 8192 tokens, 14.7 -> 12.1 us at 512,
// same bits), so this is several waves of short token walks. Measured on B200 (same box, bit-identical
// outputs): 3 per SM (one wave, long walks) 191.8 us at 8192 tokens and 17.7 us at 512; 12, 24 and 40 per SM
// 172-174 us and 12.6 us (24 best).
constexpr int kCtasPerSm = 24;

// Each thread owns one 16-byte column group and walks tokens blockIdx.y, + gridDim.y, ... (a grid of
// kCtasPerSm CTAs per SM: several waves of short walks). Slots go in groups of 8: a group's row indices
// and weights, then its rows (all in flight together), then its FP64 sums in slot order. For k <= 8 (one group) the next token's
// slot indices and weights are loaded while the current token's rows are in flight, so a thread waits for
// one round of row reads per token (the combine is bound by that latency at decode sizes). A row index past
// the last row of y is skipped and latched as bad input.
template <bool kOneGroup>   // k <= 8
__global__ void __launch_bounds__(kThreads, 4) combine_kernel(const uint16_t* __restrict__ y,
                                                           const int32_t* __restrict__ inv_perm,
                                                           const float* __restrict__ w, int64_t T, int32_t k,
                                                           int64_t H, uint16_t* __restrict__ out, uint32_t* status) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x;  // 16-byte column group
    if (c * kColsPerThread >= H) return;
    const int64_t col = c * kColsPerThread;
    const int64_t R = T * k;
    bool bad = false;
    int32_t p[8];
    float s[8];
    auto load_slots = [&](int64_t t, int j0) {
#pragma unroll
        for (int j = 0; j < 8; j++) {
            int32_t pj = j0 + j < k ? __ldg(inv_perm + t * k + j0 + j) : -1;
            if (pj >= R) {
                bad = true;
                pj = -1;
            }
            p[j] = pj;
            s[j] = j0 + j < k ? __ldg(w + t * k + j0 + j) : 0.0f;
        }
    };
    auto accumulate = [&](const uint4 (&v)[8], const int32_t (&pc)[8], const float (&sc)[8], double (&a)[8]) {
#pragma unroll
        for (int j = 0; j < 8; j++) {   // slots ascending (the oracle's order)
            if (pc[j] < 0) continue;
            const double sd = (double)sc[j];
            const uint32_t x[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int i = 0; i < 4; i++) {
                a[2 * i] = fma(sd, (double)__uint_as_float(x[i] << 16), a[2 * i]);
                a[2 * i + 1] = fma(sd, (double)__uint_as_float(x[i] & 0xFFFF0000u), a[2 * i + 1]);
            }
        }
    };
    auto store = [&](int64_t t, const double (&a)[8]) {
        uint4 o;
        o.x = f64_to_bf16_bits(a[0]) | (f64_to_bf16_bits(a[1]) << 16);
        o.y = f64_to_bf16_bits(a[2]) | (f64_to_bf16_bits(a[3]) << 16);
        o.z = f64_to_bf16_bits(a[4]) | (f64_to_bf16_bits(a[5]) << 16);
        o.w = f64_to_bf16_bits(a[6]) | (f64_to_bf16_bits(a[7]) << 16);
        *reinterpret_cast<uint4*>(out + t * H + col) = o;
    };
    int64_t t = blockIdx.y;
    if (kOneGroup && t < T) load_slots(t, 0);
    while (t < T) {
        const int64_t tn = t + gridDim.y;
        double a[8];
#pragma unroll
        for (int i = 0; i < 8; i++) a[i] = 0.0;
        for (int j0 = 0; j0 < (kOneGroup ? 1 : k); j0 += 8) {
            if (!kOneGroup) load_slots(t, j0);
            uint4 v[8];
            float sc[8];
            int32_t pc[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                pc[j] = p[j];
                sc[j] = s[j];
                v[j] = pc[j] >= 0 ? __ldcg(reinterpret_cast<const uint4*>(y + (int64_t)pc[j] * H + col))
                                  : make_uint4(0, 0, 0, 0);
            }
            if (kOneGroup && tn < T) load_slots(tn, 0);   // the next token's slots, while these rows are in flight
            accumulate(v, pc, sc, a);
        }
        store(t, a);
        t = tn;
    }
    if (bad) atomicOr(status, kStatusBadInput);
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
    // kCtasPerSm CTAs per SM in all (each thread walks tokens)
    const int64_t gx = (hvec + kThreads - 1) / kThreads;
    int64_t gy = ((int64_t)device_sm_count() * kCtasPerSm + gx - 1) / gx;
    if (gy > T) gy = T;
    if (gy > 65535) gy = 65535;
    dim3 grid((unsigned)gx, (unsigned)gy);
    uint32_t* status = status_word_ptr();
    if (!status) return NVFP4_ERR_CUDA;
    launch_pdl(k <= 8 ? combine_kernel<true> : combine_kernel<false>, dim3(grid), dim3(kThreads), 0,
               reinterpret_cast<cudaStream_t>(stream), y, inv_perm, topk_w, (int64_t)T, k, H, out, status);
    count_launch();
    return check_launch();
}

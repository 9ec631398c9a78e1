// quantize.cu -- BF16 -> NVFP4 (packed E2M1 codes, E4M3 block scales, FP32
// global scale) for one tensor.
//
// Format: two FP4 values per byte and one FP8 scale per 16 elements ("Peering
// into the CUTLASS SharedStorage", Input Knowledge Required, item 3). The
// global scale maps the tensor amax onto 6 * 448 (E2M1 max times E4M3 max) and
// is stored as the dequantisation multiplier g_dec = amax / 2688.
//
// Two memory-bound passes, no tensor cores:
//   1. amax_partial_kernel: grid-stride, 16-byte loads, packed 16-bit integer
//      max of |bf16| bit patterns (finite BF16 magnitudes order like their
//      bits), one partial per CTA.
//   2. quantize_kernel: every CTA folds the partials into the tensor amax (a
//      few KB from L2), then each thread turns one 16-element block (32 bytes
//      in) into 8 code bytes and one scale byte with the hardware satfinite
//      round-to-nearest-even conversions.
#include "common.cuh"
#include "quant_math.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxPartials = 8 * 148;

// kRaise: atomically raise partial[0] to the tensor amax instead of one partial per CTA.
template <bool kRaise>
__global__ void __launch_bounds__(kThreads) amax_partial_kernel(const uint4* __restrict__ x, int64_t nvec,
                                                                 uint32_t* __restrict__ partial) {
    pdl_launch_dependents();
    pdl_wait();
    uint32_t m = 0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
        uint4 v = __ldg(x + i);  // default caching: the quantiser reads x again right after
        m = absmax_pair(m, v.x);
        m = absmax_pair(m, v.y);
        m = absmax_pair(m, v.z);
        m = absmax_pair(m, v.w);
    }
    m = warp_max_u32(fold_pair(m));
    __shared__ uint32_t s_warp[kThreads / 32];
    if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint32_t v = threadIdx.x < kThreads / 32 ? s_warp[threadIdx.x] : 0u;
        v = warp_max_u32(v);
        if (threadIdx.x == 0) {
            if (kRaise) atomicMax(partial, v);
            else partial[blockIdx.x] = v;
        }
    }
}

// kLayout: the nvfp4_sf_layout the block scales are written in.
template <int kLayout>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const uint4* __restrict__ x, int64_t rows, int64_t K,
                                                            const float* __restrict__ gdec_in,
                                                            const uint32_t* __restrict__ partial, int npartial,
                                                            uint2* __restrict__ q, uint8_t* __restrict__ sf,
                                                            float* __restrict__ gdec_out, const uint8_t* __restrict__ pf,
                                                            int64_t pf_bytes) {
    pdl_launch_dependents();
    // the next GEMM's first weight tiles (constant: no wait needed) start streaming into L2 meanwhile
    l2_prefetch_slice(pf, pf_bytes, (int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x);
    pdl_wait();
    __shared__ float s_genc;
    if (threadIdx.x < 32) {
        float amax = 0.0f;
        if (gdec_in == nullptr) {
            uint32_t m = 0;
            for (int i = threadIdx.x; i < npartial; i += 32) m = max(m, partial[i]);
            m = warp_max_u32(m);
            amax = bf16_bits_to_f32(m);
        }
        const GlobalScale g = global_scale(amax, gdec_in);
        if (threadIdx.x == 0) {
            s_genc = g.enc;
            if (blockIdx.x == 0) *gdec_out = g.dec;
        }
    }
    __syncthreads();
    const float g_enc = s_genc;
    const int64_t blocks_per_row = K >> 4;
    const int64_t nblk = rows * blocks_per_row;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        uint2 packed;
        const uint32_t S = quantize_block(__ldcs(x + 2 * b), __ldcs(x + 2 * b + 1), g_enc, packed);
        q[b] = packed;
        int64_t sf_off;
        if (kLayout == NVFP4_SF_MMA_TILED) {
            const int64_t r = b / blocks_per_row, kb = b - r * blocks_per_row;
            const int64_t atom = (r >> 7) * (K >> 6) + (kb >> 2);
            sf_off = atom * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
        } else if (kLayout == NVFP4_SF_KSTAGE) {
            // slab of the 256-element K step kb / 16, row r's 16-byte piece, byte kb % 16
            const int64_t r = b / blocks_per_row, kb = b - r * blocks_per_row;
            sf_off = ((kb >> 4) * rows + r) * 16 + (kb & 15);
            // K % 256 == 128: the last slab's piece holds 8 scales; its other 8 bytes are zero scales
            if ((blocks_per_row & 15) == 8 && kb == blocks_per_row - 1)
                *reinterpret_cast<uint2*>(sf + sf_off + 1) = make_uint2(0u, 0u);
        } else {
            sf_off = b;
        }
        sf[sf_off] = (uint8_t)S;
    }
}

}  // namespace

static int amax_grid(int64_t nvec) {
    int64_t g = (nvec + kThreads * 4 - 1) / (kThreads * 4);
    if (g < 1) g = 1;
    if (g > kMaxPartials) g = kMaxPartials;
    return (int)g;
}

// Second pass: every CTA folds the npartial amax words (BF16 bits) into the tensor amax, then quantises.
static void launch_quantize(const uint16_t* x, int64_t rows, int64_t K, const float* global_scale_in,
                            const uint32_t* partial, int npartial, uint8_t* q, uint8_t* sf, float* global_scale_out,
                            nvfp4_sf_layout layout, cudaStream_t s, const void* l2_next = nullptr,
                            size_t l2_next_bytes = 0) {
    const int64_t nblk = rows * K / 16;
    int64_t grid_q = (nblk + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)device_sm_count() * 16;
    if (grid_q > cap) grid_q = cap;
    if (grid_q < 1) grid_q = 1;
    auto kernel = layout == NVFP4_SF_MMA_TILED ? quantize_kernel<NVFP4_SF_MMA_TILED>
                  : layout == NVFP4_SF_KSTAGE  ? quantize_kernel<NVFP4_SF_KSTAGE>
                                               : quantize_kernel<NVFP4_SF_ROWMAJOR>;
    launch_pdl(kernel, dim3((int)grid_q), dim3(kThreads), 0, s, reinterpret_cast<const uint4*>(x), rows, K,
               global_scale_in, partial, npartial, reinterpret_cast<uint2*>(q), sf, global_scale_out,
               static_cast<const uint8_t*>(l2_next), (int64_t)l2_next_bytes);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_quantize_workspace_size(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return (size_t)amax_grid(rows * K / 8) * sizeof(uint32_t);
}

extern "C" nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t rows, int64_t K, const float* global_scale_in,
                                       uint8_t* q, uint8_t* sf, float* global_scale_out, nvfp4_sf_layout layout,
                                       void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!x || !q || !sf || !global_scale_out) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_MMA_TILED && layout != NVFP4_SF_KSTAGE)
        return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (layout == NVFP4_SF_MMA_TILED && (rows % 128 != 0 || K % 64 != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (layout == NVFP4_SF_KSTAGE && K % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned8(q) || (layout == NVFP4_SF_KSTAGE && !aligned16(sf))) return NVFP4_ERR_MISALIGNED;
    if (((uintptr_t)global_scale_out & 3u) || (global_scale_in && ((uintptr_t)global_scale_in & 3u)))
        return NVFP4_ERR_MISALIGNED;
    const int64_t nvec = rows * K / 8;
    const int grid_a = amax_grid(nvec);
    if (global_scale_in == nullptr) {
        if (!ws || ws_bytes < (size_t)grid_a * sizeof(uint32_t)) return NVFP4_ERR_WORKSPACE;
        if ((uintptr_t)ws & 3u) return NVFP4_ERR_MISALIGNED;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t* partial = static_cast<uint32_t*>(ws);
    if (global_scale_in == nullptr) {
        launch_pdl(amax_partial_kernel<false>, dim3(grid_a), dim3(kThreads), 0, s, reinterpret_cast<const uint4*>(x), nvec, partial);
        count_launch();
    }
    launch_quantize(x, rows, K, global_scale_in, partial, grid_a, q, sf, global_scale_out, layout, s);
    count_launch();
    return check_launch();
}

extern "C" nvfp4_status nvfp4_quantize_from_amax_prefetch(const uint16_t* x, int64_t rows, int64_t K,
                                                          const uint32_t* amax_bits, uint8_t* q, uint8_t* sf,
                                                          float* global_scale_out, nvfp4_sf_layout layout,
                                                          const void* l2_next, size_t l2_next_bytes,
                                                          nvfp4_stream_t stream) {
    if (!x || !q || !sf || !global_scale_out || !amax_bits) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (layout != NVFP4_SF_ROWMAJOR && layout != NVFP4_SF_MMA_TILED && layout != NVFP4_SF_KSTAGE)
        return NVFP4_ERR_INVALID_ARG;
    if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (layout == NVFP4_SF_MMA_TILED && (rows % 128 != 0 || K % 64 != 0)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (layout == NVFP4_SF_KSTAGE && K % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned8(q) || (layout == NVFP4_SF_KSTAGE && !aligned16(sf))) return NVFP4_ERR_MISALIGNED;
    if (((uintptr_t)global_scale_out & 3u) || ((uintptr_t)amax_bits & 3u)) return NVFP4_ERR_MISALIGNED;
    if (l2_next == nullptr) l2_next_bytes = 0;
    if (l2_next_bytes != 0 && !aligned16(l2_next)) return NVFP4_ERR_MISALIGNED;   // bulk prefetches start on 16 B
    launch_quantize(x, rows, K, nullptr, amax_bits, 1, q, sf, global_scale_out, layout,
                    reinterpret_cast<cudaStream_t>(stream), l2_next, l2_next_bytes);
    count_launch();
    return check_launch();
}

extern "C" nvfp4_status nvfp4_quantize_from_amax(const uint16_t* x, int64_t rows, int64_t K, const uint32_t* amax_bits,
                                                 uint8_t* q, uint8_t* sf, float* global_scale_out,
                                                 nvfp4_sf_layout layout, nvfp4_stream_t stream) {
    return nvfp4_quantize_from_amax_prefetch(x, rows, K, amax_bits, q, sf, global_scale_out, layout, nullptr, 0,
                                             stream);
}

extern "C" nvfp4_status nvfp4_amax(const uint16_t* x, int64_t rows, int64_t K, uint32_t* amax_bits,
                                   nvfp4_stream_t stream) {
    if (!x || !amax_bits) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (K % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || ((uintptr_t)amax_bits & 3u)) return NVFP4_ERR_MISALIGNED;
    const int64_t nvec = rows * K / 8;
    launch_pdl(amax_partial_kernel<true>, dim3(amax_grid(nvec)), dim3(kThreads), 0,
               reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<const uint4*>(x), nvec, amax_bits);
    count_launch();
    return check_launch();
}

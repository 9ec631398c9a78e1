// pack.cu -- one-time packing of quantised weights into the layout the grouped
// GEMM streams.
//
// A weight matrix [rows, K] (rows % 128 == 0, K % 128 == 0) is cut into tiles
// of 128 rows x 256 K-elements; tile (rb, kt) is one contiguous 18,432-byte
// chunk at ((rb * ceil(K/256)) + kt) * 18432 (when K % 256 == 128 the last
// tile of each row block holds 128 K-elements and zeros -- codes +0 and
// scales 0 -- in place of the other 128, which the GEMM never multiplies):
//   bytes [0, 16384): the 128 x 128 code bytes as the tensor core reads them
//     with 128-byte swizzling -- row r at r*128, its 16-byte piece c at
//     position (c XOR (r % 8));
//   bytes [16384, 18432): the 128 x 16 scale bytes as four 512-byte atoms
//     (one per 64-element K step kc), the scale of row r, block j of step kc at
//     kc*512 + (r % 32)*16 + (r / 32)*4 + j.
// The GEMM then moves each weight stage with one contiguous bulk copy per 128
// rows: streaming contiguous 16-18 KB pieces reaches ~7.3 TB/s on B200,
// strided 128-byte row pieces (a 2-D tile of row-major weights) ~6.3 TB/s.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kTileRows = 128;
constexpr int kTileK = 256;
constexpr int kCodeBytes = kTileRows * kTileK / 2;    // 16384
constexpr int kScaleBytes = kTileRows * kTileK / 16;  // 2048
constexpr int kTileBytes = kCodeBytes + kScaleBytes;  // 18432
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) pack_weights_kernel(const uint4* __restrict__ q,
                                                                const uint32_t* __restrict__ sf, int64_t K,
                                                                int64_t tiles_k, uint8_t* __restrict__ packed) {
    const int64_t tile = blockIdx.x;
    const int64_t rb = tile / tiles_k, kt = tile - rb * tiles_k;
    uint8_t* dst = packed + tile * kTileBytes;
    const int64_t q_row_vec = K / 32;   // 16-byte pieces per packed row
    const int64_t sf_row_words = K / 64;
    // 16-byte code pieces (32 elements) and 4-byte scale words (64 elements) of this tile inside K
    const int pieces = (int)min((int64_t)8, q_row_vec - kt * 8);
    const int words = (int)min((int64_t)4, sf_row_words - kt * 4);
    // codes: 1024 pieces of 16 bytes per tile
    for (int j = threadIdx.x; j < kTileRows * 8; j += kThreads) {
        const int r = j >> 3, c = j & 7;
        const uint4 v = c < pieces ? __ldg(q + (rb * kTileRows + r) * q_row_vec + kt * 8 + c) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(dst + r * 128 + ((c ^ (r & 7)) << 4)) = v;
    }
    // scales: 512 words of 4 bytes (row r, K step kc)
    for (int j = threadIdx.x; j < kTileRows * 4; j += kThreads) {
        const int r = j >> 2, kc = j & 3;
        const uint32_t w = kc < words ? __ldg(sf + (rb * kTileRows + r) * sf_row_words + kt * 4 + kc) : 0u;
        *reinterpret_cast<uint32_t*>(dst + kCodeBytes + kc * 512 + (r & 31) * 16 + (r >> 5) * 4) = w;
    }
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t nvfp4_packed_weight_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0 || rows % kTileRows || K % (kTileK / 2)) return 0;
    return (size_t)(rows / kTileRows) * (size_t)((K + kTileK - 1) / kTileK) * kTileBytes;
}

extern "C" nvfp4_status nvfp4_pack_weights(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K,
                                           uint8_t* packed, nvfp4_stream_t stream) {
    if (!q || !sf || !packed) return NVFP4_ERR_INVALID_ARG;
    if (rows <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
    if (rows % kTileRows != 0 || K % (kTileK / 2) != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(q) || !aligned16(sf) || !aligned16(packed)) return NVFP4_ERR_MISALIGNED;
    const int64_t tiles_k = (K + kTileK - 1) / kTileK;
    const int64_t tiles = (rows / kTileRows) * tiles_k;
    if (tiles > INT32_MAX) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    pack_weights_kernel<<<(unsigned)tiles, kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint32_t*>(sf), K, tiles_k, packed);
    count_launch();
    return check_launch();
}

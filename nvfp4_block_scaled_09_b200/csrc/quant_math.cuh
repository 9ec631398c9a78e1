// quant_math.cuh -- the NVFP4 quantiser's per-block arithmetic, shared by the quantise kernels and the
// permute that quantises while it gathers (the same steps, so the same bytes).
//
// Format: two FP4 values per byte and one FP8 scale per 16 elements ("Peering into the CUTLASS
// SharedStorage", Input Knowledge Required, item 3); the global scale maps the tensor amax onto
// 6 * 448 (E2M1 max times E4M3 max).
#pragma once

#include "common.cuh"

namespace nvfp4 {

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Largest |x| over a packed pair of BF16 values, kept packed (two u16 lanes).
__device__ __forceinline__ uint32_t absmax_pair(uint32_t acc, uint32_t w) { return __vmaxu2(acc, w & 0x7FFF7FFFu); }

__device__ __forceinline__ uint32_t fold_pair(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Four FP32 values -> four E2M1 pairs packed little-endian: value 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float (&y)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return out;
}

struct GlobalScale {
    float enc, dec;
};

__device__ __forceinline__ GlobalScale global_scale(float amax, const float* gdec_in) {
    GlobalScale g;
    if (gdec_in != nullptr) {
        g.dec = *gdec_in;
        g.enc = __fdiv_rn(1.0f, g.dec);
    } else if (amax == 0.0f) {
        g.enc = 1.0f;
        g.dec = 1.0f;
    } else {
        g.enc = __fdiv_rn(2688.0f, amax);
        g.dec = __fdiv_rn(amax, 2688.0f);
    }
    return g;
}

// One 16-element block (v0, v1: its 32 bytes of BF16) -> 8 code bytes in `packed` and the E4M3 scale byte
// (returned): block amax, scale = RNE(amax / 6 * g_enc), codes = RNE(x * g_enc / scale) as E2M1.
__device__ __forceinline__ uint32_t quantize_block(uint4 v0, uint4 v1, float g_enc, uint2& packed) {
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) m = absmax_pair(m, w[i]);
    const float amax_b = bf16_bits_to_f32(fold_pair(m));
    float f;
    const uint32_t S = block_scale(amax_b, g_enc, f);
    packed = make_uint2(0u, 0u);
    if (S != 0u) {
        float y[8];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            y[2 * i] = __fmul_rn(bf16_bits_to_f32(w[i] & 0xFFFFu), f);
            y[2 * i + 1] = __fmul_rn(bf16_bits_to_f32(w[i] >> 16), f);
        }
        packed.x = f32x8_to_e2m1x8(y);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            y[2 * i] = __fmul_rn(bf16_bits_to_f32(w[4 + i] & 0xFFFFu), f);
            y[2 * i + 1] = __fmul_rn(bf16_bits_to_f32(w[4 + i] >> 16), f);
        }
        packed.y = f32x8_to_e2m1x8(y);
    }
    return S;
}

}  // namespace nvfp4

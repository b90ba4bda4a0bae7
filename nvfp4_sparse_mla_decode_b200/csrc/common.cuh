// common.cuh -- constants and small device helpers shared by the kernels of
// libnvfp4mla (NVFP4 codec on the GPU side; the CPU oracle has its own).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/nvfp4mla.h"

namespace nvfp4mla {

constexpr int kRowBytes = NVFP4MLA_ROW_BYTES;          // 352
constexpr int kStagedRowBytes = NVFP4MLA_STAGED_ROW_BYTES;  // 576
constexpr int kLatent = NVFP4MLA_LATENT;                // 512
constexpr int kRope = NVFP4MLA_ROPE;                    // 64
constexpr int kDim = kLatent + kRope;                   // 576
constexpr int kGroup = NVFP4MLA_GROUP;                  // 16
constexpr int kScaleOff = 256;                          // byte offset of the 32 scales
constexpr int kRopeOff = 288;                           // byte offset of the 64 RoPE bytes
constexpr int kMaxTopk = NVFP4MLA_MAX_TOPK;

// ---------------------------------------------------------------- encoders
// E4M3 ("FN": bias 7, no infinities, 0x7F NaN, max 448), round to nearest
// even, saturating to +-448.  The sign bit is the input's sign.
__device__ __forceinline__ uint32_t e4m3_rne_sat(float x) {
    const uint32_t sign = (__float_as_uint(x) >> 24) & 0x80u;
    const float a = fabsf(x);
    if (a != a) return 0x7Fu;
    if (a > 448.0f) return sign | 0x7Eu;
    const int e = (int)((__float_as_uint(a) >> 23) & 0xFFu) - 127;  // floor(log2 a); -127 for 0/denormal
    const int q = (e < -6 ? -6 : e) - 3;                              // exponent of one code step
    // a * 2^-q is exact (power-of-two scaling, in range); round it to an
    // integer number of steps, ties to even.
    const float steps = rintf(a * __uint_as_float((uint32_t)(127 - q) << 23));
    const uint32_t n = (uint32_t)steps;
    uint32_t code = (e < -6) ? n : (((uint32_t)(e + 7) << 3) + (n - 8u));
    if (code > 0x7Eu) code = 0x7Eu;
    return sign | code;
}

// E2M1 (bias 1; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), round to nearest even,
// saturating to +-6; the sign bit is the input's sign.  The thresholds are
// the midpoints between neighbouring magnitudes; a midpoint goes to the code
// with an even mantissa bit.
__device__ __forceinline__ uint32_t e2m1_rne_sat(float y) {
    const uint32_t sign = (__float_as_uint(y) >> 28) & 0x8u;
    const float m = fabsf(y);
    uint32_t c;
    if (m <= 0.25f) c = 0;
    else if (m < 0.75f) c = 1;
    else if (m <= 1.25f) c = 2;
    else if (m < 1.75f) c = 3;
    else if (m <= 2.5f) c = 4;
    else if (m < 3.5f) c = 5;
    else if (m <= 5.0f) c = 6;
    else c = 7;
    return sign | c;
}

// Exact value of an E4M3 code as float (bias 7; subnormals 2^-6 * m/8).
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
    const uint32_t e = (code >> 3) & 15u, m = code & 7u;
    float mag = (e == 0) ? (float)m * 0.001953125f  // 2^-9
                         : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return (code & 0x80u) ? -mag : mag;
}

// ---------------------------------------------------------------- decoders
// Four packed E2M1 byte pairs (8 values) -> four f16x2 (low nibble -> low half).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(w));
}
// Two E4M3 bytes (low byte -> low half) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t d;
    asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(d) : "r"(two));
    return d;
}
// Eight E4M3 bytes (two words) -> four f16x2.
__device__ __forceinline__ void e4m3x8_to_f16x8(uint32_t lo, uint32_t hi, uint32_t (&o)[4]) {
    o[0] = e4m3x2_to_f16x2(lo & 0xFFFFu);
    o[1] = e4m3x2_to_f16x2(lo >> 16);
    o[2] = e4m3x2_to_f16x2(hi & 0xFFFFu);
    o[3] = e4m3x2_to_f16x2(hi >> 16);
}
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

}  // namespace nvfp4mla

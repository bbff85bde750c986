// nvfp4_block.cuh -- the NVFP4 encoding of one 16-element block of bf16 values, shared
// by the activation quantizer and the GEMM epilogue that re-quantizes its output
// ("BFL (fp8r / nvfp4)", nvfp4 format bullet: E2M1 values, one E4M3 scale per 16
// elements, an fp32 global scale).  Every step is one IEEE binary32 operation rounded to
// nearest even, no flush to zero:
//   t = 6g ; s = t > 0 ? amax/t : 0 ; sb = E4M3(s) ; d = dec(sb)*g ;
//   d == 0 -> codes 0 ; else code_i = E2M1(x_i * min(1/d, FLT_MAX)).
#pragma once

#include <cfloat>
#include <cstdint>

#include "bsp_ptx.cuh"

namespace bsp {

// max of two pairs of non-negative bf16 (NaN loses to a number, as fmaxf)
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// (a0 * r, a1 * r), each an IEEE binary32 multiply rounded to nearest even
__device__ __forceinline__ void mul2_rn(float a0, float a1, float r, float& y0, float& y1)
{
    asm("{\n\t.reg .b64 a, b, d;\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "mov.b64 b, {%4, %4};\n\t"
        "mul.rn.f32x2 d, a, b;\n\t"
        "mov.b64 {%0, %1}, d;\n\t}"
        : "=f"(y0), "=f"(y1)
        : "f"(a0), "f"(a1), "f"(r));
}

// Encode one block given as 8 words of two bf16 each (element 2j in the low half of
// word j).  Returns the 8 code bytes (element 2j in the low nibble) and the E4M3 scale
// byte in sb.  t = 6g is passed in.  amax is taken on the bf16 bit patterns (|x| is the
// pattern with the sign cleared, and the largest |x| is exact in bf16), so it equals the
// binary32 max of |x|; the products x * (1/d) are binary32 multiplies two at a time.
__device__ __forceinline__ uint2 nvfp4_encode_block16(const uint32_t (&v)[8], float g, float t,
                                                      uint32_t& sb)
{
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = max_bf16x2(m2, v[i] & 0x7FFF7FFFu);
    m2 = max_bf16x2(m2, __byte_perm(m2, 0, 0x1032));
    const float amax = __uint_as_float(m2 << 16);
    const float s = (t > 0.0f) ? __fdiv_rn(amax, t) : 0.0f;
    sb = cvt_e4m3x2(s, 0.0f) & 0xFFu;
    const float d = __fmul_rn(e4m3_to_f32(sb), g);
    uint2 w = make_uint2(0, 0);
    if (d != 0.0f) {
        const float r = fminf(__frcp_rn(d), FLT_MAX);
        float y[8];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            mul2_rn(bf16lo_to_f32(v[i]), bf16hi_to_f32(v[i]), r, y[2 * i], y[2 * i + 1]);
        w.x = cvt_e2m1x8(y);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            mul2_rn(bf16lo_to_f32(v[4 + i]), bf16hi_to_f32(v[4 + i]), r, y[2 * i], y[2 * i + 1]);
        w.y = cvt_e2m1x8(y);
    }
    return w;
}

// Byte offset of block-scale (row, kb) in the MMA layout of a [rows][K/16] scale array
// with kb4 = ceil(K/64) four-byte columns per 128-row tile: 512-byte chunks of 128 rows
// x 4 blocks, row r at (r%32)*16 + ((r/32)%4)*4 inside its chunk.
__host__ __device__ __forceinline__ int64_t sf_mma_offset(int64_t row, int64_t kb, int64_t kb4)
{
    return ((row >> 7) * kb4 + (kb >> 2)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 +
           (kb & 3);
}

}  // namespace bsp

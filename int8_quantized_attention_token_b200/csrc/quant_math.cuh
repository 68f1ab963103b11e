// quant_math.cuh -- the symmetric INT8 quantiser's per-element arithmetic
// (IntAttention: A Fully Integer Attention Pipeline for Efficient Edge
// Inference, section 2.1, eq. 3), shared by the standalone quantisation
// kernels and the attention kernel's in-kernel Q quantiser so that both give
// bit-identical codes and scales.  The rounding contract and its proof sketch
// are in quantize.cu's header comment.
#ifndef INTFA_QUANT_MATH_CUH_
#define INTFA_QUANT_MATH_CUH_

#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace intfa {
namespace qmath {

constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
// Rounding residuals beyond this magnitude (within 2^-14 of a half-integer)
// send an element to the IEEE quotient; see quantize.cu's header comment.
constexpr float kNearTie = 0.5f - 1.0f / 16384.0f;

// fl32(a / 127) for fp16 magnitudes a (see the header comment).
__device__ __forceinline__ float div127(float a) {
    const float c = 1.0f / 127.0f;
    const float q0 = a * c;
    const float r = fmaf(-q0, 127.0f, a);
    return fmaf(r, c, q0);
}

// Approximate 1 / s (relative error <= 2^-23); 0 for s == 0.
__device__ __forceinline__ float rcp_or_zero(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return s != 0.0f ? r : 0.0f;
}

// The code of x as the low byte of a float's bit pattern (see above); s == 0
// (r == 0) gives code 0.
__device__ __forceinline__ uint32_t code_bits(float x, float s, float r) {
    const float y = x * r;
    float t = y + kRound;
    const float res = y - (t - kRound);
    if (fabsf(res) > kNearTie) t = __fdiv_rn(x, s) + kRound;
    return __float_as_uint(t);
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __half22float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ float absmax8(const float (&f)[8]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// 8 codes packed little-endian into two words.
__device__ __forceinline__ uint2 codes8(const float (&f)[8], float s, float r) {
    uint32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = code_bits(f[i], s, r);
    return make_uint2(prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u),
                      prmt(prmt(t[4], t[5], 0x0040u), prmt(t[6], t[7], 0x0040u), 0x5410u));
}

}  // namespace qmath
}  // namespace intfa

#endif  // INTFA_QUANT_MATH_CUH_

// gelu.cuh -- GELU of a BF16 value, rounded once to BF16, for the GEMM
// epilogue that feeds the next linear layer of a feed-forward block.
//
// GELU(x) = x * Phi(x), Phi the standard normal CDF (the exact-erf form).
// Page "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化", section 2.1, quantizes
// the fully connected layers of the diffusion transformer's backbone but does
// not name the activation between the two layers of its feed-forward block;
// the exact-erf GELU is the reading taken here.  The result is the BF16 value
// nearest to the exact GELU of the BF16 input (ties to even; no input is an
// exact tie except where noted below).
//
// Only about 3.3K of the 65536 BF16 inputs need a transcendental evaluation:
//   |x| < 2^-10        GELU(x) = x/2 + x^2/sqrt(2 pi) - ..., and the second
//                      term is below half a BF16 unit of x/2, so the result is
//                      x/2, except that x/2 itself can be exactly half-way
//                      between two BF16 values (subnormal x with an odd last
//                      bit); GELU(x) - x/2 > 0 then rounds it toward +inf.
//   x >= 4             x * (1 - Phi(x)) < 1.3e-4 is below half a unit of x:
//                      the result is x (and +inf for +inf).
//   x <= -16           |GELU(x)| < 1e-56, far below the smallest BF16
//                      subnormal: the result is -0 (and -0 for -inf).
//   otherwise          a table of the 1536 positive magnitudes in
//                      [2^-10, 4) and the 1792 negative ones in [2^-10, 16),
//                      built in shared memory by each CTA that needs it.
// A table entry is x erfc(-x / sqrt 2) / 2 in binary64 (CUDA's erfc), rounded
// to BF16 by the round-to-odd method (Boldo and Melquiond): binary64 ->
// binary32 toward zero with the last bit forced to 1 when inexact, then
// binary32 -> BF16 to nearest even.  Binary32 keeps 16 more bits than BF16,
// so the two steps round exactly as one binary64 -> BF16 rounding would.
#pragma once
#include <cstdint>

namespace nvq {

constexpr uint32_t kGeluTabLo = 0x3A80u;      // BF16 magnitude of 2^-10
constexpr uint32_t kGeluPosHi = 0x4080u;      // 4.0: positive inputs at or above are returned as is
constexpr uint32_t kGeluNegHi = 0x4180u;      // 16.0: negative inputs at or below give -0
constexpr int kGeluTabPos = (int)(kGeluPosHi - kGeluTabLo);   // 1536
constexpr int kGeluTabNeg = (int)(kGeluNegHi - kGeluTabLo);   // 1792
constexpr int kGeluTabEntries = kGeluTabPos + kGeluTabNeg;
constexpr int kGeluTabBytes = kGeluTabEntries * 2;

// Correctly rounded BF16 GELU of the BF16 bit pattern h, evaluated in binary64.
__device__ __noinline__ uint32_t gelu_bf16_binary64(uint32_t h) {
    const double x = (double)__uint_as_float(h << 16);
    const double y = 0.5 * x * erfc(-x * 0.70710678118654752440);
    float f = __double2float_rz(y);
    if ((double)f != y) f = __uint_as_float(__float_as_uint(f) | 1u);
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

// Table entry i: positive magnitudes first, then negative ones.
__device__ __forceinline__ void gelu_table_fill(uint16_t* tab, uint32_t t, uint32_t nthreads) {
    for (uint32_t i = t; i < (uint32_t)kGeluTabEntries; i += nthreads) {
        const uint32_t h = i < (uint32_t)kGeluTabPos ? kGeluTabLo + i : 0x8000u | (kGeluTabLo + i - kGeluTabPos);
        tab[i] = (uint16_t)gelu_bf16_binary64(h);
    }
}

// GELU of the BF16 bit pattern h (low 16 bits), as a BF16 bit pattern.
__device__ __forceinline__ uint32_t gelu_bf16(uint32_t h, const uint16_t* tab) {
    const uint32_t a = h & 0x7FFFu, neg = h >> 15;
    const uint32_t hi = neg ? kGeluNegHi : kGeluPosHi;
    if (a >= kGeluTabLo && a < hi) return tab[(neg ? (uint32_t)kGeluTabPos : 0u) + (a - kGeluTabLo)];
    if (a < kGeluTabLo) {
        // x/2 is exact in binary32; its low 16 bits are 0 or exactly half a
        // BF16 unit, and only the latter rounds (up for x > 0, down in
        // magnitude for x < 0)
        const uint32_t u = __float_as_uint(__uint_as_float(h << 16) * 0.5f);
        return (u >> 16) + ((u >> 15) & 1u & (neg ^ 1u));
    }
    if (a > 0x7F80u) return (h & 0x8000u) | 0x7FC0u;   // NaN: the quiet NaN of that sign
    return neg ? 0x8000u : h;
}

// GELU of both BF16 halves of a 32-bit word.
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w, const uint16_t* tab) {
    return gelu_bf16(w & 0xFFFFu, tab) | (gelu_bf16(w >> 16, tab) << 16);
}

// Test hook: out[i] = GELU(in[i]) through the same table and lookup as the
// GEMM epilogue (each CTA builds its own table).
__global__ void __launch_bounds__(256) probe_gelu_kernel(const uint16_t* __restrict__ in, uint32_t n,
                                                         uint16_t* __restrict__ out) {
    __shared__ uint16_t tab[kGeluTabEntries];
    gelu_table_fill(tab, threadIdx.x, blockDim.x);
    __syncthreads();
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        out[i] = (uint16_t)gelu_bf16(in[i], tab);
}

}  // namespace nvq

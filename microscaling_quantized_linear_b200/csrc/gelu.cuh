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
// Most inputs come from a table held in shared memory by each CTA that
// needs it: the 3840 BF16 magnitudes in [2^-20, 1024), for each sign.
//   2^-20 <= |x| < 2^-10   GELU(x) = x/2 + x^2/sqrt(2 pi) - ..., and the second
//                          term is below half a BF16 unit of x/2 (exact here):
//                          the entry is x/2.
//   4 <= x                 x * (1 - Phi(x)) < 1.3e-4 is below half a unit of x:
//                          the entry is x.
//   x <= -16               |GELU(x)| < 1e-56, far below the smallest BF16
//                          subnormal: the entry is -0.
//   otherwise              x erfc(-x / sqrt 2) / 2 in binary64 (CUDA's erfc),
//                          rounded to BF16 by the round-to-odd method (Boldo
//                          and Melquiond): binary64 -> binary32 toward zero
//                          with the last bit forced to 1 when inexact, then
//                          binary32 -> BF16 to nearest even.  Binary32 keeps
//                          16 more bits than BF16, so the two steps round
//                          exactly as one binary64 -> BF16 rounding would.
// The other inputs take closed forms:
//   |x| < 2^-20            x/2, which can be exactly half-way between two BF16
//                          values (subnormal x with an odd last bit); GELU(x) -
//                          x/2 > 0 then rounds it toward +inf.
//   x >= 1024              x (+inf for +inf).
//   x <= -1024             -0 (-0 for -inf too).
//   NaN                    the quiet NaN of the same sign.
#pragma once
#include <cstdint>

namespace nvq {

constexpr uint32_t kGeluTabLo = 0x3580u;      // BF16 magnitude of 2^-20
constexpr uint32_t kGeluTabHi = 0x4480u;      // 1024.0
constexpr uint32_t kGeluErfcLo = 0x3A80u;     // 2^-10: evaluated from here ...
constexpr uint32_t kGeluPosId = 0x4080u;      // ... up to 4 for x > 0 (x itself above)
constexpr uint32_t kGeluNegZero = 0x4180u;    // ... and 16 for x < 0 (-0 above)
constexpr int kGeluTabSide = (int)(kGeluTabHi - kGeluTabLo);    // 3840 magnitudes per sign
constexpr int kGeluTabEntries = 2 * kGeluTabSide;               // positive, then negative
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

__device__ __forceinline__ void gelu_table_fill(uint16_t* tab, uint32_t t, uint32_t nthreads) {
    for (uint32_t i = t; i < (uint32_t)kGeluTabEntries; i += nthreads) {
        const uint32_t sign = i < (uint32_t)kGeluTabSide ? 0u : 0x8000u;
        const uint32_t a = kGeluTabLo + (sign ? i - kGeluTabSide : i);
        // below 2^-10: x/2, the exponent field less one (the result is normal)
        uint32_t g;
        if (a < kGeluErfcLo) g = sign | (a - 0x80u);
        else if (!sign && a >= kGeluPosId) g = a;
        else if (sign && a >= kGeluNegZero) g = 0x8000u;
        else g = gelu_bf16_binary64(sign | a);
        tab[i] = (uint16_t)g;
    }
}

// GELU of a BF16 bit pattern h outside the table.
__device__ __forceinline__ uint32_t gelu_bf16_outside(uint32_t h) {
    const uint32_t a = h & 0x7FFFu, neg = h >> 15;
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

// Table position of magnitude a (clamped into the table) and whether a is
// outside it (u >= kGeluTabSide).
__device__ __forceinline__ uint32_t gelu_slot(uint32_t a, uint32_t neg, uint32_t& u) {
    u = a - kGeluTabLo;                                   // wraps below 2^-20
    return min(u, (uint32_t)kGeluTabSide - 1u) + neg * (uint32_t)kGeluTabSide;
}

// GELU of the BF16 bit pattern h (low 16 bits, upper bits zero).
__device__ __forceinline__ uint32_t gelu_bf16(uint32_t h, const uint16_t* tab) {
    uint32_t u;
    const uint32_t r = tab[gelu_slot(h & 0x7FFFu, h >> 15, u)];
    return u < (uint32_t)kGeluTabSide ? r : gelu_bf16_outside(h);
}

// GELU of both BF16 halves of a 32-bit word (exact for every input).
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w, const uint16_t* tab) {
    return gelu_bf16(w & 0xFFFFu, tab) | (gelu_bf16(w >> 16, tab) << 16);
}

// GELU, in place, of the 32 BF16 values in w[0..15] (element 2e in the low
// half of w[e]).  A first pass takes the smallest and largest magnitude of
// the 32 values; when all lie in the table (the common case for activations)
// each value costs one index computation and one shared-memory load, all 32
// loads issued before any result is used; otherwise every value takes the
// exact per-value path (gelu_bf16x2).
__device__ __forceinline__ void gelu_bf16x32(uint32_t (&w)[16], const uint16_t* tab) {
    uint32_t mx = 0, mn = 0x7FFF7FFFu;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        const uint32_t a = w[e] & 0x7FFF7FFFu;
        mx = __vmaxu2(mx, a);
        mn = __vminu2(mn, a);
    }
    const bool inside = min(mn & 0xFFFFu, mn >> 16) >= kGeluTabLo && max(mx & 0xFFFFu, mx >> 16) < kGeluTabHi;
    if (__builtin_expect(inside, 1)) {
        // h in [LO, HI) -> h - LO;  h in [0x8000 | LO, 0x8000 | HI) -> h - LO - 0x8000 + side
        constexpr uint32_t kNegShift = 0x8000u - (uint32_t)kGeluTabSide;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t hl = w[e] & 0xFFFFu, hh = w[e] >> 16;
            const uint32_t lo = tab[hl - kGeluTabLo - (hl >> 15) * kNegShift];
            const uint32_t hi = tab[hh - kGeluTabLo - (hh >> 15) * kNegShift];
            w[e] = lo | (hi << 16);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) w[e] = gelu_bf16x2(w[e], tab);
    }
}

// Test hook: out[i] = GELU(in[i]) through the same table and the same
// 32-value lookup (gelu_bf16x32) as the GEMM epilogue; each CTA builds its
// own table.  Inputs are taken 32 at a time (in[32b + 2e] in the low half of
// word e), a short last group padded with zeros.
__global__ void __launch_bounds__(256) probe_gelu_kernel(const uint16_t* __restrict__ in, uint32_t n,
                                                         uint16_t* __restrict__ out) {
    __shared__ uint16_t tab[kGeluTabEntries];
    gelu_table_fill(tab, threadIdx.x, blockDim.x);
    __syncthreads();
    for (uint32_t b = blockIdx.x * blockDim.x + threadIdx.x; b * 32 < n; b += gridDim.x * blockDim.x) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t i = 32 * b + 2 * e;
            w[e] = (i < n ? in[i] : 0u) | (i + 1 < n ? (uint32_t)in[i + 1] << 16 : 0u);
        }
        gelu_bf16x32(w, tab);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t i = 32 * b + 2 * e;
            if (i < n) out[i] = (uint16_t)(w[e] & 0xFFFFu);
            if (i + 1 < n) out[i + 1] = (uint16_t)(w[e] >> 16);
        }
    }
}

}  // namespace nvq

// quantize.cuh -- BF16 -> NVFP4 / MXFP8 quantize-and-pack kernels.
//
// NVFP4 (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍", section NVFP4量化格式;
// page "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化", section 3.1):
//   pass 1  amax_partials_kernel: per-CTA max|x| -> workspace[cta]
//   pass 2  nvfp4_quantize_kernel: every CTA reduces the partials to the
//           tensor amax (a few KB, L2-resident), derives g_enc / g_dec, then
//           quantizes one 16-element block per thread: block amax -> E4M3
//           scale -> E2M1 codes, 8 code bytes per thread, the 4 scale bytes
//           of 4 neighbouring blocks gathered into one 32-bit store in the
//           128x4 tile order.
// MXFP8 (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍", section MXFP8量化格式):
//   mxfp8_quantize_kernel: one 32-element block per thread, E8M0 exponent
//   from the block maximum's exponent bits, E4M3 codes of x * 2^-X.
//
// All scale arithmetic is FP32 round-to-nearest-even in a fixed order, with
// no contraction, so results are bit-identical to the CPU oracle.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace nvq {

constexpr int kAmaxThreads = 256;
constexpr int kMaxAmaxPartials = 1024;        // workspace = kMaxAmaxPartials * 4 bytes
constexpr int kQuantThreads = 256;
constexpr float kAmaxFloor = 0x1p-100f;       // below this the tensor quantizes to zero

// bf16 bits (low 16 of u) -> float
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// max over the two 16-bit magnitudes packed in u
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t u) {
    return __vmaxu2(acc, u & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t fold2(uint32_t m2) {
    return max(m2 & 0xFFFFu, m2 >> 16);
}

// Block-wide max of one value per thread; result valid in every thread.
template <int THREADS>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red /* THREADS/32 */) {
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t w = (lane < THREADS / 32) ? red[lane] : 0u;
    w = __reduce_max_sync(0xFFFFFFFFu, w);
    __syncthreads();
    return w;
}

// Offset of scale (row r, column c) in the 128x4 tile order, C/4 = ctiles.
__device__ __forceinline__ uint32_t sf_tile_offset(uint32_t r, uint32_t c, uint32_t ctiles) {
    return ((r >> 7) * ctiles + (c >> 2)) * 512u + (r & 31u) * 16u + ((r & 127u) >> 5) * 4u + (c & 3u);
}

// E4M3 (non-negative) code -> float, exact.
__device__ __forceinline__ float e4m3_decode_pos(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0x1p-9f;
}

// ------------------------------------------------------------------ amax
// x viewed as rows of `vecs_per_row` 16-byte vectors with a row pitch of
// `pitch_vecs` vectors; partial[blockIdx.x] = max |x| bits (BF16 magnitude).
__global__ void __launch_bounds__(kAmaxThreads)
amax_partials_kernel(const uint4* __restrict__ x, uint32_t rows, uint32_t vecs_per_row,
                     uint32_t pitch_vecs, uint32_t* __restrict__ partial) {
    __shared__ uint32_t red[kAmaxThreads / 32];
    uint32_t m2 = 0;
    const uint32_t total = rows * vecs_per_row;
    const uint32_t stride = gridDim.x * kAmaxThreads;
    uint32_t i = blockIdx.x * kAmaxThreads + threadIdx.x;
    if (pitch_vecs == vecs_per_row) {
        // contiguous: 4 independent 16-byte loads in flight per thread
        for (; i + 3 * stride < total; i += 4 * stride) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldg(x + i + u * stride);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                m2 = absmax2(absmax2(absmax2(absmax2(m2, v[u].x), v[u].y), v[u].z), v[u].w);
        }
        for (; i < total; i += stride) {
            uint4 v = __ldg(x + i);
            m2 = absmax2(absmax2(absmax2(absmax2(m2, v.x), v.y), v.z), v.w);
        }
    } else {
        for (; i < total; i += stride) {
            const uint32_t r = i / vecs_per_row, c = i - r * vecs_per_row;
            uint4 v = __ldg(x + (size_t)r * pitch_vecs + c);
            m2 = absmax2(absmax2(absmax2(absmax2(m2, v.x), v.y), v.z), v.w);
        }
    }
    const uint32_t m = block_max_u32<kAmaxThreads>(fold2(m2), red);
    if (threadIdx.x == 0) partial[blockIdx.x] = m;
}

// ------------------------------------------------------------------ NVFP4
// One thread = one 16-element block.  Block b of the tensor is (row b / nblk,
// column b % nblk) with nblk = K / 16; its codes are bytes [8b, 8b + 8).
__global__ void __launch_bounds__(kQuantThreads)
nvfp4_quantize_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ g_dec_out,
                      const uint32_t* __restrict__ partial, uint32_t npartial,
                      const float* __restrict__ calib_amax, unsigned int* __restrict__ status) {
    __shared__ uint32_t red[kQuantThreads / 32];
    float amax;
    if (calib_amax != nullptr) {
        amax = *calib_amax;
    } else {
        uint32_t m = 0;
        for (uint32_t i = threadIdx.x; i < npartial; i += kQuantThreads) m = max(m, partial[i]);
        m = block_max_u32<kQuantThreads>(m, red);
        if (m >= 0x7F80u && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, 2u);
        amax = __uint_as_float(m << 16);
    }
    const bool zero_tensor = !(amax >= kAmaxFloor);
    const float g_enc = __fdiv_rn(2688.0f, amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_dec_out = zero_tensor ? 0.0f : __fdiv_rn(amax, 2688.0f);

    const uint32_t total = rows * nblk;
    const uint32_t ctiles = nblk >> 2;
    for (uint32_t b = blockIdx.x * kQuantThreads + threadIdx.x; b - threadIdx.x < total;
         b += gridDim.x * kQuantThreads) {
        const bool active = b < total;       // whole warps stay in the loop for the shuffles
        uint32_t r = 0, c = 0;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (active) {
            r = b / nblk;
            c = b - r * nblk;
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
            v0 = __ldg(src);
            v1 = __ldg(src + 1);
        }
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) m2 = absmax2(m2, w[i]);
        const float bmax = __uint_as_float(fold2(m2) << 16);

        uint32_t sc = 0, lo = 0, hi = 0;
        if (!zero_tensor) {
            const float s = __fmul_rn(__fdiv_rn(bmax, 6.0f), g_enc);
            sc = cvt_e4m3x2(0.0f, s) & 0xFFu;
            const float scv = e4m3_decode_pos(sc);
            if (scv != 0.0f) {
                const float rr = __fdiv_rn(g_enc, scv);
                uint32_t q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    q[i] = cvt_e2m1x2(__fmul_rn(bf16hi(w[i]), rr), __fmul_rn(bf16lo(w[i]), rr));
                lo = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
                hi = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
            }
        }
        // gather the scales of 4 neighbouring blocks (c % 4 == 0..3, same row)
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
        if (active) {
            *reinterpret_cast<uint2*>(codes + (size_t)b * 8) = make_uint2(lo, hi);
            if ((c & 3u) == 0)
                *reinterpret_cast<uint32_t*>(sf + sf_tile_offset(r, c, ctiles)) =
                    sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
}

// ------------------------------------------------------------------ MXFP8
// One thread = one 32-element block.  Block b is (row b / nblk, column
// b % nblk), nblk = K / 32; its codes are bytes [32b, 32b + 32).
__global__ void __launch_bounds__(kQuantThreads)
mxfp8_quantize_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
    const uint32_t total = rows * nblk;
    const uint32_t ctiles = nblk >> 2;
    for (uint32_t b = blockIdx.x * kQuantThreads + threadIdx.x; b - threadIdx.x < total;
         b += gridDim.x * kQuantThreads) {
        const bool active = b < total;
        uint32_t r = 0, c = 0;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = 0;
        if (active) {
            r = b / nblk;
            c = b - r * nblk;
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint4 v = __ldg(src + u);
                w[4 * u] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
            }
        }
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) m2 = absmax2(m2, w[i]);
        const uint32_t mb = fold2(m2);               // BF16 magnitude bits of the block max
        int X;
        if (mb == 0) {
            X = -127;
        } else {
            const int E = (int)(mb >> 7);
            const int e = E ? E - 127 : (31 - __clz((int)(mb & 0x7F))) - 133;
            X = min(max(e - 8, -127), 127);
        }
        const uint32_t sc = (uint32_t)(X + 127);
        const float mult = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, X <= 119
        uint32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t p0 = cvt_e4m3x2(__fmul_rn(bf16hi(w[2 * i]), mult), __fmul_rn(bf16lo(w[2 * i]), mult));
            const uint32_t p1 = cvt_e4m3x2(__fmul_rn(bf16hi(w[2 * i + 1]), mult), __fmul_rn(bf16lo(w[2 * i + 1]), mult));
            q[i] = p0 | (p1 << 16);
        }
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
        if (active) {
            uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)b * 32);
            dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
            dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
            if ((c & 3u) == 0)
                *reinterpret_cast<uint32_t*>(sf + sf_tile_offset(r, c, ctiles)) =
                    sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
}

// ------------------------------------------------------------------ probe
__global__ void probe_convert_kernel(const float* __restrict__ in, uint32_t n,
                                     uint8_t* __restrict__ e2m1, uint8_t* __restrict__ e4m3) {
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float v = in[i];
        e2m1[i] = (uint8_t)(cvt_e2m1x2(0.0f, v) & 0xFu);
        e4m3[i] = (uint8_t)(cvt_e4m3x2(0.0f, v) & 0xFFu);
    }
}

}  // namespace nvq

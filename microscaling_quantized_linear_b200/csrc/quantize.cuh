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
constexpr int kMaxAmaxPartials = 1024;        // u32 partial maxima of the two-pass path
constexpr int kMaxFusedCtas = 1024;           // u64 epoch-tagged slots of the one-pass path
constexpr size_t kWorkspaceSlotsOffset = 0;
constexpr size_t kWorkspacePartialsOffset = kMaxFusedCtas * 8;
constexpr size_t kWorkspaceBytes = kWorkspacePartialsOffset + kMaxAmaxPartials * 4;
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

// Quantize one 16-element block (w[0..7] = 16 BF16 values) with the given
// global encode scale; returns the E4M3 scale code, writes the 8 code bytes.
__device__ __forceinline__ uint32_t nvfp4_block(const uint32_t (&w)[8], float g_enc, uint32_t& lo, uint32_t& hi) {
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = absmax2(m2, w[i]);
    const float bmax = __uint_as_float(fold2(m2) << 16);
    const float s = __fmul_rn(__fdiv_rn(bmax, 6.0f), g_enc);
    const uint32_t sc = cvt_e4m3x2(0.0f, s) & 0xFFu;
    const float scv = e4m3_decode_pos(sc);
    lo = hi = 0;
    if (scv != 0.0f) {
        const float rr = __fdiv_rn(g_enc, scv);
        uint32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            q[i] = cvt_e2m1x2(__fmul_rn(bf16hi(w[i]), rr), __fmul_rn(bf16lo(w[i]), rr));
        lo = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
        hi = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
    }
    return sc;
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
        // contiguous: 8 independent 16-byte loads in flight per thread
        for (; i + 7 * stride < total; i += 8 * stride) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(x + i + u * stride);
#pragma unroll
            for (int u = 0; u < 8; ++u)
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
__global__ void __launch_bounds__(kQuantThreads, 8)
nvfp4_quantize_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ g_dec_out,
                      const uint32_t* __restrict__ partial, uint32_t npartial,
                      const float* __restrict__ calib_amax, unsigned int* __restrict__ status) {
    __shared__ uint32_t red[kQuantThreads / 32];
    const uint32_t total = rows * nblk;
    // the first block's loads do not depend on the amax: issue them first
    uint32_t b = blockIdx.x * kQuantThreads + threadIdx.x;
    uint4 p0 = make_uint4(0, 0, 0, 0), p1 = p0;
    if (b < total) {
        const uint32_t r = b / nblk, c = b - r * nblk;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
        p0 = __ldg(src);
        p1 = __ldg(src + 1);
    }
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

    const uint32_t ctiles = nblk >> 2;
    for (bool first = true; b - threadIdx.x < total; b += gridDim.x * kQuantThreads, first = false) {
        const bool active = b < total;       // whole warps stay in the loop for the shuffles
        uint32_t r = 0, c = 0;
        uint4 v0 = p0, v1 = p1;
        if (active) {
            r = b / nblk;
            c = b - r * nblk;
            if (!first) {
                const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
                v0 = __ldg(src);
                v1 = __ldg(src + 1);
            }
        }
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t sc = 0, lo = 0, hi = 0;
        if (!zero_tensor) sc = nvfp4_block(w, g_enc, lo, hi);
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

// ------------------------------------------------------------------ NVFP4, one pass
// For tensors whose rows fit in the shared memory of one CTA per SM: every
// CTA copies its rows into shared memory once (bulk copies, 4 chunks with
// their own mbarriers so the block maxima are taken while later chunks are
// still landing), publishes its partial amax in an epoch-tagged 64-bit slot
// of the workspace, waits (bounded) until every CTA's slot carries this
// call's epoch, and quantizes from shared memory.  HBM sees exactly one read
// of the activation.  Must be launched cooperatively (all CTAs co-resident).
constexpr int kFusedThreads = 1024;
constexpr int kFusedChunks = 4;
constexpr uint64_t kFusedWaitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// Two 16-byte halves of the 32-byte block at smem byte offset 32*b.  Threads
// 4..7 of every 8 read the halves in the opposite order, which makes each
// 8-thread shared-memory phase touch 8 distinct 4-bank groups.
__device__ __forceinline__ void lds_block32(const uint8_t* base, uint32_t b, uint4& v0, uint4& v1) {
    const uint4* p = reinterpret_cast<const uint4*>(base + (size_t)b * 32);
    const uint32_t sw = (threadIdx.x >> 2) & 1u;
    const uint4 first = p[sw];
    const uint4 second = p[sw ^ 1u];
    v0 = sw ? second : first;
    v1 = sw ? first : second;
}

__global__ void __launch_bounds__(kFusedThreads, 1)
nvfp4_quantize_fused_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t K, uint32_t ldx,
                            uint32_t rows_per_cta, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                            float* __restrict__ g_dec_out, unsigned long long* __restrict__ slots,
                            uint32_t epoch, unsigned int* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ __align__(8) uint64_t bars[kFusedChunks];
    __shared__ uint32_t red[kFusedThreads / 32];
    __shared__ int s_timeout;

    const uint32_t r0 = blockIdx.x * rows_per_cta;
    const uint32_t nr = min(rows_per_cta, rows - r0);
    const uint32_t nblk = K >> 4;
    const uint32_t row_bytes = K * 2;
    const uint32_t rows_per_chunk = (nr + kFusedChunks - 1) / kFusedChunks;
    if (threadIdx.x == 0) {
        s_timeout = 0;
        for (int c = 0; c < kFusedChunks; ++c) mbar_init(smem_u32(&bars[c]), 1);
        fence_mbarrier_init();
        for (int c = 0; c < kFusedChunks; ++c) {
            const uint32_t ra = min(nr, c * rows_per_chunk), rb = min(nr, (c + 1) * rows_per_chunk);
            const uint32_t bar = smem_u32(&bars[c]);
            mbar_arrive_expect_tx(bar, (rb - ra) * row_bytes);
            if (ldx == K) {
                if (rb > ra)
                    bulk_load(smem_u32(tile + (size_t)ra * row_bytes), x + (size_t)(r0 + ra) * K,
                              (rb - ra) * row_bytes, bar);
            } else {
                for (uint32_t r = ra; r < rb; ++r)
                    bulk_load(smem_u32(tile + (size_t)r * row_bytes), x + (size_t)(r0 + r) * ldx, row_bytes, bar);
            }
        }
    }
    __syncthreads();

    // partial amax, chunk by chunk as the copies land
    uint32_t m2 = 0;
    for (int c = 0; c < kFusedChunks; ++c) {
        const uint32_t ra = min(nr, c * rows_per_chunk), rb = min(nr, (c + 1) * rows_per_chunk);
        if (!mbar_wait_bounded(smem_u32(&bars[c]), 0, &s_timeout, kFusedWaitNs)) s_timeout = 1;
        if (s_timeout) break;
        for (uint32_t b = ra * nblk + threadIdx.x; b < rb * nblk; b += kFusedThreads) {
            uint4 v0, v1;
            lds_block32(tile, b, v0, v1);
            m2 = absmax2(absmax2(absmax2(absmax2(m2, v0.x), v0.y), v0.z), v0.w);
            m2 = absmax2(absmax2(absmax2(absmax2(m2, v1.x), v1.y), v1.z), v1.w);
        }
    }
    const uint32_t cta_max = block_max_u32<kFusedThreads>(fold2(m2), red);
    if (threadIdx.x == 0)
        st_release_u64(slots + blockIdx.x, ((unsigned long long)epoch << 32) | cta_max);

    // every CTA's partial, tagged with this call's epoch
    uint32_t m = 0;
    if (threadIdx.x < gridDim.x) {
        const unsigned long long* slot = slots + threadIdx.x;
        unsigned long long v = ld_acquire_u64(slot);
        if ((uint32_t)(v >> 32) != epoch) {
            const uint64_t t0 = globaltimer_ns();
            while ((uint32_t)((v = ld_acquire_u64(slot)) >> 32) != epoch) {
                if (s_timeout || globaltimer_ns() - t0 > kFusedWaitNs) {
                    s_timeout = 1;
                    break;
                }
            }
        }
        m = (uint32_t)(v & 0xFFFFFFFFull);
    }
    const uint32_t amax_bits = block_max_u32<kFusedThreads>(m, red);
    if (s_timeout) {                                  // a copy or a peer never arrived: write nothing
        if (threadIdx.x == 0) atomicOr(status, 1u);
        // let every issued copy land before the CTA exits
        if (threadIdx.x == 0) {
            int never = 0;
            for (int c = 0; c < kFusedChunks; ++c) mbar_wait_bounded(smem_u32(&bars[c]), 0, &never, kFusedWaitNs);
        }
        __syncthreads();
        return;
    }
    if (amax_bits >= 0x7F80u && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, 2u);
    const float amax = __uint_as_float(amax_bits << 16);
    const bool zero_tensor = !(amax >= kAmaxFloor);
    const float g_enc = __fdiv_rn(2688.0f, amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_dec_out = zero_tensor ? 0.0f : __fdiv_rn(amax, 2688.0f);

    const uint32_t total = nr * nblk;
    const uint32_t ctiles = nblk >> 2;
    for (uint32_t base = 0; base < total; base += kFusedThreads) {
        const uint32_t b = base + threadIdx.x;
        const bool active = b < total;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (active) lds_block32(tile, b, v0, v1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t lo = 0, hi = 0, sc = 0;
        if (!zero_tensor) sc = nvfp4_block(w, g_enc, lo, hi);
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
        if (active) {
            const uint32_t rl = b / nblk, c = b - rl * nblk, r = r0 + rl;
            *reinterpret_cast<uint2*>(codes + (size_t)r * (K >> 1) + (size_t)c * 8) = make_uint2(lo, hi);
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

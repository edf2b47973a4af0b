// quantize.cuh -- BF16 -> NVFP4 / MXFP8 quantize-and-pack kernels.
//
// NVFP4 (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍", section NVFP4量化格式;
// page "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化", section 3.1), per
// 16-element block along K, in FP32 round-to-nearest-even:
//   s = (b / 6) * g_enc, sc = E4M3(s), r = g_enc / E4M3(sc), q_i = E2M1(x_i * r)
// with b the block's max |x| and g_enc = 2688 / amax of the tensor.
//   one pass   nvfp4_quantize_fused_kernel (rows fit on chip; the default there)
//   two pass   amax_partials_kernel, then nvfp4_quantize_kernel
//   calibrated nvfp4_quantize_kernel alone, amax given by the caller
// MXFP8 (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍", section MXFP8量化格式):
//   mxfp8_quantize_kernel: one 32-element block per thread, E8M0 exponent
//   from the block maximum's exponent bits, E4M3 codes of x * 2^-X.
//
// Exactness with fewer instructions: both divisions of the NVFP4 rule come
// from small per-CTA tables that hold correctly rounded quotients.
//   b / 6:       b = M * 2^(E-134) with M the 8-bit BF16 significand, so
//                fl(b/6) = fl(M/6) * 2^(E-134) exactly whenever the result
//                is a normal float (E >= 8); smaller E divides directly.
//   g_enc / sc:  sc takes one of 127 values, so r comes from a 127-entry
//                table computed once per CTA with a correctly rounded divide.
// Products use packed f32x2 multiplies (IEEE round-to-nearest-even, like the
// scalar ones); every result is bit-identical to the CPU oracle.
#pragma once
#include <cstdint>
#include "debug.cuh"
#include "ptx.cuh"

namespace nvq {

constexpr int kAmaxThreads = 256;
constexpr int kMaxAmaxPartials = 1024;        // u32 partial maxima of the two-pass path
constexpr int kMaxFusedCtas = 256;            // generation-tagged slots of the one-pass path
constexpr int kFusedSlotStride = 16;          // u64 per slot: one 128-byte line each, so polls spread over L2
// Workspace: the one-pass slots, the two-pass partial maxima, then the
// one-pass generation word on a line of its own.  The caller zero-fills it
// once before its first use; every call leaves it valid for the next.
constexpr size_t kWorkspaceSlotsOffset = 0;
constexpr size_t kWorkspacePartialsOffset = (size_t)kMaxFusedCtas * kFusedSlotStride * 8;
constexpr size_t kWorkspaceGenOffset = kWorkspacePartialsOffset + kMaxAmaxPartials * 4;
constexpr size_t kWorkspaceBytes = kWorkspaceGenOffset + 128;
constexpr int kQuantThreads = 256;
constexpr float kAmaxFloor = 0x1p-100f;       // below this the tensor quantizes to zero

// Bits of the device status word (the NVQ_STATUS_* values of nvq.h).
constexpr unsigned int kStatusTimeout = 1u;
constexpr unsigned int kStatusNonfinite = 2u;
constexpr unsigned int kStatusWorkspace = 4u;

// max over the two 16-bit magnitudes packed in u
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t u) {
    return __vmaxu2(acc, u & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t fold2(uint32_t m2) {
    return max(m2 & 0xFFFFu, m2 >> 16);
}

// BF16 magnitude bits of the largest |x| among the 16 values in w[0..7].
__device__ __forceinline__ uint32_t block16_max(const uint32_t (&w)[8]) {
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = absmax2(m2, w[i]);
    return fold2(m2);
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

// Scale rows past `rows`, up to the next multiple of 128, are zero (the
// tensor-core tile holds 128 rows).  One 32-bit word = the 4 scale bytes of
// one row in one column tile; thread `t` of `nthreads` writes its share.
__device__ __forceinline__ void zero_pad_scale_rows(uint8_t* sf, uint32_t rows, uint32_t ctiles, uint32_t t,
                                                    uint32_t nthreads, unsigned int* status) {
    const uint32_t pad_rows = ((rows + 127u) & ~127u) - rows;
    for (uint32_t i = t; i < pad_rows * ctiles; i += nthreads) {
        const uint32_t r = rows + i / ctiles, ct = i - (i / ctiles) * ctiles;
        const uint32_t off = sf_tile_offset(r, 4 * ct, ctiles);
        if (in_bounds(off, 4, sf_extent(rows, ctiles), status)) *reinterpret_cast<uint32_t*>(sf + off) = 0u;
    }
}

// E4M3 (non-negative) code -> float, exact.
__device__ __forceinline__ float e4m3_decode_pos(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0x1p-9f;
}

// ------------------------------------------------------------------ NVFP4 block
// Per-CTA tables: d6[t] = fl((128 + t) / 6); rtab[c] = fl(g_enc / E4M3(c)).
__device__ __forceinline__ void init_d6(float* d6) {
    if (threadIdx.x < 128) d6[threadIdx.x] = __fdiv_rn((float)(128 + threadIdx.x), 6.0f);
}

__device__ __forceinline__ void init_rtab(float* rtab, float g_enc) {
    if (threadIdx.x < 128)
        rtab[threadIdx.x] = threadIdx.x ? __fdiv_rn(g_enc, e4m3_decode_pos(threadIdx.x)) : 0.0f;
}

// fl32(b / 6) for b given by its BF16 magnitude bits mb.
__device__ __forceinline__ float div6(uint32_t mb, const float* d6) {
    const uint32_t E = mb >> 7;
    if (E >= 8) return __fmul_rn(d6[mb & 0x7Fu], __uint_as_float((E - 7u) << 23));
    return __fdiv_rn(__uint_as_float(mb << 16), 6.0f);
}

// One 16-element block given d = fl(b / 6) for its block max b, the 16 BF16
// values in w[0..7].  Returns the E4M3 scale code; lo/hi receive the 16 E2M1
// codes.  g_enc == 0 (a zero tensor) gives scale 0 and zero codes.
__device__ __forceinline__ uint32_t nvfp4_block_d(float d, const uint32_t (&w)[8], float g_enc, const float* rtab,
                                                  uint32_t& lo, uint32_t& hi) {
    const float s = __fmul_rn(d, g_enc);
    const uint32_t sc = cvt_e4m3x2(0.0f, s) & 0xFFu;
    const float r = rtab[sc];
    float2 p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) p[i] = bf16x2_mul(w[i], r);
    lo = cvt_e2m1x8(p[0].x, p[0].y, p[1].x, p[1].y, p[2].x, p[2].y, p[3].x, p[3].y);
    hi = cvt_e2m1x8(p[4].x, p[4].y, p[5].x, p[5].y, p[6].x, p[6].y, p[7].x, p[7].y);
    if (sc == 0) lo = hi = 0;                         // scale rounded to zero: zero codes (no -0)
    return sc;
}

// Two blocks at once: both E4M3 scales from one conversion.
__device__ __forceinline__ uint32_t nvfp4_block_pair_d(float d0, float d1, const uint32_t (&w0)[8],
                                                       const uint32_t (&w1)[8], float g_enc, const float* rtab,
                                                       uint32_t& lo0, uint32_t& hi0, uint32_t& lo1, uint32_t& hi1) {
    const uint32_t pair = cvt_e4m3x2(__fmul_rn(d1, g_enc), __fmul_rn(d0, g_enc));
    const uint32_t sc0 = pair & 0xFFu, sc1 = pair >> 8;
    const float r0 = rtab[sc0], r1 = rtab[sc1];
    float2 p[8], q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        p[i] = bf16x2_mul(w0[i], r0);
        q[i] = bf16x2_mul(w1[i], r1);
    }
    lo0 = cvt_e2m1x8(p[0].x, p[0].y, p[1].x, p[1].y, p[2].x, p[2].y, p[3].x, p[3].y);
    hi0 = cvt_e2m1x8(p[4].x, p[4].y, p[5].x, p[5].y, p[6].x, p[6].y, p[7].x, p[7].y);
    lo1 = cvt_e2m1x8(q[0].x, q[0].y, q[1].x, q[1].y, q[2].x, q[2].y, q[3].x, q[3].y);
    hi1 = cvt_e2m1x8(q[4].x, q[4].y, q[5].x, q[5].y, q[6].x, q[6].y, q[7].x, q[7].y);
    if (sc0 == 0) lo0 = hi0 = 0;
    if (sc1 == 0) lo1 = hi1 = 0;
    return pair;
}

// The same block given its block max bits mb.
__device__ __forceinline__ uint32_t nvfp4_block(uint32_t mb, const uint32_t (&w)[8], float g_enc,
                                                const float* d6, const float* rtab, uint32_t& lo, uint32_t& hi) {
    return nvfp4_block_d(div6(mb, d6), w, g_enc, rtab, lo, hi);
}

__device__ __forceinline__ float encode_scale(float amax) {
    return amax >= kAmaxFloor ? __fdiv_rn(2688.0f, amax) : 0.0f;
}

__device__ __forceinline__ float decode_scale(float amax) {
    return amax >= kAmaxFloor ? __fdiv_rn(amax, 2688.0f) : 0.0f;
}

// ------------------------------------------------------------------ amax
// x viewed as rows of `vecs_per_row` 16-byte vectors with a row pitch of
// `pitch_vecs` vectors; partial[blockIdx.x] = max |x| bits (BF16 magnitude).
__global__ void __launch_bounds__(kAmaxThreads)
amax_partials_kernel(const uint4* __restrict__ x, uint32_t rows, uint32_t vecs_per_row,
                     uint32_t pitch_vecs, uint32_t* __restrict__ partial, uint32_t capacity,
                     unsigned int* __restrict__ status) {
    __shared__ uint32_t red[kAmaxThreads / 32];
    griddep_wait();                       // x may come from the previous grid
    griddep_launch();                     // the quantize pass may start its prologue
    uint32_t m2 = 0;
    const uint32_t total = rows * vecs_per_row;
    const uint32_t stride = gridDim.x * kAmaxThreads;
    const uint64_t x_vecs = pitched_extent(rows, vecs_per_row, pitch_vecs);
    uint32_t i = blockIdx.x * kAmaxThreads + threadIdx.x;
    if (pitch_vecs == vecs_per_row) {
        // contiguous: batches of 8 independent 16-byte loads, all issued
        // before any is used (predicated at the tail, so a thread with fewer
        // than 8 vectors still has all of them in flight at once)
        for (; i < total; i += 8 * stride) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (i + u * stride < total && in_bounds(i + u * stride, 1, x_vecs, status))
                           ? __ldg(x + i + u * stride)
                           : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                m2 = absmax2(absmax2(absmax2(absmax2(m2, v[u].x), v[u].y), v[u].z), v[u].w);
        }
    } else {
        for (; i < total; i += stride) {
            const uint32_t r = i / vecs_per_row, c = i - r * vecs_per_row;
            const uint64_t off = (uint64_t)r * pitch_vecs + c;
            const uint4 v = in_bounds(off, 1, x_vecs, status) ? __ldg(x + off) : make_uint4(0, 0, 0, 0);
            m2 = absmax2(absmax2(absmax2(absmax2(m2, v.x), v.y), v.z), v.w);
        }
    }
    const uint32_t m = block_max_u32<kAmaxThreads>(fold2(m2), red);
    if (threadIdx.x == 0 && in_bounds(blockIdx.x, 1, capacity, status)) partial[blockIdx.x] = m;
}

// ------------------------------------------------------------------ NVFP4, streaming
// One thread = two 16-element blocks per iteration (b and b - stride, both
// loaded before either is computed).  Block b is (row b / nblk, column
// b % nblk), nblk = K / 16; its codes are bytes [8b, 8b + 8).  The amax is the
// reduction of the two-pass partials, or *calib_amax.
// The grid walks the tensor from its end to its start: after the amax pass,
// which reads x from start to end, the rows read last are the likeliest
// still in L2, so they are quantized first.  Within a warp the blocks stay
// in ascending order (the scale gather below needs four neighbours).
__device__ __forceinline__ void block_step_down(uint32_t& r, uint32_t& c, uint32_t qs, uint32_t rs, uint32_t nblk) {
    if (c < rs) {
        c += nblk - rs;
        r -= qs + 1;
    } else {
        c -= rs;
        r -= qs;
    }
}

__global__ void __launch_bounds__(kQuantThreads, 6)
nvfp4_quantize_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, float* __restrict__ g_dec_out,
                      const uint32_t* __restrict__ partial, uint32_t npartial,
                      const float* __restrict__ calib_amax, unsigned int* __restrict__ status) {
    __shared__ uint32_t red[kQuantThreads / 32];
    __shared__ float d6[128], rtab[128];
    const uint32_t total = rows * nblk;
    const uint32_t stride = gridDim.x * kQuantThreads;
    const uint32_t qs = stride / nblk, rs = stride - qs * nblk;
    const uint64_t x_elems = pitched_extent(rows, nblk * 16, ldx);
    // This thread's blocks are b0 + k * stride; the CTA walks k from its
    // last (nk - 1) down to 0, two per iteration: b = b0 + k * stride and
    // b1 = b - stride.  Only at k = nk - 1 can b lie past the end.
    const uint32_t base_cta = blockIdx.x * kQuantThreads;
    const uint32_t nk = total > base_cta ? (total - base_cta + stride - 1) / stride : 0;
    int32_t k = (int32_t)nk - 1;
    uint32_t b = base_cta + threadIdx.x + (uint32_t)(k > 0 ? k : 0) * stride;
    uint32_t r = b / nblk, c = b - r * nblk;
    uint32_t r1 = r, c1 = c;
    block_step_down(r1, c1, qs, rs, nblk);       // block b - stride (not used when k < 1)
    // Calibrated: x may come from the previous grid, so nothing is read
    // before it has completed.  Dynamic: the previous grid is this call's amax
    // pass, which only reads x and lets this grid start once it has itself
    // waited for x's producer, so the first iteration's loads go first.
    if (calib_amax != nullptr) griddep_wait();
    uint4 v[4];
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    {
        const bool a0 = k >= 0 && b < total, a1 = k >= 1;
        const uint4* s0 = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
        const uint4* s1 = reinterpret_cast<const uint4*>(x + (size_t)r1 * ldx + (size_t)c1 * 16);
        const bool l0 = a0 && in_bounds((uint64_t)r * ldx + c * 16, 16, x_elems, status);
        const bool l1 = a1 && in_bounds((uint64_t)r1 * ldx + c1 * 16, 16, x_elems, status);
        v[0] = l0 ? __ldg(s0) : zero4;
        v[1] = l0 ? __ldg(s0 + 1) : zero4;
        v[2] = l1 ? __ldg(s1) : zero4;
        v[3] = l1 ? __ldg(s1 + 1) : zero4;
    }
    init_d6(d6);
    // x is final (the amax pass that may still be running only reads it);
    // the partial maxima and every output are touched only after this wait.
    griddep_wait();
    griddep_launch();
    float amax;
    if (calib_amax != nullptr) {
        amax = *calib_amax;
    } else {
        uint32_t m = 0;
        for (uint32_t i = threadIdx.x; i < npartial; i += kQuantThreads) m = max(m, partial[i]);
        m = block_max_u32<kQuantThreads>(m, red);
        if (m >= 0x7F80u && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusNonfinite);
        amax = __uint_as_float(m << 16);
    }
    const float g_enc = encode_scale(amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_dec_out = decode_scale(amax);
    init_rtab(rtab, g_enc);
    __syncthreads();

    const uint32_t ctiles = nblk >> 2;
    for (bool first = true; k >= 0; k -= 2, first = false) {
        const bool a0 = b < total, a1 = k >= 1;      // whole warps stay in the loop for the shuffles
        if (!first) {
            const uint4* s0 = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
            const uint4* s1 = reinterpret_cast<const uint4*>(x + (size_t)r1 * ldx + (size_t)c1 * 16);
            const bool l0 = a0 && in_bounds((uint64_t)r * ldx + c * 16, 16, x_elems, status);
            const bool l1 = a1 && in_bounds((uint64_t)r1 * ldx + c1 * 16, 16, x_elems, status);
            v[0] = l0 ? __ldg(s0) : zero4;
            v[1] = l0 ? __ldg(s0 + 1) : zero4;
            v[2] = l1 ? __ldg(s1) : zero4;
            v[3] = l1 ? __ldg(s1 + 1) : zero4;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t bu = u ? b - stride : b, ru = u ? r1 : r, cu = u ? c1 : c;
            const bool active = u ? a1 : a0;
            const uint4 p0 = v[2 * u], p1 = v[2 * u + 1];
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            uint32_t lo, hi;
            const uint32_t sc = nvfp4_block(block16_max(w), w, g_enc, d6, rtab, lo, hi);
            // gather the scales of 4 neighbouring blocks (c % 4 == 0..3, same row)
            const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
            const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
            const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
            if (active) {
                if (in_bounds((uint64_t)bu * 8, 8, (uint64_t)total * 8, status))
                    *reinterpret_cast<uint2*>(codes + (size_t)bu * 8) = make_uint2(lo, hi);
                const uint32_t so = sf_tile_offset(ru, cu, ctiles);
                if ((cu & 3u) == 0 && in_bounds(so, 4, sf_extent(rows, ctiles), status))
                    *reinterpret_cast<uint32_t*>(sf + so) = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
            }
        }
        if (k >= 2) {                                // the next pair: b - 2 stride, b - 3 stride
            b -= 2 * stride;
            r = r1;
            c = c1;
            block_step_down(r, c, qs, rs, nblk);
            r1 = r;
            c1 = c;
            block_step_down(r1, c1, qs, rs, nblk);
        }
    }
    zero_pad_scale_rows(sf, rows, ctiles, blockIdx.x * kQuantThreads + threadIdx.x, stride, status);
}

// ------------------------------------------------------------------ NVFP4, small tensors
// One cluster of kClusterCtas CTAs quantizes a tensor of at most
// kClusterMaxBlocks 16-blocks in one launch: each thread holds up to
// kClusterBlocksPerThread blocks in registers, each CTA reduces its maximum,
// the CTAs exchange their maxima through distributed shared memory (all into
// CTA 0's array, one cluster barrier), and every thread quantizes the blocks
// it holds.  No workspace, no second read of the tensor, no grid barrier.
constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 1024;
constexpr int kClusterBlocksPerThread = 4;
constexpr uint32_t kClusterMaxBlocks = (uint32_t)kClusterCtas * kClusterThreads * kClusterBlocksPerThread;

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kClusterThreads, 1)
nvfp4_quantize_cluster_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                              float* __restrict__ g_dec_out, unsigned int* __restrict__ status) {
    __shared__ uint32_t red[kClusterThreads / 32];
    __shared__ uint32_t cta_max[kClusterCtas];             // used in CTA 0: one slot per CTA
    __shared__ float d6[128], rtab[128];
    const uint32_t rank = cluster_ctarank();
    const uint32_t nthr = kClusterCtas * kClusterThreads;
    const uint32_t tid = rank * kClusterThreads + threadIdx.x;
    const uint32_t total = rows * nblk;
    griddep_wait();                                        // x may come from the previous grid
    griddep_launch();
    uint4 v[2 * kClusterBlocksPerThread];
    const uint4 zero4 = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < kClusterBlocksPerThread; ++i) {
        const uint32_t b = tid + (uint32_t)i * nthr;
        if (b < total && in_bounds((uint64_t)(b / nblk) * ldx + (b % nblk) * 16, 16,
                                   pitched_extent(rows, nblk * 16, ldx), status)) {
            const uint32_t r = b / nblk, c = b - r * nblk;
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 16);
            v[2 * i] = __ldg(src);
            v[2 * i + 1] = __ldg(src + 1);
        } else {
            v[2 * i] = v[2 * i + 1] = zero4;
        }
    }
    init_d6(d6);
    uint32_t mb[kClusterBlocksPerThread], m = 0;
#pragma unroll
    for (int i = 0; i < kClusterBlocksPerThread; ++i) {
        const uint32_t w[8] = {v[2 * i].x, v[2 * i].y, v[2 * i].z, v[2 * i].w,
                               v[2 * i + 1].x, v[2 * i + 1].y, v[2 * i + 1].z, v[2 * i + 1].w};
        mb[i] = block16_max(w);
        m = max(m, mb[i]);
    }
    m = block_max_u32<kClusterThreads>(m, red);
    if (threadIdx.x == 0) st_shared_cluster_u32(mapa_shared(smem_u32(&cta_max[rank]), 0), m);
    cluster_sync();                                        // CTA 0's array complete (release / acquire)
    uint32_t all = threadIdx.x < kClusterCtas ? ld_shared_cluster_u32(mapa_shared(smem_u32(&cta_max[threadIdx.x]), 0))
                                              : 0u;
    all = __reduce_max_sync(0xFFFFFFFFu, all);            // warp 0 holds the tensor's max
    if (threadIdx.x == 0) red[0] = all;
    cluster_sync();                                        // every CTA has read CTA 0's array
    const uint32_t amax_bits = red[0];
    if (amax_bits >= 0x7F80u && tid == 0) atomicOr(status, 2u);
    const float amax = __uint_as_float(amax_bits << 16);
    const float g_enc = encode_scale(amax);
    if (tid == 0) *g_dec_out = decode_scale(amax);
    init_rtab(rtab, g_enc);
    __syncthreads();
    const uint32_t ctiles = nblk >> 2;
#pragma unroll
    for (int i = 0; i < kClusterBlocksPerThread; ++i) {
        const uint32_t b = tid + (uint32_t)i * nthr;
        if (b - threadIdx.x % 32 >= total) break;          // whole warps past the end stop together
        const bool active = b < total;
        const uint32_t r = b / nblk, c = b - r * nblk;
        const uint32_t w[8] = {v[2 * i].x, v[2 * i].y, v[2 * i].z, v[2 * i].w,
                               v[2 * i + 1].x, v[2 * i + 1].y, v[2 * i + 1].z, v[2 * i + 1].w};
        uint32_t lo, hi;
        const uint32_t sc = nvfp4_block(mb[i], w, g_enc, d6, rtab, lo, hi);
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
        if (active) {
            if (in_bounds((uint64_t)b * 8, 8, (uint64_t)total * 8, status))
                *reinterpret_cast<uint2*>(codes + (size_t)b * 8) = make_uint2(lo, hi);
            const uint32_t so = sf_tile_offset(r, c, ctiles);
            if ((c & 3u) == 0 && in_bounds(so, 4, sf_extent(rows, ctiles), status))
                *reinterpret_cast<uint32_t*>(sf + so) = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
    }
    zero_pad_scale_rows(sf, rows, ctiles, tid, nthr, status);
}

// ------------------------------------------------------------------ NVFP4, one pass
// For tensors whose rows fit in the shared memory of one CTA per SM: every
// CTA copies its rows into shared memory once (each thread copies its own
// blocks with 16-byte asynchronous copies, all issued at once, one commit
// group per block, and takes each block's maximum and fl(b/6) as its group
// lands), publishes its partial amax in a tagged 64-bit slot of the
// workspace, waits (bounded) until every CTA's slot carries this call's tag,
// and quantizes from shared memory.  HBM sees exactly one read of the
// activation.  Every CTA must be resident at once: at most one CTA per SM.
//
// The tag comes from a generation word in the workspace, never from the
// host, so a launch replayed from a CUDA graph is as correct as a fresh one.
// A call reads the word g (zero in a fresh workspace) and tags its slots
// with E = g + 1.  Every tag an earlier call wrote is <= g, so no stale slot
// can pass for this call's.  Once CTA 0 has seen every slot tagged E it
// raises the word to E; every CTA read g before publishing, so all CTAs of
// the call agree on E.  A CTA whose wait gives up raises the word to its own
// tag too, so the next call's tag is above every tag written in this one,
// whichever CTAs gave up; it then takes the amax by reading the whole tensor
// itself, so its outputs are exact all the same, and reports
// NVQ_STATUS_TIMEOUT.  A word at or above 2^48 - 1 (2^48 calls away from a
// zero-filled workspace) was not left by this library: every CTA takes the
// direct amax and the call reports NVQ_STATUS_WORKSPACE.
constexpr int kFusedThreads = 1024;
constexpr int kFusedMaxBlocks = 8;                 // 16-blocks per thread: rows_per_cta * K / 16 <= 8192
constexpr uint64_t kFusedWaitNs = 2000000000ull;   // 2 s
constexpr unsigned long long kGenMax = (1ull << 48) - 1;   // a slot holds a 48-bit tag above a 16-bit maximum

// The slot word carries its tag and its value together, so relaxed
// single-copy-atomic 64-bit accesses suffice: nothing else is published.
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// The generation word is raised with a relaxed maximum.  CTA 0 raises it to
// E only after it has read every slot tagged E, and a CTA's tag is computed
// from the word it read: for a CTA of the same call to read the raised word,
// its own slot would have to hold a tag derived from that read, which CTA 0
// could not have seen before raising it (the memory model's no-thin-air
// rule), so no fence is needed, and no thread waits for one.
__device__ __forceinline__ void red_relaxed_max_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("red.relaxed.gpu.global.max.u64 [%0], %1;" :: "l"(p), "l"(v) : "memory");
}

// BF16 magnitude bits of max |x| over the whole [rows, K] tensor (pitch ldx),
// read by one CTA: the one-pass kernel's amax when its wait gives up.
__device__ __forceinline__ uint32_t cta_tensor_absmax(const uint16_t* __restrict__ x, uint32_t rows, uint32_t K,
                                                      uint32_t ldx, uint32_t* red, unsigned int* status) {
    const uint32_t vpr = K >> 3;                        // 16-byte vectors per row
    const uint32_t total = rows * vpr;
    uint32_t m2 = 0;
    for (uint32_t i = threadIdx.x; i < total; i += kFusedThreads) {
        const uint32_t r = i / vpr, c = i - r * vpr;
        if (!in_bounds((uint64_t)r * ldx + c * 8, 8, pitched_extent(rows, K, ldx), status)) continue;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + (size_t)r * ldx) + c);
        m2 = absmax2(absmax2(absmax2(absmax2(m2, v.x), v.y), v.z), v.w);
    }
    return block_max_u32<kFusedThreads>(fold2(m2), red);
}

// Shared-memory layout of the one-pass kernel's tile: the CTA's rows in
// row-major order, cut into 64-byte groups of two 16-element blocks (blocks
// 2g and 2g + 1), the four 16-byte chunks of group g stored in the order
// chunk ^ ((g >> 1) & 3).  A warp whose consecutive lanes read the same chunk
// of consecutive groups then touches eight different 16-byte bank groups in
// every quarter-warp phase, and each thread reads its chunks in their logical
// order.  Block b's two halves are its group's chunks 2(b & 1) and 2(b & 1) + 1.
__device__ __forceinline__ uint32_t group_chunk(uint32_t g, uint32_t k) {
    return 64u * g + 16u * (k ^ ((g >> 1) & 3u));
}

// Shared memory the one-pass kernel needs for rows_per_cta rows of K: the
// BF16 tile and fl(b / 6) of every block's max b.
__host__ __device__ constexpr size_t fused_smem_bytes(size_t rows_per_cta, size_t K) {
    return 128 /*align*/ + rows_per_cta * K * 2 /*tile*/ + rows_per_cta * (K / 16) * 4 /*fl(b/6)*/;
}

__global__ void __launch_bounds__(kFusedThreads, 1)
nvfp4_quantize_fused_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t K, uint32_t ldx,
                            uint32_t rows_per_cta, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                            float* __restrict__ g_dec_out, unsigned long long* __restrict__ slots,
                            unsigned long long* __restrict__ gen, uint64_t wait_ns,
                            unsigned int* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const uint32_t nblk = K >> 4;
    float* bdiv6 = reinterpret_cast<float*>(tile + (size_t)rows_per_cta * K * 2);
    __shared__ uint32_t red[kFusedThreads / 32];
    __shared__ uint32_t s_pmax[kMaxFusedCtas / 32];
    __shared__ float d6[128], rtab[128];
    __shared__ int s_timeout;
    __shared__ unsigned long long s_gen;

    // x may come from the previous grid, and that grid may still read the
    // outputs: nothing global is touched before it has completed
    griddep_wait();
    griddep_launch();
    const uint32_t r0 = blockIdx.x * rows_per_cta;
    const uint32_t nr = min(rows_per_cta, rows - r0);
    const uint32_t total = nr * nblk;
    // Thread t copies blocks t, t + 1024, ... (the ones it quantizes later),
    // one commit group per block slot so that each can be used as it lands;
    // slots past the thread's blocks commit empty groups.
#pragma unroll
    for (int i = 0; i < kFusedMaxBlocks; ++i) {
        const uint32_t b = threadIdx.x + (uint32_t)i * kFusedThreads;
        const uint32_t rl = b / nblk, c = b - rl * nblk;
        if (b < total && in_bounds((uint64_t)(r0 + rl) * ldx + c * 16, 16, pitched_extent(rows, K, ldx), status)) {
            const uint16_t* src = x + (size_t)(r0 + rl) * ldx + (size_t)c * 16;
            const uint32_t t0 = smem_u32(tile);
            cp_async16(t0 + group_chunk(b >> 1, 2 * (b & 1)), src);          // the block's two halves,
            cp_async16(t0 + group_chunk(b >> 1, 2 * (b & 1) + 1), src + 8);  // one 32-byte source
        }
        cp_async_commit();
    }
    if (threadIdx.x == 0) s_timeout = 0;
    init_d6(d6);
    __syncthreads();
    // The generation this call starts from; no CTA of the call can raise it
    // before every CTA has read it.  Thread 0 reads it here, after its copies
    // and the barrier, and needs the value only when it publishes, so the
    // load's latency hides under the copies'.  A relaxed load suffices: the
    // slot it publishes carries a tag computed from the value read, and that
    // data dependency keeps the publication after the read.
    unsigned long long g_seen = 0;
    if (threadIdx.x == 0) g_seen = ld_relaxed_u64(gen);

    // block maxima and fl(b/6), block by block as the copies land
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < kFusedMaxBlocks; ++i) {
        switch (i) {            // at most kFusedMaxBlocks - 1 - i groups may still be pending
            case 0: cp_async_wait<kFusedMaxBlocks - 1>(); break;
            case 1: cp_async_wait<kFusedMaxBlocks - 2>(); break;
            case 2: cp_async_wait<kFusedMaxBlocks - 3>(); break;
            case 3: cp_async_wait<kFusedMaxBlocks - 4>(); break;
            case 4: cp_async_wait<kFusedMaxBlocks - 5>(); break;
            case 5: cp_async_wait<kFusedMaxBlocks - 6>(); break;
            case 6: cp_async_wait<kFusedMaxBlocks - 7>(); break;
            default: cp_async_wait<0>(); break;
        }
        const uint32_t b = threadIdx.x + (uint32_t)i * kFusedThreads;
        if (b < total) {
            const uint4 v0 = *reinterpret_cast<const uint4*>(tile + group_chunk(b >> 1, 2 * (b & 1)));
            const uint4 v1 = *reinterpret_cast<const uint4*>(tile + group_chunk(b >> 1, 2 * (b & 1) + 1));
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const uint32_t mb = block16_max(w);
            bdiv6[b] = div6(mb, d6);           // the scale's first step, done while copies land
            m = max(m, mb);
        }
    }
    if (threadIdx.x == 0) s_gen = g_seen;
    const uint32_t cta_max = block_max_u32<kFusedThreads>(m, red);   // (its barriers publish s_gen)
    const unsigned long long g0 = s_gen;
    const bool trusted = g0 < kGenMax;
    const unsigned long long tag = g0 + 1;
    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t npoll = (gridDim.x + 31) >> 5;
    if (trusted) {
        if (threadIdx.x == 0 && in_bounds(blockIdx.x, 1, kMaxAmaxPartials, status))
            st_relaxed_u64(slots + (size_t)blockIdx.x * kFusedSlotStride, (tag << 16) | cta_max);
        // Every CTA's partial, tagged with this call's tag.  Warp w polls
        // slots 32w .. 32w + 31, one per lane, so a polling round costs one
        // L2 round trip; the other warps wait at the barrier below.
        if (warp < npoll) {
            volatile int* timeout = &s_timeout;
            const uint32_t j = warp * 32 + lane;
            bool done = j >= gridDim.x;
            uint32_t mine = 0;
            const uint64_t t0 = globaltimer_ns();
            uint32_t spins = 0;
            while (true) {
                if (!done) {
                    const unsigned long long v = ld_relaxed_u64(slots + (size_t)j * kFusedSlotStride);
                    if ((v >> 16) == tag) {
                        mine = (uint32_t)(v & 0xFFFFull);
                        done = true;
                    }
                }
                if (__all_sync(0xFFFFFFFFu, done)) break;
                // decided by lane 0 so the warp leaves together; the clock
                // is read in the first round and every 8th after it (a round is one
                // L2 round trip)
                int give_up = 0;
                if (lane == 0 && (spins++ & 7u) == 0) give_up = *timeout || globaltimer_ns() - t0 > wait_ns;
                if (__shfl_sync(0xFFFFFFFFu, give_up, 0)) {
                    if (lane == 0) *timeout = 1;
                    break;
                }
            }
            mine = __reduce_max_sync(0xFFFFFFFFu, mine);
            if (lane == 0) s_pmax[warp] = mine;
        }
    }
    __syncthreads();
    uint32_t amax_bits = 0;
    if (!trusted || s_timeout) {
        // The barrier is off (a peer never arrived within the limit, or the
        // generation word is not one this library left): the amax straight
        // from x, so the outputs are exact all the same.
        if (threadIdx.x == 0) {
            atomicOr(status, trusted ? kStatusTimeout : kStatusWorkspace);
            if (trusted) red_relaxed_max_u64(gen, tag);
        }
        amax_bits = cta_tensor_absmax(x, rows, K, ldx, red, status);
    } else {
        for (uint32_t i = 0; i < npoll; ++i) amax_bits = max(amax_bits, s_pmax[i]);
        if (blockIdx.x == 0 && threadIdx.x == 0) red_relaxed_max_u64(gen, tag);
    }
    if (amax_bits >= 0x7F80u && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusNonfinite);
    const float amax = __uint_as_float(amax_bits << 16);
    const float g_enc = encode_scale(amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_dec_out = decode_scale(amax);
    init_rtab(rtab, g_enc);
    __syncthreads();

    // Encode: thread t takes the 2-block groups g = t, t + 1024, ..., two
    // groups per iteration, both read before either is computed.  A group's
    // 16 code bytes leave in one store; the 4 scale bytes of blocks 4j ..
    // 4j + 3 (groups 2j, 2j + 1: lanes l, l + 1) in one 32-bit store by the
    // even lane.  Groups never straddle rows (K / 16 is a multiple of 4).
    const uint32_t ctiles = nblk >> 2;
    const uint32_t ngroups = total >> 1;
    const uint32_t qs = 2 * kFusedThreads / nblk, rs = 2 * kFusedThreads - qs * nblk;   // one group stride, in blocks
    uint32_t rl = 2 * threadIdx.x / nblk, c = 2 * threadIdx.x - rl * nblk;            // first block of group t
    const float2* bd2 = reinterpret_cast<const float2*>(bdiv6);
    uint8_t* code_cta = codes + (size_t)r0 * nblk * 8;
    for (uint32_t base = 0; base < ngroups; base += 2 * kFusedThreads) {
        uint32_t rlu[2], cu[2];
        rlu[0] = rl;
        cu[0] = c;
        rlu[1] = rl + qs;
        cu[1] = c + rs;
        if (cu[1] >= nblk) {
            cu[1] -= nblk;
            ++rlu[1];
        }
        uint4 v[2][4];
        float2 d[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t g = base + u * kFusedThreads + threadIdx.x;
            d[u] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int k = 0; k < 4; ++k) v[u][k] = make_uint4(0, 0, 0, 0);
            if (g < ngroups) {
#pragma unroll
                for (int k = 0; k < 4; ++k) v[u][k] = *reinterpret_cast<const uint4*>(tile + group_chunk(g, k));
                d[u] = bd2[g];
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const uint32_t g = base + u * kFusedThreads + threadIdx.x;
            const bool active = g < ngroups;         // whole warps stay for the shuffle
            const uint32_t w0[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                                    v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
            const uint32_t w1[8] = {v[u][2].x, v[u][2].y, v[u][2].z, v[u][2].w,
                                    v[u][3].x, v[u][3].y, v[u][3].z, v[u][3].w};
            uint32_t lo0, hi0, lo1, hi1;
            const uint32_t pair = nvfp4_block_pair_d(d[u].x, d[u].y, w0, w1, g_enc, rtab, lo0, hi0, lo1, hi1);
            const uint32_t next = __shfl_down_sync(0xFFFFFFFFu, pair, 1);
            if (active) {
                if (in_bounds((uint64_t)r0 * nblk * 8 + (uint64_t)g * 16, 16, (uint64_t)rows * nblk * 8, status))
                    *reinterpret_cast<uint4*>(code_cta + (size_t)g * 16) = make_uint4(lo0, hi0, lo1, hi1);
                const uint32_t so = sf_tile_offset(r0 + rlu[u], cu[u], ctiles);
                if ((g & 1u) == 0 && in_bounds(so, 4, sf_extent(rows, ctiles), status))
                    *reinterpret_cast<uint32_t*>(sf + so) = pair | (next << 16);
            }
        }
        // advance by two group strides
        rl = rlu[1] + qs;
        c = cu[1] + rs;
        if (c >= nblk) {
            c -= nblk;
            ++rl;
        }
    }
    zero_pad_scale_rows(sf, rows, ctiles, blockIdx.x * kFusedThreads + threadIdx.x, gridDim.x * kFusedThreads,
                        status);
}

// ------------------------------------------------------------------ MXFP8
// One 32-element block, its 32 BF16 values in w[0..15] (element 2i in the
// low half of w[i]).  ELEM 0: E4M3 elements (largest 448 = 1.75 * 2^8);
// ELEM 1: E5M2 (largest 57344 = 1.75 * 2^15).  RULE 0: X = floor(log2 b) -
// emax (OCP); RULE 1: the smallest X with b <= largest * 2^X, i.e. one more
// than the floor value when b's significand exceeds 1.75 (both largest
// values are 1.75 * 2^emax), so no element saturates.  Returns the E8M0
// scale byte X + 127; q receives the 32 element codes, 4 per word.
template <int ELEM, int RULE>
__device__ __forceinline__ uint32_t mx_block(const uint32_t (&w)[16], uint32_t (&q)[8]) {
    constexpr int EMAX = ELEM == 0 ? 8 : 15;
    uint32_t m2 = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) m2 = absmax2(m2, w[i]);
    const uint32_t mb = fold2(m2);                   // BF16 magnitude bits of the block max
    int X;
    if (mb == 0) {
        X = -127;
    } else {
        const int E = (int)(mb >> 7);
        const uint32_t mant = mb & 0x7Fu;
        const int p = 31 - __clz((int)mant);          // subnormal: leading one of the mantissa
        const int e = E ? E - 127 : p - 133;
        int up = 0;
        if (RULE == 1) up = E ? (mant > 96u) : (4u * mant > (7u << p));   // significand > 1.75
        X = min(max(e - EMAX + up, -127), 127);
    }
    const float mult = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, -127 <= X <= 121
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 p0 = bf16x2_mul(w[2 * i], mult);
        const float2 p1 = bf16x2_mul(w[2 * i + 1], mult);
        q[i] = ELEM == 0 ? cvt_e4m3x4(p0.x, p0.y, p1.x, p1.y) : cvt_e5m2x4(p0.x, p0.y, p1.x, p1.y);
    }
    return (uint32_t)(X + 127);
}

// One thread = one 32-element block (mx_block above).  Block b is
// (row b / nblk, column b % nblk), nblk = K / 32; its codes are bytes
// [32b, 32b + 32).
template <int ELEM, int RULE>
__global__ void __launch_bounds__(kQuantThreads)
mxfp8_quantize_kernel(const uint16_t* __restrict__ x, uint32_t rows, uint32_t nblk, uint32_t ldx,
                      uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, unsigned int* __restrict__ status) {
    griddep_wait();                              // x may come from the previous grid
    griddep_launch();
    const uint32_t total = rows * nblk;
    const uint32_t ctiles = nblk >> 2;
    const uint32_t stride = gridDim.x * kQuantThreads;
    const uint32_t qs = stride / nblk, rs = stride - qs * nblk;
    uint32_t b = blockIdx.x * kQuantThreads + threadIdx.x;
    uint32_t r = b / nblk, c = b - r * nblk;
    for (; b - threadIdx.x < total; b += stride) {
        const bool active = b < total;
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = 0;
        if (active && in_bounds((uint64_t)r * ldx + c * 32, 32, pitched_extent(rows, nblk * 32, ldx), status)) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)r * ldx + (size_t)c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint4 v = __ldg(src + u);
                w[4 * u] = v.x; w[4 * u + 1] = v.y; w[4 * u + 2] = v.z; w[4 * u + 3] = v.w;
            }
        }
        uint32_t q[8];
        const uint32_t sc = mx_block<ELEM, RULE>(w, q);
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
        if (active) {
            if (in_bounds((uint64_t)b * 32, 32, (uint64_t)total * 32, status)) {
                uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)b * 32);
                dst[0] = make_uint4(q[0], q[1], q[2], q[3]);
                dst[1] = make_uint4(q[4], q[5], q[6], q[7]);
            }
            const uint32_t so = sf_tile_offset(r, c, ctiles);
            if ((c & 3u) == 0 && in_bounds(so, 4, sf_extent(rows, ctiles), status))
                *reinterpret_cast<uint32_t*>(sf + so) = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        }
        r += qs;
        c += rs;
        if (c >= nblk) {
            c -= nblk;
            ++r;
        }
    }
    zero_pad_scale_rows(sf, rows, ctiles, blockIdx.x * kQuantThreads + threadIdx.x, stride, status);
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

// Test hook for the bounded waits: one thread waits, through the same
// mbar_wait_bounded the GEMM pipelines use, on a shared-memory mbarrier that
// nothing arrives on.  When the wait gives up after limit_ns it sets
// NVQ_STATUS_TIMEOUT (bit 0) in the status word, as a GEMM role would, and the
// kernel returns normally.  *waited receives the nanoseconds spent.
// One failing bounds check and nothing else: the debug build's report path
// (the status bit) without any memory access.  In the normal build the
// check compiles away and the kernel does nothing.
__global__ void probe_bounds_kernel(unsigned int* __restrict__ status) {
    if (threadIdx.x == 0) (void)in_bounds(1, 1, 1, status);
}

__global__ void probe_wait_kernel(uint64_t limit_ns, unsigned int* __restrict__ status,
                                  unsigned long long* __restrict__ waited) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int never;
    if (threadIdx.x != 0) return;
    never = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbarrier_init();
    const uint64_t t0 = globaltimer_ns();
    if (!mbar_wait_bounded(smem_u32(&bar), 0, &never, limit_ns)) atomicOr(status, 1u);
    *waited = globaltimer_ns() - t0;
}

}  // namespace nvq

/*
 * nvq.h -- C ABI of the B200 (sm_100a) microscaling-quantized linear layer.
 *
 * The layer has two parts (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍",
 * section "MXFP8和NVFP4技术背景解析"; page "NVIDIA Blackwell平台FP4量化技术解析与
 * 图像生成优化", section 3.1):
 *   1. dynamic activation quantization, BF16 -> NVFP4 (E2M1 values in
 *      16-element blocks, an E4M3 block scale, one FP32 per-tensor global
 *      scale) or BF16 -> MXFP8 (E4M3 values in 32-element blocks, an E8M0
 *      block scale);
 *   2. the block-scaled GEMM that multiplies the quantized activations by
 *      pre-quantized weights on the tensor cores and writes BF16.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or keeps them.  It allocates no device memory of
 *    its own.  Its device state is static device variables, present on every
 *    GPU that loads the library: one status word per GPU, read by
 *    nvq_device_status(), and the 4 KB scratch array of
 *    nvfp4_quantize_noalloc().  The library looks up their device addresses
 *    once per GPU and keeps them; a device reset (cudaDeviceReset) invalidates
 *    them, so no library call may follow one in the same process.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  The return value reports only host-side argument
 *    checks and launch errors.  Errors found by the host launch nothing.
 *  - Matrices are row-major.  BF16 tensors are [rows, K] with a row pitch
 *    `ld` in elements.  Quantized codes are dense: an NVFP4 row is K/2 bytes
 *    (element 2j in the low nibble of byte j, 2j+1 in the high nibble), an
 *    MXFP8 row is K bytes of E4M3 (or E5M2, format NVQ_MXFP8_E5M2).
 *  - Block scales form a logical matrix S[rows][K / block] of bytes (E4M3 for
 *    NVFP4, E8M0 for MXFP8) stored in the 128x4 tile order the sm_100
 *    block-scaled tensor-core instructions read: tiles of 128 rows x 4
 *    scale columns, 512 bytes each, tile (r/128, c/4) at
 *    ((r/128) * (C/4) + c/4) * 512, and inside a tile row r, column c at
 *    (r%32)*16 + ((r%128)/32)*4 + (c%4), where C = K / block.  The tiles
 *    cover the rows rounded up to 128 ("block alignment must be a multiple
 *    of 128", NVIDIA Blackwell平台FP4量化技术解析与图像生成优化, section 5.2);
 *    the quantizers write zero into the rows past the tensor's last row.
 *  - Shape contract: any row count (M, N >= 0; a ragged count is padded
 *    only in the scale tiles); K a positive multiple of 64 (NVFP4) or 128
 *    (MXFP8) so scale columns fill whole tiles; every BF16 pitch a multiple
 *    of 8 elements and >= K; all pointers 16-byte aligned; rows * K < 2^31.
 *    Otherwise NVQ_ERR_SHAPE / NVQ_ERR_ALIGN, and nothing is launched.
 *    M == 0 (an empty batch) is accepted and launches nothing.
 *  - The device must be compute capability 10.0 (B200, sm_100a), else
 *    NVQ_ERR_ARCH.
 *  - Inputs must be finite.  A NaN or infinity in a tensor handed to
 *    nvfp4_quantize sets NVQ_STATUS_NONFINITE in the device status word; the
 *    codes written for such a tensor are unspecified.
 */
#ifndef NVQ_H
#define NVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NVQ_API __attribute__((visibility("default")))
#else
#define NVQ_API
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* nvq_stream_t;

/* NVQ_MXFP8_E5M2: MXFP8 with E5M2 elements (page "NVIDIA量化推理：5步极速优化显存+
 * 成功率翻倍", section MXFP8量化格式, names E4M3 and E5M2 as the element types). */
typedef enum { NVQ_NVFP4 = 0, NVQ_MXFP8 = 1, NVQ_MXFP8_E5M2 = 2 } nvq_format;

/* MXFP8 block-exponent rule (mxfp8_quantize_ex).  FLOOR is the OCP rule
 * X = floor(log2(block max)) - emax (elements in [max, 2*max) * 2^X
 * saturate); CEIL takes the smallest X with block max <= max * 2^X, so no
 * element saturates.  emax = 8 (E4M3, max 448), 15 (E5M2, max 57344). */
enum { NVQ_SCALE_FLOOR = 0, NVQ_SCALE_CEIL = 1 };

/* Return codes (host side). */
enum {
    NVQ_OK = 0,
    NVQ_ERR_NULL = -1,      /* a required pointer is NULL */
    NVQ_ERR_SHAPE = -2,     /* a size or pitch breaks the shape contract */
    NVQ_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned */
    NVQ_ERR_ARCH = -4,      /* current device is not compute capability 10.0 */
    NVQ_ERR_CUDA = -5,      /* a CUDA runtime/driver call or launch failed */
    NVQ_ERR_FORMAT = -7     /* unknown nvq_format value */
};

/* Bits of the device status word (nvq_device_status). */
enum {
    NVQ_STATUS_TIMEOUT = 1,     /* a bounded wait inside a kernel gave up (see the entry points) */
    NVQ_STATUS_NONFINITE = 2,   /* nvfp4_quantize saw a NaN/Inf amax */
    NVQ_STATUS_WORKSPACE = 4,   /* nvfp4_quantize was given a workspace it did not leave (not zero-filled) */
    NVQ_STATUS_BOUNDS = 8       /* debug build only: a kernel's bounds check failed (nvq_debug_build) */
};

/* Bytes of the code buffer for a [rows, K] tensor: rows*K/2 (NVFP4), rows*K (MXFP8, either element). */
NVQ_API size_t nvq_codes_bytes(int format, int64_t rows, int64_t K);

/* Bytes of the swizzled scale buffer: ceil(rows/128)*128 * ceil((K/block)/4)*4,
 * block = 16 (NVFP4) or 32 (MXFP8). */
NVQ_API size_t nvq_scale_bytes(int format, int64_t rows, int64_t K);

/* Bytes of device scratch that nvfp4_quantize / quantize_weight(NVQ_NVFP4)
 * need: the per-CTA partial maxima of the tensor and the tagged slots and
 * generation word of the one-pass kernel's grid barrier.  Constant for the
 * life of the library.  A workspace must be zero-filled once before its
 * first use (nvq_workspace_init, or any memset to zero); every call leaves
 * it ready for the next, so it is never cleared again.  Calls that can run
 * at the same time (different streams, no ordering) must not share one. */
NVQ_API size_t nvq_workspace_bytes(void);

/* nvq_workspace_init -- zero-fills a workspace of nvq_workspace_bytes() bytes
 * (asynchronously on `stream`), as its first use requires.  No counterpart
 * on the pages.  NVQ_ERR_NULL / NVQ_ERR_ALIGN / NVQ_ERR_CUDA. */
NVQ_API int nvq_workspace_init(void* workspace, nvq_stream_t stream);

/*
 * nvfp4_quantize -- dynamic BF16 -> NVFP4 activation quantization.
 * Page "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化", section 3.1: the
 * run-time quantizer turns a BF16 input into [FP4 data, FP8 block scales,
 * FP32 global scale]; page "NVIDIA量化推理：5步极速优化显存+成功率翻倍",
 * step 2: the per-tensor scale is computed from the live activation.
 *
 *   x            [M, K] BF16, row pitch ldx elements (read only)
 *   codes        out, nvq_codes_bytes(NVQ_NVFP4, M, K) bytes
 *   scales       out, nvq_scale_bytes(NVQ_NVFP4, M, K) bytes (E4M3, tile order)
 *   global_scale out, one float: the decode scale g_dec = amax / 2688
 *   calib_amax   NULL for the dynamic path (amax taken from x).  Otherwise a
 *                device float holding a calibrated per-tensor amax (page
 *                "FP8量化技术提升SD3.5...", section 校准): the amax pass is
 *                skipped; elements beyond the calibrated range saturate.
 *   workspace    device scratch of nvq_workspace_bytes(), zero-filled before
 *                its first use (see nvq_workspace_bytes); must not be shared
 *                by two calls that can run at the same time.  Required on the
 *                dynamic path; with calib_amax it is not read (may be NULL).
 *
 * Arithmetic, in FP32 round-to-nearest-even, bit-exact with the CPU oracle:
 *   g_enc = 2688 / amax, g_dec = amax / 2688; per 16-block along K,
 *   b = max|x|, sc = E4M3(b / 6 * g_enc), r = g_enc / sc, q = E2M1(x * r)
 *   (round to nearest even, saturate, sign kept).  A block whose scale
 *   rounds to zero gets zero codes.  amax < 2^-100 (zero included) gives
 *   all-zero codes and scales and g_dec = 0.
 *
 * The dynamic path takes one of three kernels by size: one cluster of CTAs
 * for small tensors; one pass (amax and quantization in one launch, x read
 * once) when one CTA per SM can hold its rows in shared memory; else an amax
 * pass and a quantize pass.  All give the same bits.  The one-pass kernel's
 * CTAs exchange partial maxima through the workspace and so must all be
 * resident at once; kernels on other streams that hold SMs can delay some of
 * them.  A CTA that has waited past the limit (2 s) reads the amax from x
 * itself: the results stay exact, the call is slower, and NVQ_STATUS_TIMEOUT
 * is set.  A graph capture of this call replays correctly: the barrier's
 * state lives in the workspace.  A workspace that was not zero-filled can
 * make the one-pass kernel report NVQ_STATUS_WORKSPACE (results then still
 * exact) or, undetectably, use a stale partial maximum.
 */
NVQ_API int nvfp4_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                   uint8_t* codes, uint8_t* scales, float* global_scale,
                   const float* calib_amax, void* workspace, nvq_stream_t stream);

/*
 * mxfp8_quantize -- BF16 -> MXFP8 (E4M3 elements, E8M0 scale per 32-block).
 * Page "NVIDIA量化推理：5步极速优化显存+成功率翻倍", section "MXFP8量化格式"
 * (OCP 8-bit microscaling format).  Per 32-block along K: X = floor(log2(max
 * |x|)) - 8 clamped to [-127, 127] (-127 for an all-zero block), scale byte
 * X + 127, q = E4M3(x * 2^-X) rounded to nearest even and saturated at 448.
 *
 *   x       [M, K] BF16, row pitch ldx elements
 *   codes   out, nvq_codes_bytes(NVQ_MXFP8, M, K) bytes
 *   scales  out, nvq_scale_bytes(NVQ_MXFP8, M, K) bytes (E8M0, tile order)
 */
NVQ_API int mxfp8_quantize(const void* x, int64_t M, int64_t K, int64_t ldx,
                   uint8_t* codes, uint8_t* scales, nvq_stream_t stream);

/*
 * mxfp8_quantize_ex -- mxfp8_quantize with a choice of element type and
 * block-exponent rule (page "NVIDIA量化推理：5步极速优化显存+成功率翻倍",
 * section MXFP8量化格式: E4M3 or E5M2 elements under one 8-bit shared
 * exponent per 32 values).
 *
 *   elem_format  NVQ_MXFP8 (E4M3 elements) or NVQ_MXFP8_E5M2 (E5M2: 1 sign,
 *                5 exponent, 2 mantissa bits, bias 15, largest 57344)
 *   scale_rule   NVQ_SCALE_FLOOR or NVQ_SCALE_CEIL (see above)
 * Per 32-block: X from the rule, clamped to [-127, 127] (-127 for an
 * all-zero block), scale byte X + 127, q = ELEM(x * 2^-X) rounded to nearest
 * even and saturated.  Other arguments and errors as mxfp8_quantize; an
 * unknown elem_format or scale_rule gives NVQ_ERR_FORMAT.
 */
NVQ_API int mxfp8_quantize_ex(const void* x, int64_t M, int64_t K, int64_t ldx,
                      uint8_t* codes, uint8_t* scales, int elem_format, int scale_rule,
                      nvq_stream_t stream);

/*
 * quantize_weight -- offline weight quantization ("double quantization" of
 * BF16 weights into FP4 data + FP8 scales, page "NVIDIA Blackwell平台FP4量化
 * 技术解析与图像生成优化", section 3.1), run once at load time.  Same
 * arithmetic as nvfp4_quantize / mxfp8_quantize applied to W [N, K]; for
 * NVFP4 the global scale is the weight's own static g_dec.
 *
 *   format        NVQ_NVFP4, NVQ_MXFP8 or NVQ_MXFP8_E5M2 (floor block exponent)
 *   global_scale  NVFP4: out, required.  MXFP8: ignored (may be NULL).
 *   workspace     NVFP4: required (nvq_workspace_bytes(), zero-filled before
 *                 its first use).  MXFP8: ignored.
 */
NVQ_API int quantize_weight(int format, const void* w, int64_t N, int64_t K, int64_t ldw,
                    uint8_t* codes, uint8_t* scales, float* global_scale,
                    void* workspace, nvq_stream_t stream);

/*
 * block_scaled_linear -- D = A * B^T on the block-scaled tensor cores
 * (page "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化", section 3.1: FP4
 * operands with FP8 block scales consumed by the 5th-generation tensor
 * cores; page "NVIDIA量化推理：5步极速优化显存+成功率翻倍": every nn.Linear of
 * the transformer becomes a quantized linear).
 *
 *   D[m, n] = bf16( alpha * sum_k a(m,k) * sa(m, k/bs) * b(n,k) * sb(n, k/bs) + bias[n] )
 *   with alpha = a_global[0] * b_global[0] for NVFP4 and 1 for MXFP8.
 *
 *   a_codes, a_scales   quantized activations [M, K] (nvfp4_quantize/mxfp8_quantize)
 *   a_global            NVFP4: device float g_dec of A.  MXFP8: ignored.
 *   b_codes, b_scales   quantized weights [N, K] (quantize_weight)
 *   b_global            NVFP4: device float g_dec of B.  MXFP8: ignored.
 *   bias                NULL or BF16 [N]
 *   format              NVQ_NVFP4, NVQ_MXFP8 (E4M3 x E4M3) or NVQ_MXFP8_E5M2 (E5M2 x E5M2)
 *   out                 BF16 [M, N], row pitch ldo elements (ldo >= N, multiple of 8)
 *   M, N                M any, N a multiple of 8 (ragged tiles read zeros past the
 *                       end and store nothing there; bias is read only for n < N;
 *                       the store of a row's last chunk is clipped at 16 bytes);
 *                       K a multiple of 256 (NVFP4) or 128 (MXFP8)
 *
 * Accumulation is FP32 in tensor memory; the order of the K sum is the
 * hardware's.  At a short M (at most 32 rows) the K range may be split over
 * a cluster of CTAs whose FP32 partial sums are then added in a fixed order
 * (nvq_gemm_plan reports the choice).  Results match the FP64 sum over the
 * dequantized operands to a relative error (normalised by the output row's
 * L2 norm) of 2e-3.
 * Pipeline waits inside the kernel are bounded (4 s, or nvq_set_wait_limit);
 * if one gives up, the kernel sets NVQ_STATUS_TIMEOUT, writes nothing further
 * (the output is then unspecified) and exits after waiting, again bounded,
 * for its own copies and tensor-core work in flight.
 */
NVQ_API int block_scaled_linear(int format,
                        const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global,
                        const void* bias, void* out, int64_t ldo,
                        int64_t M, int64_t N, int64_t K, nvq_stream_t stream);

/*
 * nvq_gemm_plan -- the kernel block_scaled_linear launches for a shape on
 * the current device: output tile tile_m x tile_n (tile_m 256 = CTA pairs,
 * 128 = one CTA per tile) and k_split CTAs per tile summing disjoint K
 * ranges (1 = no split).  Host-only: launches nothing, allocates nothing.
 *
 *   format               as block_scaled_linear
 *   M, N, K              as block_scaled_linear (M >= 1)
 *   tile_m, tile_n, k_split  out, host pointers
 *
 * Returns NVQ_OK, NVQ_ERR_FORMAT, NVQ_ERR_NULL, NVQ_ERR_SHAPE (the shape
 * block_scaled_linear would reject), NVQ_ERR_ARCH or NVQ_ERR_CUDA (no
 * device); outputs are written only on NVQ_OK.
 */
NVQ_API int nvq_gemm_plan(int format, int64_t M, int64_t N, int64_t K, int* tile_m, int* tile_n, int* k_split);

/*
 * nvq_gemm_plan_host -- the same choice for stated device facts instead of
 * the current device's, so that it can be reasoned about (and tested)
 * without a GPU.  Host-only.
 *
 *   num_sms        SMs of the device (> 0)
 *   max_clusters   host int[3][9]: [w][s] = the most clusters of s CTAs with
 *                  w-wide tiles the device holds at once, w = 0 / 1 / 2 for
 *                  128 / 192 / 256 (cudaOccupancyMaxActiveClusters at one CTA
 *                  per SM); entries s < 2 are not read
 *   use_pairs      0 forbids CTA pairs (as NVQ_GEMM_PAIRS=0 does)
 *   use_splitk     0 forbids the K split (as NVQ_GEMM_SPLITK=0 does)
 *
 * Returns as nvq_gemm_plan, without NVQ_ERR_ARCH / NVQ_ERR_CUDA;
 * NVQ_ERR_SHAPE also for num_sms <= 0.
 */
NVQ_API int nvq_gemm_plan_host(int format, int64_t M, int64_t N, int64_t K, int num_sms, const int* max_clusters,
                               int use_pairs, int use_splitk, int* tile_m, int* tile_n, int* k_split);

/*
 * block_scaled_linear_gelu_mxfp8 -- the first linear of a feed-forward block
 * with the next layer's activation quantization fused into its epilogue:
 *
 *   D[m, n]  = bf16( alpha * sum_k a(m,k) sa(m,k/bs) b(n,k) sb(n,k/bs) + bias[n] )
 *              exactly as block_scaled_linear computes it (D is not written)
 *   G[m, n]  = GELU(D[m, n]) = D * Phi(D), Phi the standard normal CDF (the
 *              exact-erf form), rounded once to BF16
 *   y_codes, y_scales = mxfp8_quantize(G): per 32 consecutive columns of a
 *              row, X = floor(log2(max |G|)) - 8, scale byte X + 127, codes
 *              E4M3(G * 2^-X) (round to nearest even, saturate at 448)
 *
 * The output is the quantized activation of the following linear (format
 * NVQ_MXFP8, K of that layer = N of this one), so the BF16 activation between
 * the two layers never reaches memory (page "NVIDIA Blackwell平台FP4量化技术解析
 * 与图像生成优化", section 2.1: the transformer's fully connected layers run in
 * FP4; the activation between them is not named on the pages, and the exact-erf
 * GELU is the reading taken).
 *
 *   format            NVQ_NVFP4 or NVQ_MXFP8 (A and B operands, as block_scaled_linear)
 *   a_*, b_*, bias    as block_scaled_linear
 *   y_codes           out, [M, N] E4M3 bytes, dense (nvq_codes_bytes(NVQ_MXFP8, M, N))
 *   y_scales          out, nvq_scale_bytes(NVQ_MXFP8, M, N) bytes (E8M0, tile
 *                     order; rows M .. ceil(M/128)*128 - 1 written as zero)
 *   M, N, K           M any, N a multiple of 128 (whole scale tiles of the next
 *                     layer), K a multiple of 256 (NVFP4) or 128 (MXFP8)
 *
 * For every BF16 value of D the GELU is the correctly rounded one, so y_codes
 * and y_scales are a function of D alone; D itself carries the GEMM's
 * tolerance (see block_scaled_linear).  Errors: as block_scaled_linear, and
 * NVQ_ERR_FORMAT for NVQ_MXFP8_E5M2 operands.
 */
NVQ_API int block_scaled_linear_gelu_mxfp8(int format,
                        const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global,
                        const void* bias, uint8_t* y_codes, uint8_t* y_scales,
                        int64_t M, int64_t N, int64_t K, nvq_stream_t stream);

/*
 * nvfp4_linear_short_m -- the NVFP4 linear of a short batch (M <= 16) in one
 * launch: the dynamic activation quantization of nvfp4_quantize and the
 * block-scaled GEMM of block_scaled_linear, fused, for latency at short
 * batches (batch 1 of the pages' FLUX runs, page "Modelos de Difusão"; the
 * small-batch latency discussion of page "NVIDIA量化推理：5步极速优化显存+成功率
 * 翻倍").  Every CTA of the split-K GEMM quantizes the rows of its own share
 * of K into its pipeline stages, with the arithmetic of nvfp4_quantize, while
 * the weight streams in.  The amax: up to 4 rows every CTA reads the whole
 * activation; above 4 rows each CTA takes the max over its own share and the
 * CTAs of a cluster (whose shares cover K) exchange these partial maxima
 * through distributed shared memory.  If that exchange's bounded wait gives
 * up, the CTA reads the whole activation instead (the result stays exact) and
 * NVQ_STATUS_TIMEOUT is set.
 *
 *   out = block_scaled_linear(NVQ_NVFP4, nvfp4_quantize(x), w) bit for bit:
 *   the same codes, scales and global scale, the same split-K order.
 *
 *   x          in, BF16 [M, K], row pitch ldx elements (ldx >= K, a multiple
 *              of 8), 16-byte aligned
 *   M, K, N    1 <= M <= 16 (0 is a no-op); K a multiple of 256; N a
 *              multiple of 8
 *   b_*        the weight as quantize_weight(NVQ_NVFP4) wrote it, [N, K]
 *   bias       optional BF16 [N] (NULL for none)
 *   out, ldo   out, BF16 [M, N] with row pitch ldo (>= N, a multiple of 8)
 *   a_codes, a_scales, a_global
 *              optional outs (each may be NULL): the activation's codes,
 *              scales (tile order, padding rows zero) and global scale, as
 *              nvfp4_quantize would write them
 *
 * The fused launch exists only where block_scaled_linear would split K
 * across a cluster (nvq_gemm_plan returns k_split > 1) and every CTA's share
 * of the K stages fits its pipeline at once; otherwise it returns
 * NVQ_ERR_SHAPE and launches nothing, and the caller takes the two calls.
 * A NaN/Inf amax sets NVQ_STATUS_NONFINITE.  Other errors as nvfp4_quantize
 * and block_scaled_linear.
 */
NVQ_API int nvfp4_linear_short_m(const void* x, int64_t M, int64_t K, int64_t ldx, const uint8_t* b_codes,
                                 const uint8_t* b_scales, const float* b_global, const void* bias, void* out,
                                 int64_t ldo, int64_t N, uint8_t* a_codes, uint8_t* a_scales, float* a_global,
                                 nvq_stream_t stream);

/*
 * nvq_device_status -- synchronizes `stream`, then returns the current
 * device's status word (NVQ_STATUS_* bits, 0 = clean) and clears it.
 * Returns NVQ_ERR_CUDA (< 0) if the synchronization or the read fails.
 */
NVQ_API int nvq_device_status(nvq_stream_t stream);

/* Human-readable name of a return code. */
NVQ_API const char* nvq_status_string(int code);

/*
 * nvq_set_wait_limit -- test hook (no counterpart on the pages).  Sets, for
 * the whole process, the limit of the bounded waits between the roles of a
 * kernel that later launches use: the GEMM pipeline waits (default 4 s) and
 * the one-pass quantizer's grid barrier (default 2 s).  0 restores the
 * defaults; at most 4e9 (else NVQ_ERR_SHAPE).  It lets a test make those
 * waits run out on purpose and check that the kernel reports
 * NVQ_STATUS_TIMEOUT and returns, with the context intact.  The waits with
 * which a kernel drains its own copies and tensor-core work before it exits
 * keep their 4 s limit.  Launches already issued are not affected.
 */
NVQ_API int nvq_set_wait_limit(uint64_t limit_ns);

/*
 * nvq_wait_limit -- the limit nvq_set_wait_limit last set (0: the defaults).
 * Its initial value comes from the environment variable NVQ_WAIT_LIMIT_NS
 * (decimal nanoseconds, at most 4e9), read once when the library loads; an
 * unset, malformed or larger value leaves the defaults.  No device needed.
 */
NVQ_API uint64_t nvq_wait_limit(void);

/*
 * nvfp4_quantize_noalloc -- nvfp4_quantize for callers that cannot allocate
 * device memory.  The pages have no counterpart to this entry point.
 *
 * Some callers cannot call cudaMalloc, nor hand the library a workspace:
 * code that runs inside a host framework which owns all device memory and
 * offers its plug-ins neither an allocator nor a scratch buffer, or code on
 * a latency-critical path where a device allocation (and the synchronisation
 * it can imply) is not acceptable.  This variant takes the same inputs and
 * outputs as nvfp4_quantize on the dynamic path (no calibrated amax) and
 * needs no workspace: its scratch -- the amax pass's partial maxima, at most
 * NVQ_NOALLOC_MAX_PARTIALS 32-bit words (4 KB) -- is a static array inside
 * the library, resident on every GPU that loads the library until the
 * process exits.  It allocates nothing and calls no allocating routine.
 *
 *   Same arguments, layouts, arithmetic and results as nvfp4_quantize with
 *   calib_amax == NULL (bit-identical codes, scales and global scale).
 *   The first call on a device (the current device) looks up the scratch
 *   array's device address; make that first call before any stream capture.
 *   Every call on a device shares the one scratch array: two calls whose
 *   work can overlap on the GPU (different streams, no ordering between
 *   them) race on it and may produce wrong results.  Calls ordered on one
 *   stream are safe.  The scratch keeps the last call's contents; nothing in
 *   it needs to start at zero, because every call rewrites every partial it
 *   reads.
 *   The amax pass sizes its grid to the scratch: one CTA per partial
 *   maximum, never more than NVQ_NOALLOC_MAX_PARTIALS CTAs (each reads more
 *   rows when the tensor is large), so every tensor that the shape contract
 *   admits (rows * K < 2^31) fits; anything larger is NVQ_ERR_SHAPE and
 *   launches nothing.  Errors otherwise as nvfp4_quantize (without a
 *   workspace to check).  The scratch address is looked up once per device,
 *   like the status word: a device reset invalidates it.
 */
#define NVQ_NOALLOC_MAX_PARTIALS 1024
NVQ_API int nvfp4_quantize_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx,
                                   uint8_t* codes, uint8_t* scales, float* global_scale,
                                   nvq_stream_t stream);

/*
 * nvq_probe_convert -- conversion self-test (no counterpart on the pages).
 * Runs the device's FP32 -> E2M1 and FP32 -> E4M3 round-to-nearest-even,
 * saturating conversions that the quantize kernels use on n inputs, so
 * tests can compare them with the CPU oracle on every tie and edge case.
 *   in         n floats (device)
 *   e2m1_out   n bytes (device), code in the low nibble
 *   e4m3_out   n bytes (device)
 */
NVQ_API int nvq_probe_convert(const float* in, int64_t n, uint8_t* e2m1_out, uint8_t* e4m3_out,
                      nvq_stream_t stream);

/*
 * nvq_probe_gelu -- GELU self-test (no counterpart on the pages).  Runs the
 * BF16 GELU of block_scaled_linear_gelu_mxfp8's epilogue (same table, same
 * lookup) on n BF16 bit patterns, so tests can compare all 65536 inputs with
 * the CPU oracle.
 *   in    n BF16 values (device)
 *   out   n BF16 values (device)
 */
NVQ_API int nvq_probe_gelu(const uint16_t* in, int64_t n, uint16_t* out, nvq_stream_t stream);

/*
 * nvq_probe_wait -- bounded-wait self-test (no counterpart on the pages).
 * Launches one thread that waits, with the same bounded wait every GEMM
 * pipeline stage uses, on an mbarrier that nothing arrives on.  After
 * limit_ns of wall time the wait gives up, sets NVQ_STATUS_TIMEOUT in the
 * device status word (read it with nvq_device_status) and the kernel returns
 * normally, so the context stays usable.  Nothing faults, traps or hangs.
 *   limit_ns    the wait's limit, at most 1e9 (else NVQ_ERR_SHAPE)
 *   waited_ns   device pointer to one 64-bit word: the nanoseconds waited
 */
NVQ_API int nvq_probe_wait(uint64_t limit_ns, unsigned long long* waited_ns, nvq_stream_t stream);

/*
 * nvq_debug_build -- 1 in the debug build of this library (libnvq_debug.so,
 * compiled with NVQ_DEBUG), 0 in the normal one (no counterpart on the
 * pages).  In the debug build every kernel checks, before each global
 * access whose address it computes from its indices, that the accessed bytes
 * lie inside the buffer the call passed (its extent follows from the call's
 * sizes: rows, K, pitches, tile counts).  A failed check sets
 * NVQ_STATUS_BOUNDS in the device status word and skips the access: a store
 * writes nothing, a load reads zeros, and a skipped bulk copy into a
 * pipeline stage is counted on the stage's barrier without data, so no wait
 * runs out because of it.  Nothing traps.  Results are otherwise identical
 * to the normal build's.  The normal build contains no checks.
 */
NVQ_API int nvq_debug_build(void);

/*
 * nvq_probe_bounds -- bounds-check self-test (no counterpart on the pages).
 * Launches one kernel that evaluates one failing bounds check and makes no
 * memory access.  In the debug build the device status word then holds
 * NVQ_STATUS_BOUNDS (read it with nvq_device_status); in the normal build it
 * stays clean.
 */
NVQ_API int nvq_probe_bounds(nvq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVQ_H */

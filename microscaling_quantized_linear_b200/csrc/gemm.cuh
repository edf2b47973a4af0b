// gemm.cuh -- block-scaled GEMM on the sm_100a 5th-generation tensor cores.
//
//   D[M, N] = bf16( alpha * A[M, K] . B[N, K]^T + bias[N] )
//
// A and B are quantized operands (NVFP4: E2M1 codes + E4M3 scales per 16 of
// K; MXFP8: E4M3 codes + E8M0 scales per 32 of K), both K-major ("TN").
// The tensor core applies the block scales itself (tcgen05.mma
// kind::mxf4nvf4 / kind::mxf8f6f4 with .block_scale), so no dequantized copy
// of either operand ever exists (page "NVIDIA Blackwell平台FP4量化技术解析与图像
// 生成优化", section 3.1: FP4 decoded to BF16 inside the SM).
//
// Structure: one persistent CTA per SM, 12-13 warps, output tiles 128 x BN.
//   warp 0  TMA producer: per pipeline stage one 128 x 128-byte tile of A,
//           one BN x 128-byte tile of B (tensor maps, 128-byte swizzle), and
//           the matching 512-byte scale tiles (plain bulk copies: the global
//           128x4 tile order is exactly what tensor memory wants).
//   warp 1  allocates tensor memory; one lane issues the MMAs into an FP32
//           accumulator in tensor memory; tcgen05.commit frees the stage.
//           With two accumulators (BN = 128 or 192) the MMAs of tile i+1 run
//           while the epilogue drains tile i.
//   warps 10+ scale-factor copy warps, one per 128-row block of scales of a
//           stage (A, then B): tcgen05.cp into a tensor-memory scale slot.
//           Each copy instruction occupies its issuing thread for ~100
//           cycles while the MMA warp's instructions run in parallel, so the
//           copies are spread over several warps and kept off the MMA warp.
//   warps 2-9  epilogue, two warps per tensor-memory lane quarter: tensor
//           memory -> registers (tcgen05.ld), scale by alpha, add bias,
//           round to BF16, release the accumulator, then stage 32 x 32
//           sub-tiles in 64-byte-swizzled shared memory for TMA stores.
// At a short M the same kernel (SPLITK) runs one cluster of CTAs per output
// tile instead, each CTA over a share of K, the partial sums added through
// distributed shared memory (see bsgemm_kernel).
// Every mbarrier wait is bounded in wall time; a wait that gives up sets the
// status word and an abort flag that releases the other roles.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "gelu.cuh"
#include "ptx.cuh"
#include "quantize.cuh"

namespace nvq {

// Limit of the waits with which a CTA drains its own in-flight copies and
// tensor-core work before it exits.  The pipeline waits take theirs from
// GemmParams::wait_ns (the same 4 s unless a test shortens it).
constexpr uint64_t kWaitLimitNs = 4000000000ull;   // 4 s per wait
// Warp roles: 0 TMA producer, 1 MMA issuer, 2..9 epilogue (two warps per
// tensor-memory lane quarter, each owning half of the tile's columns),
// 10.. scale-factor copy warps.
constexpr int kEpiWarps = 8;
constexpr int kFirstSfWarp = 2 + kEpiWarps;

// alpha * acc + bias for 32 accumulator columns (c .. c+31 of the tile),
// rounded to BF16 pairs; products as packed f32x2 multiplies (RNE per lane).
// Bias entries at tile columns >= nlim (past N) are not read.
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&r)[32], float alpha, const __nv_bfloat16* bias_tile,
                                               int c, int nlim, uint32_t (&packed)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float2 v = f32x2_mul(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]), alpha);
        if (bias_tile) {
            const int n = c + 2 * e;
            if (n + 1 < nlim) {
                const __nv_bfloat162 bb = *reinterpret_cast<const __nv_bfloat162*>(bias_tile + n);
                v.x = __fadd_rn(v.x, __bfloat162float(bb.x));
                v.y = __fadd_rn(v.y, __bfloat162float(bb.y));
            } else if (n < nlim) {
                v.x = __fadd_rn(v.x, __bfloat162float(bias_tile[n]));
            }
        }
        const __nv_bfloat162 o = __floats2bfloat162_rn(v.x, v.y);
        packed[e] = *reinterpret_cast<const uint32_t*>(&o);
    }
}

// Drains one 32-row x BN/2-column share of an accumulator.  Tensor-memory
// chunks are read two at a time; every pair but the last is converted to
// BF16 before the next is read, and the accumulator is released as soon as
// the last pair is in registers (its conversion follows the release), so the
// MMAs of the next tile wait for the loads and one conversion only.  The
// BF16 sub-tiles are then written via the warp's 64-byte-swizzled staging
// buffer and TMA stores.
// Output of the epilogue that quantizes for the next layer (EPI 1):
// GELU of the BF16 result, then MXFP8 (E4M3 elements, OCP floor exponent)
// per 32 consecutive columns, the codes dense [m, n] and the E8M0 scales in
// the 128x4 tile order of an [m, n/32] scale matrix (rows m .. m_pad - 1 of
// the last row tile zero).
struct EpiQuant {
    uint8_t* codes;
    uint8_t* sf;
    uint32_t n, m, m_pad;
    unsigned int* status;   // bounds checks of the debug build
};

template <int BN, int EPI>
__device__ __forceinline__ void drain_accumulator(uint32_t tmem_acc_q, int half, int lane, float alpha,
                                                  const __nv_bfloat16* bias_tile, uint8_t* staging,
                                                  const CUtensorMap* tmap_d, int32_t row0, uint32_t n0,
                                                  int nlim, uint32_t release_bar, bool release_remote,
                                                  const EpiQuant& eq, const uint16_t* gelu_tab) {
    constexpr int NC = BN / 64;                          // 32-column chunks per warp
    constexpr int JL = (NC - 1) & ~1;                    // first chunk of the last pair
    const int c0 = half * (BN / 2);
    uint32_t packed[NC][16];
#pragma unroll
    for (int j = 0; j < JL; j += 2) {
        uint32_t r0[32], r1[32];
        tc_ld_32x32b_x32(tmem_acc_q + c0 + 32 * j, r0);
        tc_ld_32x32b_x32(tmem_acc_q + c0 + 32 * (j + 1), r1);
        tc_wait_ld();
        epilogue_chunk(r0, alpha, bias_tile, c0 + 32 * j, nlim, packed[j]);
        epilogue_chunk(r1, alpha, bias_tile, c0 + 32 * (j + 1), nlim, packed[j + 1]);
    }
    {
        uint32_t r0[32], r1[32];
        tc_ld_32x32b_x32(tmem_acc_q + c0 + 32 * JL, r0);
        if (JL + 1 < NC) tc_ld_32x32b_x32(tmem_acc_q + c0 + 32 * (JL + 1), r1);
        tc_wait_ld();
        // The release signal carries no data: tcgen05.wait::ld has returned,
        // so every load of this share has read the accumulator before the
        // arrive executes, and the MMA lane only has to be ordered after that
        // (its tcgen05.fence::after_thread_sync).  Hence a relaxed arrive; a
        // release arrive at cluster scope stalled the warp for about 1,700
        // cycles.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if (release_remote) mbar_arrive_relaxed_cluster(release_bar);
            else mbar_arrive_relaxed(release_bar);
        }
        epilogue_chunk(r0, alpha, bias_tile, c0 + 32 * JL, nlim, packed[JL]);
        if (JL + 1 < NC) epilogue_chunk(r1, alpha, bias_tile, c0 + 32 * (JL + 1), nlim, packed[JL + 1 < NC ? JL + 1 : JL]);
    }
    if constexpr (EPI == 1) {
        // One thread = one row; each 32-column chunk is one MXFP8 block.  The
        // NC scale bytes of the row's share are consecutive in the tile order
        // (the share starts at a multiple of 4 blocks for BN 256, of 2 for
        // BN 128), so they go out in one store.
        static_assert(NC == 2 || NC == 4, "MXFP8 epilogue: 128- or 256-wide tiles");
        const uint32_t row = (uint32_t)row0 + (uint32_t)lane;
        const uint32_t cfirst = n0 + (uint32_t)c0;
        if (cfirst >= eq.n || row >= eq.m_pad) return;
        uint32_t scw = 0;
        if (row < eq.m) {
            uint8_t* dst = eq.codes + (size_t)row * eq.n + cfirst;
#pragma unroll
            for (int j = 0; j < NC; ++j) {
                uint32_t q[8];
                gelu_bf16x32(packed[j], gelu_tab);
                scw |= mx_block<0, 0>(packed[j], q) << (8 * j);
                if (in_bounds((uint64_t)row * eq.n + cfirst + 32 * j, 32, (uint64_t)eq.m * eq.n, eq.status)) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * j);
                    d4[0] = make_uint4(q[0], q[1], q[2], q[3]);
                    d4[1] = make_uint4(q[4], q[5], q[6], q[7]);
                }
            }
        }
        const uint32_t so = sf_tile_offset(row, cfirst / 32, eq.n / 128);
        if (!in_bounds(so, NC, sf_extent(eq.m_pad, eq.n / 128), eq.status)) return;
        uint8_t* sfp = eq.sf + so;
        if (NC == 4) *reinterpret_cast<uint32_t*>(sfp) = scw;
        else *reinterpret_cast<uint16_t*>(sfp) = (uint16_t)scw;
        return;
    }
    const uint32_t swz = (uint32_t)((lane >> 1) & 3);     // 64-byte swizzle of this thread's row
#pragma unroll
    for (int j = 0; j < NC; ++j) {
        if (lane == 0) bulk_wait_group_read<0>();         // the previous store has read the buffer
        __syncwarp();
#pragma unroll
        for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4*>(staging + lane * 64 + 16 * ((uint32_t)v ^ swz)) =
                make_uint4(packed[j][4 * v], packed[j][4 * v + 1], packed[j][4 * v + 2], packed[j][4 * v + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmap_d, smem_u32(staging), (int32_t)(n0 + c0 + 32 * j), row0);
            bulk_commit_group();
        }
    }
}

// Rows of the output that the split-K kernel takes (one short row block).
constexpr uint32_t kSplitKRows = 32;

// SPLIT_ROWS: 0 for the persistent kernel; 16 or 32 for the split-K kernel
// at M <= SPLIT_ROWS (the rows its receive area holds).
template <int FMT, int BN_, int SPLIT_ROWS = 0, bool FUSEQ = false>
struct GemmCfg {
    static constexpr bool SPLITK = SPLIT_ROWS > 0;
    // fused short-M path: d6 and rtab tables (128 floats each) and a
    // reduction slot per epilogue warp, after the barriers
    static constexpr int SCRATCH_BYTES = FUSEQ ? 1280 : 0;
    static constexpr int BM = 128;
    static constexpr int BN = BN_;
    static constexpr int KBYTES = 128;                       // bytes of K per stage (one swizzle atom)
    static constexpr int BK = FMT == 0 ? 256 : 128;          // K elements per stage
    static constexpr int MMA_K = FMT == 0 ? 64 : 32;         // K elements per instruction
    static constexpr int KSTEPS = BK / MMA_K;                // 4 instructions per stage
    static constexpr int MMA_K_BYTES = KBYTES / KSTEPS;      // 32
    static constexpr int SF_BLOCK = FMT == 0 ? 16 : 32;
    static constexpr int SF_ATOMS = BK / SF_BLOCK / 4;       // 128x4 scale tiles per 128 rows per stage
    static constexpr int SFB_H = BN == 128 ? 1 : 2;          // 128-row scale tiles spanned by a B tile
    // Split-K stages only the activation's first 32 rows (M <= 32; the box
    // past M reads zeros).  The MMA still spans 128 rows: its rows 32..127
    // read the stage's B tile, and those accumulator rows are never read.
    static constexpr int A_ROWS = SPLITK ? 32 : BM;
    static constexpr int A_BYTES = A_ROWS * KBYTES;
    static constexpr int B_BYTES = BN * KBYTES;
    static constexpr int SFA_BYTES = SF_ATOMS * 512;
    static constexpr int SFB_BYTES = SFB_H * SF_ATOMS * 512;
    static constexpr int AB_BYTES = A_BYTES + B_BYTES;       // per stage, on full[s]
    static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;   // per stage, on sfdata[s]
    static constexpr int STAGE_BYTES = (AB_BYTES + SF_BYTES + 1023) / 1024 * 1024;
    static constexpr int OFF_B = A_BYTES;
    static constexpr int OFF_SFA = A_BYTES + B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + SFA_BYTES;
    // epilogue staging: 8 warps x (32 rows x 64 bytes)
    static constexpr int EPI_BUF_BYTES = 32 * 64;
    static constexpr int EPI_BYTES = kEpiWarps * EPI_BUF_BYTES;
    // split-K: the receive area for the partial sums that the cluster's CTAs
    // push here (SPLIT_ROWS rows of BN FP32 values, plus the padding of the
    // per-rank slots) takes the place of the staging area, which that kernel
    // does not use
    static constexpr int RECV_BYTES = SPLITK ? SPLIT_ROWS * BN * 4 + 2048 : 0;
    static constexpr int EPI_AREA = SPLITK ? RECV_BYTES : EPI_BYTES;
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int FIXED_BYTES = 1024 /*align*/ + 512 /*barriers*/ + EPI_AREA + SCRATCH_BYTES;
    // tensor-memory columns: accumulator(s), then scale factors of A and B
    static constexpr int SFA_COLS = FMT == 0 ? 4 * KSTEPS : 4;
    static constexpr int SFB_COLS_PER_MMA = 4 * SFB_H;
    static constexpr int SFB_COLS = FMT == 0 ? SFB_COLS_PER_MMA * KSTEPS : SFB_COLS_PER_MMA;
    // Each pipeline stage owns one tensor-memory scale slot (SF_COLS columns,
    // filled by the copy warps ahead of the MMAs), so the stage count is
    // bounded by shared memory and by the columns left beside the
    // accumulator(s); two accumulators only when at least 4 slots remain.
    static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED_BYTES) / STAGE_BYTES;
    // A split-K CTA owns one tile: one accumulator, and up to 8 stages (its
    // share of K is short, so the more of it in flight at once the better).
    static constexpr int ACC_BUFS = SPLITK ? 1 : ((512 - 2 * BN) / SF_COLS >= 4 ? 2 : 1);
    static constexpr int SLOTS_FIT = (512 - ACC_BUFS * BN) / SF_COLS;
    static constexpr int STAGES_MIN2 = STAGES_FIT < SLOTS_FIT ? STAGES_FIT : SLOTS_FIT;
    static constexpr int STAGES_CAP = SPLITK ? 8 : 6;
    static constexpr int STAGES = STAGES_MIN2 > STAGES_CAP ? STAGES_CAP : STAGES_MIN2;
    static constexpr int OFF_EPI = STAGES * STAGE_BYTES;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED_BYTES;
    static constexpr int TM_SF = ACC_BUFS * BN;            // slot s at TM_SF + s * SF_COLS
    static constexpr int TM_USED = ACC_BUFS * BN + STAGES * SF_COLS;
    static constexpr int TM_COLS = TM_USED <= 256 ? 256 : 512;
    // copy jobs per stage: the A scales, then each 128-row block of B scales;
    // one warp per job (a tcgen05.cp takes ~100 cycles to issue, so the jobs
    // run in parallel warps, off the MMA warp's path)
    static constexpr int SF_WARPS = 1 + SFB_H;
    static constexpr int THREADS = 32 * (kFirstSfWarp + SF_WARPS);
    // instruction descriptor: A/B format (E2M1 = 1 for mxf4nvf4, E4M3 = 0 for
    // mxf8f6f4) in bits 7-9 / 10-12, K-major A and B, N >> 3 in bits 17-22,
    // scale format (0 = UE4M3, 1 = UE8M0) in bit 23, M >> 4 in bits 24-28.
    static constexpr uint32_t IDESC =
        (FMT != 1 ? (1u << 7) | (1u << 10) : 0u) |   // A, B type: E2M1 (NVFP4) / E5M2 (FMT 2); 0 = E4M3
        ((uint32_t)(BN >> 3) << 17) |
        (FMT == 0 ? 0u : (1u << 23)) |
        ((uint32_t)(BM >> 4) << 24);
    static_assert(BN == 128 || BN == 192 || BN == 256, "tile width");
    static_assert(TM_USED <= 512, "tensor memory overflow");
    static_assert(STAGES >= 3, "too few pipeline stages");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory overflow");
};

struct GemmParams {
    union {
        const uint8_t* sfa;
        const uint16_t* x;       // fused short-M path: the BF16 activation [m_total, K], pitch ldx
    };
    const uint8_t* sfb;
    union {
        const float* a_global;
        float* a_global_out;     // fused short-M path: where the activation's global scale goes (or null)
    };
    const float* b_global;
    const __nv_bfloat16* bias;
    unsigned int* status;
    uint32_t num_m_blocks, num_n_blocks, num_k_tiles;
    uint32_t sf_ctiles;          // (K / SF_BLOCK) / 4: scale tiles per 128 rows
    uint32_t n_total;            // N: output columns past it are neither stored nor biased
    uint32_t sfa_rtiles, sfb_rtiles;   // 128-row scale tiles in the A and B scale buffers
    // quantizing epilogue (EPI 1) only: MXFP8 codes [m_total, n_total] and
    // scales of GELU(D), m_pad = m_total rounded up to 128.  Fused short-M
    // path: the activation's NVFP4 codes and scales (either may be null)
    uint8_t* q_codes;
    uint8_t* q_sf;
    uint32_t m_total;
    union {
        uint32_t m_pad;
        uint32_t ldx;            // fused short-M path: the activation's row pitch in elements
    };
    // split-K kernels only: CTAs per cluster, each summing one contiguous
    // share of the K tiles of the cluster's output tile; D is stored with
    // plain stores (out, ldo elements per row)
    uint32_t k_split = 1;
    __nv_bfloat16* out = nullptr;
    uint32_t ldo = 0;
    // limit of every pipeline wait in ns (a role that gives up sets the
    // status word and the abort flag); the drain waits keep kWaitLimitNs.
    // 32 bits, in the struct's tail padding: the kernels' code is the same
    // size as without it.
    uint32_t wait_ns = (uint32_t)kWaitLimitNs;
};
static_assert(sizeof(GemmParams) == 128, "GemmParams keeps its 128 bytes");

// Split-K exchange for one output tile of at most kSplitKRows rows.  The
// tile's 4-column groups are numbered row-major (group idx = row * BN/4 +
// column/4) and cut into `split` contiguous shares of `per` groups; CTA rank
// r of the cluster finishes share r.  Every CTA pushes its FP32 partial of
// share r into slot (its own rank) of CTA r's receive area; a slot covers
// the share's aligned groups of eight, with group idx stored at position
// (idx & ~7) | ((idx ^ row) & 7) from the share's first aligned group, so
// that the pushes of one row per lane hit all banks.
struct SplitShares {
    uint32_t total, per, slot;   // groups in the tile, per share, per slot (16 bytes each)
};

template <int BN>
__device__ __forceinline__ SplitShares split_shares(uint32_t rows, uint32_t split) {
    SplitShares sh;
    sh.total = rows * (BN / 4);
    sh.per = (sh.total + split - 1) / split;
    sh.slot = ((sh.per + 7) & ~7u) + 8;
    return sh;
}

// Position (in 16-byte groups) of group idx, of tile row `row`, within its
// slot; b8 = the owner's first group rounded down to a multiple of eight.
__device__ __forceinline__ uint32_t split_pos(uint32_t idx, uint32_t row, uint32_t b8) {
    return ((idx & ~7u) | ((idx ^ row) & 7u)) - b8;
}

// CTA `rank` finishes its share from its receive area (every slot filled):
// the partials summed in rank order, times alpha, plus bias, rounded to BF16
// and stored.  Groups at columns >= n_total are not stored.
template <int BN>
__device__ __forceinline__ void splitk_finish(uint32_t recv, const SplitShares& sh, uint32_t rank, uint32_t split,
                                              uint32_t n0, uint32_t n_total, float alpha,
                                              const __nv_bfloat16* bias, __nv_bfloat16* out, uint32_t ldo,
                                              uint32_t tid, uint32_t nthreads, unsigned int* status) {
    constexpr uint32_t F = BN / 4;
    const uint64_t out_elems = pitched_extent(sh.total / F, n_total, ldo);
    const uint32_t begin = rank * sh.per;
    const uint32_t end = min(sh.total, begin + sh.per);
    for (uint32_t idx = begin + tid; idx < end; idx += nthreads) {
        const uint32_t row = idx / F, n = n0 + 4 * (idx % F);
        const uint32_t off = recv + split_pos(idx, row, begin & ~7u) * 16;
        float4 acc = ld_shared_f4(off);
        for (uint32_t r = 1; r < split; ++r) {
            const float4 v = ld_shared_f4(off + r * sh.slot * 16);
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
        }
        if (n >= n_total) continue;
        float o[4] = {__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha), __fmul_rn(acc.z, alpha),
                      __fmul_rn(acc.w, alpha)};
        if (bias) {
            const __nv_bfloat162 b01 = *reinterpret_cast<const __nv_bfloat162*>(bias + n);
            const __nv_bfloat162 b23 = *reinterpret_cast<const __nv_bfloat162*>(bias + n + 2);
            o[0] = __fadd_rn(o[0], __bfloat162float(b01.x));
            o[1] = __fadd_rn(o[1], __bfloat162float(b01.y));
            o[2] = __fadd_rn(o[2], __bfloat162float(b23.x));
            o[3] = __fadd_rn(o[3], __bfloat162float(b23.y));
        }
        const __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
        if (in_bounds((uint64_t)row * ldo + n, 4, out_elems, status))
            *reinterpret_cast<uint2*>(out + (size_t)row * ldo + n) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
    }
}

// Fused short-M path: the activation's dynamic NVFP4 quantization inside the
// split-K GEMM, by the epilogue warps (idle until the accumulator is ready)
// while the B tiles load.  For more than kShortAmaxRows rows every CTA takes
// the max |x| of its own K tiles' columns and sends it with st.async to every
// CTA of its cluster (the cluster's shares cover K, so each CTA then holds
// the tensor's amax; the receiving mbarrier expects one 4-byte value per
// CTA); for fewer rows each CTA reads the whole activation, which is cheaper
// than the exchange's latency.  Then every CTA quantizes the
// rows of its own K tiles with the same arithmetic as the quantize kernels,
// writing the E2M1 codes into its stages' A tiles (the 128-byte swizzle the
// MMA reads: 16-byte chunk c of row r at chunk c ^ (r % 8)) and the E4M3
// scales into their A scale tiles (128x4 order), then counts one arrival per
// stage on full[] and sfdata[] once the tiles are written.  Rows M..31 of
// the A tiles are left as they are: they only feed accumulator rows that
// nothing reads.  With q_codes / q_sf / a_global_out set, the CTAs of the
// first cluster also write the codes, scales (padding rows zero) and g_dec,
// exactly as nvfp4_quantize would.  With the exchange (more than
// kShortAmaxRows rows) this waits on the cluster barrier's first phase before
// the first st.async, and the caller does not wait on it again.  If the wait for the cluster's maxima gives up, the amax comes
// from the whole activation read here (exact all the same) and the status
// word records the timeout.  Returns g_dec.  Threads tid 0..255.
constexpr uint32_t kShortAmaxRows = 4;

template <typename C>
__device__ __forceinline__ float fused_quantize_a(const GemmParams& p, uint8_t* smem, float* scratch,
                                                  uint32_t kt_begin, uint32_t kt_end, bool first_cluster,
                                                  uint32_t tid, uint32_t full0, uint32_t sfdata0, uint32_t amaxbar,
                                                  uint32_t rank, const volatile int* abort_flag,
                                                  bool& amax_got) {
    constexpr uint32_t NT = 32 * kEpiWarps;
    float* d6 = scratch;
    float* rtab = scratch + 128;
    uint32_t* red = reinterpret_cast<uint32_t*>(scratch + 256);
    uint32_t* slots = reinterpret_cast<uint32_t*>(scratch + 264);      // one per CTA of the cluster
    volatile uint32_t* gave_up = reinterpret_cast<volatile uint32_t*>(scratch + 274);
    const uint32_t rows = p.m_total;
    const uint32_t K = p.num_k_tiles * 256u;
    const uint64_t x_elems = pitched_extent(rows, K, p.ldx);
    // max |x| over this CTA's K tiles (or the whole tensor): batches of 8
    // independent 16-byte loads per thread, all issued before any is used
    const bool shared_amax = rows > kShortAmaxRows;
    const uint32_t vps = shared_amax ? (kt_end - kt_begin) * 32 : K / 8;   // 16-byte vectors per row read
    const uint32_t c0 = shared_amax ? kt_begin * 32 : 0;
    uint32_t m2 = 0;
    for (uint32_t i0 = tid; i0 < rows * vps; i0 += 8 * NT) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t i = i0 + u * NT, r = i / vps, c = c0 + (i - r * vps);
            v[u] = (i < rows * vps && in_bounds((uint64_t)r * p.ldx + c * 8, 8, x_elems, p.status))
                       ? __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)r * p.ldx) + c)
                       : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) m2 = absmax2(absmax2(absmax2(absmax2(m2, v[u].x), v[u].y), v[u].z), v[u].w);
    }
    uint32_t m = __reduce_max_sync(0xFFFFFFFFu, fold2(m2));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    if (tid < 128) d6[tid] = __fdiv_rn((float)(128 + tid), 6.0f);
    if (tid == 0) *gave_up = 0;
    named_barrier_sync(3, NT);
    m = 0;
    if (!shared_amax) {
#pragma unroll
        for (int w = 0; w < kEpiWarps; ++w) m = max(m, red[w]);
        amax_got = true;
    } else {
    cluster_wait();                           // every CTA's amax barrier is initialised
    if (tid == 0) {
#pragma unroll
        for (int w = 0; w < kEpiWarps; ++w) m = max(m, red[w]);
        for (uint32_t r = 0; r < p.k_split; ++r)
            st_async_u32(mapa_shared(smem_u32(slots + rank), r), m, mapa_shared(amaxbar, r));
    }
    if (!mbar_wait_bounded_cluster(amaxbar, 0, abort_flag, p.wait_ns)) *gave_up = 1;
    named_barrier_sync(3, NT);                // one decision for all: the branches below hold barriers
    amax_got = *gave_up == 0;
    m = 0;
    if (amax_got) {
        for (uint32_t r = 0; r < p.k_split; ++r) m = max(m, slots[r]);
    } else {
        // a CTA of the cluster did not send: the amax from the whole tensor
        if (tid == 0) atomicOr(p.status, kStatusTimeout);
        const uint32_t vpr = K / 8;
        uint32_t a2 = 0;
        for (uint32_t i = tid; i < rows * vpr; i += NT) {
            const uint32_t r = i / vpr, c = i - r * vpr;
            if (in_bounds((uint64_t)r * p.ldx + c * 8, 8, x_elems, p.status)) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x + (size_t)r * p.ldx) + c);
                a2 = absmax2(absmax2(absmax2(absmax2(a2, v.x), v.y), v.z), v.w);
            }
        }
        named_barrier_sync(3, NT);            // everyone has read red[] above
        const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, fold2(a2));
        if ((tid & 31) == 0) red[tid >> 5] = wm;
        named_barrier_sync(3, NT);
#pragma unroll
        for (int w = 0; w < kEpiWarps; ++w) m = max(m, red[w]);
    }
    }
    if (m >= 0x7F80u && first_cluster && cluster_ctarank() == 0 && tid == 0) atomicOr(p.status, kStatusNonfinite);
    const float amax = __uint_as_float(m << 16);
    const float g_enc = encode_scale(amax);
    const float g_dec = decode_scale(amax);
    if (tid >= 128) {
        const uint32_t c = tid - 128;
        rtab[c] = c ? __fdiv_rn(g_enc, e4m3_decode_pos(c)) : 0.0f;
    }
    named_barrier_sync(3, NT);
    // this CTA's K tiles: stage s holds K tile kt_begin + s
    const uint32_t share = kt_end - kt_begin;
    const uint32_t ctiles = K / 64;
    // two blocks per thread per iteration, both loaded before either is used
    const uint32_t nblocks = rows * share * 16;
    for (uint32_t u0 = tid; u0 < nblocks; u0 += 2 * NT) {
        uint4 v[4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t u = u0 + h * NT;
            const uint32_t r = u / (share * 16), rem = u - r * (share * 16);
            const uint32_t col = (kt_begin + (rem >> 4)) * 256 + (rem & 15u) * 16;
            const bool ld = u < nblocks && in_bounds((uint64_t)r * p.ldx + col, 16, x_elems, p.status);
            const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)r * p.ldx + col);
            v[2 * h] = ld ? __ldg(src) : make_uint4(0, 0, 0, 0);
            v[2 * h + 1] = ld ? __ldg(src + 1) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
        const uint32_t u = u0 + h * NT;
        if (u >= nblocks) break;
        const uint32_t r = u / (share * 16), rem = u - r * (share * 16);
        const uint32_t st = rem >> 4, b = rem & 15u, kt = kt_begin + st;
        const uint32_t col = kt * 256 + b * 16;
        const uint32_t w[8] = {v[2 * h].x, v[2 * h].y, v[2 * h].z, v[2 * h].w,
                               v[2 * h + 1].x, v[2 * h + 1].y, v[2 * h + 1].z, v[2 * h + 1].w};
        uint32_t lo, hi;
        const uint32_t sc = nvfp4_block(block16_max(w), w, g_enc, d6, rtab, lo, hi);
        const uint32_t stage = smem_u32(smem + st * C::STAGE_BYTES);
        const uint32_t chunk = b >> 1;
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};"
                     :: "r"(stage + r * 128 + ((chunk ^ (r & 7u)) << 4) + ((b & 1u) << 3)), "r"(lo), "r"(hi)
                     : "memory");
        asm volatile("st.shared.u8 [%0], %1;"
                     :: "r"(stage + C::OFF_SFA + (b >> 2) * 512 + r * 16 + (b & 3u)), "r"(sc) : "memory");
        if (first_cluster) {
            if (p.q_codes && in_bounds((uint64_t)r * (K / 2) + col / 2, 8, (uint64_t)rows * (K / 2), p.status))
                *reinterpret_cast<uint2*>(p.q_codes + (size_t)r * (K / 2) + col / 2) = make_uint2(lo, hi);
            const uint32_t so = sf_tile_offset(r, col / 16, ctiles);
            if (p.q_sf && in_bounds(so, 1, sf_extent(rows, ctiles), p.status)) p.q_sf[so] = (uint8_t)sc;
        }
        }
    }
    if (first_cluster && cluster_ctarank() == 0) {
        if (p.q_sf) zero_pad_scale_rows(p.q_sf, rows, ctiles, tid, NT, p.status);
        if (p.a_global_out && tid == 0) *p.a_global_out = g_dec;
    }
    fence_proxy_async_smem();                 // the tiles, to the tensor core and the scale copies
    named_barrier_sync(3, NT);
    if (tid == 0)
        for (uint32_t st = 0; st < share; ++st) {
            mbar_arrive(full0 + 8 * st);
            mbar_arrive(sfdata0 + 8 * st);
        }
    return g_dec;
}

// Scale-factor copy warp `job` (0: A scales, 1..SFB_H: B scale row block
// job-1) for one pipeline stage: shared memory -> tensor-memory slot.
template <typename C, bool PAIR>
__device__ __forceinline__ void sf_copy_job(int job, uint32_t st, uint32_t sf_slot) {
    if (job == 0) {
#pragma unroll
        for (int a = 0; a < C::SF_ATOMS; ++a) {
            const uint64_t d = smem_desc(st + C::OFF_SFA + 512 * a, 16, 128, 0);
            if (PAIR) tc_cp_pair_32x128b_warpx4(sf_slot + 4 * a, d);
            else tc_cp_32x128b_warpx4(sf_slot + 4 * a, d);
        }
    } else {
        const int h = job - 1;
#pragma unroll
        for (int a = 0; a < C::SF_ATOMS; ++a) {
            const uint64_t d = smem_desc(st + C::OFF_SFB + h * C::SF_ATOMS * 512 + 512 * a, 16, 128, 0);
            const uint32_t t = sf_slot + C::SFA_COLS + C::SFB_COLS_PER_MMA * a + 4 * h;
            if (PAIR) tc_cp_pair_32x128b_warpx4(t, d);
            else tc_cp_32x128b_warpx4(t, d);
        }
    }
}

// EPI 0: D = bf16(alpha A.B^T + bias) through tmap_d.  EPI 1: D is not
// written; GELU(D) leaves as MXFP8 codes and scales (EpiQuant), and the
// epilogue warps' staging area holds the GELU table instead.
// SPLIT_ROWS > 0 (EPI 0, M <= SPLIT_ROWS): the grid is one cluster of p.k_split
// CTAs per output tile.  CTA rank r of a cluster runs the mainloop over the
// r-th contiguous share of the K tiles into its own accumulator.  Its
// epilogue warps read the accumulator once and lay each share of it out in
// the CTA's free pipeline stages, and one bulk copy per share sends it into
// the receive area of the CTA that finishes that share; every CTA then waits
// on one mbarrier for the copies of the whole cluster and finishes its share
// (splitk_finish).  A cluster barrier split into arrive and wait guards the
// exchange: its first phase makes the receive barriers' initialisation
// visible before any copy, its second keeps every CTA alive until every
// CTA's copies have landed.  Before it waits for the previous grid, one
// epilogue warp asks L2 for the CTA's whole B share, so at a short M the
// weight stream overlaps the producer of A.
// FUSEQ (NVFP4 split-K only): the activation arrives as BF16 (p.x) and is
// quantized inside the kernel (fused_quantize_a); tmap_a is not used.
template <int FMT, int BN, int EPI, int SPLIT_ROWS = 0, bool FUSEQ = false>
__global__ void __launch_bounds__(GemmCfg<FMT, BN>::THREADS, 1)
bsgemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
              const __grid_constant__ CUtensorMap tmap_d, const GemmParams p) {
    using C = GemmCfg<FMT, BN, SPLIT_ROWS, FUSEQ>;
    constexpr bool SPLITK = SPLIT_ROWS > 0;
    static_assert(EPI == 0 || kGeluTabBytes <= C::EPI_BYTES, "GELU table must fit the staging area");
    static_assert(!SPLITK || EPI == 0, "split-K: plain epilogue only");
    static_assert(!FUSEQ || (SPLITK && FMT == 0), "fused activation quantization: NVFP4 split-K only");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_EPI + C::EPI_AREA);
    // The MMA lane waits once per stage (the tensor pipe holds little more
    // than one MMA in flight, so its barrier checks are idle pipe time):
    //   full[s]   A and B tiles landed (tx) + the copy warps' commits of the
    //             stage's scales into tensor-memory slot s
    //   sfdata[s] the stage's scale tiles landed (tx): the copy warps' wait
    //   empty[s]  the stage's MMAs completed: frees shared-memory stage s
    //             and scale slot s
    const uint32_t full0 = smem_u32(bars);                 // [STAGES]
    const uint32_t empty0 = full0 + 8 * C::STAGES;         // [STAGES]
    const uint32_t sfdata0 = empty0 + 8 * C::STAGES;       // [STAGES]
    const uint32_t tfull0 = sfdata0 + 8 * C::STAGES;       // [2]  MMA -> epilogue
    const uint32_t tempty0 = tfull0 + 8 * 2;               // [2]  epilogue -> MMA
    const uint32_t drain = tempty0 + 8 * 2;                // MMA warp's own completion
    const uint32_t sfdrain = drain + 8;                    // copy warps' own completion
    const uint32_t recvbar = sfdrain + 8;                  // split-K: the cluster's pushes landed (tx)
    const uint32_t amaxbar = smem_u32(bars + 64) + 1088;   // fused short-M: the cluster's partial maxima (tx)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 3 * C::STAGES + 7);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* never = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1 + C::SF_WARPS + (FUSEQ ? 1 : 0));
            mbar_init(empty0 + 8 * s, 1);
            mbar_init(sfdata0 + 8 * s, FUSEQ ? 2 : 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_init(sfdrain, C::SF_WARPS);
        if (FUSEQ) {
            mbar_init(amaxbar, 1);
            if (p.m_total > kShortAmaxRows) mbar_arrive_expect_tx(amaxbar, p.k_split * 4);
        }
        if (SPLITK) {
            // expects one whole slot from every CTA of the cluster, its own included
            const SplitShares sh = split_shares<BN>(min(p.m_total, (uint32_t)SPLIT_ROWS), p.k_split);
            mbar_init(recvbar, 1);
            mbar_arrive_expect_tx(recvbar, p.k_split * sh.slot * 16);
        }
        *abort_flag = 0;
        *never = 0;
        fence_mbarrier_init();
    }
    // Tiles and K tiles of this CTA: persistent CTAs stride over the tiles
    // with all K tiles each; a split-K cluster owns one tile and CTA rank
    // ks of it the K tiles [kt_begin, kt_end).
    const uint32_t num_tiles = p.num_m_blocks * p.num_n_blocks;
    const uint32_t ks = SPLITK ? cluster_ctarank() : 0;
    const uint32_t tile_first = SPLITK ? blockIdx.x / p.k_split : blockIdx.x;
    const uint32_t tile_step = SPLITK ? num_tiles : gridDim.x;
    const uint32_t kt_begin = SPLITK ? ks * p.num_k_tiles / p.k_split : 0;
    const uint32_t kt_end = SPLITK ? (ks + 1) * p.num_k_tiles / p.k_split : p.num_k_tiles;
    if (warp == 0 && lane == 0) {
        if (!FUSEQ) prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
        if (EPI == 0 && !SPLITK) prefetch_tensormap(&tmap_d);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_holder), C::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (SPLITK) cluster_arrive_relaxed();   // this CTA's receive barrier is initialised
    const uint32_t tmem = *tmem_holder;
    bool split_got = true;                  // split-K: this thread's wait for the pushes ended in time
    if (SPLITK && warp == kFirstSfWarp - 1 && lane == 0 && tile_first < num_tiles) {
        // the weight share into L2, from an epilogue warp (idle until the
        // accumulator is ready), so the prologue of the other roles does not
        // wait for the prefetch instructions to issue
        const uint32_t nb = tile_first / p.num_m_blocks;
        const uint32_t a0 = (nb * BN) / 128;
        for (uint32_t kt = kt_begin; kt < kt_end; ++kt) {
            prefetch_l2_tile_2d(&tmap_b, (int32_t)(kt * C::KBYTES), (int32_t)(nb * BN));
#pragma unroll
            for (int h = 0; h < C::SFB_H; ++h) {
                const uint32_t bt = min(a0 + h, p.sfb_rtiles - 1);
                const uint64_t sfb_off = ((uint64_t)bt * p.sf_ctiles + (uint64_t)kt * C::SF_ATOMS) * 512;
                if (in_bounds(sfb_off, C::SF_ATOMS * 512, (uint64_t)p.sfb_rtiles * p.sf_ctiles * 512, p.status))
                    prefetch_l2_bulk(p.sfb + sfb_off, C::SF_ATOMS * 512);
            }
        }
    }
    // everything above overlaps the previous grid; no global data is read
    // or written before it has completed (the split-K prefetch only warms
    // L2, the device's point of coherence).  The next grid in the stream may
    // then launch: its CTAs wait at their own griddepcontrol.wait until this
    // grid has completed, so only its launch latency overlaps this grid.
    griddep_wait();
    griddep_launch();
    const uint32_t total_iters =
        ((num_tiles > tile_first) ? (num_tiles - tile_first + tile_step - 1) / tile_step : 0) * (kt_end - kt_begin);

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = tile_first; tile < num_tiles && ok; tile += tile_step) {
                const uint32_t mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
                const uint32_t a0 = (nb * BN) / 128;             // first 128-row scale tile of B
                for (uint32_t kt = kt_begin; kt < kt_end; ++kt) {
                    const uint32_t s = it % C::STAGES, use = it / C::STAGES;
                    if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t fb = full0 + 8 * s, sb = sfdata0 + 8 * s;
                    // (fused activation quantization: the epilogue warps write
                    // the A tile and its scales, and arrive on both barriers)
                    mbar_arrive_expect_tx(sb, C::SF_BYTES - (FUSEQ ? C::SFA_BYTES : 0));
                    mbar_arrive_expect_tx(fb, C::AB_BYTES - (FUSEQ ? C::A_BYTES : 0));
                    // scale tiles first: the copy warps need them before the MMAs
                    // can run.  Plain bulk copies have no out-of-range fill: a B
                    // tile that runs past N (its rows are not stored) reads the
                    // last scale tile.
                    const uint64_t sfa_off = ((uint64_t)mb * p.sf_ctiles + (uint64_t)kt * C::SF_ATOMS) * 512;
                    if (FUSEQ) {
                    } else if (in_bounds(sfa_off, C::SFA_BYTES, (uint64_t)p.sfa_rtiles * p.sf_ctiles * 512, p.status)) {
                        bulk_load(st + C::OFF_SFA, p.sfa + sfa_off, C::SFA_BYTES, sb);
                    } else {
                        mbar_complete_tx(sb, C::SFA_BYTES);     // counted without data: no wait runs out
                    }
#pragma unroll
                    for (int h = 0; h < C::SFB_H; ++h) {
                        const uint32_t bt = min(a0 + h, p.sfb_rtiles - 1);
                        const uint64_t sfb_off = ((uint64_t)bt * p.sf_ctiles + (uint64_t)kt * C::SF_ATOMS) * 512;
                        if (in_bounds(sfb_off, C::SF_ATOMS * 512, (uint64_t)p.sfb_rtiles * p.sf_ctiles * 512,
                                      p.status))
                            bulk_load(st + C::OFF_SFB + h * C::SF_ATOMS * 512, p.sfb + sfb_off, C::SF_ATOMS * 512,
                                      sb);
                        else
                            mbar_complete_tx(sb, C::SF_ATOMS * 512);
                    }
                    if (!FUSEQ) tma_load_2d(st, &tmap_a, fb, (int32_t)(kt * C::KBYTES), (int32_t)(mb * C::BM));
                    tma_load_2d(st + C::OFF_B, &tmap_b, fb, (int32_t)(kt * C::KBYTES), (int32_t)(nb * BN));
                    ++it;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            // every load this thread issued must land before the CTA exits
            for (uint32_t j = it > (uint32_t)C::STAGES ? it - C::STAGES : 0; j < it; ++j) {
                mbar_wait_bounded(sfdata0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1, never, kWaitLimitNs);
                mbar_wait_bounded(full0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1, never, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0, t_local = 0;
            bool ok = true;
            for (uint32_t tile = tile_first; tile < num_tiles && ok; tile += tile_step, ++t_local) {
                const uint32_t buf = C::ACC_BUFS == 2 ? (t_local & 1) : 0;
                const uint32_t use = C::ACC_BUFS == 2 ? (t_local >> 1) : t_local;
                if (use > 0 && !mbar_wait_bounded(tempty0 + 8 * buf, (use - 1) & 1, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t nb = tile / p.num_m_blocks;
                const uint32_t sfb_shift = ((nb * BN) % 128) / 32;   // B tile starting mid scale tile (BN = 192)
                const uint32_t d_tmem = tmem + buf * BN;
                for (uint32_t kt = kt_begin; kt < kt_end; ++kt, ++it) {
                    const uint32_t s = it % C::STAGES, su = it / C::STAGES;
                    if (!mbar_wait_bounded(full0 + 8 * s, su & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t sfa_t = tmem + C::TM_SF + s * C::SF_COLS;
                    const uint32_t sfb_t = sfa_t + C::SFA_COLS;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        const uint64_t adesc = smem_desc(st + k * C::MMA_K_BYTES, 16, 1024, 2);
                        const uint64_t bdesc = smem_desc(st + C::OFF_B + k * C::MMA_K_BYTES, 16, 1024, 2);
                        const uint32_t acc = (kt != kt_begin) || k != 0;
                        if (FMT == 0) {
                            tc_mma_nvf4(d_tmem, adesc, bdesc, C::IDESC, sfa_t + 4 * k,
                                        sfb_t + C::SFB_COLS_PER_MMA * k + sfb_shift, acc);
                        } else {
                            const uint32_t id = C::IDESC | ((uint32_t)k << 29) | ((uint32_t)k << 4);
                            tc_mma_mxf8(d_tmem, adesc, bdesc, id, sfa_t | ((uint32_t)k << 30),
                                        (sfb_t + sfb_shift) | ((uint32_t)k << 30), acc);
                        }
                    }
                    tc_commit(empty0 + 8 * s);        // shared-memory stage and scale slot free
                }
                if (!ok) break;
                tc_commit(tfull0 + 8 * buf);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            tc_commit(drain);
            mbar_wait_bounded(drain, 0, never, kWaitLimitNs);
        }
    } else if (warp >= kFirstSfWarp) {
        // ---------------------------------------------------------- scale-factor copy warps
        if (lane == 0) {
            const int job = warp - kFirstSfWarp;
            bool ok = true;
            for (uint32_t it = 0; it < total_iters; ++it) {
                const uint32_t s = it % C::STAGES, su = it / C::STAGES;
                // slot s is free once the MMAs of its previous use completed
                if ((su > 0 && !mbar_wait_bounded(empty0 + 8 * s, (su - 1) & 1, abort_flag, p.wait_ns)) ||
                    !mbar_wait_bounded(sfdata0 + 8 * s, su & 1, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                sf_copy_job<C, false>(job, smem_u32(smem + s * C::STAGE_BYTES), tmem + C::TM_SF + s * C::SF_COLS);
                tc_commit(full0 + 8 * s);             // the copies' share of the MMA's wait
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            tc_commit(sfdrain);
            mbar_wait_bounded(sfdrain, 0, never, kWaitLimitNs);
        }
    } else {
        // ---------------------------------------------------------- epilogue (warps 2-9)
        const int q = warp & 3;                       // tensor-memory lane quarter of this warp
        const int half = (warp - 2) >> 2;             // which half of the tile's columns
        float a_dec;
        bool amax_got = true;
        if constexpr (FUSEQ)
            a_dec = fused_quantize_a<C>(p, smem, reinterpret_cast<float*>(bars + 64), kt_begin, kt_end,
                                        tile_first == 0, threadIdx.x - 64, full0, sfdata0, amaxbar, ks,
                                        abort_flag, amax_got);
        else
            a_dec = FMT == 0 ? *p.a_global : 1.0f;
        const float alpha = FMT == 0 ? __fmul_rn(a_dec, *p.b_global) : 1.0f;
        uint8_t* staging = smem + C::OFF_EPI + (warp - 2) * C::EPI_BUF_BYTES;
        const uint16_t* gelu_tab = reinterpret_cast<const uint16_t*>(smem + C::OFF_EPI);
        const EpiQuant eq = {p.q_codes, p.q_sf, p.n_total, p.m_total, p.m_pad, p.status};
        if (EPI == 1) {
            // built while the first tile's MMAs run (the epilogue warps are
            // idle until then); the other roles never touch it
            gelu_table_fill(reinterpret_cast<uint16_t*>(smem + C::OFF_EPI), threadIdx.x - 64, 32 * kEpiWarps);
            named_barrier_sync(1, 32 * kEpiWarps);
        }
        if constexpr (SPLITK) {
            // Rows < SPLIT_ROWS: the first tensor-memory lane quarter holds
            // them all, so the two warps with q == 0 read the accumulator
            // (one row per lane, half of the columns each).  They lay each
            // owner's share out in this CTA's own pipeline stages (free once
            // the MMAs completed), in the slot layout of the owner's receive
            // area, and one thread then sends each slot with one bulk copy
            // that completes on the owner's receive barrier.
            const uint32_t rows = min(p.m_total, (uint32_t)SPLIT_ROWS);
            const SplitShares sh = split_shares<BN>(rows, p.k_split);
            const uint32_t recv = smem_u32(smem + C::OFF_EPI);
            const uint32_t outbox = smem_u32(smem);           // slot for owner j at j * slot * 16
            // one decision per warp: the tensor-memory loads below are warp-wide
            const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(tfull0, 0, abort_flag, p.wait_ns));
            // every receive barrier of the cluster is initialised (the fused
            // path with the amax exchange has waited for this already)
            if (!FUSEQ || p.m_total <= kShortAmaxRows) cluster_wait();
            if (!ok) {
                // the slots still go out (their contents unspecified), so
                // every receive barrier completes
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            if (q == 0 && ok) {
                // A lane's BN/8 groups are consecutive, so the owner only
                // steps on at a share boundary.
                const uint32_t row = lane;
                uint32_t idx = row * (BN / 4) + half * (BN / 8);
                uint32_t owner = idx / sh.per;
                uint32_t bound = (owner + 1) * sh.per;
                uint32_t b8 = (owner * sh.per) & ~7u;
                uint32_t obase = outbox + owner * sh.slot * 16;
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < BN / 2; c0 += 64) {   // 64 columns per load batch
                    const int nc = BN / 2 - c0 < 64 ? BN / 2 - c0 : 64;
                    uint32_t r[64];
                    tc_ld_32x32b_x32(tmem + half * (BN / 2) + c0, *reinterpret_cast<uint32_t(*)[32]>(r));
                    if (nc > 32)
                        tc_ld_32x32b_x32(tmem + half * (BN / 2) + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
                    tc_wait_ld();
                    if (row < rows) {
#pragma unroll
                        for (int v = 0; v < nc / 4; ++v, ++idx) {
                            if (idx == bound) {
                                ++owner;
                                b8 = bound & ~7u;
                                bound += sh.per;
                                obase = outbox + owner * sh.slot * 16;
                            }
                            st_shared_f4(obase + split_pos(idx, row, b8) * 16,
                                         make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
                        }
                    }
                }
                fence_proxy_async_smem();     // the slots, to the bulk copies
            }
            named_barrier_sync(2, 32 * kEpiWarps);
            if (threadIdx.x == 64) {
                for (uint32_t j = 0; j < p.k_split; ++j)
                    bulk_copy_to_cluster(mapa_shared(recv + ks * sh.slot * 16, j), outbox + j * sh.slot * 16,
                                         sh.slot * 16, mapa_shared(recvbar, j));
            }
            split_got = mbar_wait_bounded_cluster(recvbar, 0, abort_flag, p.wait_ns);
            if (!split_got) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
                // the copies into this CTA were all issued; let them land
                mbar_wait_bounded_cluster(recvbar, 0, never, kWaitLimitNs);
            } else {
                splitk_finish<BN>(recv, sh, ks, p.k_split, (tile_first / p.num_m_blocks) * BN, p.n_total, alpha,
                                  p.bias, p.out, p.ldo, threadIdx.x - 64, 32 * kEpiWarps, p.status);
            }
            // (fused: a wait for the cluster's maxima that gave up lets the
            // values already sent land first)
            if (FUSEQ && !amax_got) mbar_wait_bounded_cluster(amaxbar, 0, never, kWaitLimitNs);
            __syncwarp();
            cluster_arrive_relaxed();         // this CTA's share has arrived: its copies out have been read
        }
        uint32_t t_local = 0;
        for (uint32_t tile = SPLITK ? num_tiles : tile_first; tile < num_tiles; tile += tile_step, ++t_local) {
            const uint32_t mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
            const uint32_t buf = C::ACC_BUFS == 2 ? (t_local & 1) : 0;
            const uint32_t use = C::ACC_BUFS == 2 ? (t_local >> 1) : t_local;
            if (!mbar_wait_bounded(tfull0 + 8 * buf, use & 1, abort_flag, p.wait_ns)) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
                break;
            }
            tc_fence_after();
            const uint32_t n0 = nb * BN;
            drain_accumulator<BN, EPI>(tmem + ((uint32_t)(32 * q) << 16) + buf * BN, half, lane, alpha,
                                       p.bias ? p.bias + n0 : nullptr, staging, &tmap_d,
                                       (int32_t)(mb * C::BM + 32 * q), n0, (int)(p.n_total - n0), tempty0 + 8 * buf,
                                       false, eq, gelu_tab);
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    if constexpr (SPLITK) {
        // The roles outside the exchange pass the first phase of the cluster
        // barrier and arrive on the second here; the epilogue warps did both
        // around the exchange, arriving once their CTA's receive barrier
        // completed (every copy into it landed, so every copy out of its
        // sender's shared memory has been read).  Every wait above is
        // bounded, so each thread of the cluster arrives, and no CTA exits
        // while a copy into or out of its shared memory is in flight.
        __syncwarp();
        if (warp < 2 || warp >= kFirstSfWarp) {
            cluster_wait();
            cluster_arrive_relaxed();
        }
        cluster_wait();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TM_COLS);
    }
}

}  // namespace nvq

// gemm_pair.cuh -- block-scaled GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same product as gemm.cuh, D = bf16(alpha * A . B^T + bias), on output tiles
// of 256 x BN (BN = 256, or 192 with two tensor-memory accumulators so the
// epilogue of one tile overlaps the MMAs of the next) computed by a cluster
// of two CTAs on two SMs:
//   CTA r (r = 0, 1) stages rows [128r, 128r + 128) of the A tile and rows
//   [r BN/2, (r+1) BN/2) of the B tile in its own shared memory, holds the
//   scale tiles of its 128 A rows and of all BN B rows, and owns accumulator
//   rows [128r, 128r + 128) in its own tensor memory.
//   The leader (r = 0) alone issues tcgen05.cp (both CTAs' scales into both
//   tensor memories, from its scale-copy warps) and the 256 x BN x K MMAs
//   (from its MMA warp); the MMA commits arrive on the barriers of both CTAs
//   (.multicast::cluster on the commit).
//   Both CTAs' tile loads complete on the leader's barriers (.cta_group::2
//   tensor loads; no load multicast anywhere).  The A and B tiles of a
//   stage land on full[s], which also counts the copy warps' commits, so
//   the MMA lane waits once per stage: it issues the MMAs one after another
//   (the tensor pipe holds little more than one in flight), so every barrier
//   check in its loop is time the pipe stands idle.  Stage s owns scale slot
//   s in tensor memory, and one commit per stage frees both.
//   The scale tiles travel apart from A and B: a producer warp of their own
//   fills a ring of scale slots in shared memory (longer than the stages)
//   as soon as the copies out of a slot have completed, so a stage's scales
//   are in shared memory well before its tensor-memory slot frees, and the
//   copy warps move them the moment it does.  The copy path (scale load,
//   wake-up, twelve tcgen05.cp per stage, completion) otherwise sat on the
//   critical path of every stage.
//   Each CTA drains its own accumulator half; the peer's epilogue warps
//   arrive remotely on the leader's accumulator-empty barrier.
// Per SM this halves the B bytes staged from L2 and the tensor-core
// instructions issued for the same work, compared with one 128 x BN tile
// per SM.  All waits are bounded (status word + abort flag), as in gemm.cuh.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "gemm.cuh"
#include "ptx.cuh"

namespace nvq {

template <int FMT, int BN_>
struct PairCfg {
    static constexpr int BM = 256;                           // rows per pair; 128 per CTA
    static constexpr int BN = BN_;
    static constexpr int BN_HALF = BN / 2;                   // B rows staged per CTA
    static constexpr int KBYTES = 128;
    static constexpr int BK = FMT == 0 ? 256 : 128;
    static constexpr int MMA_K = FMT == 0 ? 64 : 32;
    static constexpr int KSTEPS = BK / MMA_K;
    static constexpr int MMA_K_BYTES = KBYTES / KSTEPS;
    static constexpr int SF_BLOCK = FMT == 0 ? 16 : 32;
    static constexpr int SF_ATOMS = BK / SF_BLOCK / 4;
    static constexpr int SF_CHUNK = SF_ATOMS * 512;          // scale bytes per 128 rows per stage
    static constexpr int SFB_H = 2;                          // 128-row scale tiles spanned by the B tile
    static constexpr int A_BYTES = 128 * KBYTES;
    static constexpr int B_BYTES = BN_HALF * KBYTES;
    static constexpr int SFA_BYTES = SF_CHUNK;
    static constexpr int SFB_BYTES = SFB_H * SF_CHUNK;
    static constexpr int AB_BYTES = A_BYTES + B_BYTES;                    // per CTA per stage
    static constexpr int SF_BYTES = SFA_BYTES + SFB_BYTES;                  // per CTA per stage
    // The A/B tiles of a stage and its scale tiles live apart: stages of
    // A and B, and a longer ring of scale slots that runs ahead of them, so
    // the copies of a stage's scales into tensor memory can start the moment
    // its tensor-memory slot is free instead of after a load issued then.
    static constexpr int STAGE_BYTES = (AB_BYTES + 1023) / 1024 * 1024;
    static constexpr int OFF_B = A_BYTES;
    static constexpr int SF_SLOT_BYTES = (SF_BYTES + 127) / 128 * 128;
    static constexpr int OFF_SFA = 0;                        // within a scale slot
    static constexpr int OFF_SFB = SFA_BYTES;
    static constexpr int EPI_BUF_BYTES = 32 * 64;
    static constexpr int EPI_BYTES = kEpiWarps * EPI_BUF_BYTES;
    static constexpr int BAR_BYTES = 1024;
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int FIXED_BYTES = 1024 /*align*/ + BAR_BYTES + EPI_BYTES;
    static constexpr int SFA_COLS = FMT == 0 ? 4 * KSTEPS : 4;
    static constexpr int SFB_COLS_PER_MMA = 4 * SFB_H;
    static constexpr int SFB_COLS = FMT == 0 ? SFB_COLS_PER_MMA * KSTEPS : SFB_COLS_PER_MMA;
    static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
    // Each stage owns one tensor-memory scale slot, so the stage count is
    // bounded by the columns left beside the accumulator(s) and by shared
    // memory with at least kMinRing scale slots; the ring takes what is
    // left.  Two accumulators only when at least 4 slots remain.
    static constexpr int kMinRing = 8;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED_BYTES - kMinRing * SF_SLOT_BYTES) / STAGE_BYTES;
    static constexpr int ACC_BUFS = (512 - 2 * BN) / SF_COLS >= 4 ? 2 : 1;
    static constexpr int SLOTS_FIT = (512 - ACC_BUFS * BN) / SF_COLS;
    static constexpr int STAGES_MIN2 = STAGES_FIT < SLOTS_FIT ? STAGES_FIT : SLOTS_FIT;
    static constexpr int STAGES = STAGES_MIN2 > 8 ? 8 : STAGES_MIN2;
    static constexpr int RING_FIT = (SMEM_LIMIT - FIXED_BYTES - STAGES * STAGE_BYTES) / SF_SLOT_BYTES;
    static constexpr int SF_RING = RING_FIT > 16 ? 16 : RING_FIT;
    static constexpr int OFF_SF = STAGES * STAGE_BYTES;
    static constexpr int OFF_EPI = (OFF_SF + SF_RING * SF_SLOT_BYTES + 1023) / 1024 * 1024;
    static constexpr int SMEM_BYTES = OFF_EPI + EPI_BYTES + BAR_BYTES + 1024 /*align*/;
    static constexpr int TM_SF = ACC_BUFS * BN;
    static constexpr int TM_USED = ACC_BUFS * BN + STAGES * SF_COLS;
    static constexpr int TM_COLS = TM_USED <= 256 ? 256 : 512;
    static constexpr int SF_WARPS = 1 + SFB_H;             // copy warps (used in the leader)
    static constexpr int SCALE_WARP = kFirstSfWarp + SF_WARPS;   // loads the scale tiles (both CTAs)
    static constexpr int THREADS = 32 * (SCALE_WARP + 1);
    static constexpr uint32_t IDESC =
        (FMT != 1 ? (1u << 7) | (1u << 10) : 0u) |   // A, B type: E2M1 (NVFP4) / E5M2 (FMT 2); 0 = E4M3
        ((uint32_t)(BN >> 3) << 17) |
        (FMT == 0 ? 0u : (1u << 23)) |
        ((uint32_t)(BM >> 4) << 24);
    static_assert(BN == 256 || BN == 192, "pair tiles are 256 x 256 or 256 x 192");
    static_assert(TM_USED <= 512, "tensor memory overflow");
    static_assert(STAGES >= 4, "too few pipeline stages");
    static_assert(SF_RING >= STAGES, "the scale ring must be at least as long as the stages");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory overflow");
    static_assert((2 * STAGES + 2 * SF_RING + 6) * 8 + 12 <= BAR_BYTES, "barrier area");
};

// EPI as in bsgemm_kernel: 0 writes D, 1 writes MXFP8 codes and scales of GELU(D).
template <int FMT, int BN, int EPI>
__global__ void __launch_bounds__(PairCfg<FMT, BN>::THREADS, 1)
bsgemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                   const __grid_constant__ CUtensorMap tmap_d, const GemmParams p) {
    using C = PairCfg<FMT, BN>;
    static_assert(EPI == 0 || (BN == 256 && kGeluTabBytes <= C::EPI_BYTES), "GELU table must fit the staging area");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_EPI + C::EPI_BYTES);
    // full[s]:     A and B tiles of both CTAs landed (tx) + the scale copies
    //              into slot s committed (one arrival per copy warp): the MMA
    //              warp's single wait per stage
    // empty[s]:    the stage's MMAs completed (commit multicast to both CTAs):
    //              frees shared-memory stage s and tensor-memory scale slot s
    // sffull[r]:   both CTAs' scale tiles in ring slot r landed (tx)
    // sfempty[r]:  the copies out of ring slot r completed (commits
    //              multicast to both CTAs, one per copy warp): frees slot r
    const uint32_t full0 = smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * C::STAGES;
    const uint32_t sffull0 = empty0 + 8 * C::STAGES;
    const uint32_t sfempty0 = sffull0 + 8 * C::SF_RING;
    const uint32_t tfull0 = sfempty0 + 8 * C::SF_RING;
    const uint32_t tempty0 = tfull0 + 8 * 2;
    const uint32_t drain = tempty0 + 8 * 2;
    const uint32_t sfdrain = drain + 8;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 2 * C::SF_RING + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* never = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();               // 0 = leader
    const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1 + C::SF_WARPS);
            mbar_init(empty0 + 8 * s, 1);
        }
        for (int r = 0; r < C::SF_RING; ++r) {
            mbar_init(sffull0 + 8 * r, 1);
            mbar_init(sfempty0 + 8 * r, C::SF_WARPS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull0 + 8 * b, 1);
            mbar_init(tempty0 + 8 * b, 2 * kEpiWarps);     // the epilogue warps of both CTAs
        }
        mbar_init(drain, 1);
        mbar_init(sfdrain, C::SF_WARPS);
        *abort_flag = 0;
        *never = 0;
        fence_mbarrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_a);
        prefetch_tensormap(&tmap_b);
        prefetch_tensormap(&tmap_sfa);
        prefetch_tensormap(&tmap_sfb);
        if (EPI == 0) prefetch_tensormap(&tmap_d);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_holder), C::TM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();                                        // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // everything above overlaps the previous grid; no global data is
    // touched before it has completed.  The next grid in the stream may then
    // launch: its CTAs wait at their own griddepcontrol.wait until this grid
    // has completed, so only its launch latency overlaps this grid.
    griddep_wait();
    griddep_launch();
    const uint32_t num_tiles = p.num_m_blocks * p.num_n_blocks;   // 256 x BN tiles
    const uint32_t total_iters = ((num_tiles > pair) ? (num_tiles - pair + npairs - 1) / npairs : 0) * p.num_k_tiles;

    if (warp == 0) {
        // ---------------------------------------------------------- producer (both CTAs)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = pair; tile < num_tiles && ok; tile += npairs) {
                const uint32_t mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
                const int32_t arow = (int32_t)(mb * 256 + 128 * rank);
                const int32_t brow = (int32_t)(nb * BN + C::BN_HALF * rank);
                for (uint32_t kt = 0; kt < p.num_k_tiles; ++kt) {
                    const uint32_t s = it % C::STAGES, use = it / C::STAGES;
                    if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = smem_u32(smem + s * C::STAGE_BYTES);
                    const uint32_t fb = mapa_shared(full0 + 8 * s, 0);     // the leader's barrier
                    if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * C::AB_BYTES);
                    tma_load_2d_pair(st, &tmap_a, fb, (int32_t)(kt * C::KBYTES), arow);
                    tma_load_2d_pair(st + C::OFF_B, &tmap_b, fb, (int32_t)(kt * C::KBYTES), brow);
                    ++it;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            // Neither CTA leaves while a load it issued may still be in flight.
            if (rank == 0) {    // the leader's barriers count both CTAs' bytes: wait for the last stages
                for (uint32_t j = it > (uint32_t)C::STAGES ? it - C::STAGES : 0; j < it; ++j)
                    mbar_wait_bounded(full0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1, never, kWaitLimitNs);
            } else {
                // The peer's loads complete on the leader's barriers, which it
                // cannot wait on; the MMAs that consume a stage complete only
                // after its loads landed, and their commit reaches this CTA's
                // empty[s].  (After an abort that commit may never come: the
                // bounded wait then ends long after any load has landed.)
                for (uint32_t j = it > (uint32_t)C::STAGES ? it - C::STAGES : 0; j < it; ++j)
                    mbar_wait_bounded(empty0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1, never, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer (leader only)
        if (lane == 0 && rank == 0) {
            uint32_t it = 0, t_local = 0;
            bool ok = true;
            for (uint32_t tile = pair; tile < num_tiles && ok; tile += npairs, ++t_local) {
                const uint32_t buf = C::ACC_BUFS == 2 ? (t_local & 1) : 0;
                const uint32_t use = C::ACC_BUFS == 2 ? (t_local >> 1) : t_local;
                if (use > 0 && !mbar_wait_bounded(tempty0 + 8 * buf, (use - 1) & 1, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * BN;
                // a 192-wide B tile may start half-way through a 128-row scale tile
                const uint32_t sfb_shift = (((tile / p.num_m_blocks) * BN) % 128) / 32;
                for (uint32_t kt = 0; kt < p.num_k_tiles; ++kt, ++it) {
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
                        const uint32_t acc = (kt | (uint32_t)k) != 0;
                        if (FMT == 0) {
                            tc_mma_nvf4_pair(d_tmem, adesc, bdesc, C::IDESC, sfa_t + 4 * k,
                                             sfb_t + C::SFB_COLS_PER_MMA * k + sfb_shift, acc);
                        } else {
                            const uint32_t id = C::IDESC | ((uint32_t)k << 29) | ((uint32_t)k << 4);
                            tc_mma_mxf8_pair(d_tmem, adesc, bdesc, id, sfa_t | ((uint32_t)k << 30),
                                             (sfb_t + sfb_shift) | ((uint32_t)k << 30), acc);
                        }
                    }
                    tc_commit_pair_mc(empty0 + 8 * s, 0x3);     // frees stage and scale slot in both CTAs
                }
                if (!ok) break;
                tc_commit_pair_mc(tfull0 + 8 * buf, 0x3);       // accumulator ready in both CTAs
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            tc_commit_pair(drain);
            mbar_wait_bounded(drain, 0, never, kWaitLimitNs);
        }
    } else if (warp == C::SCALE_WARP) {
        // ---------------------------------------------------------- scale-tile producer (both CTAs)
        // Runs up to SF_RING stages ahead: a ring slot is reloaded as soon
        // as the copies out of it have completed.
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tile = pair; tile < num_tiles && ok; tile += npairs) {
                const uint32_t mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
                const uint32_t sfa_atom = mb * 2 + rank;              // this CTA's 128 A rows
                const uint32_t sfb_atom = (nb * BN) / 128;            // first scale tile of the B tile
                for (uint32_t kt = 0; kt < p.num_k_tiles; ++kt) {
                    const uint32_t r = it % C::SF_RING, ru = it / C::SF_RING;
                    if (ru > 0 && !mbar_wait_bounded(sfempty0 + 8 * r, (ru - 1) & 1, abort_flag, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t slot = smem_u32(smem + C::OFF_SF + r * C::SF_SLOT_BYTES);
                    const uint32_t sb = mapa_shared(sffull0 + 8 * r, 0);   // the leader's barrier
                    if (rank == 0) mbar_arrive_expect_tx(sffull0 + 8 * r, 2 * C::SF_BYTES);
                    // the scale tensors are viewed as rows of 256 bytes
                    tma_load_2d_pair(slot + C::OFF_SFA, &tmap_sfa, sb, 0,
                                     (int32_t)(((size_t)sfa_atom * p.sf_ctiles + (size_t)kt * C::SF_ATOMS) * 2));
#pragma unroll
                    for (int h = 0; h < C::SFB_H; ++h)
                        tma_load_2d_pair(slot + C::OFF_SFB + h * C::SF_CHUNK, &tmap_sfb, sb, 0,
                                         (int32_t)(((size_t)(sfb_atom + h) * p.sf_ctiles + (size_t)kt * C::SF_ATOMS) * 2));
                    ++it;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            // Its own loads must land before the CTA leaves: the leader's
            // ring barriers count both CTAs' bytes; the copies out of a slot
            // complete only after its loads landed, and their commits reach
            // both CTAs' sfempty (after an abort they may never come: the
            // bounded wait then ends long after any load has landed).
            for (uint32_t j = it > (uint32_t)C::SF_RING ? it - C::SF_RING : 0; j < it; ++j) {
                if (rank == 0)
                    mbar_wait_bounded(sffull0 + 8 * (j % C::SF_RING), (j / C::SF_RING) & 1, never, kWaitLimitNs);
                else
                    mbar_wait_bounded(sfempty0 + 8 * (j % C::SF_RING), (j / C::SF_RING) & 1, never, kWaitLimitNs);
            }
        }
    } else if (warp >= kFirstSfWarp) {
        // ---------------------------------------------------------- scale-factor copy warps (leader)
        if (lane == 0 && rank == 0) {
            const int job = warp - kFirstSfWarp;
            bool ok = true;
            for (uint32_t it = 0; it < total_iters; ++it) {
                const uint32_t s = it % C::STAGES, su = it / C::STAGES;
                const uint32_t r = it % C::SF_RING, ru = it / C::SF_RING;
                // tensor-memory slot s is free once the MMAs of its previous
                // use completed; ring slot r holds this stage's scale tiles
                if ((su > 0 && !mbar_wait_bounded(empty0 + 8 * s, (su - 1) & 1, abort_flag, p.wait_ns)) ||
                    !mbar_wait_bounded(sffull0 + 8 * r, ru & 1, abort_flag, p.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                sf_copy_job<C, true>(job, smem_u32(smem + C::OFF_SF + r * C::SF_SLOT_BYTES),
                                     tmem + C::TM_SF + s * C::SF_COLS);
                tc_commit_pair(full0 + 8 * s);               // the copies' share of the MMA's wait
                tc_commit_pair_mc(sfempty0 + 8 * r, 0x3);    // ring slot r free in both CTAs
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status, 1u);
            }
            tc_commit_pair(sfdrain);
            mbar_wait_bounded(sfdrain, 0, never, kWaitLimitNs);
        }
    } else {
        // ---------------------------------------------------------- epilogue (both CTAs, warps 2-9)
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const float alpha = FMT == 0 ? __fmul_rn(*p.a_global, *p.b_global) : 1.0f;
        uint8_t* staging = smem + C::OFF_EPI + (warp - 2) * C::EPI_BUF_BYTES;
        const uint16_t* gelu_tab = reinterpret_cast<const uint16_t*>(smem + C::OFF_EPI);
        const EpiQuant eq = {p.q_codes, p.q_sf, p.n_total, p.m_total, p.m_pad, p.status};
        if (EPI == 1) {
            // built while the first tile's MMAs run; the other roles never touch it
            gelu_table_fill(reinterpret_cast<uint16_t*>(smem + C::OFF_EPI), threadIdx.x - 64, 32 * kEpiWarps);
            named_barrier_sync(1, 32 * kEpiWarps);
        }
        uint32_t t_local = 0;
        for (uint32_t tile = pair; tile < num_tiles; tile += npairs, ++t_local) {
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
                                       (int32_t)(mb * 256 + 128 * rank + 32 * q), n0, (int)(p.n_total - n0),
                                       mapa_shared(tempty0 + 8 * buf, 0), true, eq, gelu_tab);
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync();                                        // both CTAs done with the pair's resources
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::TM_COLS);
    }
}

}  // namespace nvq

// skinny.cuh -- the packed INT4 GEMM for few tokens (M <= 128), where the
// weight stream is the whole cost.
//
// Same result as gemm.cuh ("convrot-mlx" README, "What is included": the
// integer GEMM on packed weights, then scaling and bias):
//   acc[m][n] = sum_k qx[m][k] qw[n][k],
//   y[m][n]   = bf16_rne((float(acc) * sx[m]) * sw[n] + b[n]).
//
// With M <= 128 the 0.5 byte per weight has to stream at HBM speed, and
// every weight byte passes through the SM once.  So the layout is chosen to
// touch each weight byte as few times as possible on chip:
//   * the weights are the MMA's A operand and are widened straight into
//     TMEM (tcgen05.st): one TMA write and one shared-memory read per packed
//     byte, instead of the extra widened write and MMA read that a
//     shared-memory A operand costs;
//   * the tokens are the N side (BN = 16, 32, 64 or 128 columns), widened
//     into the 128-byte swizzled shared-memory layout like gemm.cuh's B;
//   * CTA i owns weight rows [i R, i R + R) over the whole of K, with R the
//     row count that spreads N over the SMs (a multiple of 8, at most 128):
//     one wave, no split-K reduction, every SM streaming;
//   * a stage is two K-blocks (256 codes, 128 packed bytes per row), so each
//     TMA copy moves 128 contiguous bytes of a row and every barrier
//     operation, TMEM store wait and TMA issue is paid once per 256 codes;
//   * in the whole-layer call the weights do not depend on the activation
//     prep kernel that precedes the GEMM, so the first stages of weights are
//     requested before waiting for that kernel: the weight stream overlaps
//     the prep.
// Widening, K order and the x16 scale of the int8 operands are those of
// gemm.cuh (the epilogue shifts the accumulator right by 8).
//
// CTA organisation (one CTA per SM, one tile):
//   warp 0      weight TMA producer (one thread): packed weight tiles
//               [R x 128 B] (128-byte swizzle), in a ring as deep as shared
//               memory allows;
//   warp 10     token TMA producer (one thread): packed token tiles
//               [BN x 128 B], a ring of three (they come from L2);
//   warp 1      TMEM allocator and MMA issuer (one thread): 8 MMAs of K = 32
//               per stage, A from TMEM, B from shared memory;
//   warps 2..5  token widening into the swizzled B stages;
//   warps 6..9  weight widening into the TMEM A stages (thread = weight row
//               = TMEM lane);
//   warps 2..9  then the epilogue (tcgen05.ld, scale, bias, bf16), two warps
//               per TMEM lane quarter, two tokens at a time.
// The CTA-pair form (PAIR) shares each MMA between two CTAs (see Cfg).
#pragma once

#include "gemm.cuh"

namespace skinny {

using gemm::BK;
using gemm::BKP;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpB0 = 2, kWarpA0 = 6, kWarpTmaB = 10;
constexpr int kThreads = 11 * 32;
constexpr int kMaxRows = 128;       // weight rows per CTA: the TMEM lanes
constexpr int kSKB = 2;             // K-blocks per stage
constexpr int kPKB = kSKB * BKP;    // packed bytes per row per stage (128)

// PAIR: two CTAs (a cluster) share each MMA (cta_group::2, M = 256): each
// keeps its own R weight rows in its own TMEM lanes and half of the token
// columns in its shared memory; CTA 0 issues the MMAs for both.  Half the
// MMA instructions per weight byte of the one-CTA form.
template <int BN, bool PAIR = false>
struct Cfg {
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128, "token tile of 16..128");
    static_assert(!PAIR || BN >= 32, "cta_group::2 MMAs with A in TMEM need N >= 32");
    static constexpr int CG = PAIR ? 2 : 1;           // tcgen05 CTA group
    static constexpr int BR = PAIR ? BN / 2 : BN;     // token rows held by this CTA
    static constexpr int SU = (BN == 128 && !PAIR) ? 3 : 4;   // TMEM A stages = widened B stages
    static constexpr int PA = kMaxRows * kPKB;        // packed weight stage (up to 128 rows)
    static constexpr int PB = BR * kPKB;              // packed token stage
    // Tokens and weights have rings of their own: the tokens come from L2
    // and need few stages in flight, the weight stream from HBM as many as
    // the rest of shared memory holds (up to 12: ~160 KB in flight per SM).
    static constexpr int SB = 3;
    static constexpr int SP_FIT = (232448 - (SU * kSKB * BR * BK + SB * PB + 4096)) / PA;
    static constexpr int SP = SP_FIT > 12 ? 12 : SP_FIT;
    static_assert(SP >= 3, "at least three weight stages in flight");
    static constexpr int UBH = BR * BK;               // widened token tile of one K-block
    static constexpr int UB = kSKB * UBH;             // widened token stage
    static constexpr int OFF_UB = 0;                  // 1024-aligned tiles first
    static constexpr int OFF_PA = OFF_UB + SU * UB;
    static constexpr int OFF_PB = OFF_PA + SP * PA;
    static constexpr int OFF_BAR = OFF_PB + SB * PB;
    static constexpr int NUM_BARS = 2 * SP + 2 * SB + 2 * SU + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;     // TMEM base, abort flag
    static constexpr int OFF_SX = OFF_MISC + 16;                 // token scales (fp32 x BN)
    static constexpr int SMEM_BYTES = OFF_SX + 4 * BN + 1024;   // + slack for 1024 alignment
    static constexpr uint32_t IDESC = ptx::idesc_i8(PAIR ? 256 : 128, BN);
    static constexpr int ACC_COLS = BN < 32 ? 32 : BN;          // read 32 columns at a time
    static constexpr int A_COLS = kSKB * BK / 4;                // TMEM columns of an A stage (64)
    static constexpr int A_OFF = ACC_COLS;                      // first A-stage column
    static constexpr int TMEM_NEED = A_OFF + SU * A_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                     : TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
    static_assert(UBH % 1024 == 0 && PA % 1024 == 0, "swizzled tiles stay 1024-aligned");
    static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory limit");
};

// Weight rows per CTA for N output columns on num_sms SMs.
inline int rows_per_cta(int64_t N, int num_sms) {
    int64_t r = (N + num_sms - 1) / num_sms;
    r = (r + 7) / 8 * 8;
    return static_cast<int>(r < 8 ? 8 : r > kMaxRows ? kMaxRows : r);
}

// tmA: packed weights [N][K/2], box 128 B x R rows, 128-byte swizzle.
// tmB: packed tokens [M][K/2], box 128 B x Cfg::BR rows.
// wrep: the weights are in the block-major repacked layout (3-D tmA).
// early_a: the weights were complete before the preceding kernel on the
// stream started, so they may be loaded before waiting for it.
// OUT_S32: write the integer accumulators (test hook) instead of bf16.
template <int BN, bool OUT_S32, bool PAIR = false>
__global__ void __launch_bounds__(kThreads, 1)
skinny_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              int R, int early_a, int K, int wrep, const float *__restrict__ sx,
              const float *__restrict__ sw, const uint16_t *__restrict__ bias,
              void *__restrict__ out, int M, int N) {
    using C = Cfg<BN, PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full_a = [&](int s) { return bar0 + 8u * s; };                 // weight stages
    auto empty_a = [&](int s) { return bar0 + 8u * (C::SP + s); };
    auto full_b = [&](int s) { return bar0 + 8u * (2 * C::SP + s); };   // token stages
    auto empty_b = [&](int s) { return bar0 + 8u * (2 * C::SP + C::SB + s); };
    const uint32_t bar_u = bar0 + 8u * (2 * C::SP + 2 * C::SB);
    auto full_u = [&](int s) { return bar_u + 8u * s; };                // TMEM A / widened B
    auto empty_u = [&](int s) { return bar_u + 8u * (C::SU + s); };
    const uint32_t acc_full = bar_u + 8u * (2 * C::SU);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = static_cast<int>(blockIdx.x) * R;     // first weight row of this CTA
    const int num_kp = (K / 2 + kPKB - 1) / kPKB;        // stages; K tails are zero-filled
    const uint32_t a_tx = static_cast<uint32_t>(R * kPKB);        // bytes of a weight stage
    const uint32_t b_tx = static_cast<uint32_t>(C::BR * kPKB);    // bytes of a token stage
    // Rank in the pair: CTA 0 issues the MMAs and holds the barrier that
    // gathers both CTAs' widened stages; its commits reach both CTAs.
    const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
    auto arrive_leader = [&](uint32_t bar) {
        if (PAIR && rank != 0) ptx::mbar_arrive_remote(ptx::mapa_shared(bar, 0));
        else ptx::mbar_arrive(bar);
    };

    // Thread 0 is also the weight producer: it sets up the barriers and,
    // when the weights may be read early, requests the first stages of them
    // before the rest of the set-up (TMEM allocation, the CTA barrier), so
    // the weight stream starts as early as the CTA does.
    const int early = early_a ? (num_kp < C::SP ? num_kp : C::SP) : 0;
    if (threadIdx.x == 0) {
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
        for (int s = 0; s < C::SP; ++s) {
            ptx::mbar_init(full_a(s), 1);
            ptx::mbar_init(empty_a(s), 4);    // the 4 weight widening warps
        }
        for (int s = 0; s < C::SB; ++s) {
            ptx::mbar_init(full_b(s), 1);
            ptx::mbar_init(empty_b(s), 4);    // the 4 token widening warps
        }
        for (int s = 0; s < C::SU; ++s) {
            ptx::mbar_init(full_u(s), (PAIR ? 2 : 1) * 8);
            ptx::mbar_init(empty_u(s), 1);
        }
        ptx::mbar_init(acc_full, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        for (int kp = 0; kp < early; ++kp) {
            ptx::mbar_arrive_expect_tx(full_a(kp), a_tx);
            ptx::tma_load_rows(sbase + C::OFF_PA + kp * C::PA, &tmA, full_a(kp), kp * kPKB, n0,
                               wrep);
        }
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc<C::CG>(sbase + C::OFF_MISC, C::TMEM_COLS);
        ptx::tmem_relinquish<C::CG>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) ptx::cluster_sync();   // the peer's barriers are initialised
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Let a producer's copies already in flight land before the CTA exits:
    // `issued` stages went into a ring of S slots.
    auto drain = [&](auto full, int issued, int S) {
        const int ps = issued % S;
        const uint32_t ph = static_cast<uint32_t>(issued / S) & 1u;
        for (int s = 0; s < S; ++s) {
            volatile int never = 0;
            ptx::mbar_wait(full(s), ph ^ (s < ps ? 0u : 1u), &never, 10000000ull);
        }
    };

    // The producer and MMA loops run in one thread each.
    if (warp == kWarpTma) {
        if (lane == 0) {
            // Weights that may come from the preceding kernel wait for it.
            if (!early_a) ptx::grid_dependency_wait();
            int kp = early;
            for (; kp < num_kp; ++kp) {
                const int s = kp % C::SP;
                if (!ptx::mbar_wait(empty_a(s), ((kp / C::SP) & 1) ^ 1, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(full_a(s), a_tx);
                ptx::tma_load_rows(sbase + C::OFF_PA + s * C::PA, &tmA, full_a(s), kp * kPKB, n0,
                                   wrep);
            }
            if (kp < num_kp) drain(full_a, kp, C::SP);
        }
    } else if (warp == kWarpTmaB) {
        if (lane == 0) {
            ptx::grid_dependency_wait();   // the tokens come from the preceding kernel
            int kp = 0;
            for (; kp < num_kp; ++kp) {
                const int s = kp % C::SB;
                if (!ptx::mbar_wait(empty_b(s), ((kp / C::SB) & 1) ^ 1, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(full_b(s), b_tx);
                ptx::tma_load_2d(sbase + C::OFF_PB + s * C::PB, &tmB, full_b(s), kp * kPKB,
                                 static_cast<int>(rank) * C::BR);
            }
            if (kp < num_kp) drain(full_b, kp, C::SB);
        }
    } else if (warp == kWarpMma) {
        if (lane == 0 && rank == 0) {
            auto commit_both = [&](uint32_t bar) {
                ptx::tc_commit<C::CG>(bar);
                if constexpr (PAIR) ptx::tc_commit<C::CG>(ptx::mapa_shared(bar, 1));
            };
            ptx::grid_dependency_wait();
            int us = 0;
            uint32_t ph = 0;
            for (int kp = 0; kp < num_kp; ++kp) {
                if (!ptx::mbar_wait<PAIR>(full_u(us), ph, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t a0 = tmem_base + static_cast<uint32_t>(C::A_OFF + us * C::A_COLS);
                const uint32_t b0 = sbase + C::OFF_UB + us * C::UB;
#pragma unroll
                for (int j = 0; j < kSKB * BK / 32; ++j)   // A stage: 8 columns per MMA
                    ptx::mma_i8_ts<C::CG>(tmem_base, a0 + static_cast<uint32_t>(8 * j),
                                          ptx::sw128_kmajor_desc(b0 + (j >> 2) * C::UBH + 32 * (j & 3)),
                                          C::IDESC, (kp | j) != 0 ? 1u : 0u);
                commit_both(empty_u(us));
                if (++us == C::SU) { us = 0; ph ^= 1; }
            }
            // Also the drain: TMEM is released only after every MMA completed.
            commit_both(acc_full);
            volatile int never = 0;
            ptx::mbar_wait<PAIR>(acc_full, 0, &never, 100000000ull);
        }
    } else if (warp < kWarpA0) {
        // ------------------------------------------------------ token widening
        // Thread bt takes 16-byte chunk bt & 7 of the 128 packed bytes of token
        // rows bt / 8 + 16 i (chunks 0..3 are K-block 0, 4..7 K-block 1); 16
        // is a multiple of the 8-row swizzle period, so each thread's swizzle
        // phase is fixed.
        ptx::grid_dependency_wait();
        const int bt = static_cast<int>(threadIdx.x) - kWarpB0 * 32;
        constexpr int kPerB = C::BR / 16;
        const uint32_t c8 = static_cast<uint32_t>(bt & 7);
        const uint32_t h = c8 >> 2, c = c8 & 3;
        const int row0 = bt >> 3;
        const uint32_t sw8 = static_cast<uint32_t>(row0 & 7);
        const uint32_t lo_off = ((2u * c) ^ sw8) << 4;
        const uint32_t hi_off = ((2u * c + 1u) ^ sw8) << 4;
        const uint32_t hm = 0xF0F0F0F0u;
        for (int kp = 0; kp < num_kp; ++kp) {
            const int ps = kp % C::SB, us = kp % C::SU;
            const uint32_t pph = (kp / C::SB) & 1, uph = (kp / C::SU) & 1;
            if (!ptx::mbar_wait(full_b(ps), pph, abort_flag)) break;
            if (!ptx::mbar_wait<PAIR>(empty_u(us), uph ^ 1, abort_flag)) break;
            const uint32_t pb = sbase + C::OFF_PB + ps * C::PB + row0 * kPKB + c8 * 16;
            const uint32_t ub = sbase + C::OFF_UB + us * C::UB + h * C::UBH + row0 * 128;
            uint4 w[kPerB];
#pragma unroll
            for (int i = 0; i < kPerB; ++i) w[i] = gemm::lds128(pb + i * 16 * kPKB);
#pragma unroll
            for (int i = 0; i < kPerB; ++i) {
                const uint32_t dst = ub + i * 16 * 128;
                gemm::sts128(dst + lo_off, (w[i].x << 4) & hm, (w[i].y << 4) & hm,
                             (w[i].z << 4) & hm, (w[i].w << 4) & hm);
                gemm::sts128(dst + hi_off, w[i].x & hm, w[i].y & hm, w[i].z & hm, w[i].w & hm);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(empty_b(ps));
                arrive_leader(full_u(us));
            }
        }
    } else {
        // ----------------------------------------------------- weight widening
        // Thread = weight row r of the slice = TMEM lane.  Its 128 packed bytes
        // of a stage arrive 128-byte swizzled (16-byte chunk p of row r at
        // p ^ (r & 7)), so eight consecutive rows reading the same logical
        // chunk hit all banks once.  Chunk p = 4 h + c belongs to K-block h;
        // column 32 h + 8 c + x (x < 4) of the stage holds the even codes of
        // its packed word x and column 32 h + 8 c + 4 + x the odd codes: the K
        // order of the token rows' [even, odd] 16-byte halves.  Lanes at or
        // past R store zeros.
        ptx::grid_dependency_wait();
        const int quarter = warp & 3;                  // TMEM lanes 32 quarter ..
        const int r = quarter * 32 + lane;
        // The token scales are staged in shared memory now, long before the
        // epilogue needs them.
        float *sxs = reinterpret_cast<float *>(smem + C::OFF_SX);
        if (!OUT_S32 && r < BN) sxs[r] = r < M ? sx[r] : 0.0f;
        const bool live = r < R;
        const uint32_t rsw = static_cast<uint32_t>(r & 7);
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t hm = 0xF0F0F0F0u;
        for (int kp = 0; kp < num_kp; ++kp) {
            const int ps = kp % C::SP, us = kp % C::SU;
            const uint32_t pph = (kp / C::SP) & 1, uph = (kp / C::SU) & 1;
            if (!ptx::mbar_wait(full_a(ps), pph, abort_flag)) break;
            if (!ptx::mbar_wait<PAIR>(empty_u(us), uph ^ 1, abort_flag)) break;
            ptx::tc_fence_after();
            const uint32_t src = sbase + C::OFF_PA + ps * C::PA + r * kPKB;
#pragma unroll
            for (int hh = 0; hh < kSKB; ++hh) {
                uint32_t t[32];
                if (live) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const uint32_t chunk = static_cast<uint32_t>(4 * hh + cc) ^ rsw;
                        const uint4 w = gemm::lds128(src + (chunk << 4));
                        t[8 * cc + 0] = (w.x << 4) & hm;
                        t[8 * cc + 1] = (w.y << 4) & hm;
                        t[8 * cc + 2] = (w.z << 4) & hm;
                        t[8 * cc + 3] = (w.w << 4) & hm;
                        t[8 * cc + 4] = w.x & hm;
                        t[8 * cc + 5] = w.y & hm;
                        t[8 * cc + 6] = w.z & hm;
                        t[8 * cc + 7] = w.w & hm;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) t[i] = 0u;
                }
                __syncwarp();   // tcgen05.st is warp-collective
                ptx::tmem_st_32x32b_x32(
                    lane_base + static_cast<uint32_t>(C::A_OFF + us * C::A_COLS + 32 * hh), t);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(empty_a(ps));
                arrive_leader(full_u(us));
            }
        }
    }

    // ---------------------------------------------------------------- epilogue
    // Warps 2-9, two per TMEM lane quarter: lane = output column n (a weight
    // row), accumulator columns = tokens m.  With 64 or more token columns
    // the weight warps take the even 32-column chunks and the token warps
    // the odd ones.
    if (warp >= kWarpB0 && warp < kWarpTmaB) {
        asm volatile("bar.sync 1, 256;" ::: "memory");   // sxs is written, both loops are done
        const bool wgrp = warp >= kWarpA0;
        constexpr int kStep = BN >= 64 ? 64 : 32;
        const int cbeg = (BN >= 64 && !wgrp) ? 32 : 0;
        const bool active = BN >= 64 || wgrp;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        const float *sxs = reinterpret_cast<const float *>(smem + C::OFF_SX);
        if (active && !*abort_flag && ptx::mbar_wait<PAIR>(acc_full, 0, abort_flag)) {
            ptx::tc_fence_after();
            const int n = n0 + r;
            const bool store = r < R && n < N;
            const float swn = (!OUT_S32 && store) ? sw[n] : 0.0f;
            const float bn = (!OUT_S32 && store && bias) ? gemm::bf16_to_f32(bias[n]) : 0.0f;
            constexpr int JW = BN < 32 ? BN : 32;
#pragma unroll 1
            for (int c0 = cbeg; c0 < BN; c0 += kStep) {
                uint32_t v[32];
                __syncwarp();   // tcgen05.ld is warp-collective
                ptx::tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(c0), v);
                ptx::tmem_ld_wait();
                if (!store) continue;
                if (OUT_S32) {
#pragma unroll
                    for (int j = 0; j < JW; ++j) {
                        const int m = c0 + j;
                        if (m < M)
                            reinterpret_cast<int32_t *>(out)[static_cast<size_t>(m) * N + n] =
                                static_cast<int32_t>(v[j]) >> 8;
                    }
                } else {
                    // Two tokens at a time with the packed arithmetic (and no
                    // int-to-float conversions: the conversion unit's rate,
                    // not the stores, bounded this loop).
                    uint16_t *y = reinterpret_cast<uint16_t *>(out);
#pragma unroll
                    for (int j = 0; j < JW; j += 2) {
                        const int m = c0 + j;
                        if (m < M) {
                            const uint32_t pr =
                                gemm::epi_pair_tok(v[j], v[j + 1], sxs[m], sxs[m + 1], swn, bn);
                            y[static_cast<size_t>(m) * N + n] = static_cast<uint16_t>(pr);
                            if (m + 1 < M)
                                y[static_cast<size_t>(m + 1) * N + n] = static_cast<uint16_t>(pr >> 16);
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) ptx::cluster_sync();   // the peer's MMAs and arrivals are done
    ptx::tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        ptx::tmem_dealloc<C::CG>(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace skinny

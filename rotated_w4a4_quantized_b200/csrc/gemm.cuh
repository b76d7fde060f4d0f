// gemm.cuh -- packed INT4 x INT4 GEMM on the sm_100a tensor cores, with the
// fused scale / bias / bf16 epilogue.
//
// What it computes ("convrot-mlx" README, "What is included" and "Install and
// test"): acc[m][n] = sum_k qx[m][k] qw[n][k] exactly, then
// y[m][n] = bf16_rne((float(acc) * sx[m]) * sw[n] + b[n]).
//
// The tensor pipe has no 4-bit integer operand, so packed tiles are widened
// to int8 in shared memory and fed to tcgen05.mma kind::i8 (s8 x s8 -> s32,
// accumulators in TMEM).  Widening: a packed byte holds code c0 in its low
// nibble and c1 in its high nibble (two's complement).  (byte & 0xF0) read
// as int8 is exactly 16 c1, and ((byte << 4) & 0xF0) is exactly 16 c0, so a
// 32-bit word of 8 codes widens with one AND, one SHIFT and one AND into two
// words of four int8 each: no sign-extension work.  Both operands are
// widened the same way, so the tensor cores accumulate 256 * acc; the
// epilogue shifts right by 8 (exact: |256 acc| <= 256 * 49 * 32768 < 2^31).
// The widened K order inside every 32-code block is [even codes, odd codes];
// it is the same permutation for both operands, so the dot products are
// unchanged.
//
// CTA organisation (one CTA per SM, persistent over output tiles):
//   warp 0        TMA producer: packed A [128 x 64 B] and B [BN x 64 B] tiles
//                 per K-block into a ring of packed stages;
//   warp 1        TMEM allocator and MMA issuer (one thread): 4 MMAs of K = 32
//                 per K-block into one of two TMEM accumulators;
//   warps 2..9    epilogue, two warps per TMEM lane quarter (each takes half
//                 of the tile's columns): tcgen05.ld, shift, scale, bias,
//                 bf16; full tiles leave through a swizzled shared-memory
//                 box and a TMA store;
//   warps 10..17  widening: packed stage -> int8 stage in the 128-byte
//                 swizzled K-major layout the MMA descriptors describe; the
//                 warps form groups that take alternate stages.
// Accumulators are double-buffered in TMEM so the epilogue of one tile runs
// under the main loop of the next.
//
// Split K.  Where the tiles leave the last wave of the persistent grid
// part-filled, the host may split the first `split_tiles` tiles into
// `splits` contiguous ranges of K-blocks each.  These split units come first
// in the schedule (one per CTA or pair), so their fix-up overlaps the whole
// tiles that follow.  Each epilogue warp of a split unit writes its region
// of the raw accumulators (256 x a partial sum; 32 rows x half the columns)
// to the unit's slot in the split area, then counts itself in on the
// region's counter with one atomic.  The warp that arrives last adds the
// other parts' copies of its region to its own accumulators and runs the
// epilogue on it: integer addition is exact and associative, so the result
// is bit-identical to the unsplit one in any arrival order, and no warp or
// CTA ever waits for another.  The counter wraps back to zero on the last
// arrival (atom.inc), so it is ready for the next launch.
//
// SWAP selects the skinny-M form: the weights become the 128-row MMA operand
// and the few token rows the N-side operand (BN = 16 .. 128), so the weight
// stream is split over many CTAs; the epilogue writes the transposed tile
// with direct stores.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace gemm {

constexpr int BM = 128;          // MMA M: rows of operand A per tile
constexpr int BKP = 64;          // packed bytes per row per 128-deep K-block
constexpr int BK = 128;          // int8 values per row per K-block
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpEpi0 = 2, kEpiWarps = 8;
constexpr int kWarpUnp0 = kWarpEpi0 + kEpiWarps, kUnpWarps = 8;
constexpr int kThreads = (kWarpUnp0 + kUnpWarps) * 32;    // 576
constexpr int kStoreBox = 32;    // epilogue TMA-store box: 32 rows x 32 bf16
// Split area: kSplitCounters counter words (one per split tile, CTA and
// epilogue warp), then one slot of BM x BN int32 per split unit and CTA.
constexpr int kSplitCounters = 2048;

// One unit of the persistent schedule: output tile `tile`, packed K-stages
// [kp0, kp1), and its part index (-1 for a whole tile).  Units
// 0 .. split_tiles * splits - 1 are the parts of tiles 0 .. split_tiles - 1
// (part p of tile t is unit t * splits + p); the rest are whole tiles.
struct Unit {
    int tile, kp0, kp1, part;
};

__device__ __forceinline__ Unit unit_at(int u, int split_tiles, int splits, int num_kp) {
    Unit w;
    const int nsu = split_tiles * splits;
    if (u < nsu) {
        w.tile = u / splits;
        w.part = u - w.tile * splits;
        w.kp0 = w.part * num_kp / splits;
        w.kp1 = (w.part + 1) * num_kp / splits;
    } else {
        w.tile = u - nsu + split_tiles;
        w.part = -1;
        w.kp0 = 0;
        w.kp1 = num_kp;
    }
    return w;
}

// PAIR: a 2-CTA cluster computes one 256 x BN tile with cta_group::2 MMAs;
// each CTA holds 128 rows of A (in its TMEM), BN / 2 rows of B (in its
// shared memory) and 128 rows of the accumulator.
template <int BN, bool SWAP, bool PAIR = false>
struct Cfg {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "kind::i8 with M=128 needs N%16==0");
    static_assert(!PAIR || (!SWAP && (BN == 192 || BN == 128)), "the CTA pair runs 256 x 192 or 256 x 128 tiles");
    static constexpr int CG = PAIR ? 2 : 1;          // tcgen05 CTA group
    static constexpr int TM = PAIR ? 2 * BM : BM;    // rows of A per tile
    static constexpr int BR = PAIR ? BN / 2 : BN;    // rows of B per CTA
    static_assert(BN < 64 || (BN / 2) % 32 == 0, "each epilogue half covers whole 32-column reads");
    // Packed stages keep HBM loads in flight; the narrow (skinny) tiles are
    // bound by the weight stream, so they trade widened stages for more
    // packed ones.  The wide tile keeps room for the epilogue's store boxes.
    // A widened slot comes back only after its MMAs complete (~500 cycles)
    // and the next widening (~700 cycles) is done, so narrow tiles, whose
    // MMAs are short, keep more widened slots; the packed ring keeps 100+ KB
    // of the weight stream in flight.
    // ATM: the 128 x 192 tile widens operand A straight into TMEM (the MMA
    // reads A from there), so only B passes through widened shared memory;
    // TMEM holds two 192-column accumulators plus SU 64-column A stages.
    // Its stages are two K-blocks deep (KS = 2, 128 packed bytes per row):
    // every TMA issue, barrier operation and TMEM store wait is paid once per
    // 256 codes, which the single-thread issue loops need to keep up with
    // the tensor cores.
    static constexpr bool ATM = PAIR || (!SWAP && BN == 192);
    static constexpr int KS = ATM ? 2 : 1;           // K-blocks per widened stage
    static constexpr int SP = PAIR ? 4 : ATM ? 2 : BN == 256 ? 3 : BN == 192 ? 5 : BN == 128 ? 3 : BN == 64 ? 4 : BN == 32 ? 5 : 3;
    // the 256 x 128 pair has room in TMEM for four A stages (2 x 128
    // accumulator columns + 4 x 64), the 192-wide tiles for two
    static constexpr int SU = (PAIR && BN == 128) ? 4 : ATM ? 2 : BN >= 192 ? 2 : BN == 128 ? 4 : BN == 64 ? 5 : 6;
    // The widening warps split into UG groups that take alternate stages, so
    // the hand-off latency of one stage overlaps the widening of the next.
    static constexpr int UG = (ATM || BN >= 192) ? 1 : 2;   // the TMEM-A widening runs as one group
    static_assert(SU >= UG, "each group needs a widened stage of its own");
    // Packed stages of the narrow tiles carry PKB bytes of each row (PSUB
    // K-blocks), so the weight stream is read in longer contiguous pieces;
    // the widening turns each packed stage into PSUB widened K-blocks.
    static constexpr int PKB = ATM ? 128 : (!SWAP && BN >= 192) ? 64 : BN == 16 ? 256 : 128;
    static constexpr int PSUB = ATM ? 1 : PKB / BKP;
    static constexpr int PA = BM * PKB;
    static constexpr int PB = BR * PKB;
    static constexpr int UA = ATM ? 0 : BM * BK;
    static constexpr int UBH = BR * BK;               // widened B tile of one K-block
    static constexpr int UB = KS * UBH;
    // store boxes per epilogue warp: three let the pair's epilogue (3 boxes
    // per tile and warp) issue every store without waiting for a box
    static constexpr int SB = PAIR ? 3 : 2;
    static constexpr int ST = SWAP ? 0 : kEpiWarps * SB * kStoreBox * kStoreBox * 2;
    static constexpr int OFF_UA = 0;                   // 1024-aligned tiles first
    static constexpr int OFF_UB = OFF_UA + SU * UA;
    static constexpr int OFF_ST = OFF_UB + SU * UB;
    // per-warp copies of the tile's column parameters (sw as fp32, bias as
    // bf16) for the columns that warp covers, two tiles deep
    static constexpr int CP_COLS = BN >= 64 ? BN / 2 : BN;
    static constexpr int CP_WARP = 2 * CP_COLS * 6;
    static constexpr int CP = SWAP ? 0 : kEpiWarps * CP_WARP;
    static constexpr int OFF_CP = OFF_ST + ST;
    static constexpr int OFF_PA = OFF_CP + ((CP + 1023) / 1024) * 1024;
    static constexpr int OFF_PB = OFF_PA + SP * PA;
    static constexpr int OFF_BAR = OFF_PB + SP * PB;
    static constexpr int NUM_BARS = 2 * SP + 2 * SU + 5;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + slack for 1024 alignment
    // Each accumulator buffer is read 32 columns at a time, so buffers are at
    // least 32 columns apart and the allocation covers two of them.
    static constexpr int ACC_STRIDE = BN < 32 ? 32 : BN;
    static constexpr int A_OFF = 2 * ACC_STRIDE;              // first A-stage column (ATM)
    static constexpr int A_COLS = KS * BK / 4;                 // TMEM columns of an A stage
    static constexpr int TMEM_NEED = A_OFF + (ATM ? SU * A_COLS : 0);
    static constexpr int TMEM_COLS = TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                     : TMEM_NEED <= 256 ? 256 : 512;   // power of two
    static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
    static_assert(!ATM || (PSUB == 1 && PKB == 128), "A-in-TMEM reads 128-byte swizzled packed rows");
    static constexpr int JW = BN < 32 ? BN : 32;             // valid columns per 32-wide read
    static_assert(UB % 1024 == 0, "widened B tiles must stay 1024-aligned");
    static_assert(ST % 1024 == 0, "store boxes must stay 1024-aligned");
    static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory limit");
};

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(addr));
    return r;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&h);
}

// The epilogue arithmetic, in the fixed order of the definition.
__device__ __forceinline__ float epi(uint32_t raw, float sx, float sw, float b) {
    const int acc = static_cast<int>(raw) >> 8;
    float t = __fmul_rn(__int2float_rn(acc), sx);
    t = __fmul_rn(t, sw);
    return __fadd_rn(t, b);
}

// The same arithmetic for two adjacent columns, returning their bf16 pair
// (low half = first column).  float(acc) is formed exactly without the
// conversion unit: for |acc| < 2^22 the bit pattern 0x4B400000 + acc is the
// float 1.5 * 2^23 + acc, and subtracting 1.5 * 2^23 is exact.  The last
// multiply and the bias add are scalar round-to-nearest operations: ptxas
// fuses a packed mul.rn.f32x2 feeding an add.rn.f32x2 into one fused
// multiply-add (measured on sm_100a), which rounds once instead of twice
// and, where the bias cancels the product, changes the bf16 result.
__device__ __forceinline__ uint32_t epi_pair(uint32_t r0, uint32_t r1, float sx, float sw0,
                                             float sw1, float b0, float b1) {
    float f0 = __int_as_float((static_cast<int>(r0) >> 8) + 0x4B400000);
    float f1 = __int_as_float((static_cast<int>(r1) >> 8) + 0x4B400000);
    ptx::add2(f0, f1, f0, f1, -12582912.0f, -12582912.0f);
    ptx::mul2(f0, f1, f0, f1, sx, sx);
    f0 = __fadd_rn(__fmul_rn(f0, sw0), b0);
    f1 = __fadd_rn(__fmul_rn(f1, sw1), b1);
    const __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// The same arithmetic for two tokens of one output column (the few-token
// forms, where accumulator columns are tokens): their own token scales,
// the column's weight scale and bias.
__device__ __forceinline__ uint32_t epi_pair_tok(uint32_t r0, uint32_t r1, float sx0, float sx1,
                                                 float sw, float b) {
    float f0 = __int_as_float((static_cast<int>(r0) >> 8) + 0x4B400000);
    float f1 = __int_as_float((static_cast<int>(r1) >> 8) + 0x4B400000);
    ptx::add2(f0, f1, f0, f1, -12582912.0f, -12582912.0f);
    ptx::mul2(f0, f1, f0, f1, sx0, sx1);
    f0 = __fadd_rn(__fmul_rn(f0, sw), b);
    f1 = __fadd_rn(__fmul_rn(f1, sw), b);
    const __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// OUT_S32: write the integer accumulators (test hook) instead of bf16.
// tmY (used when !SWAP && !OUT_S32 && use_tma_store): bf16 y [M][N], box
// 32 x 32, 64-byte swizzle.
template <int BN, bool SWAP, bool OUT_S32, bool PAIR = false>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmY, int use_tma_store, int rowsA, int rowsB,
            int K, const float *__restrict__ sx, const float *__restrict__ sw,
            const uint16_t *__restrict__ bias, void *__restrict__ out, int M, int N, int wrep,
            int split_tiles, int splits, uint32_t *__restrict__ split_ws) {
    using C = Cfg<BN, SWAP, PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full_p = [&](int s) { return bar0 + 8u * s; };
    auto empty_p = [&](int s) { return bar0 + 8u * (C::SP + s); };
    auto full_u = [&](int s) { return bar0 + 8u * (2 * C::SP + s); };
    auto empty_u = [&](int s) { return bar0 + 8u * (2 * C::SP + C::SU + s); };
    auto acc_full = [&](int b) { return bar0 + 8u * (2 * C::SP + 2 * C::SU + b); };
    auto acc_empty = [&](int b) { return bar0 + 8u * (2 * C::SP + 2 * C::SU + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * C::SP + 2 * C::SU + 4);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Rank in the CTA pair (0 issues the MMAs; the barriers that gather both
    // CTAs' work live in CTA 0).
    const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
    // Arrive on a barrier of CTA 0 (remote for CTA 1 of a pair).
    auto arrive_leader = [&](uint32_t bar) {
        if (PAIR && rank != 0) ptx::mbar_arrive_remote(ptx::mapa_shared(bar, 0));
        else ptx::mbar_arrive(bar);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::SP; ++s) {
            ptx::mbar_init(full_p(s), 1);
            ptx::mbar_init(empty_p(s), C::PSUB * (kUnpWarps / C::UG));
        }
        for (int s = 0; s < C::SU; ++s) {
            ptx::mbar_init(full_u(s), (PAIR ? 2 : 1) * kUnpWarps / C::UG);
            ptx::mbar_init(empty_u(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(acc_full(b), 1);
            ptx::mbar_init(acc_empty(b), (PAIR ? 2 : 1) * kEpiWarps);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
        if (!SWAP && !OUT_S32 && use_tma_store) ptx::tma_prefetch_desc(&tmY);
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
    // Everything above overlaps the tail of the kernel that produced the
    // operands (programmatic dependent launch); nothing below may run before
    // that kernel's results are visible.
    ptx::grid_dependency_wait();

    const int tiles_a = (rowsA + C::TM - 1) / C::TM;
    const int tiles_b = (rowsB + BN - 1) / BN;
    const int num_tiles = tiles_a * tiles_b;
    // Persistent schedule: unit u goes to CTA (pair) u mod the grid.
    const int num_units = num_tiles + split_tiles * (splits - 1);
    const int first_tile = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int num_kp = (K / 2 + C::PKB - 1) / C::PKB;   // packed stages per tile

    // The producer and MMA loops run in one thread each (lane 0): a warp-wide
    // mbarrier operation costs a multiple of one thread's.
    if (warp == kWarpTma) {
        int ps = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int u = first_tile; lane == 0 && u < num_units && ok; u += tile_step) {
            const Unit w = unit_at(u, split_tiles, splits, num_kp);
            const int ta = w.tile % tiles_a, tb = w.tile / tiles_a;
            for (int kp = w.kp0; kp < w.kp1; ++kp) {
                if (!ptx::mbar_wait(empty_p(ps), ph ^ 1, abort_flag)) { ok = false; break; }
                ptx::mbar_arrive_expect_tx(full_p(ps), C::PA + C::PB);
                // the weights (B, or A in the swapped form) may be repacked
                ptx::tma_load_rows(sbase + C::OFF_PA + ps * C::PA, &tmA, full_p(ps), kp * C::PKB,
                                   ta * C::TM + static_cast<int>(rank) * BM, SWAP ? wrep : 0);
                ptx::tma_load_rows(sbase + C::OFF_PB + ps * C::PB, &tmB, full_p(ps), kp * C::PKB,
                                   tb * BN + static_cast<int>(rank) * C::BR, SWAP ? 0 : wrep);
                if (++ps == C::SP) { ps = 0; ph ^= 1; }
            }
        }
        if (!ok) {
            // Let copies already in flight land before the CTA exits.
            for (int s = 0; s < C::SP; ++s) {
                volatile int never = 0;
                ptx::mbar_wait(full_p(s), ph ^ (s < ps ? 0u : 1u), &never, 10000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        // In a pair only CTA 0 issues; its commits arrive on the barriers of
        // both CTAs.
        const bool issuer = (!PAIR || rank == 0) && lane == 0;
        constexpr uint32_t idesc = ptx::idesc_i8(C::TM, BN);
        auto commit_both = [&](uint32_t bar) {
            ptx::tc_commit<C::CG>(bar);
            if constexpr (PAIR) ptx::tc_commit<C::CG>(ptx::mapa_shared(bar, 1));
        };
        int us = 0;
        uint32_t ph = 0;
        int local = 0;
        bool ok = true;
        for (int u = first_tile; issuer && u < num_units && ok; u += tile_step, ++local) {
            const Unit w = unit_at(u, split_tiles, splits, num_kp);
            const int num_kb = (w.kp1 - w.kp0) * C::PSUB;   // widened K-blocks of the unit
            const int b = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            if (!ptx::mbar_wait<PAIR>(acc_empty(b), aph ^ 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t d = tmem_base + static_cast<uint32_t>(b * C::ACC_STRIDE);
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!ptx::mbar_wait<PAIR>(full_u(us), ph, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t a0 = sbase + C::OFF_UA + us * C::UA;
                const uint32_t b0 = sbase + C::OFF_UB + us * C::UB;
#pragma unroll
                for (int j = 0; j < C::KS * BK / 32; ++j) {
                    if constexpr (C::ATM)
                        // A stage: 8 columns (32 int8 of each row) per MMA; B
                        // K-block j / 4 is its own 128-byte swizzled tile
                        ptx::mma_i8_ts<C::CG>(
                            d, tmem_base + static_cast<uint32_t>(C::A_OFF + us * C::A_COLS + 8 * j),
                            ptx::sw128_kmajor_desc(b0 + (j >> 2) * C::UBH + 32 * (j & 3)), idesc,
                            (kb | j) != 0 ? 1u : 0u);
                    else
                        ptx::mma_i8_ss(d, ptx::sw128_kmajor_desc(a0 + 32 * j),
                                       ptx::sw128_kmajor_desc(b0 + 32 * j), idesc,
                                       (kb | j) != 0 ? 1u : 0u);
                }
                commit_both(empty_u(us));
                if (++us == C::SU) { us = 0; ph ^= 1; }
            }
            if (ok) commit_both(acc_full(b));
        }
        // Wait for every MMA this thread issued before TMEM is released.
        if (issuer) {
            ptx::tc_commit<C::CG>(drain_bar);
            volatile int never = 0;
            ptx::mbar_wait(drain_bar, 0, &never, 100000000ull);
        }
    } else if (warp < kWarpUnp0) {
        // ------------------------------------------------------------ epilogue
        const int e = warp - kWarpEpi0;               // 0 .. 7
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ..
        const int half = e >> 2;                      // which half of the columns
        const int r = quarter * 32 + lane;            // row of the accumulator tile
        constexpr int kCols = BN >= 64 ? BN / 2 : BN; // columns this warp covers
        const int col_begin = BN >= 64 ? half * kCols : 0;
        const bool active = BN >= 64 || half == 0;
        const bool tma_out = !SWAP && !OUT_S32 && use_tma_store;
        const uint32_t box0 = sbase + C::OFF_ST + e * (C::SB * kStoreBox * kStoreBox * 2);
        int nstores = 0;
        int local = 0;
        for (int u = first_tile; u < num_units; u += tile_step, ++local) {
            const Unit w = unit_at(u, split_tiles, splits, num_kp);
            const int ta = w.tile % tiles_a, tb = w.tile / tiles_a;
            const int b = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            const int row0 = ta * C::TM + static_cast<int>(rank) * BM;   // this CTA's first A row
            const int arow = row0 + r;                // A row of this lane
            // The tile's column scales and bias go to shared memory (and the
            // row scale to a register) while the main loop still runs, so the
            // epilogue never waits on these loads.
            // Each warp keeps its own copy of its columns' parameters, so no
            // synchronisation beyond the warp is needed.
            float *cp_sw = reinterpret_cast<float *>(smem + C::OFF_CP + e * C::CP_WARP +
                                                     b * (C::CP_COLS * 6));
            uint16_t *cp_b = reinterpret_cast<uint16_t *>(cp_sw + C::CP_COLS);
            float sxm = 0.0f;
            if (tma_out && active) {
                for (int i = lane; i < kCols; i += 32) {
                    const int n = tb * BN + col_begin + i;
                    cp_sw[i] = n < N ? sw[n] : 0.0f;
                    cp_b[i] = (bias && n < N) ? bias[n] : static_cast<uint16_t>(0);
                }
                sxm = arow < M ? sx[arow] : 0.0f;
                __syncwarp();
            }
            if (!ptx::mbar_wait<PAIR>(acc_full(b), aph, abort_flag)) break;
            ptx::tc_fence_after();
            const uint32_t acc_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                      static_cast<uint32_t>(b * C::ACC_STRIDE);
            bool emit = true;
            if constexpr (!SWAP && BN >= 64) {
                if (w.part >= 0) {
                    // A part of a split tile: this warp's region of the raw
                    // accumulators goes to the unit's slot, 32 columns at a
                    // time as eight 16-byte words per row, word j4 of column
                    // block c of row r at ((c * 8 + j4) * BM + r) * 4
                    // (coalesced across the warp).
                    uint32_t *slot = split_ws + kSplitCounters +
                                     static_cast<size_t>(u * C::CG + static_cast<int>(rank)) * (BM * BN);
#pragma unroll 1
                    for (int c0 = col_begin; c0 < col_begin + kCols; c0 += 32) {
                        uint32_t v[32];
                        __syncwarp();
                        ptx::tmem_ld_32x32b_x32(acc_lane + static_cast<uint32_t>(c0), v);
                        ptx::tmem_ld_wait();
                        uint32_t *dst = slot + (static_cast<size_t>(c0 / 32) * 8 * BM + r) * 4;
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4)
                            ptx::st_cg_v4(dst + j4 * BM * 4, v[4 * j4], v[4 * j4 + 1], v[4 * j4 + 2],
                                          v[4 * j4 + 3]);
                    }
                    // The region is in the slot before the counter moves; the
                    // last arrival then sees every other part's copy of it.
                    __threadfence();
                    __syncwarp();
                    uint32_t old = 0;
                    if (lane == 0)
                        old = ptx::atom_inc_acq_rel(
                            split_ws + (w.tile * C::CG + static_cast<int>(rank)) * kEpiWarps + e,
                            static_cast<uint32_t>(splits - 1));
                    old = __shfl_sync(0xFFFFFFFFu, old, 0);
                    emit = old == static_cast<uint32_t>(splits - 1);
                    if (emit) __threadfence();
                }
            }
            if (active && emit) {
#pragma unroll 1
                for (int c0 = col_begin; c0 < col_begin + kCols; c0 += 32) {
                    const int bcol0 = tb * BN + c0;   // first B row of these 32 columns
                    uint32_t v[32];
                    __syncwarp();   // tcgen05.ld is warp-collective
                    ptx::tmem_ld_32x32b_x32(acc_lane + static_cast<uint32_t>(c0), v);
                    ptx::tmem_ld_wait();
                    if constexpr (!SWAP && BN >= 64) {
                        if (w.part >= 0) {
                            // last part of a split tile: add the other parts
                            for (int p = 0; p < splits; ++p) {
                                if (p == w.part) continue;
                                const uint32_t *src =
                                    split_ws + kSplitCounters +
                                    static_cast<size_t>((w.tile * splits + p) * C::CG +
                                                        static_cast<int>(rank)) * (BM * BN) +
                                    (static_cast<size_t>(c0 / 32) * 8 * BM + r) * 4;
                                // all eight loads in flight before the first add
                                uint4 q[8];
#pragma unroll
                                for (int j4 = 0; j4 < 8; ++j4) q[j4] = ptx::ld_cg_v4(src + j4 * BM * 4);
#pragma unroll
                                for (int j4 = 0; j4 < 8; ++j4) {
                                    v[4 * j4] += q[j4].x;
                                    v[4 * j4 + 1] += q[j4].y;
                                    v[4 * j4 + 2] += q[j4].z;
                                    v[4 * j4 + 3] += q[j4].w;
                                }
                            }
                        }
                    }
                    if (!SWAP && !OUT_S32 && tma_out) {
                        // 32 rows x 32 columns through a swizzled box, one TMA store
                        const int n0 = bcol0;
                        uint32_t pk[16];
                        const float4 *s4 = reinterpret_cast<const float4 *>(cp_sw + (c0 - col_begin));
                        const uint4 *b4 = reinterpret_cast<const uint4 *>(cp_b + (c0 - col_begin));
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 fa = s4[2 * i], fb = s4[2 * i + 1];
                            const uint4 u = b4[i];
                            const uint32_t bw[4] = {u.x, u.y, u.z, u.w};
                            const float swv[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                pk[4 * i + j] = epi_pair(v[8 * i + 2 * j], v[8 * i + 2 * j + 1], sxm,
                                                         swv[2 * j], swv[2 * j + 1],
                                                         __uint_as_float(bw[j] << 16),
                                                         __uint_as_float(bw[j] & 0xFFFF0000u));
                        }
                        const uint32_t box = box0 + (nstores % C::SB) * (kStoreBox * kStoreBox * 2);
                        if (lane == 0) ptx::bulk_wait_read<C::SB - 1>();   // this box's previous store
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint32_t sw16 = static_cast<uint32_t>(c ^ ((lane >> 1) & 3));
                            sts128(box + lane * 64 + sw16 * 16, pk[4 * c], pk[4 * c + 1],
                                   pk[4 * c + 2], pk[4 * c + 3]);
                        }
                        ptx::fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            ptx::tma_store_2d(&tmY, box, n0, row0 + quarter * 32);
                            ptx::bulk_commit();
                        }
                        ++nstores;
                    } else if (!SWAP) {
                        // lane = output row m, columns = output columns n
                        const int m = arow;
                        if (m >= M) continue;
                        const int n0 = bcol0;
                        if (OUT_S32) {
                            int32_t *o = reinterpret_cast<int32_t *>(out) + static_cast<size_t>(m) * N;
                            for (int j = 0; j < C::JW; ++j)
                                if (n0 + j < N) o[n0 + j] = static_cast<int32_t>(v[j]) >> 8;
                        } else {
                            const float sxm = sx[m];
                            uint16_t *o = reinterpret_cast<uint16_t *>(out) + static_cast<size_t>(m) * N;
                            for (int j = 0; j < C::JW; ++j) {
                                const int n = n0 + j;
                                if (n >= N) break;
                                const float bb = bias ? bf16_to_f32(bias[n]) : 0.0f;
                                o[n] = f32_to_bf16_rne(epi(v[j], sxm, sw[n], bb));
                            }
                        }
                    } else {
                        // lane = output column n (a weight row), columns = tokens m
                        const int n = arow;
                        if (n >= N) continue;
                        if (OUT_S32) {
                            int32_t *o = reinterpret_cast<int32_t *>(out);
                            for (int j = 0; j < C::JW; ++j) {
                                const int m = bcol0 + j;
                                if (m >= M) break;
                                o[static_cast<size_t>(m) * N + n] = static_cast<int32_t>(v[j]) >> 8;
                            }
                        } else {
                            const float swn = sw[n];
                            const float bn = bias ? bf16_to_f32(bias[n]) : 0.0f;
                            uint16_t *o = reinterpret_cast<uint16_t *>(out);
                            for (int j = 0; j < C::JW; ++j) {
                                const int m = bcol0 + j;
                                if (m >= M) break;
                                o[static_cast<size_t>(m) * N + n] =
                                    f32_to_bf16_rne(epi(v[j], sx[m], swn, bn));
                            }
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(acc_empty(b));
        }
        // The boxes must have been read before the CTA's shared memory goes;
        // the global writes complete with the grid.
        if (tma_out && lane == 0) ptx::bulk_wait_read<0>();
    } else if constexpr (C::ATM) {
        // ------------------------------------------------- widening, A in TMEM
        // A stage = two K-blocks.  Warps 0..3 of the group widen A: thread =
        // one A row (TMEM lane); its 128 packed bytes arrive 128-byte swizzled
        // (16-byte chunk p of row r at p ^ (r & 7)), so eight consecutive rows
        // reading the same logical chunk hit all banks once.  Chunk p = 4 h + c
        // is in K-block h; column 32 h + 8 c + x (x < 4) of the stage holds the
        // even codes of packed word x of the chunk and column 32 h + 8 c + 4 + x
        // its odd codes: the K order of the B rows' [even, odd] 16-byte halves.
        // Warps 4..7 widen B into the swizzled shared-memory stage, one
        // 128-byte-row tile per K-block.
        const int uw = warp - kWarpUnp0;
        int total = 0;   // widened stages this CTA runs
        for (int u = first_tile; u < num_units; u += tile_step) {
            const Unit w = unit_at(u, split_tiles, splits, num_kp);
            total += (w.kp1 - w.kp0) * C::PSUB;
        }
        const uint32_t hm = 0xF0F0F0F0u;
        if (uw < 4) {
            const int quarter = warp & 3;             // TMEM lanes 32*quarter ..
            const int r = quarter * 32 + lane;
            const uint32_t rsw = static_cast<uint32_t>(r & 7);
            const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                  static_cast<uint32_t>(C::A_OFF);
            for (int n = 0; n < total; ++n) {
                const int ps = n % C::SP, us = n % C::SU;
                const uint32_t pph = (n / C::SP) & 1, uph = (n / C::SU) & 1;
                if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) break;
                if (!ptx::mbar_wait<PAIR>(empty_u(us), uph ^ 1, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t src = sbase + C::OFF_PA + ps * C::PA + r * C::PKB;
#pragma unroll
                for (int h = 0; h < C::KS; ++h) {
                    uint32_t t[32];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t chunk = static_cast<uint32_t>(4 * h + c) ^ rsw;
                        const uint4 w = lds128(src + (chunk << 4));
                        t[8 * c + 0] = (w.x << 4) & hm;
                        t[8 * c + 1] = (w.y << 4) & hm;
                        t[8 * c + 2] = (w.z << 4) & hm;
                        t[8 * c + 3] = (w.w << 4) & hm;
                        t[8 * c + 4] = w.x & hm;
                        t[8 * c + 5] = w.y & hm;
                        t[8 * c + 6] = w.z & hm;
                        t[8 * c + 7] = w.w & hm;
                    }
                    __syncwarp();   // tcgen05.st is warp-collective
                    ptx::tmem_st_32x32b_x32(trow + static_cast<uint32_t>(us * C::A_COLS + 32 * h), t);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(empty_p(ps));
                    arrive_leader(full_u(us));
                }
            }
        } else {
            // 128 threads over BR rows x 2 K-blocks x 4 chunks of 16 bytes:
            // thread bt takes chunk c = bt & 3 of K-block h = (bt >> 2) & 1, of
            // rows 32 j + 2 q + (h ^ i) for i = 0, 1 (q = bt >> 3).  The eight
            // threads of a quarter warp then touch one row's K-block 0 and an
            // adjacent row's K-block 1: 128 distinct bytes on the packed read,
            // and chunk sets of opposite swizzle parity on the widened writes,
            // so neither access has bank conflicts.
            const int bt = threadIdx.x - (kWarpUnp0 + 4) * 32;
            constexpr int kRowBlocks = C::BR / 32;
            const uint32_t c = static_cast<uint32_t>(bt & 3);
            const int h = (bt >> 2) & 1;
            const int q2 = 2 * (bt >> 3);
            for (int n = 0; n < total; ++n) {
                const int ps = n % C::SP, us = n % C::SU;
                const uint32_t pph = (n / C::SP) & 1, uph = (n / C::SU) & 1;
                if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) break;
                if (!ptx::mbar_wait<PAIR>(empty_u(us), uph ^ 1, abort_flag)) break;
                const uint32_t pb = sbase + C::OFF_PB + ps * C::PB + h * BKP + c * 16;
                const uint32_t ub = sbase + C::OFF_UB + us * C::UB + h * C::UBH;
#pragma unroll
                for (int j = 0; j < kRowBlocks; ++j) {
                    uint4 w[2];
                    int row[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        row[i] = 32 * j + q2 + (h ^ i);
                        w[i] = lds128(pb + row[i] * C::PKB);
                    }
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const uint32_t sw8 = static_cast<uint32_t>(row[i] & 7);
                        const uint32_t dst = ub + row[i] * 128;
                        sts128(dst + (((2u * c) ^ sw8) << 4), (w[i].x << 4) & hm, (w[i].y << 4) & hm,
                               (w[i].z << 4) & hm, (w[i].w << 4) & hm);
                        sts128(dst + (((2u * c + 1u) ^ sw8) << 4), w[i].x & hm, w[i].y & hm,
                               w[i].z & hm, w[i].w & hm);
                    }
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(empty_p(ps));
                    arrive_leader(full_u(us));
                }
            }
        }
    } else {
        // ------------------------------------------------------------ widening
        // Group g of UG takes stages g, g + UG, g + 2 UG, ... (counted over all
        // tiles and K-blocks of this CTA).  Within a group, thread ut widens
        // 16-byte packed chunks ut, ut + GT, ... (GT threads per group); GT is
        // a multiple of 4 chunks per row and of 8 rows per swizzle group, so a
        // thread's chunk column and swizzle phase never change.
        constexpr int GT = kUnpWarps * 32 / C::UG;
        const int ug = (threadIdx.x - kWarpUnp0 * 32) / GT;
        const int ut = (threadIdx.x - kWarpUnp0 * 32) % GT;
        constexpr int kChunks = (BM + BN) * 4;          // 16-byte packed chunks per stage
        constexpr int kPer = (kChunks + GT - 1) / GT;
        constexpr int kRowStep = GT / 4;
        const uint32_t c = static_cast<uint32_t>(ut & 3);
        const uint32_t sw8 = static_cast<uint32_t>((ut >> 2) & 7);
        const uint32_t lo_off = ((2u * c) ^ sw8) << 4;
        const uint32_t hi_off = ((2u * c + 1u) ^ sw8) << 4;
        int total = 0;                                  // stages this CTA runs
        for (int u = first_tile; u < num_units; u += tile_step) {
            const Unit w = unit_at(u, split_tiles, splits, num_kp);
            total += (w.kp1 - w.kp0) * C::PSUB;
        }
        for (int n = ug; n < total; n += C::UG) {
            const int np = n / C::PSUB, sub = n % C::PSUB;   // packed stage, K-block in it
            const int ps = np % C::SP, us = n % C::SU;
            const uint32_t pph = (np / C::SP) & 1, uph = (n / C::SU) & 1;
            if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) break;
            if (!ptx::mbar_wait(empty_u(us), uph ^ 1, abort_flag)) break;
            const uint32_t pa = sbase + C::OFF_PA + ps * C::PA;
            const uint32_t pb = sbase + C::OFF_PB + ps * C::PB;
            const uint32_t ua = sbase + C::OFF_UA + us * C::UA;
            const uint32_t ub = sbase + C::OFF_UB + us * C::UB;
            uint4 w[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int row = (ut >> 2) + kRowStep * i;   // rows of A, then rows of B
                if (row < BM + BN) {
                    const uint32_t src = row < BM ? pa + row * C::PKB : pb + (row - BM) * C::PKB;
                    w[i] = lds128(src + sub * BKP + c * 16);
                }
            }
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int row = (ut >> 2) + kRowStep * i;
                if (row < BM + BN) {
                    const uint32_t dst = row < BM ? ua + row * 128 : ub + (row - BM) * 128;
                    const uint32_t hm = 0xF0F0F0F0u;
                    sts128(dst + lo_off, (w[i].x << 4) & hm, (w[i].y << 4) & hm,
                           (w[i].z << 4) & hm, (w[i].w << 4) & hm);
                    sts128(dst + hi_off, w[i].x & hm, w[i].y & hm, w[i].z & hm, w[i].w & hm);
                }
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(empty_p(ps));
                ptx::mbar_arrive(full_u(us));
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    // A pair's CTAs leave together: CTA 0's MMAs read CTA 1's shared memory
    // and TMEM, and CTA 1 arrives on CTA 0's barriers.
    if constexpr (PAIR) ptx::cluster_sync();
    ptx::tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        ptx::tmem_dealloc<C::CG>(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace gemm

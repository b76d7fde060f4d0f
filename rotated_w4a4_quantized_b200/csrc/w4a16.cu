// w4a16.cu -- the W4A16 variant (include/convrot_w4a16.h): bf16 activations
// rotated by the same block Hadamard as the weights, times the packed INT4
// weights, on the sm_100a tensor cores (tcgen05.mma kind::f16, bf16 x bf16
// -> fp32 in TMEM).  Built as its own library (libconvrot_w4a16.so), so it
// has its own device error word.
//
// What it computes ("convrot-mlx" README, "What is included": the W4A16
// TensorOps path beside W4A4; "Requirements": BF16 x INT4 products):
//   xr[m][k] = bf16_rne((x_m R)[k]),  R = I_G (x) H_n  (as in the W4A4 prep),
//   y[m][n]  = bf16_rne((sum_k xr[m][k] q[n][k]) * sw[n] + b[n]).
//
// Kernels:
//   rotate_bf16_kernel  the W4A4 prep kernel's row loop and butterflies
//                       (prep.cuh helpers), writing each rotated value
//                       rounded to bf16 instead of quantising the row;
//   w4a16_gemm_kernel   persistent output tiles, one CTA per SM: 128 token
//                       rows by 256 weight rows, or for few tokens 128
//                       weight rows (on the MMA's M side) by 16, 32 or 64
//                       token rows.
//
// GEMM roles (448 threads):
//   warp 0        TMA producer: per stage (one or two 64-deep K-blocks)
//                 the xr tiles [TN rows x 128 B], 128-byte swizzled,
//                 straight into the MMA layout, and the packed weight tile
//                 [WT rows x 32 or 64 B];
//   warp 1        TMEM allocator and MMA issuer (one thread): 4 MMAs of
//                 K = 16 per K-block into one of two fp32 accumulators;
//   warps 2..5    epilogue, one per TMEM lane quarter: tcgen05.ld, scale,
//                 bias, bf16, stores;
//   warps 6..13   widening: packed codes -> bf16 codes in the swizzled
//                 K-major layout of the MMA's weight operand.
//
// Widening a code to bf16 without the conversion unit: for a nibble u
// (the 4-bit two's complement code c), u ^ 8 = c + 8 in [0, 15], and the
// bf16 pattern 0x4300 | (c + 8) is the number 128 + c + 8 exactly (the bf16
// spacing in [128, 256) is 1).  One bf16x2 fused multiply-add by 1 with
// addend -136 then gives c exactly in both halves.  A packed word w holds
// codes 2j (low nibble of byte j) and 2j + 1 (high nibble); a byte permute
// of w and w >> 4 puts the two nibbles of byte j at bits 0..3 and 16..19,
// so output word j holds codes (2j, 2j + 1): the natural K order, the same
// as the activation rows, with no repacking of the weights.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <initializer_list>
#include <mutex>

#include "../../include/convrot_w4a16.h"
#include "prep.cuh"
#include "ptx.cuh"

namespace w4a16 {

// ------------------------------------------------------------------ rotation

// bf16 pair (round to nearest even), low half = first value.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Persistent over rows like the W4A4 prep kernel: K/64 threads per CTA,
// thread t owns 64 channels; the next row's copy into the stage buffer
// overlaps the current row's arithmetic.
template <int G>
__global__ void __launch_bounds__(prep::kMaxThreads)
rotate_bf16_kernel(const uint16_t *__restrict__ x, int M, int K, uint16_t *__restrict__ xr) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 1/sqrt(G), exact

    // K * 2 bytes of stage buffer, then (group 256) K * 4 bytes of exchange
    extern __shared__ uint4 stage[];

    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                     // K / 64
    const int warp = t >> 5;
    const int warp_lanes = min(32, nthreads - warp * 32);
    const uint32_t mask = warp_lanes == 32 ? 0xFFFFFFFFu : ((1u << warp_lanes) - 1u);
    const int row_chunks = nthreads * 8;                 // 16-byte chunks per row
    const uint32_t stage_s = ptx::smem_u32(stage);

    // chunk c of owner thread o's 128-byte slice lands at o * 8 + (c ^ (o mod 8))
    auto issue_row = [&](int r) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(r) * K);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int g = t + j * nthreads;
            const int owner = g >> 3, c = g & 7;
            prep::cp_async16(stage_s + static_cast<uint32_t>((owner * 8 + (c ^ (owner & 7))) * 16),
                             src + g);
        }
    };

    int row = blockIdx.x;
    if (row < M) issue_row(row);
    prep::cp_async_commit();
    // The GEMM that follows sets up while this grid runs; it reads xr only
    // after its griddepcontrol.wait (this whole grid complete).
    ptx::launch_dependents();
    for (; row < M; row += gridDim.x) {
        const int next = row + gridDim.x;
        prep::cp_async_wait_all();
        __syncthreads();

        float v[prep::kElemsPerThread];
        prep::load_row(stage, t, v);
        __syncthreads();          // the stage buffer is free again
        if (next < M) issue_row(next);
        prep::cp_async_commit();

        prep::rotate_row<G>(v, reinterpret_cast<float4 *>(stage + row_chunks), t, mask);

        // registers 16 b .. 16 b + 15 hold 16 consecutive channels
        uint16_t *dst = xr + static_cast<size_t>(row) * K;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                w[j] = bf16x2_rn(v[16 * b + 2 * j] * kNorm, v[16 * b + 2 * j + 1] * kNorm);
            uint4 *d = reinterpret_cast<uint4 *>(dst + prep::row_chan<G>(t, 16 * b));
            d[0] = make_uint4(w[0], w[1], w[2], w[3]);
            d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

// ------------------------------------------------------------------ GEMM

constexpr int KB = 64;                   // K per block: one 128-byte bf16 row
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpEpi0 = 2, kEpiWarps = 4;
constexpr int kWarpUnp0 = kWarpEpi0 + kEpiWarps, kUnpWarps = 8;
constexpr int kThreads = (kWarpUnp0 + kUnpWarps) * 32;   // 448

// Tile forms.  TN = token rows of a tile, WT = weight rows.
//   !SWAP (TN = 128, WT = 256): the token rows are the MMA's M side (A = xr,
//     loaded by TMA) and the 256 weight rows its N side (B = widened
//     weights).  Both operands come from shared memory, so the wide N side
//     halves the xr bytes read per MMA flop (a 128 x 128 tile needs the
//     whole 128 B/cycle of shared-memory bandwidth at the tensor peak).  One
//     K-block per stage leaves room for five ring stages and three widened
//     ones beside the 32 KB widened K-block.
//   SWAP (TN = 16, 32, 64: few tokens; WT = 128): the weight rows are the M
//     side (A = widened weights) and the token rows the N side (B = xr), so a
//     decode-size call still streams its weights through 128-row tiles; they
//     use the room their small token tiles leave for a deeper ring of packed
//     weights (8 or 6 stages).  Measured on 1 x 4096 -> 14336: one K-block
//     per stage with six widened stages and a 12-deep ring was slower (897
//     against 1000 GB/s of weight stream) than two K-blocks per stage with
//     two widened stages.
template <int TN, bool SWAP>
struct Cfg {
    static_assert(SWAP ? (TN == 16 || TN == 32 || TN == 64) : TN == 128, "tile forms");
    static constexpr int WT = SWAP ? 128 : 256;          // weight rows per tile
    static constexpr int MMA_N = SWAP ? TN : WT;
    static constexpr int KBS = SWAP ? 2 : 1;             // K-blocks per stage
    static constexpr int PKB = KB * KBS / 2;             // packed weight bytes per row per stage
    static constexpr int CPR = PKB / 16;                  // 16-byte packed chunks per row
    static constexpr int SU = SWAP ? 2 : 3;              // widened weight stages
    static constexpr int UB_KB = WT * 128;               // one widened K-block tile
    static constexpr int PB_ST = WT * PKB;               // packed weights of a stage
    static constexpr int UB_ST = KBS * UB_KB;            // widened weights of a stage
    static constexpr int XR_KB = TN * 128;               // one xr K-block tile
    static constexpr int XR_ST = KBS * XR_KB;
    static constexpr int SP = !SWAP ? 5 : TN <= 32 ? 8 : 6;   // ring stages (xr + packed weights)
    static_assert((WT * CPR) % (kUnpWarps * 32) == 0, "the widening covers whole stages");
    static constexpr int ACC = MMA_N < 32 ? 32 : MMA_N;  // TMEM columns per accumulator
    static constexpr int TMEM_COLS = 2 * ACC;            // two accumulators (power of two)
    static constexpr int OFF_XR = 0;                      // 1024-aligned tiles first
    static constexpr int OFF_UB = OFF_XR + SP * XR_ST;
    static constexpr int OFF_PB = OFF_UB + SU * UB_ST;
    static constexpr int OFF_BAR = OFF_PB + SP * PB_ST;
    static constexpr int NUM_BARS = 2 * SP + 2 * SU + 5;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + slack for 1024 alignment
    static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory limit");
    static_assert(XR_KB % 1024 == 0 && UB_KB % 1024 == 0 && PB_ST % 1024 == 0,
                  "swizzled tiles stay 1024-aligned");
};

// Instruction descriptor of tcgen05.mma kind::f16: D fp32, A and B bf16,
// both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4)                                   // D format f32
           | (1u << 7)                                 // A format bf16
           | (1u << 10)                                // B format bf16
           | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 x bf16 -> f32, K = 16.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

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

// Codes (2j, 2j + 1) of the packed word w (s = w >> 4) as a bf16 pair.
__device__ __forceinline__ uint32_t widen_pair(uint32_t w, uint32_t s, uint32_t sel) {
    const uint32_t biased = (__byte_perm(w, s, sel) & 0x000F000Fu) ^ 0x43084308u;   // 136 + c
    uint32_t r;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;"
        : "=r"(r)
        : "r"(biased), "r"(0x3F803F80u) /* 1, 1 */, "r"(0xC308C308u) /* -136, -136 */);
    return r;
}

// The four bf16 pairs (eight codes, natural order) of one packed word.
__device__ __forceinline__ void widen_word(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t s = w >> 4;
    o[0] = widen_pair(w, s, 0x4400u);
    o[1] = widen_pair(w, s, 0x5511u);
    o[2] = widen_pair(w, s, 0x6622u);
    o[3] = widen_pair(w, s, 0x7733u);
}

// tmA: xr bf16 [M][K], box 64 x TN, 128-byte swizzle.  tmB: qw u8
// [N][K/2], box 64 B x 128, no swizzle (3-D over the block-major repacked
// layout when wrep).  K % 64 == 0.
template <int TN, bool SWAP>
__global__ void __launch_bounds__(kThreads, 1)
w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  int M, int N, int K, int wrep, const float *__restrict__ sw,
                  const uint16_t *__restrict__ bias, uint16_t *__restrict__ y) {
    using C = Cfg<TN, SWAP>;
    constexpr int SP = C::SP, SU = C::SU, KBS = C::KBS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full_p = [&](int s) { return bar0 + 8u * s; };
    auto empty_p = [&](int s) { return bar0 + 8u * (SP + s); };
    auto full_u = [&](int s) { return bar0 + 8u * (2 * SP + s); };
    auto empty_u = [&](int s) { return bar0 + 8u * (2 * SP + SU + s); };
    auto acc_full = [&](int b) { return bar0 + 8u * (2 * SP + 2 * SU + b); };
    auto acc_empty = [&](int b) { return bar0 + 8u * (2 * SP + 2 * SU + 2 + b); };
    const uint32_t drain_bar = bar0 + 8u * (2 * SP + 2 * SU + 4);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SP; ++s) {
            ptx::mbar_init(full_p(s), 1);
            // the widening warps release the packed part, the MMAs the xr part
            ptx::mbar_init(empty_p(s), kUnpWarps + 1);
        }
        for (int s = 0; s < SU; ++s) {
            ptx::mbar_init(full_u(s), kUnpWarps);
            ptx::mbar_init(empty_u(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(acc_full(b), 1);
            ptx::mbar_init(acc_empty(b), kEpiWarps);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWarpTma && lane == 0) {
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc<1>(sbase + C::OFF_MISC, C::TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // xr comes from the preceding kernel (programmatic dependent launch)
    ptx::grid_dependency_wait();

    const int tiles_a = (M + TN - 1) / TN;           // token tiles
    const int tiles_b = (N + C::WT - 1) / C::WT;     // weight tiles
    const int num_tiles = tiles_a * tiles_b;
    const int first_tile = static_cast<int>(blockIdx.x);
    const int tile_step = static_cast<int>(gridDim.x);
    const int nkb = K / KB;                          // K-blocks per tile
    const int num_kp = (nkb + KBS - 1) / KBS;        // stages per tile
    const int my_tiles = num_tiles > first_tile ? (num_tiles - 1 - first_tile) / tile_step + 1 : 0;

    if (warp == kWarpTma) {
        int ps = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = first_tile; lane == 0 && tile < num_tiles && ok; tile += tile_step) {
            const int ta = tile % tiles_a, tb = tile / tiles_a;
            for (int kp = 0; kp < num_kp; ++kp) {
                if (!ptx::mbar_wait(empty_p(ps), ph ^ 1, abort_flag)) { ok = false; break; }
                // a last stage past the end of K carries one K-block: its
                // second xr tile is not loaded (and not multiplied); the
                // packed tile's missing half reads as zeros
                const int nk = min(KBS, nkb - kp * KBS);
                ptx::mbar_arrive_expect_tx(full_p(ps), static_cast<uint32_t>(nk * C::XR_KB + C::PB_ST));
                for (int i = 0; i < nk; ++i)
                    ptx::tma_load_2d(sbase + C::OFF_XR + ps * C::XR_ST + i * C::XR_KB, &tmA,
                                     full_p(ps), (kp * KBS + i) * KB, ta * TN);
                ptx::tma_load_rows(sbase + C::OFF_PB + ps * C::PB_ST, &tmB, full_p(ps),
                                   kp * C::PKB, tb * C::WT, wrep);
                if (++ps == SP) { ps = 0; ph ^= 1; }
            }
        }
        if (!ok) {
            // let copies already in flight land before the CTA exits
            for (int s = 0; s < SP; ++s) {
                volatile int never = 0;
                ptx::mbar_wait(full_p(s), ph ^ (s < ps ? 0u : 1u), &never, 10000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        const bool issuer = lane == 0;
        constexpr uint32_t idesc = idesc_bf16(128, C::MMA_N);
        int ps = 0, us = 0;
        uint32_t pph = 0, uph = 0;
        int local = 0;
        bool ok = true;
        for (int tile = first_tile; issuer && tile < num_tiles && ok; tile += tile_step, ++local) {
            const int b = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            if (!ptx::mbar_wait(acc_empty(b), aph ^ 1, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t d = tmem_base + static_cast<uint32_t>(b * C::ACC);
            for (int kp = 0; kp < num_kp; ++kp) {
                if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) { ok = false; break; }
                if (!ptx::mbar_wait(full_u(us), uph, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                const int nk = min(KBS, nkb - kp * KBS);
                const uint32_t x0 = sbase + C::OFF_XR + ps * C::XR_ST;
                const uint32_t w0 = sbase + C::OFF_UB + us * C::UB_ST;
                for (int i = 0; i < nk; ++i) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t xd = ptx::sw128_kmajor_desc(x0 + i * C::XR_KB + 32 * j);
                        const uint64_t wd = ptx::sw128_kmajor_desc(w0 + i * C::UB_KB + 32 * j);
                        mma_bf16_ss(d, SWAP ? wd : xd, SWAP ? xd : wd, idesc,
                                    (kp | i | j) != 0 ? 1u : 0u);
                    }
                }
                ptx::tc_commit<1>(empty_p(ps));
                ptx::tc_commit<1>(empty_u(us));
                if (++ps == SP) { ps = 0; pph ^= 1; }
                if (++us == SU) { us = 0; uph ^= 1; }
            }
            if (ok) ptx::tc_commit<1>(acc_full(b));
        }
        // every MMA this thread issued completes before TMEM is released
        if (issuer) {
            ptx::tc_commit<1>(drain_bar);
            volatile int never = 0;
            ptx::mbar_wait(drain_bar, 0, &never, 100000000ull);
        }
    } else if (warp < kWarpUnp0) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter ..
        int local = 0;
        for (int tile = first_tile; tile < num_tiles; tile += tile_step, ++local) {
            const int ta = tile % tiles_a, tb = tile / tiles_a;
            const int b = local & 1;
            const uint32_t aph = (local >> 1) & 1;
            if (!ptx::mbar_wait(acc_full(b), aph, abort_flag)) break;
            ptx::tc_fence_after();
            if constexpr (SWAP) {
                // lane = output column n (a weight row), columns = tokens
                const int n = tb * C::WT + quarter * 32 + lane;
                const float swn = n < N ? sw[n] : 0.0f;
                const float bn = (bias && n < N) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16)
                                                 : 0.0f;
#pragma unroll 1
                for (int c0 = 0; c0 < C::ACC; c0 += 32) {
                    uint32_t v[32];
                    __syncwarp();   // tcgen05.ld is warp-collective
                    ptx::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                                static_cast<uint32_t>(b * C::ACC + c0),
                                            v);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = ta * TN + c0 + j;
                        if (c0 + j < TN && m < M && n < N)
                            y[static_cast<size_t>(m) * N + n] = static_cast<uint16_t>(
                                bf16x2_rn(__fadd_rn(__fmul_rn(__uint_as_float(v[j]), swn), bn), 0.0f));
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(acc_empty(b));
                continue;
            }
            const int m = ta * TN + quarter * 32 + lane;      // this lane's output row
#pragma unroll 1
            for (int c0 = 0; c0 < C::WT; c0 += 32) {
                const int n0 = tb * C::WT + c0;
                uint32_t v[32];
                __syncwarp();   // tcgen05.ld is warp-collective
                ptx::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                            static_cast<uint32_t>(b * C::ACC + c0),
                                        v);
                ptx::tmem_ld_wait();
                // column parameters: lane l fetches column n0 + l, then broadcast
                const int nl = n0 + lane;
                const float swl = nl < N ? sw[nl] : 0.0f;
                const float bl = (bias && nl < N) ? __uint_as_float(static_cast<uint32_t>(bias[nl]) << 16)
                                                  : 0.0f;
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float s0 = __shfl_sync(0xFFFFFFFFu, swl, j);
                    const float s1 = __shfl_sync(0xFFFFFFFFu, swl, j + 1);
                    const float c0b = __shfl_sync(0xFFFFFFFFu, bl, j);
                    const float c1b = __shfl_sync(0xFFFFFFFFu, bl, j + 1);
                    const float f0 = __fadd_rn(__fmul_rn(__uint_as_float(v[j]), s0), c0b);
                    const float f1 = __fadd_rn(__fmul_rn(__uint_as_float(v[j + 1]), s1), c1b);
                    pk[j / 2] = bf16x2_rn(f0, f1);
                }
                if (m < M) {
                    uint16_t *o = y + static_cast<size_t>(m) * N + n0;
                    if (n0 + 32 <= N && (N & 7) == 0) {
                        uint4 *o4 = reinterpret_cast<uint4 *>(o);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            o4[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (n0 + j < N) o[j] = static_cast<uint16_t>(pk[j / 2] >> (16 * (j & 1)));
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(acc_empty(b));
        }
    } else {
        // ------------------------------------------------------------ widening
        // Stage = WT rows x CPR packed chunks of 16 bytes (chunk p = codes
        // 32p .. 32p + 31 = half p & 1 of K-block p >> 1).  Thread ut takes
        // chunks ut, ut + 256, ...: a quarter warp reads 128 contiguous
        // packed bytes (two 64-byte rows, or four 32-byte rows) and writes 8
        // distinct 16-byte positions of the 128-byte swizzle pattern per
        // store: with two K-blocks per stage the store order rotates by 2
        // with the K-block and the two rows have opposite swizzle parity;
        // with one, the four rows' swizzle phases differ in their low bits.
        const int ut = threadIdx.x - kWarpUnp0 * 32;
        const int total = my_tiles * num_kp;
        constexpr int kPer = C::WT * C::CPR / (kUnpWarps * 32);
        for (int n = 0; n < total; ++n) {
            const int ps = n % SP, us = n % SU;
            const uint32_t pph = (n / SP) & 1, uph = (n / SU) & 1;
            if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) break;
            if (!ptx::mbar_wait(empty_u(us), uph ^ 1, abort_flag)) break;
            const uint32_t pb = sbase + C::OFF_PB + ps * C::PB_ST;
            const uint32_t ub = sbase + C::OFF_UB + us * C::UB_ST;
#pragma unroll
            for (int it = 0; it < kPer; ++it) {
                const int idx = ut + it * kUnpWarps * 32;
                const int row = idx / C::CPR, p = idx % C::CPR;
                const uint4 w = lds128(pb + static_cast<uint32_t>(row * C::PKB + p * 16));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                const int kbi = p >> 1;
                const uint32_t half = static_cast<uint32_t>(p & 1);
                const uint32_t swz = static_cast<uint32_t>(row & 7);
                const uint32_t dst = ub + static_cast<uint32_t>(kbi * C::UB_KB + row * 128);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    // packed word q = widened chunk q; q = (i + 2 kbi) mod 4 = i ^ 2 kbi
                    const uint32_t q = static_cast<uint32_t>(i) ^ (2u * static_cast<uint32_t>(kbi));
                    uint32_t o[4];
                    widen_word(kbi ? ws[i ^ 2] : ws[i], o);
                    const uint32_t chunk = (4u * half + q) ^ swz;
                    sts128(dst + (chunk << 4), o[0], o[1], o[2], o[3]);
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
    ptx::tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        ptx::tmem_dealloc<1>(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace w4a16

// ====================================================================== host

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmemOptin = 232448;
constexpr int kRotSmemMax = kSmemOptin - 1024;

// `ready` is stored (release) only after every other field is written and
// read (acquire) before any of them, so a thread that sees it set sees the
// whole state; the first set-up on each device runs under g_mu.
struct DeviceState {
    std::atomic<bool> ready{false};
    convrot_status status = CONVROT_OK;
    int num_sms = 0;
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

template <class F>
bool set_smem(F *kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
           cudaSuccess;
}

convrot_status device_setup(int *dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONVROT_ERR_CUDA;
    *dev_out = dev;
    DeviceState &st = g_dev[dev];
    if (st.ready.load(std::memory_order_acquire)) return st.status;
    std::lock_guard<std::mutex> lock(g_mu);
    if (st.ready.load(std::memory_order_relaxed)) return st.status;
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        st.status = CONVROT_ERR_CUDA;
        st.ready.store(true, std::memory_order_release);
        return st.status;
    }
    if (major != 10 || minor != 0) {
        st.status = CONVROT_ERR_UNSUPPORTED;
        st.ready.store(true, std::memory_order_release);
        return st.status;
    }
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn) {
            st.status = CONVROT_ERR_CUDA;
            st.ready.store(true, std::memory_order_release);
            return st.status;
        }
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    bool ok = true;
    ok &= set_smem(w4a16::rotate_bf16_kernel<64>, kRotSmemMax);
    ok &= set_smem(w4a16::rotate_bf16_kernel<256>, kRotSmemMax);
    ok &= set_smem(w4a16::w4a16_gemm_kernel<128, false>, w4a16::Cfg<128, false>::SMEM_BYTES);
    ok &= set_smem(w4a16::w4a16_gemm_kernel<16, true>, w4a16::Cfg<16, true>::SMEM_BYTES);
    ok &= set_smem(w4a16::w4a16_gemm_kernel<32, true>, w4a16::Cfg<32, true>::SMEM_BYTES);
    ok &= set_smem(w4a16::w4a16_gemm_kernel<64, true>, w4a16::Cfg<64, true>::SMEM_BYTES);
    st.num_sms = sms;
    st.status = ok ? CONVROT_OK : CONVROT_ERR_CUDA;
    st.ready.store(true, std::memory_order_release);
    return st.status;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// CONVROT_OK when every non-null pointer is device (or managed) memory of
// device `dev`, CONVROT_ERR_NOT_DEVICE otherwise: host memory, another GPU's
// memory, or an address the runtime does not know.  Run before any launch,
// so a bad pointer is never handed to a tensor map or a kernel.
convrot_status check_device_ptrs(int dev, std::initializer_list<const void *> ptrs) {
    for (const void *p : ptrs) {
        if (!p) continue;
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
            cudaGetLastError();   // clear the lookup error (it is not sticky)
            return CONVROT_ERR_NOT_DEVICE;
        }
        if ((a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) || a.device != dev)
            return CONVROT_ERR_NOT_DEVICE;
    }
    return CONVROT_OK;
}
inline size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

convrot_status check_shape(int64_t rows, int64_t K, int group) {
    if (group != 64 && group != 256) return CONVROT_ERR_GROUP;
    if (rows < 0 || K < 64 || K > CONVROT_MAX_K || K % group) return CONVROT_ERR_SHAPE;
    if (rows > (int64_t(1) << 30)) return CONVROT_ERR_SHAPE;
    return CONVROT_OK;
}

convrot_status check_gemm_shape(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 64 || K > CONVROT_MAX_K || K % 64) return CONVROT_ERR_SHAPE;
    if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || M * N > (int64_t(1) << 40))
        return CONVROT_ERR_SHAPE;
    return CONVROT_OK;
}

// Resident rotation CTAs (K/64 threads, K * (2 or 6) bytes) per SM, cached
// in atomics (concurrent first callers store the same value).
int rot_ctas_per_sm(int group, int64_t K) {
    static std::atomic<int> cache[2][prep::kMaxThreads + 1];
    const int T = static_cast<int>(K / prep::kElemsPerThread);
    std::atomic<int> &entry = cache[group == 256][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        const size_t smem = static_cast<size_t>(K) * (group == 256 ? 6 : 2);
        const cudaError_t e =
            group == 64
                ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, w4a16::rotate_bf16_kernel<64>, T, smem)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, w4a16::rotate_bf16_kernel<256>, T, smem);
        slot = (e == cudaSuccess && n > 0) ? n : 1;
        entry.store(slot, std::memory_order_relaxed);
    }
    return slot;
}

convrot_status launch_rotate(int num_sms, const void *x, int64_t M, int64_t K, int group, void *xr,
                             cudaStream_t stream) {
    if (M == 0) return CONVROT_OK;
    const size_t smem = static_cast<size_t>(K) * (group == 256 ? 6 : 2);
    const int64_t resident = static_cast<int64_t>(num_sms) * rot_ctas_per_sm(group, K);
    const dim3 grid(static_cast<unsigned>(M < resident ? M : resident));
    const dim3 block(static_cast<unsigned>(K / prep::kElemsPerThread));
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    uint16_t *out = static_cast<uint16_t *>(xr);
    if (group == 64)
        w4a16::rotate_bf16_kernel<64><<<grid, block, smem, stream>>>(xx, static_cast<int>(M),
                                                                    static_cast<int>(K), out);
    else
        w4a16::rotate_bf16_kernel<256><<<grid, block, smem, stream>>>(xx, static_cast<int>(M),
                                                                     static_cast<int>(K), out);
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// TN token rows per tile; SWAP: the few-token form (weights on the MMA's M side).
template <int TN, bool SWAP>
convrot_status launch_gemm_cfg(int num_sms, const void *xr, const uint8_t *qw, const float *sw,
                               const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                               cudaStream_t stream, bool wrep) {
    using C = w4a16::Cfg<TN, SWAP>;
    CUtensorMap tmA, tmB;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(w4a16::KB), static_cast<cuuint32_t>(TN)};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(xr), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    }
    if (wrep) {
        // the block-major repacked weights: {128 bytes, N rows, ceil(K/256)
        // blocks}; a box of PKB <= 128 bytes stays inside one block
        const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N),
                                    static_cast<cuuint64_t>((K / 2 + 127) / 128)};
        const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(N) * 128};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(C::PKB), static_cast<cuuint32_t>(C::WT), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(qw), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    } else {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(C::PKB),
                                   static_cast<cuuint32_t>(C::WT)};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(qw), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    }
    const int64_t tiles = ((M + TN - 1) / TN) * ((N + C::WT - 1) / C::WT);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(w4a16::kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, w4a16::w4a16_gemm_kernel<TN, SWAP>, tmA, tmB, static_cast<int>(M),
        static_cast<int>(N), static_cast<int>(K), wrep ? 1 : 0, sw,
        static_cast<const uint16_t *>(bias),
        static_cast<uint16_t *>(y));
    return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Up to 64 tokens: the weights take the MMA's 128-row side and the tokens a
// 16-, 32- or 64-wide side; beyond that, 128 x 256 token-by-weight tiles.
convrot_status launch_gemm(int num_sms, const void *xr, const uint8_t *qw, const float *sw,
                           const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                           cudaStream_t stream, bool wrep = false) {
    if (M <= 16) return launch_gemm_cfg<16, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
    if (M <= 32) return launch_gemm_cfg<32, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
    if (M <= 64) return launch_gemm_cfg<64, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
    return launch_gemm_cfg<128, false>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
}

}  // namespace

extern "C" {

convrot_status convrot_w4a16_prepare_act(const void *x_bf16, int64_t M, int64_t K, int group,
                                         void *xr_bf16, convrot_stream_t stream) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if (M == 0) return CONVROT_OK;
    if (!x_bf16 || !xr_bf16) return CONVROT_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(xr_bf16)) return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, xr_bf16})) != CONVROT_OK) return st;
    return launch_rotate(g_dev[dev].num_sms, x_bf16, M, K, group, xr_bf16, stream);
}

size_t convrot_w4a16_workspace_size(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return round256(static_cast<size_t>(M) * static_cast<size_t>(K) * 2);
}

static convrot_status linear_prepared_impl(const void *xr_bf16, const uint8_t *qw,
                                           const float *sw, const void *bias_bf16, int64_t M,
                                           int64_t N, int64_t K, void *y_bf16,
                                           cudaStream_t stream, bool wrep) {
    convrot_status st = check_gemm_shape(M, N, K);
    if (st != CONVROT_OK) return st;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!xr_bf16 || !qw || !sw || !y_bf16) return CONVROT_ERR_NULL;
    if (!aligned16(xr_bf16) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {xr_bf16, qw, sw, bias_bf16, y_bf16})) != CONVROT_OK) return st;
    return launch_gemm(g_dev[dev].num_sms, xr_bf16, qw, sw, bias_bf16, M, N, K, y_bf16, stream,
                       wrep);
}

static convrot_status linear_impl(const void *x_bf16, const uint8_t *qw, const float *sw,
                                  const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                  int group, void *workspace, size_t ws_bytes, void *y_bf16,
                                  cudaStream_t stream, bool wrep) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if ((st = check_gemm_shape(M, N, K)) != CONVROT_OK) return st;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!x_bf16 || !qw || !sw || !y_bf16 || !workspace) return CONVROT_ERR_NULL;
    if (ws_bytes < convrot_w4a16_workspace_size(M, K) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return CONVROT_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, qw, sw, bias_bf16, workspace, y_bf16})) != CONVROT_OK)
        return st;
    if ((st = launch_rotate(g_dev[dev].num_sms, x_bf16, M, K, group, workspace, stream)) !=
        CONVROT_OK)
        return st;
    return launch_gemm(g_dev[dev].num_sms, workspace, qw, sw, bias_bf16, M, N, K, y_bf16, stream,
                       wrep);
}

convrot_status convrot_w4a16_linear_prepared(const void *xr_bf16, const uint8_t *qw,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, void *y_bf16,
                                             convrot_stream_t stream) {
    return linear_prepared_impl(xr_bf16, qw, sw, bias_bf16, M, N, K, y_bf16, stream, false);
}

convrot_status convrot_w4a16_linear_prepared_repacked(const void *xr_bf16, const uint8_t *qw_rep,
                                                      const float *sw, const void *bias_bf16,
                                                      int64_t M, int64_t N, int64_t K,
                                                      void *y_bf16, convrot_stream_t stream) {
    return linear_prepared_impl(xr_bf16, qw_rep, sw, bias_bf16, M, N, K, y_bf16, stream, true);
}

convrot_status convrot_w4a16_linear(const void *x_bf16, const uint8_t *qw, const float *sw,
                                    const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                    int group, void *workspace, size_t ws_bytes, void *y_bf16,
                                    convrot_stream_t stream) {
    return linear_impl(x_bf16, qw, sw, bias_bf16, M, N, K, group, workspace, ws_bytes, y_bf16,
                       stream, false);
}

convrot_status convrot_w4a16_linear_repacked(const void *x_bf16, const uint8_t *qw_rep,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, int group, void *workspace,
                                             size_t ws_bytes, void *y_bf16,
                                             convrot_stream_t stream) {
    return linear_impl(x_bf16, qw_rep, sw, bias_bf16, M, N, K, group, workspace, ws_bytes, y_bf16,
                       stream, true);
}

convrot_status convrot_w4a16_check_device_error(convrot_stream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return CONVROT_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_convrot_error, sizeof v) != cudaSuccess) return CONVROT_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_convrot_error, &zero, sizeof zero) != cudaSuccess)
            return CONVROT_ERR_CUDA;
        return static_cast<convrot_status>(v);
    }
    return CONVROT_OK;
}

}  // extern "C"

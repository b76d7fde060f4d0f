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

    // K * 2 bytes of stage buffer
    extern __shared__ uint4 stage[];

    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                     // K / 64
    const int warp = t >> 5;
    const int warp_lanes = min(32, nthreads - warp * 32);
    const uint32_t mask = warp_lanes == 32 ? 0xFFFFFFFFu : ((1u << warp_lanes) - 1u);
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
        prep::load_row<G>(stage, t, v);
        __syncthreads();          // the stage buffer is free again
        if (next < M) issue_row(next);
        prep::cp_async_commit();

        prep::rotate_row<G>(v, mask);

        // registers 16 b .. 16 b + 15 hold 16 consecutive channels; with
        // group 256 store d writes digit 3 = d, register block d ^ (t mod 4)
        uint16_t *dst = xr + static_cast<size_t>(row) * K;
        uint32_t w[4][8];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                w[b][i] = bf16x2_rn(v[16 * b + 2 * i] * kNorm, v[16 * b + 2 * i + 1] * kNorm);
        const int jg = (G == 256) ? (t & 3) : 0;
#pragma unroll
        for (int d = 0; d < 4; ++d) {
            const int m = d ^ jg;
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = prep::pick4(w[0][i], w[1][i], w[2][i], w[3][i], m);
            uint4 *p = reinterpret_cast<uint4 *>(dst + prep::row_chan<G>(t, 16 * m));
            p[0] = make_uint4(o[0], o[1], o[2], o[3]);
            p[1] = make_uint4(o[4], o[5], o[6], o[7]);
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


// ------------------------------------------------ few tokens, weights in TMEM
// The few-token form of the W4A4 skinny kernel, for bf16 tokens: the packed
// weights are widened to bf16 straight into TMEM (the MMA's A operand,
// 128 lanes = weight rows), so a weight byte is written once by TMA and
// read once from shared memory; the rotated tokens xr are already bf16 and
// go by TMA straight into the 128-byte swizzled K-major layout of the MMA's
// B operand.  CTA i owns weight rows [i R, i R + R) over the whole of K
// (R spreads N over the SMs): one wave, no split K.  A stage is 256 codes:
// 128 packed bytes per weight row, four 64-deep xr K-blocks.
//
// CTA organisation (12 warps):
//   warp 0      weight TMA producer (one thread), a ring as deep as shared
//               memory allows; in the whole-layer call the first stages are
//               requested before waiting for the rotation kernel;
//   warp 2      token TMA producer (one thread), a ring of three;
//   warp 1      TMEM allocator and MMA issuer: 16 MMAs of K = 16 per stage,
//               A from TMEM, B from shared memory;
//   warps 4..11 weight widening, two warps per TMEM lane quarter (thread =
//               weight row = TMEM lane; warp 4 + q takes codes 0..127 of
//               each stage, warp 8 + q codes 128..255), then the epilogue
//               (lane = output column, accumulator columns = tokens).
// Widening: packed chunk p of row r arrives at p ^ (r & 7) (128-byte
// swizzle); its 32 codes become 16 bf16 pairs in natural K order
// (widen_word), TMEM columns 16 p .. 16 p + 15 of the stage.
namespace sk {

constexpr int kWarpTmaW = 0, kWarpMma = 1, kWarpTmaX = 2, kWarpW0 = 4, kWidenWarps = 8;
constexpr int kThreads = (kWarpW0 + kWidenWarps) * 32;   // 384
constexpr int kMaxRows = 128;          // weight rows per CTA: the TMEM lanes
constexpr int kPKB = 128;              // packed weight bytes per row per stage (256 codes)
constexpr int kXKB = 4;                // 64-deep xr K-blocks per stage
constexpr int kSU = 3;                 // TMEM A stages
constexpr int kSX = 3;                 // token stages (from L2)

template <int BN>
struct Cfg {
    static_assert(BN == 16 || BN == 32 || BN == 64, "token tile of 16, 32 or 64");
    static constexpr int XKB = BN * 128;                 // one xr K-block tile (BN rows x 64 bf16)
    static constexpr int XST = kXKB * XKB;               // token stage
    static constexpr int PA = kMaxRows * kPKB;           // weight stage (up to 128 rows)
    static constexpr int SP_FIT = (232448 - (kSX * XST + 2048)) / PA;
    static constexpr int SP = SP_FIT > 12 ? 12 : SP_FIT;
    static_assert(SP >= 3, "at least three weight stages in flight");
    static constexpr int OFF_X = 0;                      // 1024-aligned tiles first
    static constexpr int OFF_PA = OFF_X + kSX * XST;
    static constexpr int OFF_BAR = OFF_PA + SP * PA;
    static constexpr int NUM_BARS = 2 * SP + 2 * kSX + 2 * kSU + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;     // TMEM base, abort flag
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;    // + slack for 1024 alignment
    static constexpr int ACC_COLS = BN < 32 ? 32 : BN;         // read 32 columns at a time
    static constexpr int A_COLS = kPKB;                        // 256 bf16 = 128 columns
    static constexpr int A_OFF = ACC_COLS;
    static constexpr int TMEM_NEED = A_OFF + kSU * A_COLS;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
    static_assert(XKB % 1024 == 0 && PA % 1024 == 0, "swizzled tiles stay 1024-aligned");
    static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory limit");
};

// D[tmem] (+)= A[tmem] * B[smem desc]^T, bf16 x bf16 -> f32, K = 16: A holds
// 8 columns (16 bf16, two per column, low half first) of each of 128 lanes.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// tmX: xr bf16 [M][K], box 64 x BN, 128-byte swizzle.  tmW: qw u8 [N][K/2],
// box 128 B x R rows, 128-byte swizzle (3-D over the repacked layout when
// wrep).  early_w: the weights were complete before the preceding kernel on
// the stream started.  K % 64 == 0; K tails past a stage read zeros.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
w4a16_skinny_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    int R, int early_w, int M, int N, int K, int wrep, const float *__restrict__ sw,
                    const uint16_t *__restrict__ bias, uint16_t *__restrict__ y) {
    using C = Cfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full_a = [&](int s) { return bar0 + 8u * s; };                  // weight stages
    auto empty_a = [&](int s) { return bar0 + 8u * (C::SP + s); };
    auto full_x = [&](int s) { return bar0 + 8u * (2 * C::SP + s); };    // token stages
    auto empty_x = [&](int s) { return bar0 + 8u * (2 * C::SP + kSX + s); };
    const uint32_t bar_u = bar0 + 8u * (2 * C::SP + 2 * kSX);
    auto full_u = [&](int s) { return bar_u + 8u * s; };                 // TMEM A stages
    auto empty_u = [&](int s) { return bar_u + 8u * (kSU + s); };
    const uint32_t acc_full = bar_u + 8u * (2 * kSU);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = static_cast<int>(blockIdx.x) * R;      // first weight row of this CTA
    const int num_kp = (K / 2 + kPKB - 1) / kPKB;         // stages
    const uint32_t a_tx = static_cast<uint32_t>(R * kPKB);

    const int early = early_w ? (num_kp < C::SP ? num_kp : C::SP) : 0;
    if (threadIdx.x == 0) {
        ptx::tma_prefetch_desc(&tmX);
        ptx::tma_prefetch_desc(&tmW);
        for (int s = 0; s < C::SP; ++s) {
            ptx::mbar_init(full_a(s), 1);
            ptx::mbar_init(empty_a(s), kWidenWarps);
        }
        for (int s = 0; s < kSX; ++s) {
            ptx::mbar_init(full_x(s), 1);
            ptx::mbar_init(empty_x(s), 1);     // the MMAs read the tokens in place
        }
        for (int s = 0; s < kSU; ++s) {
            ptx::mbar_init(full_u(s), kWidenWarps);
            ptx::mbar_init(empty_u(s), 1);
        }
        ptx::mbar_init(acc_full, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        for (int kp = 0; kp < early; ++kp) {
            ptx::mbar_arrive_expect_tx(full_a(kp), a_tx);
            ptx::tma_load_rows(sbase + C::OFF_PA + kp * C::PA, &tmW, full_a(kp), kp * kPKB, n0, wrep);
        }
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc<1>(sbase + C::OFF_MISC, C::TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
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

    if (warp == kWarpTmaW) {
        if (lane == 0) {
            if (!early_w) ptx::grid_dependency_wait();
            int kp = early;
            for (; kp < num_kp; ++kp) {
                const int s = kp % C::SP;
                if (!ptx::mbar_wait(empty_a(s), ((kp / C::SP) & 1) ^ 1, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(full_a(s), a_tx);
                ptx::tma_load_rows(sbase + C::OFF_PA + s * C::PA, &tmW, full_a(s), kp * kPKB, n0, wrep);
            }
            if (kp < num_kp) drain(full_a, kp, C::SP);
        }
    } else if (warp == kWarpTmaX) {
        if (lane == 0) {
            ptx::grid_dependency_wait();   // xr comes from the preceding kernel
            int kp = 0;
            for (; kp < num_kp; ++kp) {
                const int s = kp % kSX;
                if (!ptx::mbar_wait(empty_x(s), ((kp / kSX) & 1) ^ 1, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(full_x(s), static_cast<uint32_t>(C::XST));
#pragma unroll
                for (int i = 0; i < kXKB; ++i)   // K-blocks past K arrive as zeros
                    ptx::tma_load_2d(sbase + C::OFF_X + s * C::XST + i * C::XKB, &tmX, full_x(s),
                                     (kp * kXKB + i) * KB, 0);
            }
            if (kp < num_kp) drain(full_x, kp, kSX);
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, BN);
            int us = 0, xs = 0;
            uint32_t uph = 0, xph = 0;
            for (int kp = 0; kp < num_kp; ++kp) {
                if (!ptx::mbar_wait(full_u(us), uph, abort_flag)) break;
                if (!ptx::mbar_wait(full_x(xs), xph, abort_flag)) break;
                ptx::tc_fence_after();
                const uint32_t a0 = tmem_base + static_cast<uint32_t>(C::A_OFF + us * C::A_COLS);
                const uint32_t x0 = sbase + C::OFF_X + xs * C::XST;
#pragma unroll
                for (int j = 0; j < kXKB * KB / 16; ++j)   // A stage: 8 columns per MMA
                    mma_bf16_ts(tmem_base, a0 + static_cast<uint32_t>(8 * j),
                                ptx::sw128_kmajor_desc(x0 + (j >> 2) * C::XKB + 32 * (j & 3)), idesc,
                                (kp | j) != 0 ? 1u : 0u);
                ptx::tc_commit<1>(empty_u(us));
                ptx::tc_commit<1>(empty_x(xs));
                if (++us == kSU) { us = 0; uph ^= 1; }
                if (++xs == kSX) { xs = 0; xph ^= 1; }
            }
            // Also the drain: TMEM is released only after every MMA completed.
            ptx::tc_commit<1>(acc_full);
            volatile int never = 0;
            ptx::mbar_wait(acc_full, 0, &never, 100000000ull);
        }
    } else if (warp >= kWarpW0) {
        const int quarter = warp & 3;                  // TMEM lanes 32 quarter ..
        const int hh = (warp - kWarpW0) >> 2;          // which 128 codes of a stage
        const int r = quarter * 32 + lane;
        const bool live = r < R;
        const uint32_t rsw = static_cast<uint32_t>(r & 7);
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        // ------------------------------------------------- weight widening
        for (int kp = 0; kp < num_kp; ++kp) {
            const int ps = kp % C::SP, us = kp % kSU;
            const uint32_t pph = (kp / C::SP) & 1, uph = (kp / kSU) & 1;
            if (!ptx::mbar_wait(full_a(ps), pph, abort_flag)) break;
            if (!ptx::mbar_wait(empty_u(us), uph ^ 1, abort_flag)) break;
            ptx::tc_fence_after();
            const uint32_t src = sbase + C::OFF_PA + ps * C::PA + r * kPKB;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t t[32];
                if (live) {
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const uint32_t chunk = static_cast<uint32_t>(4 * hh + 2 * half + cc) ^ rsw;
                        const uint4 w = lds128(src + (chunk << 4));
                        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint32_t o[4];
                            widen_word(wv[x], o);
#pragma unroll
                            for (int z = 0; z < 4; ++z) t[16 * cc + 4 * x + z] = o[z];
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) t[i] = 0u;
                }
                __syncwarp();   // tcgen05.st is warp-collective
                ptx::tmem_st_32x32b_x32(
                    lane_base + static_cast<uint32_t>(C::A_OFF + us * C::A_COLS + 64 * hh + 32 * half), t);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(empty_a(ps));
                ptx::mbar_arrive(full_u(us));
            }
        }
        // --------------------------------------------------------- epilogue
        // lane = output column n (a weight row), accumulator columns =
        // tokens; with 64 tokens the two warps of a quarter take 32 each.
        const bool active = BN >= 64 || hh == 0;
        if (active && !*abort_flag && ptx::mbar_wait(acc_full, 0, abort_flag)) {
            ptx::tc_fence_after();
            const int n = n0 + r;
            const bool store = live && n < N;
            const float swn = store ? sw[n] : 0.0f;
            const float bn = (store && bias) ? __uint_as_float(static_cast<uint32_t>(bias[n]) << 16) : 0.0f;
            const int c0 = 32 * hh;
            uint32_t v[32];
            __syncwarp();   // tcgen05.ld is warp-collective
            ptx::tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(c0), v);
            ptx::tmem_ld_wait();
            constexpr int JW = BN < 32 ? BN : 32;
            if (store) {
#pragma unroll
                for (int j = 0; j < JW; ++j) {
                    const int m = c0 + j;
                    if (m < M)
                        y[static_cast<size_t>(m) * N + n] = static_cast<uint16_t>(
                            bf16x2_rn(__fadd_rn(__fmul_rn(__uint_as_float(v[j]), swn), bn), 0.0f));
                }
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

// Weight rows per CTA for N output columns on num_sms SMs (a multiple of 8,
// at most 128).
inline int rows_per_cta(int64_t N, int num_sms) {
    int64_t r = (N + num_sms - 1) / num_sms;
    r = (r + 7) / 8 * 8;
    return static_cast<int>(r < 8 ? 8 : r > kMaxRows ? kMaxRows : r);
}

}  // namespace sk

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
    ok &= set_smem(w4a16::sk::w4a16_skinny_kernel<16>, w4a16::sk::Cfg<16>::SMEM_BYTES);
    ok &= set_smem(w4a16::sk::w4a16_skinny_kernel<32>, w4a16::sk::Cfg<32>::SMEM_BYTES);
    ok &= set_smem(w4a16::sk::w4a16_skinny_kernel<64>, w4a16::sk::Cfg<64>::SMEM_BYTES);
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

// Resident rotation CTAs (K/64 threads, K * 2 bytes) per SM, cached
// in atomics (concurrent first callers store the same value).
int rot_ctas_per_sm(int group, int64_t K) {
    static std::atomic<int> cache[2][prep::kMaxThreads + 1];
    const int T = static_cast<int>(K / prep::kElemsPerThread);
    std::atomic<int> &entry = cache[group == 256][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        const size_t smem = static_cast<size_t>(K) * 2;
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
    const size_t smem = static_cast<size_t>(K) * 2;
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

// The few-token form with the weights widened into TMEM (M <= BN).
// early_w: the weights were complete before the preceding kernel on the
// stream started (the whole-layer call), so the kernel streams them before
// waiting for it.
template <int BN>
convrot_status launch_skinny_cfg(int num_sms, const void *xr, const uint8_t *qw, const float *sw,
                                 const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                                 cudaStream_t stream, bool wrep, bool early_w) {
    using C = w4a16::sk::Cfg<BN>;
    const int R = w4a16::sk::rows_per_cta(N, num_sms);
    CUtensorMap tmX, tmW;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(w4a16::KB), static_cast<cuuint32_t>(BN)};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(xr), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    }
    if (wrep) {
        // the block-major repacked weights: {128 bytes, N rows, ceil(K/256) blocks}
        const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(N),
                                    static_cast<cuuint64_t>((K / 2 + 127) / 128)};
        const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(N) * 128};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(w4a16::sk::kPKB),
                                   static_cast<cuuint32_t>(R), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (g_encode(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(qw), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    } else {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(N)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(w4a16::sk::kPKB),
                                   static_cast<cuuint32_t>(R)};
        const cuuint32_t estr[2] = {1, 1};
        if (g_encode(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(qw), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return CONVROT_ERR_CUDA;
    }
    const int64_t ctas = (N + R - 1) / R;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    cfg.blockDim = dim3(w4a16::sk::kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, w4a16::sk::w4a16_skinny_kernel<BN>, tmX, tmW, R, early_w ? 1 : 0,
        static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), wrep ? 1 : 0, sw,
        static_cast<const uint16_t *>(bias), static_cast<uint16_t *>(y));
    return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// GEMM forms: the automatic choice, the 128 x 256 token-by-weight tiles, and
// the two few-token forms (M <= 64): weights widened in shared memory (the
// 128-row tiles of w4a16_gemm_kernel) or into TMEM (w4a16_skinny_kernel).
enum Form { kFormAuto = 0, kFormTiles = 1, kFormFewSmem = 2, kFormFewTmem = 3 };

// Up to 64 tokens the few-token form with the weights in TMEM; beyond
// that, 128 x 256 token-by-weight tiles.
convrot_status launch_gemm(int num_sms, const void *xr, const uint8_t *qw, const float *sw,
                           const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                           cudaStream_t stream, bool wrep = false, bool early_w = false,
                           int form = kFormAuto) {
    if (form == kFormAuto) form = M <= 64 ? kFormFewTmem : kFormTiles;
    if ((form == kFormFewSmem || form == kFormFewTmem) && M > 64) return CONVROT_ERR_SHAPE;
    if (form == kFormFewTmem) {
        if (M <= 16)
            return launch_skinny_cfg<16>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep, early_w);
        if (M <= 32)
            return launch_skinny_cfg<32>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep, early_w);
        return launch_skinny_cfg<64>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep, early_w);
    }
    if (form == kFormFewSmem) {
        if (M <= 16) return launch_gemm_cfg<16, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
        if (M <= 32) return launch_gemm_cfg<32, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
        return launch_gemm_cfg<64, true>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
    }
    if (form == kFormTiles)
        return launch_gemm_cfg<128, false>(num_sms, xr, qw, sw, bias, M, N, K, y, stream, wrep);
    return CONVROT_ERR_SHAPE;
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
                                           cudaStream_t stream, bool wrep, int form = kFormAuto) {
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
                       wrep, false, form);
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
    // the weights were complete before the rotation kernel started
    return launch_gemm(g_dev[dev].num_sms, workspace, qw, sw, bias_bf16, M, N, K, y_bf16, stream,
                       wrep, true);
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

convrot_status convrot_w4a16_debug_gemm_form(const void *xr_bf16, const uint8_t *qw,
                                             const float *sw, const void *bias_bf16, int64_t M,
                                             int64_t N, int64_t K, int form, void *y_bf16,
                                             convrot_stream_t stream) {
    const bool wrep = (form & CONVROT_TILES_REPACKED) != 0;
    form &= ~CONVROT_TILES_REPACKED;
    if (form < kFormAuto || form > kFormFewTmem) return CONVROT_ERR_SHAPE;
    if ((form == kFormFewSmem || form == kFormFewTmem) && M > 64) return CONVROT_ERR_SHAPE;
    return linear_prepared_impl(xr_bf16, qw, sw, bias_bf16, M, N, K, y_bf16, stream, wrep, form);
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

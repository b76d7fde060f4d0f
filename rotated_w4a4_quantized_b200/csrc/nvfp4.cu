// nvfp4.cu -- the NVFP4 variant (include/convrot_nvfp4.h): rows rotated by
// the block Hadamard of the W4A4 layer, quantised to E2M1 codes with one
// E4M3 scale per 16 values and one fp32 scale per row, multiplied on the
// block-scaled FP4 tensor cores (tcgen05.mma kind::mxf4nvf4, scales read
// from TMEM).  Its own library (libconvrot_nvfp4.so) with its own device
// error word.
//
// Kernels:
//   quant_kernel      one CTA per row (persistent), K/64 threads: the W4A4
//                     prep kernel's row loop and butterflies (prep.cuh
//                     helpers), then per thread four blocks of 16 channels:
//                     block maximum -> E4M3 scale (cvt ... e4m3x2), codes by
//                     cvt ... e2m1x2 (round to nearest even, saturating), the
//                     scales written in the tensor cores' atom layout;
//   nvfp4_gemm_kernel persistent output tiles of 128 tokens x BN = 256 (or,
//                     where that grid is under half a wave, 128) weight
//                     rows, one CTA per SM:
//     warp 0      producer (one thread): per stage of 256 codes, the packed
//                 token and weight tiles by TMA (128-byte swizzle) and the
//                 tiles' scale atoms by TMA as four replicas of each copy
//                 source (see make_sf_map), all on one barrier;
//     warp 1      TMEM allocator and MMA issuer (one thread): per stage it
//                 copies the scales into TMEM (tcgen05.cp 128x256b: lane
//                 quarter q receives replica q, so row n's four scales of one
//                 64-code step sit in lane n mod 32 of every quarter, column
//                 n / 32) and issues four MMAs of K = 64 (M = 128, N = BN)
//                 into one fp32 accumulator of BN columns;
//     warps 2..5  epilogue, one per TMEM lane quarter: tcgen05.ld, (acc * sx)
//                 * sw + b, bf16, stores; then the accumulator is free.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <initializer_list>
#include <mutex>

#include "../../include/convrot_nvfp4.h"
#include "prep.cuh"
#include "ptx.cuh"

namespace nvfp4 {

// ------------------------------------------------------------ conversions

// Eight E2M1 codes of v[0..7], packed low nibble first (v[0] in bits 0..3):
// round to nearest even, saturating at +-6; the sign is kept.
__device__ __forceinline__ uint32_t e2m1x8(const float *v) {
    uint32_t out;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return out;
}

// E4M3 code of t >= 0 (round to nearest even, saturating at 448).
__device__ __forceinline__ uint32_t e4m3_code(float t) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.0f), "f"(t));
    return d & 0xFFu;
}

// The value of an E4M3 code (exact: every E4M3 value is an f16 value).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
    uint32_t h2;
    asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(code));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Byte offset of the scale of row r, block j in the atom layout.
__host__ __device__ __forceinline__ size_t sf_offset(int64_t r, int64_t j, int64_t K) {
    return static_cast<size_t>(((r >> 7) * (K >> 6) + (j >> 2)) * 512 + 16 * (r & 31) +
                               4 * ((r >> 5) & 3) + (j & 3));
}

// ------------------------------------------------------------ quantisation

// Persistent over rows like the W4A4 prep kernel: K/64 threads per CTA,
// thread t owns 64 channels; the next row's copy into the stage buffer
// overlaps the current row's arithmetic.  Shared memory: K * 2 bytes of
// stage (the digit-3 swap of group 256 runs on lane shuffles).
template <int G>
__global__ void __launch_bounds__(prep::kMaxThreads)
quant_kernel(const uint16_t *__restrict__ x, int M, int K, uint8_t *__restrict__ q,
             uint8_t *__restrict__ sf, float *__restrict__ s) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 1/sqrt(G), exact
    extern __shared__ uint4 stage[];
    __shared__ uint32_t red[prep::kMaxThreads / 32];

    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                     // K / 64
    const int warp = t >> 5, lane = t & 31;
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
    // The GEMM that follows sets up while this grid runs; it reads these
    // rows only after its griddepcontrol.wait (this whole grid complete).
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
#pragma unroll
        for (int e = 0; e < prep::kElemsPerThread; ++e) v[e] *= kNorm;   // exact

        const float m = prep::thread_absmax(v);
        uint32_t mb = __reduce_max_sync(mask, __float_as_uint(m));
        if (lane == 0) red[warp] = mb;
        __syncthreads();
        const int nwarps = (nthreads + 31) >> 5;
        for (int w = 0; w < nwarps; ++w) mb = max(mb, red[w]);
        const float a = __uint_as_float(mb);
        const float sr = a > 0.0f ? __fdiv_rn(a, 2688.0f) : 0.0f;
        const float rr = a > 0.0f ? __fdiv_rn(448.0f, a) : 0.0f;
        if (t == 0) s[row] = sr;

        // registers 16 b .. 16 b + 15 hold 16 consecutive channels: one block
        uint32_t words[8], codes[4];
        uint8_t *qrow = q + static_cast<size_t>(row) * (K / 2);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            float bm = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) bm = fmaxf(bm, fabsf(v[16 * b + i]));
            const uint32_t code = e4m3_code(__fmul_rn(bm, rr));
            const float d = __fmul_rn(e4m3_value(code), sr);
            const float inv = d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
            float w8[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w8[i] = __fmul_rn(v[16 * b + i], inv);
            words[2 * b] = e2m1x8(w8);
            words[2 * b + 1] = e2m1x8(w8 + 8);
            codes[b] = code;
        }
        // with group 256 store d writes digit 3 = d, register block d ^ (t mod 4)
        const int jg = (G == 256) ? (t & 3) : 0;
#pragma unroll
        for (int d = 0; d < 4; ++d) {
            const int m = d ^ jg;
            const int c0 = prep::row_chan<G>(t, 16 * m);   // first channel of the block
            sf[sf_offset(row, c0 / 16, K)] =
                static_cast<uint8_t>(prep::pick4(codes[0], codes[1], codes[2], codes[3], m));
            *reinterpret_cast<uint2 *>(qrow + c0 / 2) =
                make_uint2(prep::pick4(words[0], words[2], words[4], words[6], m),
                           prep::pick4(words[1], words[3], words[5], words[7], m));
        }
    }
    // The padding rows of the last 128-row group get scale code 0 (the value
    // 0), so that every byte of sf is a function of x alone.  In an atom, the
    // 16-byte chunk l holds the four scales (one 32-bit word) of each of rows
    // l, l + 32, l + 64, l + 96 of the group: a chunk whose rows are all
    // padding is cleared with one 16-byte store, the padding words of the
    // others one by one.  These stores touch no byte of a real row.  A warp
    // takes whole atoms, a lane the chunks l = lane, lane + (warp's lanes).
    const int m = M & 127;                               // real rows of the last group
    if (m != 0) {
        uint8_t *grp = sf + static_cast<size_t>(M >> 7) * (K / 64) * 512;
        const int nw = (nthreads + 31) >> 5;
        for (int a = warp + static_cast<int>(blockIdx.x) * nw; a < K / 64;
             a += static_cast<int>(gridDim.x) * nw) {
            uint8_t *atom = grp + static_cast<size_t>(a) * 512;
            for (int l = lane; l < 32; l += warp_lanes) {
                const int c0 = l >= m ? 0 : (m - l + 31) / 32;   // first padding word
                if (c0 == 0)
                    *reinterpret_cast<uint4 *>(atom + 16 * l) = make_uint4(0u, 0u, 0u, 0u);
                else
                    for (int c = c0; c < 4; ++c)
                        *reinterpret_cast<uint32_t *>(atom + 16 * l + 4 * c) = 0u;
            }
        }
    }
}

// ------------------------------------------------------------------ GEMM

constexpr int BM = 128;                  // token rows per tile (the MMA's M)
constexpr int PKB = 128;                 // packed bytes per row per stage: 256 codes
constexpr int KB = 4;                    // MMAs (K = 64) per stage
constexpr int A_ST = BM * PKB;           // 16 KB
// Scales are staged for 128-lane copies (tcgen05.cp 128x256b): a copy
// source is 128 rows x 32 bytes, row i = 32 q + l holding lane l's 16 bytes
// of two scale atoms (so each lane quarter q receives the same values, as
// the MMA reads them).  In core-matrix order (8 rows x 16 bytes) with the
// two 16-byte halves 2 KB apart and 8-row groups 128 bytes apart, replica q
// of an atom is the atom's 512 bytes verbatim at half * 2048 + q * 512, so
// one TMA (make_sf_map) fills a whole 4 KB source.
constexpr int SF_SRC = 4096;
constexpr int SFA_ST = (KB / 2) * SF_SRC;   // A: the atoms of steps 2p, 2p + 1 per source
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpEpi0 = 2, kEpiWarps = 4;
constexpr int kThreads = (kWarpEpi0 + kEpiWarps) * 32;   // 192

// Tiles of 128 tokens x BN weight rows (the MMA's N): 256, or 128 where the
// 256-wide grid would leave most SMs idle (few tokens, small layers).
//   BN = 256: a weight copy source holds the two 128-row atoms of one step;
//   BN = 128: like the tokens, the atoms of steps 2p, 2p + 1.
template <int BN>
struct GCfg {
    static_assert(BN == 128 || BN == 256, "128- or 256-wide weight tiles");
    static constexpr int B_ST = BN * PKB;                         // 32 or 16 KB
    static constexpr int SFB_ST = (BN == 256 ? KB : KB / 2) * SF_SRC;
    static constexpr int SP = BN == 256 ? 3 : 4;                   // ring stages of 72 or 48 KB
    static constexpr int OFF_A = 0;                                // 1024-aligned tiles first
    static constexpr int OFF_B = OFF_A + SP * A_ST;
    static constexpr int OFF_SFA = OFF_B + SP * B_ST;
    static constexpr int OFF_SFB = OFF_SFA + SP * SFA_ST;
    static constexpr int OFF_BAR = OFF_SFB + SP * SFB_ST;
    static constexpr int NUM_BARS = 2 * SP + 3;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;       // + slack for 1024 alignment
    static_assert(SMEM_BYTES <= 232448, "exceeds the per-CTA shared memory limit");
    static constexpr int SFB_COLS = BN / 32;                       // TMEM columns per step
    static constexpr int SF_COL = BN;                              // scales after the accumulator
    static constexpr int SF_REGION = KB * 4 + KB * SFB_COLS;       // A then B scales of a stage
    static constexpr int TMEM_NEED = SF_COL + 2 * SF_REGION;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static_assert(TMEM_NEED <= 512, "TMEM holds 512 columns");
};

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1 (1),
// both K-major, E4M3 scales (scale format 0), scale-factor ids 0, M x N,
// dense K = 64.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
    return (1u << 7)                                    // A format E2M1
           | (1u << 10)                                 // B format E2M1
           | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}

// Shared-memory descriptor of a scale copy source for tcgen05.cp: 128 rows
// of 32 bytes, no swizzle, core matrices of 8 rows x 16 bytes, the two
// 16-byte halves of a row 2 KB apart (leading offset), 8-row groups 128
// bytes apart (stride offset).
__device__ __forceinline__ uint64_t sf_src_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);   // start address
    d |= static_cast<uint64_t>(2048 >> 4) << 16;               // leading offset: the second half
    d |= static_cast<uint64_t>(128 >> 4) << 32;                // stride between 8-row groups
    d |= static_cast<uint64_t>(1) << 46;                       // descriptor version (sm_100)
    return d;                                                  // swizzle mode 0: none
}

// TMEM lanes 0..127, 8 columns <- 128 rows x 256 bits of shared memory.
// One instruction instead of the two four-column broadcast copies
// (32x128b.warpx4) it replaces: the tensor pipe spends about the same time
// on a copy of either size.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// One 4 KB scale copy source by TMA (4-D map, box 512 B x 4 replicas x 2 x 1;
// see make_sf_map).
__device__ __forceinline__ void tma_load_sf(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(0), "r"(c2), "r"(c3),
          "r"(bar)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16 E4M3 scales from TMEM.
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// tmA: codes of the tokens [M][K/2], box 128 B x 128 rows, 128-byte swizzle.
// tmB: codes of the weights [N][K/2], box 128 B x BN rows, 128-byte swizzle.
// tmSA, tmSB: the scale atoms of the tokens and of the weights (rows padded
// to 128) as copy-source replicas (make_sf_map); sx, sw: row scales.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmSA,
                  const __grid_constant__ CUtensorMap tmSB,
                  const float *__restrict__ sx, const float *__restrict__ sw,
                  const uint16_t *__restrict__ bias, uint16_t *__restrict__ y, int M, int N, int K) {
    using C = GCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto full_p = [&](int st) { return bar0 + 8u * st; };
    auto empty_p = [&](int st) { return bar0 + 8u * (C::SP + st); };
    const uint32_t acc_full = bar0 + 8u * (2 * C::SP);
    const uint32_t acc_empty = bar0 + 8u * (2 * C::SP + 1);
    const uint32_t drain_bar = bar0 + 8u * (2 * C::SP + 2);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < C::SP; ++st) {
            ptx::mbar_init(full_p(st), 1);
            ptx::mbar_init(empty_p(st), 1);
        }
        ptx::mbar_init(acc_full, 1);
        ptx::mbar_init(acc_empty, kEpiWarps);
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::tma_prefetch_desc(&tmA);
        ptx::tma_prefetch_desc(&tmB);
        ptx::tma_prefetch_desc(&tmSA);
        ptx::tma_prefetch_desc(&tmSB);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc<1>(sbase + C::OFF_MISC, C::TMEM_COLS);
        ptx::tmem_relinquish<1>();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the token operands come from the preceding kernel (programmatic dependent launch)
    ptx::grid_dependency_wait();

    const int tiles_m = (M + BM - 1) / BM, tiles_n = (N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int nkb = K / 64;                          // MMAs over K
    const int num_kp = (nkb + KB - 1) / KB;          // stages per tile

    if (warp == kWarpTma) {
        int ps = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; lane == 0 && ok && tile < num_tiles; tile += gridDim.x) {
            const int ta = tile % tiles_m, tb = tile / tiles_m;
            const int m0 = ta * BM, n0 = tb * BN;
            for (int kp = 0; kp < num_kp; ++kp) {
                if (!ptx::mbar_wait(empty_p(ps), ph ^ 1, abort_flag)) { ok = false; break; }
                const int nk = min(KB, nkb - kp * KB);       // MMA steps of this stage
                const int npairs = (nk + 1) / 2;             // token scale sources
                const int s0 = kp * KB;                      // first scale atom (step)
                // one 4 KB copy source per TMA; steps past K are not requested
                // (a pair's second step past K reads as zeros)
                const int nsrc_b = BN == 256 ? nk : npairs;  // weight scale sources
                ptx::mbar_arrive_expect_tx(full_p(ps),
                                           A_ST + C::B_ST + (npairs + nsrc_b) * SF_SRC);
                ptx::tma_load_2d(sbase + C::OFF_A + ps * A_ST, &tmA, full_p(ps), kp * PKB, m0);
                ptx::tma_load_2d(sbase + C::OFF_B + ps * C::B_ST, &tmB, full_p(ps), kp * PKB, n0);
                for (int pr = 0; pr < npairs; ++pr)
                    tma_load_sf(sbase + C::OFF_SFA + ps * SFA_ST + pr * SF_SRC, &tmSA, full_p(ps),
                                s0 + 2 * pr, m0 / 128);
                for (int j = 0; j < nsrc_b; ++j) {
                    if (BN == 256)       // step s0 + j, both 128-row halves
                        tma_load_sf(sbase + C::OFF_SFB + ps * C::SFB_ST + j * SF_SRC, &tmSB,
                                    full_p(ps), n0 / 128, s0 + j);
                    else                 // steps s0 + 2 j, + 1 of the one 128-row group
                        tma_load_sf(sbase + C::OFF_SFB + ps * C::SFB_ST + j * SF_SRC, &tmSB,
                                    full_p(ps), s0 + 2 * j, n0 / 128);
                }
                if (++ps == C::SP) { ps = 0; ph ^= 1; }
            }
        }
        if (!ok) {
            // let copies already in flight land before the CTA exits
            for (int st = 0; st < C::SP; ++st) {
                volatile int never = 0;
                ptx::mbar_wait(full_p(st), ph ^ (st < ps ? 0u : 1u), &never, 10000000ull);
            }
        }
    } else if (warp == kWarpMma) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_mxf4(BM, BN);
            int ps = 0;
            uint32_t pph = 0;
            int local = 0, kglob = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++local) {
                // the epilogue has read the previous tile's accumulator
                if (!ptx::mbar_wait(acc_empty, (local & 1) ^ 1, abort_flag)) { ok = false; break; }
                ptx::tc_fence_after();
                for (int kp = 0; kp < num_kp; ++kp, ++kglob) {
                    if (!ptx::mbar_wait(full_p(ps), pph, abort_flag)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const int nk = min(KB, nkb - kp * KB);
                    const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(C::SF_COL + (kglob & 1) * C::SF_REGION);
                    const uint32_t sfb_t = sfa_t + KB * 4;
                    const uint32_t sa = sbase + C::OFF_SFA + ps * SFA_ST;
                    const uint32_t sb = sbase + C::OFF_SFB + ps * C::SFB_ST;
                    // step j's scales: token columns sfa_t + 4 j (two steps per
                    // copy); weight columns sfb_t + 8 j (BN = 256: both 128-row
                    // halves of the tile per copy) or sfb_t + 4 j (BN = 128: two
                    // steps per copy)
                    for (int pr = 0; 2 * pr < nk; ++pr)
                        tmem_cp_sf(sfa_t + 8 * pr, sf_src_desc(sa + pr * SF_SRC));
                    for (int j = 0; j < (BN == 256 ? nk : (nk + 1) / 2); ++j)
                        tmem_cp_sf(sfb_t + 8 * j, sf_src_desc(sb + j * SF_SRC));
                    const uint32_t a0 = sbase + C::OFF_A + ps * A_ST, b0 = sbase + C::OFF_B + ps * C::B_ST;
                    for (int j = 0; j < nk; ++j)
                        mma_mxf4(tmem_base, ptx::sw128_kmajor_desc(a0 + 32 * j),
                                 ptx::sw128_kmajor_desc(b0 + 32 * j), idesc, sfa_t + 4 * j,
                                 sfb_t + C::SFB_COLS * j, (kp | j) != 0 ? 1u : 0u);
                    ptx::tc_commit<1>(empty_p(ps));
                    if (++ps == C::SP) { ps = 0; pph ^= 1; }
                }
                if (ok) ptx::tc_commit<1>(acc_full);
            }
            // every MMA this thread issued completes before TMEM is released
            ptx::tc_commit<1>(drain_bar);
            volatile int never = 0;
            ptx::mbar_wait(drain_bar, 0, &never, 100000000ull);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;                // TMEM lanes 32 quarter ..
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int ta = tile % tiles_m, tb = tile / tiles_m;
            if (!ptx::mbar_wait(acc_full, local & 1, abort_flag)) break;
            ptx::tc_fence_after();
            const int m = ta * BM + quarter * 32 + lane;    // this lane's output row
            const float sxm = m < M ? sx[m] : 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                const int n0 = tb * BN + c0;
                uint32_t v[32];
                __syncwarp();   // tcgen05.ld is warp-collective
                ptx::tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                            static_cast<uint32_t>(c0), v);
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
                    const float b0 = __shfl_sync(0xFFFFFFFFu, bl, j);
                    const float b1 = __shfl_sync(0xFFFFFFFFu, bl, j + 1);
                    const float f0 = __fadd_rn(__fmul_rn(__fmul_rn(__uint_as_float(v[j]), sxm), s0), b0);
                    const float f1 = __fadd_rn(__fmul_rn(__fmul_rn(__uint_as_float(v[j + 1]), sxm), s1), b1);
                    pk[j / 2] = bf16x2_rn(f0, f1);
                }
                if (m < M && n0 < N) {
                    uint16_t *o = y + static_cast<size_t>(m) * N + n0;
                    if (n0 + 32 <= N && (N & 7) == 0) {
                        uint4 *o4 = reinterpret_cast<uint4 *>(o);
#pragma unroll
                        for (int qd = 0; qd < 4; ++qd)
                            o4[qd] = make_uint4(pk[4 * qd], pk[4 * qd + 1], pk[4 * qd + 2], pk[4 * qd + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (n0 + j < N) o[j] = static_cast<uint16_t>(pk[j / 2] >> (16 * (j & 1)));
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(acc_empty);
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

}  // namespace nvfp4

// ====================================================================== host

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmemOptin = 232448;
constexpr int kQuantSmemMax = kSmemOptin - 1024;

// `ready` is stored (release) only after every other field is written and
// read (acquire) before any of them; the first set-up of a device runs
// under g_mu.
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
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                             &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess || !fn) {
            st.status = CONVROT_ERR_CUDA;
            st.ready.store(true, std::memory_order_release);
            return st.status;
        }
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    bool ok = true;
    ok &= set_smem(nvfp4::quant_kernel<64>, kQuantSmemMax);
    ok &= set_smem(nvfp4::quant_kernel<256>, kQuantSmemMax);
    ok &= set_smem(nvfp4::nvfp4_gemm_kernel<256>, nvfp4::GCfg<256>::SMEM_BYTES);
    ok &= set_smem(nvfp4::nvfp4_gemm_kernel<128>, nvfp4::GCfg<128>::SMEM_BYTES);
    st.num_sms = sms;
    st.status = ok ? CONVROT_OK : CONVROT_ERR_CUDA;
    st.ready.store(true, std::memory_order_release);
    return st.status;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// CONVROT_OK when every non-null pointer is device (or managed) memory of
// device `dev`, CONVROT_ERR_NOT_DEVICE otherwise.
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

convrot_status check_shape(int64_t rows, int64_t K, int group) {
    if (group != 64 && group != 256) return CONVROT_ERR_GROUP;
    if (rows < 0 || K < 64 || K > CONVROT_MAX_K || K % group || K % 64) return CONVROT_ERR_SHAPE;
    if (rows > (int64_t(1) << 30)) return CONVROT_ERR_SHAPE;
    return CONVROT_OK;
}

// Resident quantisation CTAs (K/64 threads, K * 2 bytes) per SM, cached
// in atomics (concurrent first callers store the same value).
int quant_ctas_per_sm(int group, int64_t K) {
    static std::atomic<int> cache[2][prep::kMaxThreads + 1];
    const int T = static_cast<int>(K / prep::kElemsPerThread);
    std::atomic<int> &entry = cache[group == 256][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        const size_t smem = static_cast<size_t>(K) * 2;
        const cudaError_t e =
            group == 64
                ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quant_kernel<64>, T, smem)
                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nvfp4::quant_kernel<256>, T, smem);
        slot = (e == cudaSuccess && n > 0) ? n : 1;
        entry.store(slot, std::memory_order_relaxed);
    }
    return slot;
}

convrot_status launch_quant(int num_sms, const void *x, int64_t rows, int64_t K, int group,
                            uint8_t *q, uint8_t *sf, float *s, cudaStream_t stream) {
    if (rows == 0) return CONVROT_OK;
    const size_t smem = static_cast<size_t>(K) * 2;
    const int64_t resident = static_cast<int64_t>(num_sms) * quant_ctas_per_sm(group, K);
    int64_t ctas = rows < resident ? rows : resident;
    // With padding rows in the last 128-row group, at least 16 CTAs, so that
    // each warp clears about two scale atoms of it (CTAs past the last row do
    // only that): one CTA clearing all K/64 atoms took ~4 us more at one row.
    if ((rows & 127) != 0 && ctas < 16) ctas = 16;
    const dim3 grid(static_cast<unsigned>(ctas));
    const dim3 block(static_cast<unsigned>(K / prep::kElemsPerThread));
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    if (group == 64)
        nvfp4::quant_kernel<64><<<grid, block, smem, stream>>>(xx, static_cast<int>(rows),
                                                              static_cast<int>(K), q, sf, s);
    else
        nvfp4::quant_kernel<256><<<grid, block, smem, stream>>>(xx, static_cast<int>(rows),
                                                               static_cast<int>(K), q, sf, s);
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

bool make_code_map(CUtensorMap *map, const uint8_t *base, int64_t rows, int64_t K, int box_rows) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(nvfp4::PKB), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The scale atoms of `rows` rows (padded to 128) as tcgen05.cp sources: a
// 4-D view of the atom layout (32-bit elements) whose 128 x 4 x 2 x 1 box is
// one 4 KB source in shared memory, [pair member][replica][atom, 512 bytes].
// The replica dimension has global stride 0: the same atom four times.
//   token side (b_side false): pair member = two consecutive steps,
//     dims {atom, replica, step, row group of 128}, coordinates (step, group);
//   weight side: pair member = two consecutive 128-row groups,
//     dims {atom, replica, group, step}, coordinates (group, step).
// The atom of step s, group g starts at (g * K/64 + s) * 512.
bool make_sf_map(CUtensorMap *map, const uint8_t *sf, int64_t rows, int64_t K, bool b_side) {
    const cuuint64_t ka = static_cast<cuuint64_t>(K / 64);
    const cuuint64_t groups = static_cast<cuuint64_t>((rows + 127) / 128);
    const cuuint64_t dims_a[4] = {128, 4, ka, groups};
    const cuuint64_t str_a[3] = {0, 512, ka * 512};
    const cuuint64_t dims_b[4] = {128, 4, groups, ka};
    const cuuint64_t str_b[3] = {0, ka * 512, 512};
    const cuuint32_t box[4] = {128, 4, 2, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint8_t *>(sf),
                    b_side ? dims_b : dims_a, b_side ? str_b : str_a, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
convrot_status launch_gemm_bn(int num_sms, const uint8_t *qx, const uint8_t *sfx, const float *sx,
                              const uint8_t *qw, const uint8_t *sfw, const float *sw,
                              const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                              cudaStream_t stream) {
    using C = nvfp4::GCfg<BN>;
    CUtensorMap tmA, tmB;
    CUtensorMap tmSA, tmSB;
    // weight copy sources: the two 128-row halves of a step (BN = 256) or
    // two steps of the one 128-row group (BN = 128, as on the token side)
    if (!make_code_map(&tmA, qx, M, K, nvfp4::BM) || !make_code_map(&tmB, qw, N, K, BN) ||
        !make_sf_map(&tmSA, sfx, M, K, false) || !make_sf_map(&tmSB, sfw, N, K, BN == 256))
        return CONVROT_ERR_CUDA;
    const int64_t tiles = ((M + nvfp4::BM - 1) / nvfp4::BM) * ((N + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(nvfp4::kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, nvfp4::nvfp4_gemm_kernel<BN>, tmA, tmB, tmSA, tmSB, sx, sw,
        static_cast<const uint16_t *>(bias), static_cast<uint16_t *>(y), static_cast<int>(M),
        static_cast<int>(N), static_cast<int>(K));
    return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// GEMM forms: automatic, 256- or 128-wide weight tiles.
enum GemmForm { kFormAuto = 0, kForm256 = 1, kForm128 = 2 };

// The automatic width: 128 where twice the 256-wide tiles still fit in one
// wave (few tokens, small layers: twice the SMs then stream the weights),
// else 256 (fewer scale copies per flop).
int auto_width(int64_t M, int64_t N, int num_sms) {
    const int64_t t256 = ((M + nvfp4::BM - 1) / nvfp4::BM) * ((N + 255) / 256);
    return 2 * t256 <= num_sms ? 128 : 256;
}

convrot_status launch_gemm(int num_sms, const uint8_t *qx, const uint8_t *sfx, const float *sx,
                           const uint8_t *qw, const uint8_t *sfw, const float *sw,
                           const void *bias, int64_t M, int64_t N, int64_t K, void *y,
                           cudaStream_t stream, int form = kFormAuto) {
    const int width = form == kForm256 ? 256 : form == kForm128 ? 128 : auto_width(M, N, num_sms);
    if (width == 128)
        return launch_gemm_bn<128>(num_sms, qx, sfx, sx, qw, sfw, sw, bias, M, N, K, y, stream);
    return launch_gemm_bn<256>(num_sms, qx, sfx, sx, qw, sfw, sw, bias, M, N, K, y, stream);
}

convrot_status check_gemm_shape(int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 64 || K > CONVROT_MAX_K || K % 64) return CONVROT_ERR_SHAPE;
    if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || M * N > (int64_t(1) << 40))
        return CONVROT_ERR_SHAPE;
    return CONVROT_OK;
}

}  // namespace

extern "C" {

size_t convrot_nvfp4_scale_bytes(int64_t rows, int64_t K) {
    if (rows <= 0 || K <= 0) return 0;
    return static_cast<size_t>((rows + 127) / 128 * 128) * static_cast<size_t>(K / 16);
}

size_t convrot_nvfp4_workspace_size(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return round256(static_cast<size_t>(M) * static_cast<size_t>(K / 2)) +
           round256(convrot_nvfp4_scale_bytes(M, K)) + round256(static_cast<size_t>(M) * 4);
}

convrot_status convrot_nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t K, int group,
                                      uint8_t *q, uint8_t *sf, float *s,
                                      convrot_stream_t stream) {
    convrot_status st = check_shape(rows, K, group);
    if (st != CONVROT_OK) return st;
    if (rows == 0) return CONVROT_OK;
    if (!x_bf16 || !q || !sf || !s) return CONVROT_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(q) || !aligned16(sf) || !aligned16(s))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, q, sf, s})) != CONVROT_OK) return st;
    return launch_quant(g_dev[dev].num_sms, x_bf16, rows, K, group, q, sf, s, stream);
}

static convrot_status linear_prepared_impl(const uint8_t *qx, const uint8_t *sfx, const float *sx,
                                           const uint8_t *qw, const uint8_t *sfw, const float *sw,
                                           const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                           void *y_bf16, cudaStream_t stream, int form) {
    if (form < kFormAuto || form > kForm128) return CONVROT_ERR_SHAPE;
    convrot_status st = check_gemm_shape(M, N, K);
    if (st != CONVROT_OK) return st;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!qx || !sfx || !sx || !qw || !sfw || !sw || !y_bf16) return CONVROT_ERR_NULL;
    if (!aligned16(qx) || !aligned16(sfx) || !aligned16(sx) || !aligned16(qw) ||
        !aligned16(sfw) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {qx, sfx, sx, qw, sfw, sw, bias_bf16, y_bf16})) != CONVROT_OK)
        return st;
    return launch_gemm(g_dev[dev].num_sms, qx, sfx, sx, qw, sfw, sw, bias_bf16, M, N, K, y_bf16,
                       stream, form);
}

convrot_status convrot_nvfp4_linear_prepared(const uint8_t *qx, const uint8_t *sfx,
                                             const float *sx, const uint8_t *qw,
                                             const uint8_t *sfw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, void *y_bf16, convrot_stream_t stream) {
    return linear_prepared_impl(qx, sfx, sx, qw, sfw, sw, bias_bf16, M, N, K, y_bf16, stream,
                                kFormAuto);
}

convrot_status convrot_nvfp4_debug_gemm_form(const uint8_t *qx, const uint8_t *sfx,
                                             const float *sx, const uint8_t *qw,
                                             const uint8_t *sfw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, int form, void *y_bf16,
                                             convrot_stream_t stream) {
    return linear_prepared_impl(qx, sfx, sx, qw, sfw, sw, bias_bf16, M, N, K, y_bf16, stream,
                                form);
}

convrot_status convrot_nvfp4_linear(const void *x_bf16, const uint8_t *qw, const uint8_t *sfw,
                                    const float *sw, const void *bias_bf16, int64_t M,
                                    int64_t N, int64_t K, int group, void *workspace,
                                    size_t ws_bytes, void *y_bf16, convrot_stream_t stream) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if ((st = check_gemm_shape(M, N, K)) != CONVROT_OK) return st;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!x_bf16 || !qw || !sfw || !sw || !y_bf16 || !workspace) return CONVROT_ERR_NULL;
    if (ws_bytes < convrot_nvfp4_workspace_size(M, K) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return CONVROT_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(qw) || !aligned16(sfw) || !aligned16(sw) ||
        !aligned16(y_bf16) || (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, qw, sfw, sw, bias_bf16, workspace, y_bf16})) !=
        CONVROT_OK)
        return st;
    uint8_t *qx = static_cast<uint8_t *>(workspace);
    uint8_t *sfx = qx + round256(static_cast<size_t>(M) * (K / 2));
    float *sx = reinterpret_cast<float *>(sfx + round256(convrot_nvfp4_scale_bytes(M, K)));
    if ((st = launch_quant(g_dev[dev].num_sms, x_bf16, M, K, group, qx, sfx, sx, stream)) !=
        CONVROT_OK)
        return st;
    return launch_gemm(g_dev[dev].num_sms, qx, sfx, sx, qw, sfw, sw, bias_bf16, M, N, K, y_bf16,
                       stream);
}

convrot_status convrot_nvfp4_check_device_error(convrot_stream_t stream) {
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

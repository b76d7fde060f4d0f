// decode.cuh -- the whole layer for 1..4 tokens in one kernel.
//
// Same result as prep_kernel followed by the GEMM ("convrot-mlx" README,
// "What is included": rotation, activation quantisation, the integer GEMM on
// packed weights, scaling and bias), with the same instructions for every
// step, so the codes, scales and outputs are bit-identical to the two-kernel
// path.
//
// With a handful of tokens the layer is the 0.5 B-per-weight stream and two
// fixed latencies: the prep kernel's, and the hand-off to the GEMM (the
// dependent grid waits for the whole prep grid to complete and flush).  Here
// every CTA prepares the M <= 4 activation rows itself (a few KB) while its
// slice of the weights is already streaming in, so there is one launch and
// no hand-off:
//   * CTA i owns weight rows [i R, i R + R) over the whole of K (R as for the
//     few-token GEMM: the multiple of 8 that spreads N over the SMs); warp 8
//     issues TMA copies of its packed rows into a ring of SP slots, a stage
//     being 512 contiguous bytes (1024 codes) of each of the R rows, loaded
//     as four 128-byte swizzled column blocks on one barrier.  The first SP
//     stages are requested at kernel start, right after the token rows.
//     Wide stages matter: with 128 bytes per row per stage the one-shot
//     29 MB stream of a 4096 x 14336 layer measured 3.9 TB/s, with 512
//     bytes about 5.5 TB/s;
//   * warps 0-7 first prepare the tokens: token m is handled by K/64 threads
//     exactly as in prep_kernel (staged bf16 row, radix-4 butterflies,
//     absmax, round-half-away, nibble packing), in rounds when the rows need
//     more than 256 threads, then widen the packed codes to int8 words in
//     shared memory (16 x code, even and odd codes of each packed word
//     apart, as the GEMM widens them);
//   * then thread (r, h) of warps 0-7 takes weight row r and part h of each
//     128-byte column block (2, 4 or 8 threads per row: see gemv), widens
//     its packed bytes and accumulates sum 256 q_w q_x with dp4a
//     (s8 x s8 -> s32) on the CUDA cores, exactly, in four independent
//     chains (integer sums: any order gives the same result) so that the
//     dp4a latency does not serialise the stage; with <= 4 tokens the tensor
//     core would spend its ~75-cycle minimum per 128-row MMA on 1-4 useful
//     columns, while dp4a needs about one instruction per weight byte per
//     token;
//   * the parts of each row are added and the epilogue (the GEMM's, same
//     arithmetic) writes y.
// Eligible shapes: M <= 4, K a multiple of 2048 up to 16384 (at most 256
// threads per token row; rows beyond what 256 threads hold at once are
// prepared in further rounds), and the rows' buffers fit in shared memory
// beside two ring slots; others take the two-kernel path.
#pragma once

#include "gemm.cuh"
#include "prep.cuh"
#include "skinny.cuh"

namespace decode {

constexpr int kConsumerWarps = 8;                        // 128 rows x 2 K-blocks
constexpr int kWarpTma = kConsumerWarps;
constexpr int kThreads = (kConsumerWarps + 1) * 32;      // 288
constexpr int kRows = skinny::kMaxRows;                  // weight rows per CTA at most
constexpr int kPKB = skinny::kPKB;                       // packed bytes per row per column block
constexpr int kBlocks = 4;                               // column blocks per stage
constexpr int kBarConsumers = 15;                        // named barrier: warps 0-7

// Shared memory of a launch (bytes, without the 1024 alignment slack):
// ring of SP slots of R x 512 bytes | widened tokens (MT x K) | token prep
// areas | K-half partial sums | barriers.  R is a multiple of 8, so every
// slot stays aligned to the 1024-byte swizzle atom.
inline size_t smem_bytes(int MT, int G, int K, int SP, int R) {
    const size_t prep_per_tok = static_cast<size_t>(K) * (G == 256 ? 4 : 2);
    return static_cast<size_t>(SP) * kBlocks * R * kPKB + static_cast<size_t>(MT) * K +
           MT * prep_per_tok + static_cast<size_t>(kConsumerWarps * 32) * MT * 4 + 2 * SP * 8 + 16;
}

// Consumer threads per weight row: 2 for slices of more than 64 rows, 4 for
// 33..64, 8 for up to 32 (small N), so that all 256 consumer threads work.
inline __host__ __device__ int threads_per_row(int R) { return R > 64 ? 2 : R > 32 ? 4 : 8; }

__device__ __forceinline__ void bar_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// The GEMV over the weight ring with NH consumer threads per weight row:
// thread (r = t mod 256/NH, h = t / (256/NH)) takes row r and the 8/NH
// 16-byte chunks h*8/NH .. of every 128-byte column block (chunks 0-3 are
// the block's first K-block of 128 codes, 4-7 its second), widens them and
// accumulates sum 256 q_w q_x with dp4a in four independent chains (integer
// sums: any order gives the same result).  Returns false if a wait gave up.
template <int MT, int NH>
__device__ __forceinline__ bool gemv(uint32_t sbase, int slot, int blk, uint32_t xw_s, int K,
                                     int R, int num_kp, int SP, uint32_t bar0,
                                     volatile int *abort_flag, int (&acc)[MT]) {
    constexpr int RR = kConsumerWarps * 32 / NH;         // rows covered
    constexpr int CPT = 8 / NH;                          // chunks per thread per block
    const int r = threadIdx.x % RR, h = threadIdx.x / RR;
    const uint32_t rsw = static_cast<uint32_t>(r & 7);
    const uint32_t hm = 0xF0F0F0F0u;
    int a4[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) a4[m][c] = 0;
    bool ok = true;
    for (int kp = 0; kp < num_kp; ++kp) {
        const int s = kp % SP;
        if (!ptx::mbar_wait(bar0 + 8u * s, (kp / SP) & 1, abort_flag)) { ok = false; break; }
        if (r < R) {                                     // rows past the slice only wait
#pragma unroll
            for (int q = 0; q < kBlocks; ++q) {
                const uint32_t src = sbase + s * slot + q * blk + r * kPKB;
                // widened tokens of the block: 2 K-blocks x 128 bytes per token
                const uint32_t xb = xw_s + static_cast<uint32_t>((kp * kBlocks + q) * 256);
#pragma unroll
                for (int cc = 0; cc < CPT; ++cc) {
                    const int p = h * CPT + cc;          // chunk of the block
                    const int kbp = p >> 2, c = p & 3;
                    const uint4 wv = gemm::lds128(src + ((static_cast<uint32_t>(p) ^ rsw) << 4));
                    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
                    constexpr int kChains = 4;
                    const int ch = (q * CPT + cc) % kChains;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        // words 4c .. 4c + 3 of K-block kbp: (even, odd) pairs
                        const uint32_t xa = xb + static_cast<uint32_t>(m * K + kbp * 128 + 32 * c);
                        const uint4 x0 = gemm::lds128(xa), x1 = gemm::lds128(xa + 16);
                        const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            a4[m][ch] = __dp4a(static_cast<int>((ww[j] << 4) & hm),
                                               static_cast<int>(xv[2 * j]), a4[m][ch]);
                            a4[m][ch] = __dp4a(static_cast<int>(ww[j] & hm),
                                               static_cast<int>(xv[2 * j + 1]), a4[m][ch]);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar0 + 8u * (SP + s));
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = (a4[m][0] + a4[m][1]) + (a4[m][2] + a4[m][3]);
    return ok;
}

// tmW: packed weights [N][K/2], box 128 B x R rows, 128-byte swizzle (3-D
// over the block-major repacked layout when wrep).
// x: bf16 [M][K]; y: bf16 [M][N]; sw: fp32 [N]; bias: bf16 [N] or null.
template <int MT, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmW, const uint16_t *__restrict__ x, int M,
              int N, int K, int R, int SP, int wrep, const float *__restrict__ sw,
              const uint16_t *__restrict__ bias, uint16_t *__restrict__ y) {
    static_assert(MT == 1 || MT == 2 || MT == 4, "1, 2 or 4 tokens");
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 2^-digits
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const size_t prep_per_tok = static_cast<size_t>(K) * (G == 256 ? 4 : 2);
    const int blk = R * kPKB;                            // one column block of a stage
    const int slot = kBlocks * blk;                      // ring slot bytes
    uint32_t *xw = reinterpret_cast<uint32_t *>(smem + static_cast<size_t>(SP) * slot);
    uint8_t *prep_area = reinterpret_cast<uint8_t *>(xw) + static_cast<size_t>(MT) * K;
    int32_t *accs = reinterpret_cast<int32_t *>(prep_area + MT * prep_per_tok);
    const uint32_t bar0 = ptx::smem_u32(accs + kConsumerWarps * 32 * MT);
    auto full_p = [&](int s) { return bar0 + 8u * s; };
    auto empty_p = [&](int s) { return bar0 + 8u * (SP + s); };
    __shared__ uint32_t red[MT][kConsumerWarps];
    __shared__ float sxs[MT];
    __shared__ int abort_flag_s;
    volatile int *abort_flag = &abort_flag_s;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = static_cast<int>(blockIdx.x) * R;
    const int num_kp = K / (2 * kPKB * kBlocks);         // K is a multiple of 2048
    const uint32_t stage_tx = static_cast<uint32_t>(slot);
    const uint32_t hm = 0xF0F0F0F0u;

    // The token rows are requested first, ahead of the weight burst, so that
    // their preparation is not queued behind it.  Token m is prepared by the
    // K/64 threads of slot m mod tpr, in round m / tpr.
    const int gt = K / prep::kElemsPerThread;            // threads per token (multiple of 32)
    const int tpr = (kConsumerWarps * 32) / gt;          // tokens per round (K <= 16384)
    const int slot_tok = threadIdx.x / gt, t = threadIdx.x % gt;
    if (warp < kWarpTma && slot_tok < tpr) {
        for (int tok = slot_tok; tok < M; tok += tpr) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(tok) * K);
            const uint32_t stg_s = ptx::smem_u32(prep_area + tok * prep_per_tok);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int g = t + j * gt;                // chunk index in the row
                const int owner = g >> 3, c = g & 7;
                prep::cp_async16(stg_s + static_cast<uint32_t>((owner * 8 + (c ^ (owner & 7))) * 16),
                                 src + g);
            }
        }
        prep::cp_async_commit();
    }
    if (threadIdx.x == kWarpTma * 32) {
        ptx::tma_prefetch_desc(&tmW);
        for (int s = 0; s < SP; ++s) {
            ptx::mbar_init(full_p(s), 1);
            ptx::mbar_init(empty_p(s), kConsumerWarps);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
        // The whole ring at once: the weights are this call's input.
        for (int kp = 0; kp < SP && kp < num_kp; ++kp) {
            ptx::mbar_arrive_expect_tx(full_p(kp), stage_tx);
            for (int q = 0; q < kBlocks; ++q)
                ptx::tma_load_rows(sbase + kp * slot + q * blk, &tmW, full_p(kp),
                                   (kp * kBlocks + q) * kPKB, n0, wrep);
        }
    }
    __syncthreads();

    if (warp == kWarpTma) {
        // ------------------------------------------------ producer: the refills
        if (lane == 0) {
            for (int kp = SP; kp < num_kp; ++kp) {
                const int s = kp % SP;
                if (!ptx::mbar_wait(empty_p(s), ((kp / SP) - 1) & 1, abort_flag)) break;
                ptx::mbar_arrive_expect_tx(full_p(s), stage_tx);
                for (int q = 0; q < kBlocks; ++q)
                    ptx::tma_load_rows(sbase + s * slot + q * blk, &tmW, full_p(s),
                                       (kp * kBlocks + q) * kPKB, n0, wrep);
            }
        }
        return;
    }

    // ------------------------------------------------------ token preparation
    for (int tok0 = 0; tok0 < MT; tok0 += tpr) {
        const int tok = tok0 + slot_tok;
        const int bid = 1 + slot_tok;                    // named barrier of the slot
        uint4 *stg = reinterpret_cast<uint4 *>(prep_area + tok * prep_per_tok);
        if (slot_tok >= tpr || tok >= MT) continue;
        if (tok < M) {
            prep::cp_async_wait_all();
            bar_named(bid, gt);                          // the row has landed
            float v[prep::kElemsPerThread];
            prep::load_row<G>(stg, t, v);
            bar_named(bid, gt);                          // the stage may be overwritten
            prep::rotate_row<G>(v, 0xFFFFFFFFu);
            const float m = prep::thread_absmax(v);
            uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
            if (lane == 0) red[tok][t >> 5] = mb;
            bar_named(bid, gt);
            for (int w = 0; w < gt / 32; ++w) mb = max(mb, red[tok][w]);
            const float a_u = __uint_as_float(mb);
            const float inv = a_u > 0.0f ? __fdiv_rn(7.0f, a_u) : 0.0f;
            if (t == 0) sxs[tok] = __fdiv_rn(a_u * kNorm, 7.0f);
            uint32_t packed[8];
            prep::quantize_pack(v, inv, packed);
            // widened words of K-block kb of token tok: xw[(tok * K / 128 + kb) * 32 + 2 i (+1)]
            // = even (odd) codes x 16 of packed word i of the K-block
            uint32_t *xt = xw + static_cast<size_t>(tok) * (K / 4);
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int ch = prep::row_chan<G>(t, 8 * w);
                const int kb = ch >> 7, i = (ch & 127) >> 3;
                *reinterpret_cast<uint2 *>(xt + kb * 32 + 2 * i) =
                    make_uint2((packed[w] << 4) & hm, packed[w] & hm);
            }
        } else {
            // tokens M .. MT-1 multiply as zeros
            uint4 *xt = reinterpret_cast<uint4 *>(xw + static_cast<size_t>(tok) * (K / 4));
            for (int i = t; i < K / 16; i += gt) xt[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    bar_named(kBarConsumers, kConsumerWarps * 32);       // all tokens are ready

    // ---------------------------------------------------------------- GEMV
    // Thread (r, h): weight row r of the slice and part h of every 128-byte
    // column block, with NH threads per row (threads_per_row).
    const int nh = threads_per_row(R);
    int acc[MT];
    bool ok;
    if (nh == 2)
        ok = gemv<MT, 2>(sbase, slot, blk, ptx::smem_u32(xw), K, R, num_kp, SP, bar0, abort_flag, acc);
    else if (nh == 4)
        ok = gemv<MT, 4>(sbase, slot, blk, ptx::smem_u32(xw), K, R, num_kp, SP, bar0, abort_flag, acc);
    else
        ok = gemv<MT, 8>(sbase, slot, blk, ptx::smem_u32(xw), K, R, num_kp, SP, bar0, abort_flag, acc);

    // ------------------------------------------------------------ epilogue
    // The NH parts of each row are added (exact integers) by its part 0.
    const int rr = (kConsumerWarps * 32) / nh;
    const int r = threadIdx.x % rr, h = threadIdx.x / rr;
#pragma unroll
    for (int m = 0; m < MT; ++m) accs[threadIdx.x * MT + m] = acc[m];
    bar_named(kBarConsumers, kConsumerWarps * 32);
    const int n = n0 + r;
    if (ok && h == 0 && r < R && n < N) {
        const float swn = sw[n];
        const float bn = bias ? gemm::bf16_to_f32(bias[n]) : 0.0f;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (m >= M) break;
            int32_t total = acc[m];
            for (int p = 1; p < nh; ++p) total += accs[(p * rr + r) * MT + m];
            y[static_cast<size_t>(m) * N + n] =
                gemm::f32_to_bf16_rne(gemm::epi(static_cast<uint32_t>(total), sxs[m], swn, bn));
        }
    }
}

}  // namespace decode

// prep.cuh -- fused rotation + rowwise absmax INT4 quantisation + packing.
//
// prep_kernel: K/64 threads per CTA, persistent over rows; thread t owns the
// 64 consecutive channels [64t, 64t + 64) of each row it helps with.
// prep16_kernel (end of file): the same steps with 16 channels per thread,
// for launches of up to 1024 rows, where each row's latency is the cost.
//
// Rotation.  Within a group of n = 4^k channels the normalised regular
// Hadamard is H_n = T^{(x)k} / 2^k with T = J - 2I (Comfy-Org/comfy-quants
// issue, section 2: regular Hadamard for N_0 = 4^k; "convrot-mlx" README,
// "What is included": groups of 64 and 256).  Applying T along base-4 digit d
// of the channel index is a radix-4 butterfly: for each quadruple of channels
// that differ only in digit d, y_i = (x_0 + x_1 + x_2 + x_3) - 2 x_i.  The k
// butterflies commute (every factor is the same symmetric T), so they run in
// any order: digits 0, 1, 2 live inside one thread's 64 registers; for
// n = 256 digit 3 spans the 4 threads of the group (four lanes of a warp),
// which swap quarters of their data with lane shuffles so that digit 3 also
// becomes a register stride.  The 1/2^k normalisation is exact and is folded
// into the scale (see below), so the butterflies run on unnormalised values.
//
// Quantisation ("convrot-mlx" README, "What is included": symmetric rowwise
// absmax to [-7, 7]).  With u the unnormalised rotated row and y = u 2^-k:
//   a_u = max|u|, inv = 7 / a_u (fp32, IEEE), s = (a_u 2^-k) / 7,
//   v = u * inv, q = round_half_away(v).
// Because 2^-k scaling is exact, u * (7 / a_u) is bit-identical to
// y * (7 / max|y|).  round_half_away(v) for |v| < 8 is computed as
// trunc(v + sign(v) (0.5 - 2^-25)): adding the largest float below 0.5
// (instead of 0.5) is exactly round-half-away-from-zero on fp32 inputs of
// this range (IEEE addition is symmetric in sign), and |v| <= 7 (1 + 2^-24)
// by construction, so no clamp is needed.  Codes are packed two per byte,
// low nibble = even channel.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace prep {

using ptx::add2;
using ptx::bfly2;
using ptx::mul2;

constexpr int kElemsPerThread = 64;
constexpr int kMaxThreads = 512;   // K <= 32768

// Two signed codes into one byte of the running word:
// result = (acc << 8) | ((hi & 0xF) << 4) | (lo & 0xF), saturating to [-8, 7]
// (codes here are already in [-7, 7]).
__device__ __forceinline__ uint32_t pack_nibbles(int hi, int lo, uint32_t acc) {
    uint32_t d;
    asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(hi), "r"(lo), "r"(acc));
    return d;
}

// Radix-4 butterflies with packed two-wide arithmetic.  Every packed
// operation works on the register pair (v[2i], v[2i+1]) so that values stay
// in the same aligned register pair through all stages.
//
// Digit 0 (stride 1): the quadruple {4q .. 4q+3} is two pairs; their packed
// sum gives (v0+v2, v1+v3), one scalar add completes the quadruple sum.
template <int E>
__device__ __forceinline__ void radix4_digit0(float (&v)[E]) {
#pragma unroll
    for (int b = 0; b < E; b += 4) {
        float p0, p1;
        add2(p0, p1, v[b], v[b + 1], v[b + 2], v[b + 3]);
        const float sum = p0 + p1;
        bfly2(v[b], v[b + 1], sum, sum);
        bfly2(v[b + 2], v[b + 3], sum, sum);
    }
}

// Digits with stride S = 4 or 16: the quadruples starting at b and b + 1
// (b even) run side by side in the two halves of each packed operation.
template <int S, int E>
__device__ __forceinline__ void radix4_stage(float (&v)[E]) {
#pragma unroll
    for (int b = 0; b < E; b += 2) {
        if ((b / S) % 4 != 0) continue;
        float s01a, s01b, s23a, s23b, suma, sumb;
        add2(s01a, s01b, v[b], v[b + 1], v[b + S], v[b + 1 + S]);
        add2(s23a, s23b, v[b + 2 * S], v[b + 1 + 2 * S], v[b + 3 * S], v[b + 1 + 3 * S]);
        add2(suma, sumb, s01a, s01b, s23a, s23b);
#pragma unroll
        for (int j = 0; j < 4; ++j) bfly2(v[b + j * S], v[b + 1 + j * S], suma, sumb);
    }
}

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// All but the most recent of this thread's committed groups have landed.
__device__ __forceinline__ void cp_async_wait_prior() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// ------------------------------------------------------------------------
// The steps of one row, shared by prep_kernel and the fused decode kernel
// (same instructions in the same order, so both give identical codes).
// t is the thread's index among the K/64 threads that handle the row.

// Registers v[0..63] <- the thread's 64 channels of a staged bf16 row (the
// stage layout: chunk c of thread t's 128-byte slice at position c ^ (t & 7)).
// For n = 64 register e holds channel 64 t + e.  For n = 256 the quarters
// come in the order the digit-3 swap of rotate_row needs: registers
// 16 m .. 16 m + 15 hold the thread's quarter m ^ (t mod 4), i.e. slice
// chunks i ^ 2 (t mod 4) for register chunk i.  The read key
// (t mod 8) ^ 2 (t mod 4) still differs between the 8 lanes of a quarter
// warp, so the 128-bit reads stay free of bank conflicts.
template <int G>
__device__ __forceinline__ void load_row(const uint4 *__restrict__ sb, int t,
                                         float (&v)[kElemsPerThread]) {
    const int key = (G == 256) ? ((t & 7) ^ ((t & 3) << 1)) : (t & 7);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 raw = sb[t * 8 + (i ^ key)];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// The unnormalised rotation of the thread's channels (registers as load_row
// leaves them): digits 0-2 in registers; for n = 256 the four threads of a
// group (lanes 4g .. 4g + 3 of one warp, j = t mod 4 the thread's digit 3)
// then swap quarters with lane shuffles so that digit 3 is a register
// stride too, and the last butterfly runs in registers.
//
// Why the sums are unchanged by load_row's quarter order: every radix-4
// butterfly adds its quadruple as (x_0 + x_1) + (x_2 + x_3).  With quarter
// m ^ j in register block m, the digit-2 butterfly pairs blocks {0, 1} and
// {2, 3}, i.e. quarters {j, j ^ 1} = {0, 1} or {2, 3} and the other pair:
// the same two pair sums, added the same way up to the order of operands,
// and IEEE addition is commutative bit for bit.
//
// The swap: in round m = 1, 2, 3 a thread sends block m (its quarter m ^ j,
// which lane j ^ m needs) to lane j ^ m and receives that lane's block m (its
// quarter (j ^ m) ^ m = j).  Every register index is static, so each round
// is 16 shuffles in place.  Afterwards block m holds quarter j of the thread
// with digit 3 = j ^ m, and the digit-3 butterfly pairs those threads as
// {j, j ^ 1} and {j ^ 2, j ^ 3}, again the pairs {0, 1} and {2, 3}.
// mask: the lanes of the warp that take part (whole groups).
template <int G>
__device__ __forceinline__ void rotate_row(float (&v)[kElemsPerThread], uint32_t mask) {
    radix4_digit0(v);
    radix4_stage<4>(v);
    radix4_stage<16>(v);
    if (G == 256) {
#pragma unroll
        for (int m = 1; m < 4; ++m)
#pragma unroll
            for (int r = 0; r < 16; ++r) v[16 * m + r] = __shfl_xor_sync(mask, v[16 * m + r], m);
        radix4_stage<16>(v);
    }
}

// a[m] for a lane-dependent m in 0..3, by selects (registers cannot be
// indexed at run time).  After rotate_row (n = 256) block m of thread t holds
// digit 3 = m ^ (t mod 4); picking block d ^ (t mod 4) in store d makes one
// store instruction cover digit 3 = d of every group, four contiguous runs of
// a group's lanes, instead of four places apart.
__device__ __forceinline__ uint32_t pick4(uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          int m) {
    return (m & 2) ? ((m & 1) ? a3 : a2) : ((m & 1) ? a1 : a0);
}

// Channel of register e of thread t after rotate_row: for n = 256, block
// e / 16 holds digit 3 = (e / 16) ^ j, quarter j = t mod 4 of the group's
// 64-channel blocks.
template <int G>
__device__ __forceinline__ int row_chan(int t, int e) {
    if (G == 64) return t * 64 + e;
    return (t & ~3) * 64 + 64 * ((e >> 4) ^ (t & 3)) + 16 * (t & 3) + (e & 15);
}

// The thread's max |v|: four independent chains of three-input maxima.
template <int E>
__device__ __forceinline__ float thread_absmax(const float (&v)[E]) {
    float mk[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int e = 0; e < E; e += 8)
#pragma unroll
        for (int k = 0; k < 4; ++k) mk[k] = max3(mk[k], fabsf(v[e + 2 * k]), fabsf(v[e + 2 * k + 1]));
    return max3(mk[0], mk[1], fmaxf(mk[2], mk[3]));
}

// Codes q = round_half_away(v * inv), packed two per byte (low nibble =
// even register): packed[w] holds registers 8w .. 8w + 7.
template <int E>
__device__ __forceinline__ void quantize_pack(const float (&v)[E], float inv,
                                              uint32_t (&packed)[E / 8]) {
#pragma unroll
    for (int w = 0; w < E / 8; ++w) {
        int code[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // the product is rounded to fp32 before the offset is added: scalar
            // round-to-nearest operations, which ptxas does not fuse (a packed
            // mul.rn.f32x2 feeding an add.rn.f32x2 becomes one fused
            // multiply-add on sm_100a)
            const float p = __fmul_rn(v[8 * w + j], inv);
            // add (0.5 - 2^-25) with the sign of the product, truncate
            const float c = __uint_as_float((__float_as_uint(p) & 0x80000000u) | 0x3EFFFFFFu);
            code[j] = __float2int_rz(__fadd_rn(p, c));
        }
        uint32_t word = pack_nibbles(code[7], code[6], 0u);
        word = pack_nibbles(code[5], code[4], word);
        word = pack_nibbles(code[3], code[2], word);
        packed[w] = pack_nibbles(code[1], code[0], word);
    }
}

// Stage buffers of prep_kernel: two for n = 256, one for n = 64 (each
// measured faster than the other count on 8192 x 8192: 43.9 against 45.1 us
// for n = 256; for n = 64 one buffer is 5% faster).
__host__ __device__ constexpr int stage_buffers(int G) { return G == 256 ? 2 : 1; }

// MODE 0: quantise + pack (q, s).  MODE 1: write the normalised rotated row
// as fp32 (yrot) instead.
//
// Persistent: CTA b handles rows b, b + gridDim.x, ...  Rows arrive by
// asynchronous copies while the previous row is rotated and quantised.  For
// n = 256, two stage buffers of one bf16 row each: the CTA's next two rows
// are on their way during the arithmetic, and the barrier of the row maximum
// also tells that every warp has read the current buffer, which then
// receives the row after next.  For n = 64, one buffer: the next row is
// requested as soon as the current one is in registers.  Each row is read
// with coalesced 16-byte copies (consecutive threads, consecutive chunks)
// that land so that chunk c of thread t's 128-byte slice sits at position
// c ^ (t mod 8); each thread then reads its own 64 channels with
// conflict-free 128-bit loads (load_row).
template <int G, int MODE>
__global__ void __launch_bounds__(kMaxThreads)
prep_kernel(const uint16_t *__restrict__ x, int M, int K, uint8_t *__restrict__ q,
            float *__restrict__ s, float *__restrict__ yrot, uint32_t *__restrict__ zero,
            int nzero) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    constexpr int kDigits = (G == 64) ? 3 : 4;
    // side job for the GEMM that follows: clear its split counters
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0u;
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 2^-kDigits
    constexpr int NBUF = stage_buffers(G);

    // NBUF stage buffers of K * 2 bytes
    extern __shared__ uint4 stage[];
    __shared__ uint32_t red[kMaxThreads / 32];

    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                     // K / 64
    const int warp = t >> 5, lane = t & 31;
    const int warp_lanes = min(32, nthreads - warp * 32);
    const uint32_t mask = warp_lanes == 32 ? 0xFFFFFFFFu : ((1u << warp_lanes) - 1u);
    const int row_chunks = nthreads * 8;                 // 16-byte chunks per row
    const uint32_t stage_s = ptx::smem_u32(stage);

    auto issue_row = [&](int r, int buf) {
        if (r < M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(r) * K);
            const uint32_t base = stage_s + static_cast<uint32_t>(buf * row_chunks * 16);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int g = t + j * nthreads;          // chunk index in the row
                const int owner = g >> 3, c = g & 7;
                cp_async16(base + static_cast<uint32_t>((owner * 8 + (c ^ (owner & 7))) * 16),
                           src + g);
            }
        }
        cp_async_commit();   // one group per row, empty past the end
    };

    int row = blockIdx.x;
    issue_row(row, 0);
    if (NBUF == 2) issue_row(row + gridDim.x, 1);
    // The GEMM that follows may be scheduled on the SMs this grid leaves
    // free from now on (all of this grid's CTAs are resident: the grid is
    // sized to the resident capacity).  It sets up, and streams weights that
    // do not depend on this grid, but reads these rows only after its
    // griddepcontrol.wait, which waits for this whole grid to complete.
    ptx::launch_dependents();
    for (int it = 0; row < M; row += gridDim.x, ++it) {
        const int b = NBUF == 2 ? (it & 1) : 0;
        uint4 *sb = stage + b * row_chunks;
        // this row's copies (by this thread) have landed ...
        if (NBUF == 2) cp_async_wait_prior();
        else cp_async_wait_all();
        __syncthreads();          // ... and everyone else's

        float v[kElemsPerThread];
        load_row<G>(sb, t, v);
        if (NBUF == 1) {
            __syncthreads();      // the stage buffer is free again
            issue_row(row + gridDim.x, 0);
        }
        rotate_row<G>(v, mask);
        auto chan = [&](int e) -> int { return row_chan<G>(t, e); };

        if (MODE == 1) {
            float *dst = yrot + static_cast<size_t>(row) * K;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<float4 *>(dst + chan(4 * i)) =
                    make_float4(v[4 * i] * kNorm, v[4 * i + 1] * kNorm, v[4 * i + 2] * kNorm,
                                v[4 * i + 3] * kNorm);
            if (NBUF == 2) {
                __syncthreads();  // every warp is done with buffer b
                issue_row(row + 2 * gridDim.x, b);
            }
            continue;
        }

        const float m = thread_absmax(v);
        // non-negative floats order like their bit patterns
        uint32_t mb = __reduce_max_sync(mask, __float_as_uint(m));
        if (lane == 0) red[warp] = mb;
        __syncthreads();          // the row maximum is complete (and buffer b is free)
        if (NBUF == 2) issue_row(row + 2 * gridDim.x, b);
        const int nwarps = (nthreads + 31) >> 5;
        for (int w = 0; w < nwarps; ++w) mb = max(mb, red[w]);
        const float a_u = __uint_as_float(mb);

        const float inv = a_u > 0.0f ? __fdiv_rn(7.0f, a_u) : 0.0f;
        if (t == 0) s[row] = __fdiv_rn(a_u * kNorm, 7.0f);

        uint32_t packed[8];
        quantize_pack(v, inv, packed);
        uint8_t *qrow = q + static_cast<size_t>(row) * (K / 2);
        if (kDigits == 3) {
            uint4 *dst = reinterpret_cast<uint4 *>(qrow + t * 32);
            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        } else {
            // each register block is 16 consecutive channels (8 bytes); store d
            // writes digit 3 = d, the block d ^ j
            const int j = t & 3;
#pragma unroll
            for (int d = 0; d < 4; ++d) {
                const int m = d ^ j;
                *reinterpret_cast<uint2 *>(qrow + ((t & ~3) * 64 + 64 * d + 16 * j) / 2) =
                    make_uint2(pick4(packed[0], packed[2], packed[4], packed[6], m),
                               pick4(packed[1], packed[3], packed[5], packed[7], m));
            }
        }
    }
    cp_async_wait_all();          // no copy outlives the CTA (empty groups past the end)
}


// ------------------------------------------------------------------------
// The same preparation with 16 channels per thread (K/16 threads per row),
// for latency-bound launches (few rows per SM): a quarter of the per-thread
// work per row and no shared-memory exchange.  Thread t owns channels
// [16t, 16t + 16), loaded straight from global memory (32 contiguous bytes
// per thread, coalesced).  Digits 0 and 1 of the rotation run in registers;
// digit 2 spans lanes t ^ 1, t ^ 2 (the four threads of a 64-group) and,
// for n = 256, digit 3 lanes t ^ 4, t ^ 8, as shuffles: lane l forms
// (x_l + x_l^1) + (x_l^2 + x_l^3), the same sums in the same order as the
// register butterfly (x_0 + x_1) + (x_2 + x_3) (addition commutes bitwise),
// so codes, scales and rotated values are bit-identical to prep_kernel's.
__device__ __forceinline__ void radix4_lanes(float (&v)[16], int m1, int m2) {
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
        float a0 = v[e] + __shfl_xor_sync(0xFFFFFFFFu, v[e], m1);
        float a1 = v[e + 1] + __shfl_xor_sync(0xFFFFFFFFu, v[e + 1], m1);
        const float s0 = a0 + __shfl_xor_sync(0xFFFFFFFFu, a0, m2);
        const float s1 = a1 + __shfl_xor_sync(0xFFFFFFFFu, a1, m2);
        bfly2(v[e], v[e + 1], s0, s1);
    }
}

template <int G, int MODE>
__global__ void __maxnreg__(40)
prep16_kernel(const uint16_t *__restrict__ x, int M, int K, uint8_t *__restrict__ q,
              float *__restrict__ s, float *__restrict__ yrot, uint32_t *__restrict__ zero,
              int nzero) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 2^-digits
    __shared__ uint32_t red[2][32];
    // side job for the GEMM that follows: clear its split counters
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0u;
    // blockDim.x = K/16 rounded up to whole warps; K is a multiple of 256, so
    // the padding lanes form whole 16-lane groups: they hold zeros, take part
    // in the shuffles and the maximum, and store nothing.
    const int t = threadIdx.x;
    const bool act = t < K / 16;
    const int nwarps = blockDim.x >> 5;
    const int warp = t >> 5, lane = t & 31;
    int it = 0;
    for (int row = blockIdx.x; row < M; row += gridDim.x, ++it) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(row) * K) + 2 * t;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const uint4 r0 = act ? src[0] : z, r1 = act ? src[1] : z;
        // As in prep_kernel: the GEMM that follows may be scheduled (and
        // stream its weights) from now on; it reads these rows only after
        // its griddepcontrol.wait.
        if (it == 0) ptx::launch_dependents();
        float v[16];
        const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
        radix4_digit0(v);
        radix4_stage<4>(v);
        radix4_lanes(v, 1, 2);                           // digit 2
        if (G == 256) radix4_lanes(v, 4, 8);             // digit 3
        if (MODE == 1) {
            if (!act) continue;
            float4 *dst = reinterpret_cast<float4 *>(yrot + static_cast<size_t>(row) * K) + 4 * t;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(v[4 * i] * kNorm, v[4 * i + 1] * kNorm, v[4 * i + 2] * kNorm,
                                     v[4 * i + 3] * kNorm);
            continue;
        }
        const float m = thread_absmax(v);
        uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
        if (lane == 0) red[it & 1][warp] = mb;           // two buffers: one barrier per row
        __syncthreads();
        for (int wi = 0; wi < nwarps; ++wi) mb = max(mb, red[it & 1][wi]);
        const float a_u = __uint_as_float(mb);
        const float inv = a_u > 0.0f ? __fdiv_rn(7.0f, a_u) : 0.0f;
        if (t == 0) s[row] = __fdiv_rn(a_u * kNorm, 7.0f);
        uint32_t packed[2];
        quantize_pack(v, inv, packed);
        if (act)
            *reinterpret_cast<uint2 *>(q + static_cast<size_t>(row) * (K / 2) + 8 * t) =
                make_uint2(packed[0], packed[1]);
    }
}


// ------------------------------------------------------------------------
// The same preparation with 32 channels per thread (K/32 threads per row),
// for launches of many rows: half the registers of prep_kernel per thread
// (its 64 channels need 128), so an SM holds twice the warps to hide the
// latency of the row's dependency chains.  Thread t owns channels
// [32t, 32t + 32): digits 0 and 1 of the rotation run in registers; digit 2
// (stride 16) spans the thread pair t, t ^ 1, which swap the partial sums
// x0 + x1 and x2 + x3 of each quadruple with one shuffle; for n = 256,
// digit 3 (stride 64) spans threads t, t ^ 2, t ^ 4, t ^ 6, which exchange
// quarters of their values through the row's stage buffer, so that digit 3
// becomes a register stride of 8.  Every sum is formed from the same
// operands in the same order as in prep_kernel (floating-point addition
// commutes bitwise), so codes, scales and rotated values are bit-identical
// to prep_kernel's.
//
// Shared-memory layouts (16-byte slots; thread t owns slots 4t .. 4t + 3,
// key(t) = (t >> 1) & 3):
//   row stage: chunk c (8 bf16) of thread t's 64 bytes at slot
//              4t + (c ^ key(t));
//   exchange:  in pass p, the four values 8k + 4p .. 8k + 4p + 3 of thread
//              t at slot 4t + (k ^ key(t)).
// Eight consecutive threads (a quarter warp) then touch eight distinct
// slots modulo 8 in every load and store (even threads slots 0-3, odd ones
// 4-7, each set distinct through the key): no bank conflicts.  Each thread
// writes only its own four slots, so one warp barrier per pass suffices.
__device__ __forceinline__ uint32_t key32(int t) { return static_cast<uint32_t>((t >> 1) & 3); }

// Registers v[0..31] <- the thread's 32 channels of a staged bf16 row.
__device__ __forceinline__ void load_row32(const uint4 *__restrict__ sb, int t, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 raw = sb[4 * t + (static_cast<uint32_t>(i) ^ key32(t))];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }
}

// The unnormalised rotation of the thread's 32 channels.  On return, for
// n = 64, v[e] is channel 32 t + e; for n = 256, v[8 d3 + q] is channel
// 256 g + 64 d3 + 32 h + 8 j + q, with g = t / 8, h = t mod 2 and
// j = (t / 2) mod 4 (row32_chan).
template <int G>
__device__ __forceinline__ void rotate_row32(float (&v)[32], float4 *__restrict__ xb, int t,
                                             uint32_t mask) {
    radix4_digit0(v);
    radix4_stage<4>(v);
    // digit 2: v[r] and v[16 + r] are x0, x1 (even thread) or x2, x3 (odd)
#pragma unroll
    for (int r = 0; r < 16; r += 2) {
        float a0, a1;
        add2(a0, a1, v[r], v[r + 1], v[r + 16], v[r + 17]);
        const float b0 = __shfl_xor_sync(mask, a0, 1);
        const float b1 = __shfl_xor_sync(mask, a1, 1);
        float s0, s1;
        add2(s0, s1, a0, a1, b0, b1);
        bfly2(v[r], v[r + 1], s0, s1);
        bfly2(v[r + 16], v[r + 17], s0, s1);
    }
    if (G == 256) {
        const int j = (t >> 1) & 3, gb = t & ~7, h = t & 1;
        const uint32_t kt = key32(t);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            __syncwarp(mask);     // the group's reads of the buffer (row load or pass 0) are done
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = 8 * k + 4 * p;
                xb[4 * t + (static_cast<uint32_t>(k) ^ kt)] = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
            __syncwarp(mask);
#pragma unroll
            for (int d3 = 0; d3 < 4; ++d3) {
                const int w = gb + 2 * d3 + h;
                const float4 f = xb[4 * w + (static_cast<uint32_t>(j) ^ key32(w))];
                const int e = 8 * d3 + 4 * p;
                v[e] = f.x;
                v[e + 1] = f.y;
                v[e + 2] = f.z;
                v[e + 3] = f.w;
            }
        }
        radix4_stage<8>(v);
    }
}

// Channel of register e of thread t after rotate_row32.
template <int G>
__device__ __forceinline__ int row32_chan(int t, int e) {
    if (G == 64) return t * 32 + e;
    return (t & ~7) * 32 + 64 * (e >> 3) + 32 * (t & 1) + 8 * ((t >> 1) & 3) + (e & 7);
}

// Persistent over rows with two stage buffers, as prep_kernel for n = 256:
// the next two rows arrive by asynchronous copies during the arithmetic,
// and the barrier of the row maximum also frees the buffer for the row
// after next.
template <int G, int MODE>
__global__ void __maxnreg__(64)
prep32_kernel(const uint16_t *__restrict__ x, int M, int K, uint8_t *__restrict__ q,
              float *__restrict__ s, float *__restrict__ yrot, uint32_t *__restrict__ zero,
              int nzero) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    // side job for the GEMM that follows: clear its split counters
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0u;
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 2^-digits

    extern __shared__ uint4 stage[];                       // two buffers of K * 2 bytes
    __shared__ uint32_t red[32];

    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                       // K / 32
    const int warp = t >> 5, lane = t & 31;
    const int warp_lanes = min(32, nthreads - warp * 32);
    const uint32_t mask = warp_lanes == 32 ? 0xFFFFFFFFu : ((1u << warp_lanes) - 1u);
    const int row_chunks = nthreads * 4;                   // 16-byte chunks per row
    const uint32_t stage_s = ptx::smem_u32(stage);

    auto issue_row = [&](int r, int buf) {
        if (r < M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(r) * K);
            const uint32_t base = stage_s + static_cast<uint32_t>(buf * row_chunks * 16);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int g = t + jj * nthreads;           // chunk index in the row
                const int owner = g >> 2;
                const uint32_t c = static_cast<uint32_t>(g & 3);
                cp_async16(base + static_cast<uint32_t>((owner * 4 + (c ^ key32(owner))) * 16), src + g);
            }
        }
        cp_async_commit();   // one group per row, empty past the end
    };

    int row = blockIdx.x;
    issue_row(row, 0);
    issue_row(row + gridDim.x, 1);
    // The GEMM that follows may be scheduled on the SMs this grid leaves
    // free; it reads these rows only after its griddepcontrol.wait.
    ptx::launch_dependents();
    for (int it = 0; row < M; row += gridDim.x, ++it) {
        const int b = it & 1;
        uint4 *sb = stage + b * row_chunks;
        cp_async_wait_prior();    // this row's copies (by this thread) have landed ...
        __syncthreads();          // ... and everyone else's

        float v[32];
        load_row32(sb, t, v);
        rotate_row32<G>(v, reinterpret_cast<float4 *>(sb), t, mask);
        auto chan = [&](int e) -> int { return row32_chan<G>(t, e); };

        if (MODE == 1) {
            float *dst = yrot + static_cast<size_t>(row) * K;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<float4 *>(dst + chan(4 * i)) =
                    make_float4(v[4 * i] * kNorm, v[4 * i + 1] * kNorm, v[4 * i + 2] * kNorm,
                                v[4 * i + 3] * kNorm);
            __syncthreads();      // every warp is done with buffer b
            issue_row(row + 2 * gridDim.x, b);
            continue;
        }

        const float m = thread_absmax(v);
        uint32_t mb = __reduce_max_sync(mask, __float_as_uint(m));
        if (lane == 0) red[warp] = mb;
        __syncthreads();          // the row maximum is complete (and buffer b is free)
        issue_row(row + 2 * gridDim.x, b);
        const int nwarps = (nthreads + 31) >> 5;
        for (int w = 0; w < nwarps; ++w) mb = max(mb, red[w]);
        const float a_u = __uint_as_float(mb);

        const float inv = a_u > 0.0f ? __fdiv_rn(7.0f, a_u) : 0.0f;
        if (t == 0) s[row] = __fdiv_rn(a_u * kNorm, 7.0f);

        uint32_t packed[4];
        quantize_pack(v, inv, packed);
        uint8_t *qrow = q + static_cast<size_t>(row) * (K / 2);
        if (G == 64) {
            *reinterpret_cast<uint4 *>(qrow + t * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        } else {
            // registers 8 d3 .. 8 d3 + 7 are 8 consecutive channels: 4 bytes
#pragma unroll
            for (int d3 = 0; d3 < 4; ++d3)
                *reinterpret_cast<uint32_t *>(qrow + chan(8 * d3) / 2) = packed[d3];
        }
        // red[] is rewritten only after the next row's first barrier, which
        // every thread passes after reading it here
    }
    cp_async_wait_all();          // no copy outlives the CTA (empty groups past the end)
}

}  // namespace prep

// prep.cuh -- fused rotation + rowwise absmax INT4 quantisation + packing.
//
// One CTA per row, K/64 threads; thread t owns the 64 consecutive channels
// [64t, 64t + 64) of its row, loaded with eight 128-bit loads.
//
// Rotation.  Within a group of n = 4^k channels the normalised regular
// Hadamard is H_n = T^{(x)k} / 2^k with T = J - 2I (Comfy-Org/comfy-quants
// issue, section 2: regular Hadamard for N_0 = 4^k; "convrot-mlx" README,
// "What is included": groups of 64 and 256).  Applying T along base-4 digit d
// of the channel index is a radix-4 butterfly: for each quadruple of channels
// that differ only in digit d, y_i = (x_0 + x_1 + x_2 + x_3) - 2 x_i.  The k
// butterflies commute (every factor is the same symmetric T), so they run in
// any order: digits 0, 1, 2 live inside one thread's 64 registers; for
// n = 256 digit 3 spans the 4 threads of the group and is done with two
// XOR shuffles.  The 1/2^k normalisation is exact and is folded into the
// scale (see below), so the butterflies run on unnormalised values.
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

__device__ __forceinline__ uint4 ldg_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Two signed codes into one byte of the running word:
// result = (acc << 8) | ((hi & 0xF) << 4) | (lo & 0xF), saturating to [-8, 7]
// (codes here are already in [-7, 7]).
__device__ __forceinline__ uint32_t pack_nibbles(int hi, int lo, uint32_t acc) {
    uint32_t d;
    asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(hi), "r"(lo), "r"(acc));
    return d;
}

// One radix-4 butterfly stage along the digit whose stride is S (1, 4, 16),
// two quadruples at a time.  Quadruples start at the indices b whose digit of
// stride S is 0; they are paired as (b, b + P) with P = 4 for S = 1 and
// P = 1 otherwise, so both members of a pair are quadruple starts.
template <int S>
__device__ __forceinline__ void radix4_stage(float (&v)[kElemsPerThread]) {
    constexpr int P = (S == 1) ? 4 : 1;
#pragma unroll
    for (int b = 0; b < kElemsPerThread; ++b) {
        if ((b / S) % 4 != 0 || (b / P) % 2 != 0) continue;
        const int c = b + P;
        float s01a, s01b, s23a, s23b, suma, sumb;
        add2(s01a, s01b, v[b], v[c], v[b + S], v[c + S]);
        add2(s23a, s23b, v[b + 2 * S], v[c + 2 * S], v[b + 3 * S], v[c + 3 * S]);
        add2(suma, sumb, s01a, s01b, s23a, s23b);
#pragma unroll
        for (int j = 0; j < 4; ++j) bfly2(v[b + j * S], v[c + j * S], suma, sumb);
    }
}

// MODE 0: quantise + pack (q, s).  MODE 1: write the normalised rotated row
// as fp32 (yrot) instead.
//
// Loads: the row is read with coalesced 128-bit loads (consecutive threads,
// consecutive 16-byte chunks) and written to shared memory so that chunk c of
// thread t's 128-byte slice sits at position c ^ (t mod 8); each thread then
// reads its own 64 channels back with conflict-free 128-bit loads.
template <int G, int MODE>
__global__ void __launch_bounds__(kMaxThreads)
prep_kernel(const uint16_t *__restrict__ x, int K, uint8_t *__restrict__ q,
            float *__restrict__ s, float *__restrict__ yrot) {
    static_assert(G == 64 || G == 256, "group 64 or 256");
    constexpr int kDigits = (G == 64) ? 3 : 4;
    constexpr float kNorm = (G == 64) ? 0.125f : 0.0625f;   // 2^-kDigits

    extern __shared__ uint4 stage[];                     // K * 2 bytes
    __shared__ uint32_t red[kMaxThreads / 32];

    const int row = blockIdx.x;
    const int t = threadIdx.x;
    const int nthreads = blockDim.x;                     // K / 64
    const int warp = t >> 5, lane = t & 31;
    const int warp_lanes = min(32, nthreads - warp * 32);
    const uint32_t mask = warp_lanes == 32 ? 0xFFFFFFFFu : ((1u << warp_lanes) - 1u);

    {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + static_cast<size_t>(row) * K);
        uint4 r[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) r[j] = ldg_stream(src + t + j * nthreads);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int g = t + j * nthreads;              // chunk index in the row
            const int owner = g >> 3, c = g & 7;
            stage[owner * 8 + (c ^ (owner & 7))] = r[j];
        }
    }
    __syncthreads();

    float v[kElemsPerThread];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 raw = stage[t * 8 + (i ^ (t & 7))];
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
            v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
    }

    radix4_stage<1>(v);
    radix4_stage<4>(v);
    radix4_stage<16>(v);
    if (kDigits == 4) {
        // digit 3 = lane bits 0..1: the 4 threads of this 256-channel group
#pragma unroll
        for (int e = 0; e < kElemsPerThread; e += 2) {
            float s0, s1;
            add2(s0, s1, v[e], v[e + 1], __shfl_xor_sync(mask, v[e], 1),
                 __shfl_xor_sync(mask, v[e + 1], 1));
            add2(s0, s1, s0, s1, __shfl_xor_sync(mask, s0, 2), __shfl_xor_sync(mask, s1, 2));
            bfly2(v[e], v[e + 1], s0, s1);
        }
    }

    if (MODE == 1) {
        float4 *dst = reinterpret_cast<float4 *>(yrot + static_cast<size_t>(row) * K) + t * 16;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            dst[i] = make_float4(v[4 * i] * kNorm, v[4 * i + 1] * kNorm, v[4 * i + 2] * kNorm,
                                 v[4 * i + 3] * kNorm);
        return;
    }

    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < kElemsPerThread; ++e) m = fmaxf(m, fabsf(v[e]));
    // non-negative floats order like their bit patterns
    uint32_t mb = __reduce_max_sync(mask, __float_as_uint(m));
    if (lane == 0) red[warp] = mb;
    __syncthreads();
    const int nwarps = (nthreads + 31) >> 5;
    for (int w = 0; w < nwarps; ++w) mb = max(mb, red[w]);
    const float a_u = __uint_as_float(mb);

    const float inv = a_u > 0.0f ? __fdiv_rn(7.0f, a_u) : 0.0f;
    if (t == 0) s[row] = __fdiv_rn(a_u * kNorm, 7.0f);

    uint32_t packed[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        int code[8];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            float p0, p1, h0, h1;
            mul2(p0, p1, v[8 * w + j], v[8 * w + j + 1], inv, inv);
            // add (0.5 - 2^-25) with the sign of the product, truncate
            const float c0 = __uint_as_float((__float_as_uint(p0) & 0x80000000u) | 0x3EFFFFFFu);
            const float c1 = __uint_as_float((__float_as_uint(p1) & 0x80000000u) | 0x3EFFFFFFu);
            add2(h0, h1, p0, p1, c0, c1);
            code[j] = __float2int_rz(h0);
            code[j + 1] = __float2int_rz(h1);
        }
        uint32_t word = pack_nibbles(code[7], code[6], 0u);
        word = pack_nibbles(code[5], code[4], word);
        word = pack_nibbles(code[3], code[2], word);
        packed[w] = pack_nibbles(code[1], code[0], word);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q + static_cast<size_t>(row) * (K / 2)) + t * 2;
    dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    // The GEMM that consumes these rows may be scheduled now; it still waits
    // for this whole grid to complete before reading them.
    ptx::launch_dependents();
}

}  // namespace prep

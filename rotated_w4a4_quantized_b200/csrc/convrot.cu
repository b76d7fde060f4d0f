// convrot.cu -- the C ABI declared in include/convrot.h: argument checks,
// launch configuration and TMA descriptors around the prep and GEMM kernels.
// One translation unit, so the device error word is a single symbol.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <initializer_list>
#include <mutex>

#include "../../include/convrot.h"
#include "gemm.cuh"
#include "prep.cuh"
#include "ptx.cuh"
#include "skinny.cuh"
#include "decode.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kSmemOptin = 232448;   // per-CTA shared memory limit (sm_100)
// dynamic shared memory the prep kernels may use (their static part is < 1 KB)
constexpr int kPrepSmemMax = kSmemOptin - 1024;

// `ready` is stored (release) only after every other field is written and
// read (acquire) before any of them, so a thread that sees it set sees the
// whole state; the first set-up on each device runs under g_mu.
struct DeviceState {
    std::atomic<bool> ready{false};
    convrot_status status = CONVROT_OK;
    int num_sms = 0;
    int pair_clusters = 0;   // co-resident 2-CTA clusters of the pair GEMM (0: none)
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

// Per-device one-time set-up: capability check, SM count, kernel attributes.
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
    ok &= set_smem(prep::prep_kernel<64, 0>, kPrepSmemMax);
    ok &= set_smem(prep::prep_kernel<256, 0>, kPrepSmemMax);
    ok &= set_smem(prep::prep_kernel<64, 1>, kPrepSmemMax);
    ok &= set_smem(prep::prep_kernel<256, 1>, kPrepSmemMax);
    ok &= set_smem(prep::prep32_kernel<256, 0>, kPrepSmemMax);
    ok &= set_smem(prep::prep32_kernel<256, 1>, kPrepSmemMax);
    ok &= set_smem(gemm::gemm_kernel<256, false, false>, gemm::Cfg<256, false>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<256, false, true>, gemm::Cfg<256, false>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<192, false, false>, gemm::Cfg<192, false>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<192, false, true>, gemm::Cfg<192, false>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<16, true, false>, gemm::Cfg<16, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<32, true, false>, gemm::Cfg<32, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<64, true, false>, gemm::Cfg<64, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<128, true, false>, gemm::Cfg<128, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<16, true, true>, gemm::Cfg<16, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<32, true, true>, gemm::Cfg<32, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<64, true, true>, gemm::Cfg<64, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<128, true, true>, gemm::Cfg<128, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<192, false, false, true>, gemm::Cfg<192, false, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<192, false, true, true>, gemm::Cfg<192, false, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<128, false, false, true>, gemm::Cfg<128, false, true>::SMEM_BYTES);
    ok &= set_smem(gemm::gemm_kernel<128, false, true, true>, gemm::Cfg<128, false, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<16, false>, skinny::Cfg<16>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<32, false>, skinny::Cfg<32>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<64, false>, skinny::Cfg<64>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<128, false>, skinny::Cfg<128>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<16, true>, skinny::Cfg<16>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<32, true>, skinny::Cfg<32>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<64, true>, skinny::Cfg<64>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<128, true>, skinny::Cfg<128>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<32, false, true>, skinny::Cfg<32, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<64, false, true>, skinny::Cfg<64, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<128, false, true>, skinny::Cfg<128, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<32, true, true>, skinny::Cfg<32, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<64, true, true>, skinny::Cfg<64, true>::SMEM_BYTES);
    ok &= set_smem(skinny::skinny_kernel<128, true, true>, skinny::Cfg<128, true>::SMEM_BYTES);
    ok &= set_smem(decode::decode_kernel<1, 64>, kPrepSmemMax);
    ok &= set_smem(decode::decode_kernel<2, 64>, kPrepSmemMax);
    ok &= set_smem(decode::decode_kernel<4, 64>, kPrepSmemMax);
    ok &= set_smem(decode::decode_kernel<1, 256>, kPrepSmemMax);
    ok &= set_smem(decode::decode_kernel<2, 256>, kPrepSmemMax);
    ok &= set_smem(decode::decode_kernel<4, 256>, kPrepSmemMax);
    if (ok) {
        // How many CTA pairs fit on the device at once (pairs need two SMs
        // of one GPC); the pair GEMM's persistent grid is that many clusters.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1));
        cfg.blockDim = dim3(gemm::kThreads);
        cfg.dynamicSmemBytes = gemm::Cfg<192, false, true>::SMEM_BYTES;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, gemm::gemm_kernel<192, false, false, true>, &cfg) !=
            cudaSuccess) {
            cudaGetLastError();   // clear it: the 1-CTA kernels remain
            n = 0;
        }
        st.pair_clusters = n;
    }
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

convrot_status check_shape(int64_t rows, int64_t K, int group) {
    if (group != 64 && group != 256) return CONVROT_ERR_GROUP;
    if (rows < 0 || K < 64 || K > CONVROT_MAX_K || K % group) return CONVROT_ERR_SHAPE;
    if (rows > (int64_t(1) << 30)) return CONVROT_ERR_SHAPE;
    return CONVROT_OK;
}

// Shared memory of one prep CTA: one or two staged bf16 rows (the group-256
// exchange reuses the current row's buffer).
size_t prep_smem(int64_t K, int group) {
    return static_cast<size_t>(K) * 2 * prep::stage_buffers(group);
}

// Resident prep CTAs per SM for a (group, mode, K) launch, cached.  The
// cache entries are atomics: concurrent first callers may both compute an
// entry, and they store the same value.
int prep_ctas_per_sm(int group, int mode, int64_t K) {
    static std::atomic<int> cache[2][2][prep::kMaxThreads + 1];
    const int T = static_cast<int>(K / prep::kElemsPerThread);
    std::atomic<int> &entry = cache[group == 256][mode][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        cudaError_t e;
        const size_t smem = prep_smem(K, group);
        if (group == 64)
            e = mode ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep_kernel<64, 1>, T, smem)
                     : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep_kernel<64, 0>, T, smem);
        else
            e = mode ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep_kernel<256, 1>, T, smem)
                     : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep_kernel<256, 0>, T, smem);
        slot = (e == cudaSuccess && n > 0) ? n : 1;
        entry.store(slot, std::memory_order_relaxed);
    }
    return slot;
}

// Resident 32-channel prep CTAs (K/32 threads, two staged rows) per SM for
// group 256, cached (as above).
int prep32_ctas_per_sm(int mode, int64_t K) {
    static std::atomic<int> cache[2][1025];
    const int T = static_cast<int>(K / 32);
    std::atomic<int> &entry = cache[mode][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        const size_t smem = static_cast<size_t>(K) * 4;
        const cudaError_t e =
            mode ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep32_kernel<256, 1>, T, smem)
                 : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep32_kernel<256, 0>, T, smem);
        slot = (e == cudaSuccess && n > 0) ? n : 1;
        entry.store(slot, std::memory_order_relaxed);
    }
    return slot;
}

// Resident 16-channel prep CTAs (K/16 threads) per SM, cached (as above).
int prep16_ctas_per_sm(int group, int mode, int64_t K) {
    static std::atomic<int> cache[2][2][1025];
    const int T = static_cast<int>((K / 16 + 31) / 32 * 32);
    std::atomic<int> &entry = cache[group == 256][mode][T];
    int slot = entry.load(std::memory_order_relaxed);
    if (slot == 0) {
        int n = 0;
        cudaError_t e;
        if (group == 64)
            e = mode ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep16_kernel<64, 1>, T, 0)
                     : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep16_kernel<64, 0>, T, 0);
        else
            e = mode ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep16_kernel<256, 1>, T, 0)
                     : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, prep::prep16_kernel<256, 0>, T, 0);
        slot = (e == cudaSuccess && n > 0) ? n : 1;
        entry.store(slot, std::memory_order_relaxed);
    }
    return slot;
}

// zero / nzero: words the kernel sets to 0 on the way (the split counters
// of the GEMM that follows), or nullptr / 0.
convrot_status launch_prep(int num_sms, const void *x, int64_t rows, int64_t K, int group,
                           uint8_t *q, float *s, float *yrot, cudaStream_t stream,
                           uint32_t *zero = nullptr, int nzero = 0) {
    if (rows == 0) return CONVROT_OK;
    const int mode = yrot ? 1 : 0;
    // Up to 1024 rows the launch is latency-bound (a row or two per CTA):
    // 16 channels per thread shorten each row's arithmetic four-fold
    // (1024 x 3072: 4.5 -> 4.1 us; 16 x 4096: 2.4 -> 2.1 us).  Beyond that the
    // 64-channel kernel, with fewer instructions per element, is faster.
    if (K <= 16384 && rows <= 1024) {
        const int64_t resident16 = static_cast<int64_t>(num_sms) * prep16_ctas_per_sm(group, mode, K);
        const dim3 grid16(static_cast<unsigned>(rows < resident16 ? rows : resident16));
        const dim3 block16(static_cast<unsigned>((K / 16 + 31) / 32 * 32));
        const uint16_t *xx = static_cast<const uint16_t *>(x);
        const int m = static_cast<int>(rows), k = static_cast<int>(K);
        if (yrot) {
            if (group == 64) prep::prep16_kernel<64, 1><<<grid16, block16, 0, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
            else prep::prep16_kernel<256, 1><<<grid16, block16, 0, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        } else {
            if (group == 64) prep::prep16_kernel<64, 0><<<grid16, block16, 0, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
            else prep::prep16_kernel<256, 0><<<grid16, block16, 0, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        }
        return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
    }
    if (group == 256 && K <= 3072) {
        // Beyond 1024 rows of up to 3072 channels, group 256: 32 channels per
        // thread, twice the resident warps of the 64-channel kernel.  Measured
        // (rows x K, us, 64- against 32-channel): 4608 x 3072 13.9 / 12.9,
        // 1536 x 3072 6.5 / 6.0, 3000 x 1024 6.1 / 4.7; on longer rows the
        // per-row costs spread over fewer channels per thread lose:
        // 2048 x 4096 8.4 / 8.7, 8192 x 8192 45.1 / 50.6.
        const int64_t resident32 = static_cast<int64_t>(num_sms) * prep32_ctas_per_sm(mode, K);
        const dim3 grid32(static_cast<unsigned>(rows < resident32 ? rows : resident32));
        const dim3 block32(static_cast<unsigned>(K / 32));
        const size_t smem32 = static_cast<size_t>(K) * 4;   // two staged bf16 rows
        const uint16_t *xx = static_cast<const uint16_t *>(x);
        const int m = static_cast<int>(rows), k = static_cast<int>(K);
        if (yrot)
            prep::prep32_kernel<256, 1><<<grid32, block32, smem32, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        else
            prep::prep32_kernel<256, 0><<<grid32, block32, smem32, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
    }
    const size_t smem = prep_smem(K, group);
    const int64_t resident = static_cast<int64_t>(num_sms) * prep_ctas_per_sm(group, mode, K);
    const dim3 grid(static_cast<unsigned>(rows < resident ? rows : resident));
    const dim3 block(static_cast<unsigned>(K / prep::kElemsPerThread));
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    const int m = static_cast<int>(rows), k = static_cast<int>(K);
    if (yrot) {
        if (group == 64) prep::prep_kernel<64, 1><<<grid, block, smem, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        else prep::prep_kernel<256, 1><<<grid, block, smem, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
    } else {
        if (group == 64) prep::prep_kernel<64, 0><<<grid, block, smem, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
        else prep::prep_kernel<256, 0><<<grid, block, smem, stream>>>(xx, m, k, q, s, yrot, zero, nzero);
    }
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Packed rows [rows][K/2] (rep = false), or the block-major repacked layout
// of the same bytes (rep = true): 3-D {128 bytes, rows, ceil(K/256) blocks},
// boxes of box_bytes <= 128 inside one block.
bool make_map(CUtensorMap *map, const uint8_t *base, int64_t rows, int64_t K, int box_bytes,
              int box_rows, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE,
              bool rep = false) {
    if (rep) {
        if (box_bytes > 128) return false;
        const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows),
                                    static_cast<cuuint64_t>((K / 2 + 127) / 128)};
        const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(rows) * 128};
        const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_bytes),
                                   static_cast<cuuint32_t>(box_rows), 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 output y [M][N] for the epilogue's TMA stores: 32 x 32 boxes,
// 64-byte swizzle (needs N % 8 == 0 so that rows start 16-byte aligned).
bool make_out_map(CUtensorMap *map, void *y, int64_t M, int64_t N) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(gemm::kStoreBox),
                               static_cast<cuuint32_t>(gemm::kStoreBox)};
    const cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// slots: CTAs (CTA pairs when PAIR) the persistent grid may use.
// wrep: the weights (qB, or qA in the swapped forms) are repacked.
// split_tiles, splits, split_ws: the split-K plan (gemm.cuh, "Split K");
// split_tiles = 0 runs every tile whole.
template <int BN, bool SWAP, bool OUT_S32, bool PAIR = false>
convrot_status launch_gemm_cfg(int slots, const uint8_t *qA, const uint8_t *qB, int64_t rowsA,
                               int64_t rowsB, int64_t K, const float *sx, const float *sw,
                               const void *bias, void *out, int64_t M, int64_t N,
                               cudaStream_t stream, bool wrep = false, int split_tiles = 0,
                               int splits = 1, uint32_t *split_ws = nullptr) {
    using C = gemm::Cfg<BN, SWAP, PAIR>;
    CUtensorMap tmA, tmB, tmY;
    constexpr int pkb = C::PKB;
    // A widened into TMEM reads its packed rows 128-byte swizzled.
    const CUtensorMapSwizzle swa = C::ATM ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
    if (wrep && pkb > 128) return CONVROT_ERR_UNSUPPORTED;   // boxes wider than a block
    if (!make_map(&tmA, qA, rowsA, K, pkb, gemm::BM, swa, SWAP && wrep) ||
        !make_map(&tmB, qB, rowsB, K, pkb, C::BR, CU_TENSOR_MAP_SWIZZLE_NONE, !SWAP && wrep))
        return CONVROT_ERR_CUDA;
    int use_tma_store = 0;
    if (!SWAP && !OUT_S32 && N % 8 == 0) {
        if (!make_out_map(&tmY, out, M, N)) return CONVROT_ERR_CUDA;
        use_tma_store = 1;
    } else {
        tmY = tmA;   // unused by the kernel
    }
    if (split_tiles > 0 && (SWAP || BN < 64 || !split_ws || splits < 2)) return CONVROT_ERR_UNSUPPORTED;
    const int64_t tiles = ((rowsA + C::TM - 1) / C::TM) * ((rowsB + BN - 1) / BN);
    const int64_t units = tiles + static_cast<int64_t>(split_tiles) * (splits - 1);
    const int grid = static_cast<int>(units < slots ? units : slots) * C::CG;
    // Programmatic dependent launch: the GEMM's set-up (barriers, TMEM,
    // descriptor prefetch) overlaps the end of the preceding kernel on the
    // stream (normally the prep kernel); the kernel waits for that grid's
    // results before its first load.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(gemm::kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = C::CG;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, gemm::gemm_kernel<BN, SWAP, OUT_S32, PAIR>, tmA, tmB, tmY, use_tma_store,
        static_cast<int>(rowsA), static_cast<int>(rowsB), static_cast<int>(K), sx, sw,
        static_cast<const uint16_t *>(bias), out, static_cast<int>(M), static_cast<int>(N),
        wrep ? 1 : 0, split_tiles, split_tiles > 0 ? splits : 1, split_ws);
    return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Skinny GEMM (M <= 128): one CTA per slice of R weight rows, weights
// widened into TMEM.  weights_ready: the weights were complete before the
// preceding kernel on the stream (the prep kernel of the same call) started,
// so the kernel may start streaming them before that kernel finishes.
template <int BN, bool OUT_S32, bool PAIR = false>
convrot_status launch_skinny_cfg(int num_sms, const uint8_t *qx, const float *sx,
                                 const uint8_t *qw, const float *sw, const void *bias, int64_t M,
                                 int64_t N, int64_t K, void *out, bool weights_ready,
                                 cudaStream_t stream, bool wrep) {
    using C = skinny::Cfg<BN, PAIR>;
    const int R = skinny::rows_per_cta(N, num_sms);
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, qw, N, K, skinny::kPKB, R, CU_TENSOR_MAP_SWIZZLE_128B, wrep) ||
        !make_map(&tmB, qx, M, K, skinny::kPKB, C::BR))
        return CONVROT_ERR_CUDA;
    int64_t ctas = (N + R - 1) / R;
    if (PAIR) ctas += ctas & 1;   // whole pairs (a trailing CTA past N only waits and exits)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas));
    cfg.blockDim = dim3(skinny::kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = PAIR ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(
        &cfg, skinny::skinny_kernel<BN, OUT_S32, PAIR>, tmA, tmB, R, weights_ready ? 1 : 0,
        static_cast<int>(K), wrep ? 1 : 0, sx, sw, static_cast<const uint16_t *>(bias), out, static_cast<int>(M),
        static_cast<int>(N));
    return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

template <bool OUT_S32>
convrot_status launch_skinny(int num_sms, const uint8_t *qx, const float *sx, const uint8_t *qw,
                             const float *sw, const void *bias, int64_t M, int64_t N, int64_t K,
                             void *out, bool weights_ready, cudaStream_t stream, bool pair = false,
                             bool wrep = false) {
    if (pair) {
        if (M <= 32)
            return launch_skinny_cfg<32, OUT_S32, true>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                                        weights_ready, stream, wrep);
        if (M <= 64)
            return launch_skinny_cfg<64, OUT_S32, true>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                                        weights_ready, stream, wrep);
        return launch_skinny_cfg<128, OUT_S32, true>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                                     weights_ready, stream, wrep);
    }
    if (M <= 16)
        return launch_skinny_cfg<16, OUT_S32>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                              weights_ready, stream, wrep);
    if (M <= 32)
        return launch_skinny_cfg<32, OUT_S32>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                              weights_ready, stream, wrep);
    if (M <= 64)
        return launch_skinny_cfg<64, OUT_S32>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                              weights_ready, stream, wrep);
    return launch_skinny_cfg<128, OUT_S32>(num_sms, qx, sx, qw, sw, bias, M, N, K, out,
                                           weights_ready, stream, wrep);
}

// Up to this many tokens the GEMM is the few-token (weight-streaming) form.
constexpr int64_t kSkinnyMaxM = 128;

// GEMM forms: the automatic choice, the three token-major tile shapes, and
// the two few-token forms (M <= 128).
enum TileChoice {
    kTilesAuto = 0, kTiles128x256 = 1, kTiles128x192 = 2, kTiles256x192Pair = 3,
    kSkinnyTmem = 4, kSkinnySmem = 5, kTiles256x128Pair = 6, kSkinnyPair = 7
};

// Split-K area handed to the token-major GEMM: counters, then partial slots
// (gemm.cuh, "Split K").  bytes = 0: no split.
struct SplitArea {
    uint32_t *ws = nullptr;
    size_t bytes = 0;
    int force_tiles = -1;   // >= 0: this plan instead of the planner's (test hook)
    int force_splits = 1;
};

// Partial slots (one per split unit and CTA) of BM x BN int32 that fit in
// a split area of `bytes` (0: no area).
int64_t split_capacity(size_t bytes, int BN) {
    if (bytes < CONVROT_SPLIT_COUNTER_BYTES) return 0;
    return static_cast<int64_t>((bytes - CONVROT_SPLIT_COUNTER_BYTES) /
                                (static_cast<size_t>(gemm::BM) * BN * 4));
}
int64_t split_capacity(const SplitArea &a, int BN) { return a.ws ? split_capacity(a.bytes, BN) : 0; }

// The planner: `tiles` output tiles (BM x bn int32 accumulators per CTA) of
// `num_kp` packed K-stages each on `slots` CTAs (pairs of cg CTAs).  Whole
// waves stay whole; the `rem` tiles of a part-filled last wave may be split
// into s parts (2 <= s <= 4, every part at least two stages, rem * s units
// within one wave and the area), which the schedule runs first.  `cost` =
// the busiest CTA's K-stages plus the split's own cost in stages: writing,
// fencing and reading back the partial sums, measured on a B200 as about 3
// stages plus 0.6 stage per MB of partials (e.g. the 1536 x 12288 -> 3072
// layer: 59.7 us unsplit, 44.1 us in 3 parts; the 512 x 4096 -> 2048 layer,
// one part-filled wave of 16-stage tiles: 14.8 us unsplit, 15.7 us in 3
// parts).  The split with the lowest cost is taken if it beats no split.
struct SplitPlan {
    int split_tiles = 0, splits = 1;
    int64_t cost = 0;   // K-stages of the busiest CTA, plus the split's cost
};

SplitPlan plan_split(int64_t tiles, int64_t slots, int64_t num_kp, int64_t capacity, int cg,
                     int bn) {
    SplitPlan p;
    if (slots <= 0) {   // no co-resident CTAs of this form: one tile after another
        p.cost = tiles * num_kp;
        return p;
    }
    const int64_t full = tiles / slots, rem = tiles % slots;
    p.cost = (full + (rem ? 1 : 0)) * num_kp;
    if (rem == 0 || capacity <= 0 || rem * cg * gemm::kEpiWarps > gemm::kSplitCounters) return p;
    int64_t smax = std::min<int64_t>(slots / rem, 4);
    smax = std::min<int64_t>(smax, num_kp / 2);
    smax = std::min<int64_t>(smax, capacity / (rem * cg));
    for (int64_t sp = 2; sp <= smax; ++sp) {
        const int64_t partial_bytes = rem * sp * cg * gemm::BM * bn * 4;
        const int64_t cost = full * num_kp + (num_kp + sp - 1) / sp + 3 +
                             (partial_bytes * 6 + 5000000) / 10000000;
        if (cost < p.cost) {
            p.split_tiles = static_cast<int>(rem);
            p.splits = static_cast<int>(sp);
            p.cost = cost;
        }
    }
    return p;
}

// The token-major tile shape and split-K plan for (M, N, K) on `pairs` CTA
// pairs (0: none) and `sms` SMs, with a split area of `area_bytes`
// (host-only: no device needed).  tiles = kTilesAuto picks the shape.
struct GemmPlan {
    int tiles = kTilesAuto;
    SplitPlan split;
};

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, int64_t pairs, int64_t sms, size_t area_bytes,
                   int tiles) {
    struct Shape {
        int64_t ntiles, slots, num_kp, capacity;
        int cg, bn;
    };
    const auto shape_of = [&](int t) {
        const bool pair = t == kTiles256x128Pair || t == kTiles256x192Pair;
        const int bn = (t == kTiles256x128Pair) ? 128 : (t == kTiles128x256) ? 256 : 192;
        const int tm = pair ? 256 : 128;
        const int pkb = (t == kTiles128x256) ? 64 : 128;
        return Shape{((M + tm - 1) / tm) * ((N + bn - 1) / bn), pair ? pairs : sms,
                     (K / 2 + pkb - 1) / pkb, split_capacity(area_bytes, bn), pair ? 2 : 1, bn};
    };
    const auto shape_plan = [&](int t) {
        const Shape h = shape_of(t);
        return plan_split(h.ntiles, h.slots, h.num_kp, h.capacity, h.cg, h.bn);
    };
    GemmPlan g;
    g.tiles = tiles;
    if (g.tiles == kTilesAuto) {
        // Measured on layers of 1024-8192 tokens and K 3072-12288: the
        // 256 x 192 pair beats both single-CTA shapes everywhere (each SM
        // widens half of B and the tensor core reads A from TMEM).  The cost
        // of a choice is the busiest CTA's K-stages (waves, less what split K
        // takes off the last one) times a stage's time.
        if (pairs > 0) {
            // A 256 x 128 pair tile takes ~0.9 of a 256 x 192 one's time
            // (measured on 1024-8192 tokens), so the narrower tile wins only
            // where the 192-wide grid wastes most of a last wave that split K
            // does not recover.
            const int64_t c192 = shape_plan(kTiles256x192Pair).cost * 10;
            const int64_t c128 = shape_plan(kTiles256x128Pair).cost * 9;
            g.tiles = c128 < c192 ? kTiles256x128Pair : kTiles256x192Pair;
        } else {
            // a 128-code stage takes ~940 cycles on 128 x 256 tiles (both
            // operands widened in shared memory), a 256-code stage ~1340 on
            // 128 x 192 (A in TMEM)
            const int64_t c_ss = shape_plan(kTiles128x256).cost * 940;
            const int64_t c_atm = shape_plan(kTiles128x192).cost * 1340;
            g.tiles = c_atm <= c_ss ? kTiles128x192 : kTiles128x256;
        }
    }
    if (g.tiles == kTiles256x128Pair || g.tiles == kTiles256x192Pair || g.tiles == kTiles128x192 ||
        g.tiles == kTiles128x256)
        g.split = shape_plan(g.tiles);
    return g;
}

// Path choice: up to 128 tokens the few-token form (weights on the 128-row
// MMA side, widened into TMEM, one CTA per slice of weight rows); otherwise
// tokens on the M side, with the tile shape (and split-K plan) that finishes
// first (plan_gemm).
template <bool OUT_S32>
convrot_status launch_gemm(const DeviceState &ds, const uint8_t *qx, const float *sx,
                           const uint8_t *qw, const float *sw, const void *bias, int64_t M,
                           int64_t N, int64_t K, void *out, cudaStream_t stream,
                           int tiles = kTilesAuto, bool weights_ready = false,
                           bool wrep = false, const SplitArea &area = SplitArea()) {
    const int num_sms = ds.num_sms;
    // Few tokens: the weight-streaming form.  (The CTA-pair form measured
    // the same at 128 tokens and slower below: each SM's tensor core does
    // the same work per weight byte either way.)
    if (tiles == kTilesAuto && M <= kSkinnyMaxM) tiles = kSkinnyTmem;
    if (tiles == kSkinnyTmem && M > 128) return CONVROT_ERR_SHAPE;
    if (tiles == kSkinnySmem && M > 128) return CONVROT_ERR_SHAPE;
    if (tiles == kSkinnyPair && M > 128) return CONVROT_ERR_SHAPE;
    if (tiles == kSkinnyPair && ds.pair_clusters <= 0) return CONVROT_ERR_UNSUPPORTED;
    if (tiles == kSkinnyTmem || tiles == kSkinnyPair)
        return launch_skinny<OUT_S32>(num_sms, qx, sx, qw, sw, bias, M, N, K, out, weights_ready,
                                      stream, tiles == kSkinnyPair, wrep);
    if (tiles == kSkinnySmem) {
        if (M <= 16)
            return launch_gemm_cfg<16, true, OUT_S32>(num_sms, qw, qx, N, M, K, sx, sw, bias, out, M,
                                                      N, stream, wrep);
        if (M <= 32)
            return launch_gemm_cfg<32, true, OUT_S32>(num_sms, qw, qx, N, M, K, sx, sw, bias, out, M,
                                                      N, stream, wrep);
        if (M <= 64)
            return launch_gemm_cfg<64, true, OUT_S32>(num_sms, qw, qx, N, M, K, sx, sw, bias, out, M,
                                                      N, stream, wrep);
        return launch_gemm_cfg<128, true, OUT_S32>(num_sms, qw, qx, N, M, K, sx, sw, bias, out, M, N,
                                                   stream, wrep);
    }
    if (tiles != kTilesAuto && tiles != kTiles256x128Pair && tiles != kTiles256x192Pair &&
        tiles != kTiles128x192 && tiles != kTiles128x256)
        return CONVROT_ERR_SHAPE;
    const GemmPlan gp = plan_gemm(M, N, K, ds.pair_clusters, num_sms, area.ws ? area.bytes : 0, tiles);
    tiles = gp.tiles;
    SplitPlan plan = gp.split;
    if (area.force_tiles > 0) {
        // a given plan: every part at least one K-stage, every slot and
        // counter inside the area
        const bool pair = tiles == kTiles256x128Pair || tiles == kTiles256x192Pair;
        const int bn = (tiles == kTiles256x128Pair) ? 128 : (tiles == kTiles128x256) ? 256 : 192;
        const int tm = pair ? 256 : 128;
        const int pkb = (tiles == kTiles128x256) ? 64 : 128;
        const int64_t ntiles = ((M + tm - 1) / tm) * ((N + bn - 1) / bn);
        const int64_t num_kp = (K / 2 + pkb - 1) / pkb;
        const int64_t cg = pair ? 2 : 1;
        const int64_t ft = area.force_tiles, fs = area.force_splits;
        if (ft > ntiles || fs < 2 || fs > num_kp || ft * cg * gemm::kEpiWarps > gemm::kSplitCounters ||
            ft * fs * cg > split_capacity(area, bn))
            return CONVROT_ERR_SHAPE;
        plan.split_tiles = area.force_tiles;
        plan.splits = area.force_splits;
    } else if (area.force_tiles == 0) {
        plan.split_tiles = 0;
        plan.splits = 1;
    }
    const int st = plan.split_tiles, sp = plan.splits;
    if (tiles == kTiles256x128Pair) {
        if (ds.pair_clusters <= 0) return CONVROT_ERR_UNSUPPORTED;
        return launch_gemm_cfg<128, false, OUT_S32, true>(ds.pair_clusters, qx, qw, M, N, K, sx, sw,
                                                          bias, out, M, N, stream, wrep, st, sp,
                                                          area.ws);
    }
    if (tiles == kTiles256x192Pair) {
        if (ds.pair_clusters <= 0) return CONVROT_ERR_UNSUPPORTED;
        return launch_gemm_cfg<192, false, OUT_S32, true>(ds.pair_clusters, qx, qw, M, N, K, sx, sw,
                                                          bias, out, M, N, stream, wrep, st, sp,
                                                          area.ws);
    }
    if (tiles == kTiles128x192)
        return launch_gemm_cfg<192, false, OUT_S32>(num_sms, qx, qw, M, N, K, sx, sw, bias, out, M,
                                                    N, stream, wrep, st, sp, area.ws);
    return launch_gemm_cfg<256, false, OUT_S32>(num_sms, qx, qw, M, N, K, sx, sw, bias, out, M, N,
                                                stream, wrep, st, sp, area.ws);
}

// The one-kernel path for 1..4 tokens (decode.cuh): token rows prepared in
// every CTA, GEMV on the CUDA cores.  Returns the ring depth (stages of 16 KB)
// that fits, or 0 when the shape takes the two-kernel path.
// R: weight rows per CTA (the ring slots are R x 128 bytes).
int decode_stages(int64_t M, int64_t K, int group, int R = decode::kRows) {
    if (M < 1 || M > 4 || K % 2048 != 0) return 0;
    const int MT = M <= 1 ? 1 : M <= 2 ? 2 : 4;
    if (K / prep::kElemsPerThread > decode::kConsumerWarps * 32) return 0;   // K <= 16384
    // Three slots of 512 bytes per row (~160 KB per SM in flight) stream as
    // fast as the whole slice at once and leave room for long rows.
    const int num_kp = static_cast<int>(K / (2 * decode::kPKB * decode::kBlocks));
    int sp = num_kp < 3 ? num_kp : 3;
    while (sp >= 2 && decode::smem_bytes(MT, group, static_cast<int>(K), sp, R) + 1024 >
                          static_cast<size_t>(kPrepSmemMax))
        --sp;
    return sp >= 2 ? sp : 0;
}

template <int MT, int G>
convrot_status launch_decode_cfg(int num_sms, int SP, const void *x, const uint8_t *qw,
                                 const float *sw, const void *bias, int64_t M, int64_t N,
                                 int64_t K, void *y, cudaStream_t stream, bool wrep) {
    const int R = skinny::rows_per_cta(N, num_sms);
    CUtensorMap tmW;
    if (!make_map(&tmW, qw, N, K, decode::kPKB, R, CU_TENSOR_MAP_SWIZZLE_128B, wrep))
        return CONVROT_ERR_CUDA;
    const size_t smem = decode::smem_bytes(MT, G, static_cast<int>(K), SP, R) + 1024;
    const dim3 grid(static_cast<unsigned>((N + R - 1) / R));
    decode::decode_kernel<MT, G><<<grid, decode::kThreads, smem, stream>>>(
        tmW, static_cast<const uint16_t *>(x), static_cast<int>(M), static_cast<int>(N),
        static_cast<int>(K), R, SP, wrep ? 1 : 0, sw, static_cast<const uint16_t *>(bias),
        static_cast<uint16_t *>(y));
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

convrot_status launch_decode(int num_sms, int SP, const void *x, const uint8_t *qw, const float *sw,
                             const void *bias, int64_t M, int64_t N, int64_t K, int group, void *y,
                             cudaStream_t stream, bool wrep = false) {
    if (group == 64) {
        if (M <= 1) return launch_decode_cfg<1, 64>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
        if (M <= 2) return launch_decode_cfg<2, 64>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
        return launch_decode_cfg<4, 64>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
    }
    if (M <= 1) return launch_decode_cfg<1, 256>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
    if (M <= 2) return launch_decode_cfg<2, 256>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
    return launch_decode_cfg<4, 256>(num_sms, SP, x, qw, sw, bias, M, N, K, y, stream, wrep);
}

convrot_status check_gemm_args(const uint8_t *qx, const uint8_t *qw, int64_t M, int64_t N,
                               int64_t K) {
    if (!qx || !qw) return CONVROT_ERR_NULL;
    if (M < 0 || N < 0 || K < 64 || K > CONVROT_MAX_K || K % 64) return CONVROT_ERR_SHAPE;
    if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30) || M * N > (int64_t(1) << 40))
        return CONVROT_ERR_SHAPE;
    if (!aligned16(qx) || !aligned16(qw)) return CONVROT_ERR_ALIGN;
    return CONVROT_OK;
}

inline size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

static_assert(gemm::kSplitCounters * 4 == CONVROT_SPLIT_COUNTER_BYTES, "split counter bytes");

// Workspace of the prepared activations (codes, then scales); the split
// area, where there is one, follows.
size_t prepared_bytes(int64_t M, int64_t K) {
    return round256(static_cast<size_t>(M) * static_cast<size_t>(K / 2)) +
           round256(static_cast<size_t>(M) * sizeof(float));
}

// steps 3-4 on prepared operands; wrep: qw is in the repacked layout
convrot_status linear_prepared_impl(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                    const float *sw, const void *bias_bf16, int64_t M, int64_t N,
                                    int64_t K, void *y_bf16, cudaStream_t stream, bool wrep,
                                    const SplitArea &area = SplitArea()) {
    if (M < 0 || N < 0) return CONVROT_ERR_SHAPE;
    if (M == 0 || N == 0) return CONVROT_OK;
    convrot_status st = check_gemm_args(qx, qw, M, N, K);
    if (st != CONVROT_OK) return st;
    if (!sx || !sw || !y_bf16) return CONVROT_ERR_NULL;
    if (!aligned16(sx) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {qx, sx, qw, sw, bias_bf16, y_bf16, area.ws})) != CONVROT_OK)
        return st;
    return launch_gemm<false>(g_dev[dev], qx, sx, qw, sw, bias_bf16, M, N, K, y_bf16, stream,
                              kTilesAuto, false, wrep, area);
}

// steps 1-4; wrep: qw is in the repacked layout
convrot_status linear_impl(const void *x_bf16, const uint8_t *qw, const float *sw,
                           const void *bias_bf16, int64_t M, int64_t N, int64_t K, int group,
                           void *workspace, size_t ws_bytes, void *y_bf16, cudaStream_t stream,
                           bool wrep) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if (N < 0) return CONVROT_ERR_SHAPE;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!x_bf16 || !qw || !sw || !y_bf16 || !workspace) return CONVROT_ERR_NULL;
    const size_t base = prepared_bytes(M, K);
    if (ws_bytes < base || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return CONVROT_ERR_WORKSPACE;
    if (!aligned16(x_bf16) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    if ((st = check_gemm_args(qw, qw, M, N, K)) != CONVROT_OK) return st;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, qw, sw, bias_bf16, workspace, y_bf16})) != CONVROT_OK)
        return st;
    // 1..4 tokens: one kernel (the workspace is not touched).  Eligibility
    // is decided for the largest slice (128 rows), so that it depends on
    // (M, K, group) alone, as convrot_linear_single_kernel reports it; the
    // ring then takes what the actual slice leaves.
    if (decode_stages(M, K, group) > 0)
        if (const int sp = decode_stages(M, K, group, skinny::rows_per_cta(N, g_dev[dev].num_sms)))
            return launch_decode(g_dev[dev].num_sms, sp, x_bf16, qw, sw, bias_bf16, M, N, K,
                                 group, y_bf16, stream, wrep);
    uint8_t *qx = static_cast<uint8_t *>(workspace);
    float *sx = reinterpret_cast<float *>(qx + round256(static_cast<size_t>(M) * (K / 2)));
    // The split area, when the workspace holds one and the token-major GEMM
    // runs; the prep kernel zeroes its counters.
    SplitArea area;
    if (M > kSkinnyMaxM && ws_bytes >= base + CONVROT_SPLIT_AREA_BYTES) {
        area.ws = reinterpret_cast<uint32_t *>(qx + base);
        area.bytes = CONVROT_SPLIT_AREA_BYTES;
    }
    if ((st = launch_prep(g_dev[dev].num_sms, x_bf16, M, K, group, qx, sx, nullptr, stream,
                          area.ws, area.ws ? gemm::kSplitCounters : 0)) != CONVROT_OK)
        return st;
    return launch_gemm<false>(g_dev[dev], qx, sx, qw, sw, bias_bf16, M, N, K, y_bf16, stream,
                              kTilesAuto, true, wrep, area);
}

// The reversible block-major repack (16 bytes per thread, grid-stride).
// Forward: chunk i of the repacked layout is 16-byte chunk j = i mod 8 of
// 128-byte block b of row n, (b, n) = (i / 8) divmod N, zero past the row's
// end.  Inverse: chunk i of the canonical layout (row n = i / row16) reads
// its chunk of its block.
__global__ void repack_kernel(const uint4 *__restrict__ in, uint4 *__restrict__ out, int64_t N,
                              int64_t row16, int64_t nblk, int inverse) {
    const int64_t total = inverse ? N * row16 : nblk * N * 8;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += step) {
        if (!inverse) {
            const int64_t j = i & 7, t = i >> 3;
            const int64_t b = t / N, n = t - b * N;
            const int64_t c16 = b * 8 + j;               // 16-byte chunk of the row
            out[i] = c16 < row16 ? in[n * row16 + c16] : make_uint4(0u, 0u, 0u, 0u);
        } else {
            const int64_t n = i / row16, c16 = i - n * row16;
            out[i] = in[((c16 >> 3) * N + n) * 8 + (c16 & 7)];
        }
    }
}

convrot_status repack_common(const uint8_t *in, int64_t N, int64_t K, uint8_t *out,
                             cudaStream_t stream, int inverse) {
    if (N < 0 || K < 64 || K > CONVROT_MAX_K || K % 64 || N > (int64_t(1) << 30))
        return CONVROT_ERR_SHAPE;
    if (N == 0) return CONVROT_OK;
    if (!in || !out) return CONVROT_ERR_NULL;
    if (!aligned16(in) || !aligned16(out)) return CONVROT_ERR_ALIGN;
    const size_t canon = static_cast<size_t>(N) * static_cast<size_t>(K / 2);
    const size_t rep = convrot_repacked_weight_size(N, K);
    const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
    const size_t na = inverse ? rep : canon, nb = inverse ? canon : rep;
    if (a < b + nb && b < a + na) return CONVROT_ERR_OVERLAP;
    int dev;
    convrot_status st = device_setup(&dev);
    if (st != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {in, out})) != CONVROT_OK) return st;
    const int64_t row16 = K / 32, nblk = (K / 2 + 127) / 128;
    repack_kernel<<<g_dev[dev].num_sms * 8, 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(in), reinterpret_cast<uint4 *>(out), N, row16, nblk, inverse);
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

}  // namespace

extern "C" {

const char *convrot_status_string(convrot_status s) {
    switch (s) {
        case CONVROT_OK: return "CONVROT_OK";
        case CONVROT_ERR_NULL: return "CONVROT_ERR_NULL: a required pointer is NULL";
        case CONVROT_ERR_GROUP: return "CONVROT_ERR_GROUP: group must be 64 or 256";
        case CONVROT_ERR_SHAPE: return "CONVROT_ERR_SHAPE: bad shape (K % group, K range, sizes)";
        case CONVROT_ERR_ALIGN: return "CONVROT_ERR_ALIGN: pointer not 16-byte aligned";
        case CONVROT_ERR_WORKSPACE: return "CONVROT_ERR_WORKSPACE: workspace too small or misaligned";
        case CONVROT_ERR_CUDA: return "CONVROT_ERR_CUDA: a CUDA call or launch failed";
        case CONVROT_ERR_DEVICE_TIMEOUT: return "CONVROT_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
        case CONVROT_ERR_UNSUPPORTED: return "CONVROT_ERR_UNSUPPORTED: needs an sm_100 device";
        case CONVROT_ERR_SCRATCH_LIMIT:
            return "CONVROT_ERR_SCRATCH_LIMIT: larger than the built-in scratch array";
        case CONVROT_ERR_NOT_DEVICE:
            return "CONVROT_ERR_NOT_DEVICE: a pointer is not memory of the current device";
        case CONVROT_ERR_OVERLAP:
            return "CONVROT_ERR_OVERLAP: input and output buffers overlap";
    }
    return "CONVROT_ERR_UNKNOWN";
}

convrot_status convrot_quantize_weight(const void *w_bf16, int64_t N, int64_t K, int group,
                                       uint8_t *qw, float *sw, convrot_stream_t stream) {
    convrot_status st = check_shape(N, K, group);
    if (st != CONVROT_OK) return st;
    if (N == 0) return CONVROT_OK;
    if (!w_bf16 || !qw || !sw) return CONVROT_ERR_NULL;
    if (!aligned16(w_bf16) || !aligned16(qw) || (reinterpret_cast<uintptr_t>(sw) & 3u))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {w_bf16, qw, sw})) != CONVROT_OK) return st;
    return launch_prep(g_dev[dev].num_sms, w_bf16, N, K, group, qw, sw, nullptr, stream);
}

convrot_status convrot_prepare_act(const void *x_bf16, int64_t M, int64_t K, int group, uint8_t *qx,
                                   float *sx, convrot_stream_t stream) {
    return convrot_quantize_weight(x_bf16, M, K, group, qx, sx, stream);
}

size_t convrot_linear_workspace_size(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return prepared_bytes(M, K) + (M > kSkinnyMaxM ? CONVROT_SPLIT_AREA_BYTES : 0);
}

convrot_status convrot_linear_prepared(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                       const float *sw, const void *bias_bf16, int64_t M, int64_t N,
                                       int64_t K, void *y_bf16, convrot_stream_t stream) {
    return linear_prepared_impl(qx, sx, qw, sw, bias_bf16, M, N, K, y_bf16, stream, false);
}

convrot_status convrot_linear_prepared_split(const uint8_t *qx, const float *sx,
                                             const uint8_t *qw, const float *sw,
                                             const void *bias_bf16, int64_t M, int64_t N,
                                             int64_t K, void *split_ws, size_t split_bytes,
                                             void *y_bf16, convrot_stream_t stream) {
    SplitArea area;
    if (split_ws) {
        if (split_bytes < CONVROT_SPLIT_AREA_BYTES || (reinterpret_cast<uintptr_t>(split_ws) & 255u))
            return CONVROT_ERR_WORKSPACE;
        area.ws = static_cast<uint32_t *>(split_ws);
        area.bytes = CONVROT_SPLIT_AREA_BYTES;
    }
    return linear_prepared_impl(qx, sx, qw, sw, bias_bf16, M, N, K, y_bf16, stream, false, area);
}

convrot_status convrot_linear(const void *x_bf16, const uint8_t *qw, const float *sw,
                              const void *bias_bf16, int64_t M, int64_t N, int64_t K, int group,
                              void *workspace, size_t ws_bytes, void *y_bf16,
                              convrot_stream_t stream) {
    return linear_impl(x_bf16, qw, sw, bias_bf16, M, N, K, group, workspace, ws_bytes, y_bf16,
                       stream, false);
}

size_t convrot_repacked_weight_size(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>((K / 2 + 127) / 128) * 128;
}

convrot_status convrot_repack_weight(const uint8_t *qw, int64_t N, int64_t K, uint8_t *qw_rep,
                                     convrot_stream_t stream) {
    return repack_common(qw, N, K, qw_rep, stream, 0);
}

convrot_status convrot_unpack_weight(const uint8_t *qw_rep, int64_t N, int64_t K, uint8_t *qw,
                                     convrot_stream_t stream) {
    return repack_common(qw_rep, N, K, qw, stream, 1);
}

convrot_status convrot_linear_repacked(const void *x_bf16, const uint8_t *qw_rep, const float *sw,
                                       const void *bias_bf16, int64_t M, int64_t N, int64_t K,
                                       int group, void *workspace, size_t ws_bytes, void *y_bf16,
                                       convrot_stream_t stream) {
    return linear_impl(x_bf16, qw_rep, sw, bias_bf16, M, N, K, group, workspace, ws_bytes, y_bf16,
                       stream, true);
}

convrot_status convrot_linear_prepared_repacked(const uint8_t *qx, const float *sx,
                                                const uint8_t *qw_rep, const float *sw,
                                                const void *bias_bf16, int64_t M, int64_t N,
                                                int64_t K, void *y_bf16, convrot_stream_t stream) {
    return linear_prepared_impl(qx, sx, qw_rep, sw, bias_bf16, M, N, K, y_bf16, stream, true);
}

int convrot_linear_single_kernel(int64_t M, int64_t K, int group) {
    if (check_shape(M, K, group) != CONVROT_OK) return 0;
    return decode_stages(M, K, group) > 0 ? 1 : 0;
}

convrot_status convrot_debug_rotate_f32(const void *x_bf16, int64_t M, int64_t K, int group,
                                        float *y_rot, convrot_stream_t stream) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if (M == 0) return CONVROT_OK;
    if (!x_bf16 || !y_rot) return CONVROT_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(y_rot)) return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, y_rot})) != CONVROT_OK) return st;
    return launch_prep(g_dev[dev].num_sms, x_bf16, M, K, group, nullptr, nullptr, y_rot, stream);
}

convrot_status convrot_debug_gemm_s32(const uint8_t *qx, const uint8_t *qw, int64_t M, int64_t N,
                                      int64_t K, int32_t *acc, convrot_stream_t stream) {
    if (M < 0 || N < 0) return CONVROT_ERR_SHAPE;
    if (M == 0 || N == 0) return CONVROT_OK;
    convrot_status st = check_gemm_args(qx, qw, M, N, K);
    if (st != CONVROT_OK) return st;
    if (!acc) return CONVROT_ERR_NULL;
    if (!aligned16(acc)) return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {qx, qw, acc})) != CONVROT_OK) return st;
    return launch_gemm<true>(g_dev[dev], qx, nullptr, qw, nullptr, nullptr, M, N, K, acc,
                             stream);
}

convrot_status convrot_debug_gemm_tiles(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                        const float *sw, const void *bias_bf16, int64_t M,
                                        int64_t N, int64_t K, int tiles, int out_s32, void *out,
                                        convrot_stream_t stream) {
    if (M < 0 || N < 0) return CONVROT_ERR_SHAPE;
    const bool wrep = (tiles & CONVROT_TILES_REPACKED) != 0;
    tiles &= ~CONVROT_TILES_REPACKED;
    if (tiles < kTilesAuto || tiles > kSkinnyPair) return CONVROT_ERR_SHAPE;
    if (M == 0 || N == 0) return CONVROT_OK;
    convrot_status st = check_gemm_args(qx, qw, M, N, K);
    if (st != CONVROT_OK) return st;
    if (!out || (!out_s32 && (!sx || !sw))) return CONVROT_ERR_NULL;
    if (!aligned16(out) || (!out_s32 && (!aligned16(sx) || !aligned16(sw) ||
                                         (bias_bf16 && !aligned16(bias_bf16)))))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {qx, qw, out})) != CONVROT_OK) return st;
    if (!out_s32 && (st = check_device_ptrs(dev, {sx, sw, bias_bf16})) != CONVROT_OK) return st;
    if (out_s32)
        return launch_gemm<true>(g_dev[dev], qx, nullptr, qw, nullptr, nullptr, M, N, K, out, stream,
                                 tiles, false, wrep);
    return launch_gemm<false>(g_dev[dev], qx, sx, qw, sw, bias_bf16, M, N, K, out, stream, tiles,
                              false, wrep);
}

convrot_status convrot_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int pairs, int sms,
                                       size_t split_bytes, int *tiles, int *split_tiles,
                                       int *splits) {
    if (!tiles || !split_tiles || !splits) return CONVROT_ERR_NULL;
    if (M < 0 || N < 0 || K < 64 || K > CONVROT_MAX_K || K % 64 || pairs < 0 || sms <= 0)
        return CONVROT_ERR_SHAPE;
    if (M <= kSkinnyMaxM) {   // the few-token form: one CTA per slice of weight rows
        *tiles = kSkinnyTmem;
        *split_tiles = 0;
        *splits = 1;
        return CONVROT_OK;
    }
    const GemmPlan g = plan_gemm(M, N, K, pairs, sms, split_bytes, kTilesAuto);
    *tiles = g.tiles;
    *split_tiles = g.split.split_tiles;
    *splits = g.split.splits;
    return CONVROT_OK;
}

convrot_status convrot_debug_gemm_split(const uint8_t *qx, const float *sx, const uint8_t *qw,
                                        const float *sw, const void *bias_bf16, int64_t M,
                                        int64_t N, int64_t K, int tiles, int split_tiles,
                                        int splits, void *split_ws, size_t split_bytes,
                                        int out_s32, void *out, convrot_stream_t stream) {
    if (M < 0 || N < 0) return CONVROT_ERR_SHAPE;
    const bool wrep = (tiles & CONVROT_TILES_REPACKED) != 0;
    tiles &= ~CONVROT_TILES_REPACKED;
    if (tiles != kTilesAuto && tiles != kTiles128x256 && tiles != kTiles128x192 &&
        tiles != kTiles256x192Pair && tiles != kTiles256x128Pair)
        return CONVROT_ERR_SHAPE;
    if (split_tiles < -1 || (split_tiles > 0 && splits < 2)) return CONVROT_ERR_SHAPE;
    if (M <= kSkinnyMaxM) return CONVROT_ERR_SHAPE;   // the token-major forms only
    if (N == 0) return CONVROT_OK;
    convrot_status st = check_gemm_args(qx, qw, M, N, K);
    if (st != CONVROT_OK) return st;
    if (!out || !split_ws || (!out_s32 && (!sx || !sw))) return CONVROT_ERR_NULL;
    if (split_bytes < CONVROT_SPLIT_COUNTER_BYTES || (reinterpret_cast<uintptr_t>(split_ws) & 255u))
        return CONVROT_ERR_WORKSPACE;
    if (!aligned16(out) || (!out_s32 && (!aligned16(sx) || !aligned16(sw) ||
                                         (bias_bf16 && !aligned16(bias_bf16)))))
        return CONVROT_ERR_ALIGN;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {qx, qw, out, split_ws})) != CONVROT_OK) return st;
    if (!out_s32 && (st = check_device_ptrs(dev, {sx, sw, bias_bf16})) != CONVROT_OK) return st;
    SplitArea area;
    area.ws = static_cast<uint32_t *>(split_ws);
    area.bytes = split_bytes;
    area.force_tiles = split_tiles;
    area.force_splits = splits;
    if (out_s32)
        return launch_gemm<true>(g_dev[dev], qx, nullptr, qw, nullptr, nullptr, M, N, K, out, stream,
                                 tiles, false, wrep, area);
    return launch_gemm<false>(g_dev[dev], qx, sx, qw, sw, bias_bf16, M, N, K, out, stream, tiles,
                              false, wrep, area);
}

convrot_status convrot_check_device_error(convrot_stream_t stream) {
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

// The timeout probe: one thread waits on a barrier nothing signals.
__global__ void timeout_probe_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    const uint32_t b = ptx::smem_u32(&bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(b, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) ptx::mbar_wait(b, 0, &abort_flag, limit_ns);
}

extern "C" convrot_status convrot_debug_timeout_probe(int64_t timeout_ns,
                                                      convrot_stream_t stream) {
    int dev;
    convrot_status st = device_setup(&dev);
    if (st != CONVROT_OK) return st;
    if (timeout_ns < 1000) timeout_ns = 1000;
    if (timeout_ns > 5000000000ll) timeout_ns = 5000000000ll;
    timeout_probe_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(timeout_ns));
    return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// convrot_linear_noalloc: the whole layer with the library's own scratch.
//
// For callers that cannot hand out device memory (a plugin inside a runtime
// that owns all allocations, or a path that must not call cudaMalloc because
// it can synchronise the device).  The packed activation codes and scales
// live in this fixed file-scope array instead of a caller's workspace.  In
// host code `g_noalloc_scratch` names only a host-side stand-in for the
// symbol, so its real device address is looked up once per device with
// cudaGetSymbolAddress and that address is what the kernels receive.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[CONVROT_NOALLOC_SCRATCH_BYTES];

namespace {
std::atomic<void *> g_noalloc_addr[kMaxDevices];

// Device address of the scratch array on `dev` (the current device).  The
// first call on a device performs the lookup; it must not run during stream
// capture.
convrot_status noalloc_scratch(int dev, uint8_t **out) {
    void *p = g_noalloc_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_mu);
        p = g_noalloc_addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
                return CONVROT_ERR_CUDA;
            g_noalloc_addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = static_cast<uint8_t *>(p);
    return CONVROT_OK;
}
}  // namespace

extern "C" convrot_status convrot_linear_noalloc(const void *x_bf16, const uint8_t *qw,
                                                 const float *sw, const void *bias_bf16, int64_t M,
                                                 int64_t N, int64_t K, int group, void *y_bf16,
                                                 convrot_stream_t stream) {
    convrot_status st = check_shape(M, K, group);
    if (st != CONVROT_OK) return st;
    if (N < 0) return CONVROT_ERR_SHAPE;
    if (M == 0 || N == 0) return CONVROT_OK;
    if (!x_bf16 || !qw || !sw || !y_bf16) return CONVROT_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(qw) || !aligned16(sw) || !aligned16(y_bf16) ||
        (bias_bf16 && !aligned16(bias_bf16)))
        return CONVROT_ERR_ALIGN;
    if ((st = check_gemm_args(qw, qw, M, N, K)) != CONVROT_OK) return st;
    if (prepared_bytes(M, K) > CONVROT_NOALLOC_SCRATCH_BYTES) return CONVROT_ERR_SCRATCH_LIMIT;
    int dev;
    if ((st = device_setup(&dev)) != CONVROT_OK) return st;
    if ((st = check_device_ptrs(dev, {x_bf16, qw, sw, bias_bf16, y_bf16})) != CONVROT_OK) return st;
    // 1..4 tokens: the same one-kernel form as convrot_linear, which needs no
    // scratch at all.
    if (decode_stages(M, K, group) > 0)
        if (const int sp = decode_stages(M, K, group, skinny::rows_per_cta(N, g_dev[dev].num_sms)))
            return launch_decode(g_dev[dev].num_sms, sp, x_bf16, qw, sw, bias_bf16, M, N, K,
                                 group, y_bf16, stream);
    uint8_t *qx = nullptr;
    if ((st = noalloc_scratch(dev, &qx)) != CONVROT_OK) return st;
    // Every byte of qx and sx read by the GEMM is written by the prep kernel
    // first, so leftovers of an earlier call never reach the result.
    float *sx = reinterpret_cast<float *>(qx + round256(static_cast<size_t>(M) * (K / 2)));
    if ((st = launch_prep(g_dev[dev].num_sms, x_bf16, M, K, group, qx, sx, nullptr, stream)) != CONVROT_OK)
        return st;
    return launch_gemm<false>(g_dev[dev], qx, sx, qw, sw, bias_bf16, M, N, K, y_bf16,
                              stream, kTilesAuto, true);
}

// switch_tc_host.cuh -- host side of the tensor-core switch: which ranks it
// takes, the TMA tensor maps of each (layer, target) weight, and the launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "common.cuh"
#include "switch_fold.cuh"
#include "switch_tc.cuh"
#include "switch_tc2.cuh"

namespace adafuse {

// The tensor-core kernel needs TMA-legal strides: rank a multiple of 8, or
// below 8 with B read from a copy whose rows are padded to 8.
inline int tc_kp_for(int r) {
    if (r < 1 || r > 64) return 0;
    if (r < 8) return 16;
    return r % 8 != 0 ? 0 : r <= 16 ? 16 : r <= 32 ? 32 : 64;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// Blocked maps (one TMA operation per W tile and per expert's A columns)
// need every weight's in to be a multiple of 64.
inline bool blocked_maps_ok(const PairDesc* pairs, int64_t n) {
    for (int64_t i = 0; i < n; ++i)
        if (pairs[i].in % 64 != 0) return false;
    return true;
}

// The W map alone (slot 0), plain or blocked; the re-base source W0 uses it
// too.  Plain: W [out, in], box 64 x 128 (cols x rows).  Blocked: W viewed as
// [in/64][out][64] (block stride 128 bytes, row stride 2*in), box 64 x 128 x 2,
// which lands in shared memory as two 64-column halves 16 KB apart, the plain
// layout of a wide tile.  128B swizzle either way.
inline bool encode_w_map(EncodeTiledFn enc, const void* W, int64_t out, int64_t in, bool blk,
                         CUtensorMap* m) {
    const cuuint32_t ones[3] = {1, 1, 1};
    if (blk) {
        const cuuint64_t dims[3] = {64, (cuuint64_t)out, (cuuint64_t)(in / 64)};
        const cuuint64_t strides[2] = {(cuuint64_t)in * 2, 128};
        const cuuint32_t box[3] = {64, 128, 2};
        return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(W), dims, strides,
                   box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
               CUDA_SUCCESS;
    }
    const cuuint64_t dims[2] = {(cuuint64_t)in, (cuuint64_t)out};
    const cuuint64_t strides[1] = {(cuuint64_t)in * 2};
    const cuuint32_t box[2] = {64, 128};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box,
               ones, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// The kMapsPerPair maps of one (layer, target):
// [0] W (encode_w_map);
// [1] A [E, r, in]: box 64 x rows x 1, 128B swizzle (rows past r read as zero);
// [2] B [E, out, r]: box KP x 128 x 1, swizzle = KP*2 bytes (cols past r read as zero);
// [3] blocked only: A viewed as [E][in/64][r][64], box 64 x rows x 2 x 1, the
//     two 64-column halves of one expert's slice in one operation (zeroed
//     when plain).
inline bool encode_pair_maps(EncodeTiledFn enc, const PairDesc& pd, int E, int r, int kp,
                             bool blk, CUtensorMap out[kMapsPerPair]) {
    const cuuint32_t ones[4] = {1, 1, 1, 1};
    const cuuint32_t a_rows = (cuuint32_t)(r <= 8 ? 8 : kp);
    if (!encode_w_map(enc, pd.W, pd.out, pd.in, blk, &out[0])) return false;
    std::memset(&out[3], 0, sizeof(CUtensorMap));
    if (blk) {
        const cuuint64_t dims[4] = {64, (cuuint64_t)r, (cuuint64_t)(pd.in / 64), (cuuint64_t)E};
        const cuuint64_t strides[3] = {(cuuint64_t)pd.in * 2, 128, (cuuint64_t)pd.in * r * 2};
        const cuuint32_t box[4] = {64, a_rows, 2, 1};
        if (enc(&out[3], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, (void*)pd.A, dims, strides, box,
                ones, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)pd.in, (cuuint64_t)r, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)pd.in * 2, (cuuint64_t)pd.in * r * 2};
        // ranks up to 8 fetch an 8-row box, other ranks a KP-row box; rows
        // past r read as zero
        const cuuint32_t box[3] = {64, a_rows, 1};
        if (enc(&out[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)pd.A, dims, strides, box,
                ones, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    if (r < 8) {
        // B rows of 2r bytes are not a legal TMA stride; the rank <= 8 path
        // bulk-copies the padded rows instead and never uses this map
        std::memset(&out[2], 0, sizeof(CUtensorMap));
        return true;
    }
    {
        const cuuint64_t dims[3] = {(cuuint64_t)r, (cuuint64_t)pd.out, (cuuint64_t)E};
        const cuuint64_t strides[2] = {(cuuint64_t)r * 2, (cuuint64_t)pd.out * r * 2};
        const cuuint32_t box[3] = {(cuuint32_t)kp, 128, 1};
        const CUtensorMapSwizzle sw = kp == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                    : kp == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_128B;
        if (enc(&out[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void*)pd.B, dims, strides, box,
                ones, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    return true;
}

// One launch of the tensor-core switch: persistent grid (one CTA per SM, at
// most one per tile), dynamic shared memory opted in once per device.
template <int KP, bool BBULK>
cudaError_t launch_switch_tc(const TcParams& prm, int device, int sm_count, cudaStream_t s) {
    const int smem = (int)TcConfig<KP, BBULK>::kSmemBytes;
    static int configured_for = -1;  // device ordinal the attribute was set on
    if (configured_for != device) {
        cudaError_t e = cudaFuncSetAttribute(switch_tc_kernel<KP, BBULK>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured_for = device;
    }
    const int64_t n = prm.t_end - prm.t_begin;
    const unsigned grid = (unsigned)(n < sm_count ? n : sm_count);
    switch_tc_kernel<KP, BBULK><<<grid, kTcThreads, smem, s>>>(prm);
    return cudaGetLastError();
}

// The folded tensor-core switch (ranks <= 8): the fold launch over the
// weights [w0, w0 + nw) the tiles belong to, then the switch launch, both on
// `s`.
inline cudaError_t launch_switch_fold(const TcParams& prm, int64_t w0, int64_t nw, int r,
                                      int device, int sm_count, cudaStream_t s) {
    const int smem = (int)FoldConfig::kSmemBytes;
    static int configured_for = -1;  // device ordinal the attribute was set on
    if (configured_for != device) {
        cudaError_t e = cudaFuncSetAttribute(switch_fold_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        configured_for = device;
    }
    const unsigned gy = (unsigned)(nw < 65535 ? nw : 65535);
    fold_operands_kernel<<<dim3(96, gy), kFoldThreads, 0, s>>>(prm.pairs, w0, nw, r, prm.prev,
                                                               prm.cur, prm.slots, prm.E, prm.s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = prm.t_end - prm.t_begin;
    const unsigned grid = (unsigned)(n < sm_count ? n : sm_count);
    switch_fold_kernel<<<grid, kTcThreads, smem, s>>>(prm);
    return cudaGetLastError();
}

// Co-resident CTA pairs of the pair kernel on this device (a persistent grid
// must not exceed it, or the clusters that do not fit run after the others).
template <int KP>
cudaError_t pair_kernel_clusters(int sm_count, int* clusters) {
    const int smem = (int)Tc2Config<KP>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(switch_tc2_kernel<KP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(sm_count & ~1));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, switch_tc2_kernel<KP>, &cfg);
    if (e != cudaSuccess) return e;
    *clusters = n;
    return n > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// One launch of the pair kernel: `clusters` CTA pairs (at most one per block
// of the table), each persistent over a strided share of the blocks.
template <int KP>
cudaError_t launch_switch_tc2(const TcParams& prm, int clusters, cudaStream_t s) {
    const int smem = (int)Tc2Config<KP>::kSmemBytes;
    const int64_t n = prm.t_end - prm.t_begin;
    const int64_t nc = n < clusters ? n : clusters;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * nc));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, switch_tc2_kernel<KP>, prm);
}

}  // namespace adafuse

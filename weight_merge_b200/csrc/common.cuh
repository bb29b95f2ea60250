// common.cuh -- device-side types shared by the pre-gate and switch kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "adafuse.h"

namespace adafuse {

// Edge of one segment-table tile of W (rows x cols).
constexpr int kTile = 128;

// One (layer, target) weight as the kernels see it.
struct PairDesc {
    uint16_t* W;         // [out, in] bf16 bits
    const uint16_t* A;   // [E, r, in]
    const uint16_t* B;   // [E, out, r]
    const uint16_t* W0;  // [out, in] pristine base for the re-base switch (or null)
    int32_t out;
    int32_t in;
    int32_t layer;
    int32_t target;
};

// One segment-table entry: which weight, which 128x128 tile of it.
//   x = index into the PairDesc array | (1 << 31) when the tile's second
//       64-column half starts inside the weight (col0 + 64 < in)
//   y = (row tile << 16) | col tile
using TileEntry = uint2;
constexpr uint32_t kTileWideBit = 0x80000000u;
constexpr uint32_t kTilePairMask = 0x7fffffffu;

// The union of the previous and the current route, as coefficients:
// c_e = s * (g_cur(e) - g_prev(e)) for each distinct expert, zeros dropped.
struct Coefs {
    int n;
    int e[4];
    float c[4];
};

// Read and check both routes, then build the coefficient list.  Every
// thread of every CTA computes the same result from the same 32 bytes, so
// either all CTAs write W or none does.  Returns a status bit set (0 = ok).
__device__ __forceinline__ int build_coefs(const adafuse_route* prev,
                                           const adafuse_route* cur, int E,
                                           float s, Coefs& cf) {
    int status = 0;
    int ue[4];
    float ug[4];
    int n = 0;
    auto add = [&](int e, float g) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < n && ue[i] == e) { ug[i] += g; return; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i == n) { ue[i] = e; ug[i] = g; }
        ++n;
    };
    // current token's experts enter with +g, previous token's with -g
#pragma unroll
    for (int side = 0; side < 2; ++side) {
        const adafuse_route* rt = side == 0 ? cur : prev;
        if (rt == nullptr) continue;
        const int4 raw = __ldg(reinterpret_cast<const int4*>(rt));
        const int idx[2] = {raw.x, raw.y};
        const float gate[2] = {__int_as_float(raw.z), __int_as_float(raw.w)};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (idx[j] < -1 || idx[j] >= E) { status |= ADAFUSE_STATUS_BAD_EXPERT; continue; }
            if (idx[j] < 0) continue;
            if (!isfinite(gate[j])) { status |= ADAFUSE_STATUS_BAD_GATE; continue; }
            add(idx[j], side == 0 ? gate[j] : -gate[j]);
        }
    }
    cf.n = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        cf.e[i] = 0;
        cf.c[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i >= n) continue;
        const float c = s * ug[i];
        if (c == 0.f) continue;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (k == cf.n) { cf.e[k] = ue[i]; cf.c[k] = c; }
        ++cf.n;
    }
    return status;
}

}  // namespace adafuse

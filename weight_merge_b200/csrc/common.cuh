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
    const uint16_t* Bk;  // [E, out, 8] B with 16-byte rows for the rank <= 8 tensor-core
                         // path: B itself at rank 8, a zero-padded copy below
    uint16_t* Af;        // rank <= 8: the folded-coefficient operand the fold launch
                         // writes before each folded switch (or null)
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
// Routes hold 2 slots (top-2) or up to 4 (top-k), so at most 8 experts.
// CAP is the list's capacity: 4 for top-2 routes, 8 for top-k routes.
constexpr int kMaxCoefs = 8;
template <int CAP>
struct CoefsT {
    int n;
    int e[CAP];
    float c[CAP];
};
using Coefs = CoefsT<4>;
using Coefs8 = CoefsT<kMaxCoefs>;

// Entry i of the coefficient list (i warp- and launch-uniform), without
// dynamic indexing into the arrays (which would put them in local memory).
template <int CAP>
__device__ __forceinline__ int coef_expert(const CoefsT<CAP>& cf, int i) {
    int e = cf.e[0];
#pragma unroll
    for (int j = 1; j < CAP; ++j)
        if (i == j) e = cf.e[j];
    return e;
}
template <int CAP>
__device__ __forceinline__ float coef_value(const CoefsT<CAP>& cf, int i) {
    float c = cf.c[0];
#pragma unroll
    for (int j = 1; j < CAP; ++j)
        if (i == j) c = cf.c[j];
    return c;
}

// Read and check both routes, then build the coefficient list.  A route of
// `slots` slots (2 or 4) is idx[slots] int32 followed by gate[slots] fp32:
// adafuse_route for 2 slots, adafuse_route4 for 4.  Every thread of every
// CTA computes the same result from the same bytes, so either all CTAs write
// W or none does.  Returns a status bit set (0 = ok).
template <int SLOTS, int CAP>
__device__ __forceinline__ int build_coefs_slots(const int32_t* prev, const int32_t* cur, int E,
                                                 float s, CoefsT<CAP>& cf) {
    static_assert(SLOTS == 2 || SLOTS == 4, "slots");
    static_assert(CAP >= 2 * SLOTS && CAP <= kMaxCoefs, "capacity");
    int status = 0;
    int ue[CAP];
    float ug[CAP];
    int n = 0;
    auto add = [&](int e, float g) {
#pragma unroll
        for (int i = 0; i < CAP; ++i)
            if (i < n && ue[i] == e) { ug[i] += g; return; }
#pragma unroll
        for (int i = 0; i < CAP; ++i)
            if (i == n) { ue[i] = e; ug[i] = g; }
        ++n;
    };
    // current token's experts enter with +g, previous token's with -g
#pragma unroll
    for (int side = 0; side < 2; ++side) {
        const int32_t* rt = side == 0 ? cur : prev;
        if (rt == nullptr) continue;
        int idx[SLOTS];
        float gate[SLOTS];
        if constexpr (SLOTS == 2) {
            const int4 raw = __ldg(reinterpret_cast<const int4*>(rt));
            idx[0] = raw.x; idx[1] = raw.y;
            gate[0] = __int_as_float(raw.z); gate[1] = __int_as_float(raw.w);
        } else {
            const int4 ri = __ldg(reinterpret_cast<const int4*>(rt));
            const int4 rg = __ldg(reinterpret_cast<const int4*>(rt) + 1);
            idx[0] = ri.x; idx[1] = ri.y; idx[2] = ri.z; idx[3] = ri.w;
            gate[0] = __int_as_float(rg.x); gate[1] = __int_as_float(rg.y);
            gate[2] = __int_as_float(rg.z); gate[3] = __int_as_float(rg.w);
        }
#pragma unroll
        for (int j = 0; j < SLOTS; ++j) {
            if (idx[j] < -1 || idx[j] >= E) { status |= ADAFUSE_STATUS_BAD_EXPERT; continue; }
            if (idx[j] < 0) continue;
            if (!isfinite(gate[j])) { status |= ADAFUSE_STATUS_BAD_GATE; continue; }
            add(idx[j], side == 0 ? gate[j] : -gate[j]);
        }
    }
    cf.n = 0;
#pragma unroll
    for (int i = 0; i < CAP; ++i) {
        cf.e[i] = 0;
        cf.c[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < CAP; ++i) {
        if (i >= n) continue;
        const float c = s * ug[i];
        if (c == 0.f) continue;
#pragma unroll
        for (int k = 0; k < CAP; ++k)
            if (k == cf.n) { cf.e[k] = ue[i]; cf.c[k] = c; }
        ++cf.n;
    }
    return status;
}

__device__ __forceinline__ int build_coefs(const int32_t* prev, const int32_t* cur, int slots,
                                           int E, float s, Coefs8& cf) {
    return slots == 4 ? build_coefs_slots<4>(prev, cur, E, s, cf)
                      : build_coefs_slots<2>(prev, cur, E, s, cf);
}

// The top-2 form (adafuse_route records).
__device__ __forceinline__ int build_coefs(const adafuse_route* prev, const adafuse_route* cur,
                                           int E, float s, Coefs& cf) {
    return build_coefs_slots<2>(reinterpret_cast<const int32_t*>(prev),
                                reinterpret_cast<const int32_t*>(cur), E, s, cf);
}

}  // namespace adafuse

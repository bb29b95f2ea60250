// switch_mma.cuh -- fused adapter switch, register-streaming variant
// (mma.sync m16n8k16 / m16n8k8, bf16 inputs, fp32 accumulators).
//
// AdaFuse (gist.science technical summary, section 2-na): one launch walks the
// segment table of every (layer, target) weight and applies, in place,
//   W <- bf16_rne(W + sum_e c_e (B_e A_e)),  c_e = s (g_cur(e) - g_prev(e)).
//
// Work unit: one 128x128 W tile.  CTA = 8 warps; warp w owns tile rows
// [16w, 16w+16) and all 128 columns, as four 32-column groups.  Lane (g, t)
// (g = lane/4, t = lane%4) owns, per group, the 16-byte W chunks at rows g and
// g+8, columns [8t, 8t+8) -- so one warp-wide 16-byte access covers 8 rows x 64
// contiguous bytes and W never passes through shared memory.
//
// To make the mma.sync accumulator land exactly on those chunks, the columns
// of A_e fed to the MMA are permuted: the accumulator of n-tile j, column
// 2t+b, is W column 8t + 2j + b of the group, so the B-operand column n of
// n-tile j is A_e column 8(n/2) + 2j + (n%2).  A 16-byte load of one A_e row
// then serves all four n-tiles (one byte-permute each).
//
// Each expert has its own fp32 accumulator, scaled by c_e in fp32 after its
// K = rank reduction; the expert sum is added to float(W) and rounded once.
// The CTA is persistent over a strided slice of the tile list; while group k
// of tile i is being finished, group k of tile i+gridDim is already being
// loaded (rolling register prefetch keeps 32 KB of W reads in flight per CTA).
#pragma once

#include "common.cuh"

namespace adafuse {

constexpr int kSwitchThreads = 256;

__device__ __forceinline__ void mma_k16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_k8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint4 ld_stream_16(const uint16_t* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void st_stream_16(uint16_t* p, uint4 v) {
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// B_e[row, k..k+1] packed (k in the low half); zero past the rank or the rows.
__device__ __forceinline__ uint32_t ld_b_pair(const uint16_t* brow, int k, int r, bool row_ok,
                                              bool r_even) {
    if (!row_ok || k >= r) return 0u;
    if (r_even) return __ldg(reinterpret_cast<const uint32_t*>(brow + k));
    const uint32_t lo = __ldg(reinterpret_cast<const unsigned short*>(brow + k));
    const uint32_t hi = (k + 1 < r) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(brow + k + 1)) : 0u;
    return lo | (hi << 16);
}

// One A_e row, 8 columns (16 bytes); zero past the rank or the columns.
__device__ __forceinline__ uint4 ld_a_row8(const uint16_t* arow, int k, int r, bool col_ok) {
    if (!col_ok || k >= r) return make_uint4(0u, 0u, 0u, 0u);
    return __ldg(reinterpret_cast<const uint4*>(arow));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// bf16x2 word -> two floats (exact widening)
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<const uint32_t*>(&v);
}

struct TileCoord {
    const uint16_t* A;
    const uint16_t* B;
    uint16_t* W;          // written
    const uint16_t* Wsrc; // read: W itself, or the pristine base when re-basing
    int out, in;
    int row0, col0;
};

__device__ __forceinline__ TileCoord load_tile(const PairDesc* __restrict__ pairs,
                                               const TileEntry* __restrict__ tiles, int64_t i,
                                               bool rebase) {
    const TileEntry te = __ldg(tiles + i);
    const PairDesc* pd = pairs + (te.x & kTilePairMask);
    TileCoord tc;
    tc.W = pd->W;
    tc.Wsrc = rebase ? pd->W0 : pd->W;
    tc.A = pd->A;
    tc.B = pd->B;
    tc.out = pd->out;
    tc.in = pd->in;
    tc.row0 = (int)(te.y >> 16) * kTile;
    tc.col0 = (int)(te.y & 0xffffu) * kTile;
    return tc;
}

// KP: per-expert contraction depth rounded up to 8, 16, 32 or 64.
// rebase: read W from the pristine base W0 instead of W itself (prev is null),
// so W <- rne(W0 + dW_cur); then even an empty route writes (it copies W0).
// SLOTS: route slots (2 for top-2 routes, 4 for top-k), so at most 2 * SLOTS experts.
template <int KP, int SLOTS>
__global__ void __launch_bounds__(kSwitchThreads, 2)
switch_mma_kernel(const PairDesc* __restrict__ pairs, const TileEntry* __restrict__ tiles,
                  int64_t t_begin, int64_t t_end, const int32_t* prev, const int32_t* cur,
                  int E, int r, float s, int32_t* status, int rebase) {
    CoefsT<2 * SLOTS> cf;
    const int st = build_coefs_slots<SLOTS>(prev, cur, E, s, cf);
    if (st != 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, st);
        return;
    }
    if (cf.n == 0 && !rebase) return;  // identity switch: nothing to write

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
    const bool r_even = (r & 1) == 0;

    int64_t tile = t_begin + blockIdx.x;
    if (tile >= t_end) return;
    TileCoord tc = load_tile(pairs, tiles, tile, rebase != 0);

    uint4 wv[4][2];
#pragma unroll
    for (int cg = 0; cg < 4; ++cg)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = tc.row0 + 16 * warp + g + 8 * hh;
            const int col = tc.col0 + 32 * cg + 8 * t;
            wv[cg][hh] = (row < tc.out && col < tc.in)
                             ? ld_stream_16(tc.Wsrc + (int64_t)row * tc.in + col)
                             : make_uint4(0u, 0u, 0u, 0u);
        }

    for (;;) {
        const int64_t next = tile + gridDim.x;
        const bool has_next = next < t_end;
        TileCoord tn = tc;
        if (has_next) tn = load_tile(pairs, tiles, next, rebase != 0);

        const int rowA = tc.row0 + 16 * warp + g;  // rows rowA and rowA + 8
        const bool okA0 = rowA < tc.out, okA1 = rowA + 8 < tc.out;

#pragma unroll
        for (int cg = 0; cg < 4; ++cg) {
            const int colc = tc.col0 + 32 * cg + 8 * (g >> 1);  // this lane's A_e chunk
            const bool col_ok = colc < tc.in;
            float tot[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) tot[j][q] = 0.f;

#pragma unroll
            for (int ei = 0; ei < 2 * SLOTS; ++ei) {
                if (ei >= cf.n) break;
                const int e = cf.e[ei];
                const uint16_t* Be = tc.B + (int64_t)e * tc.out * r;
                const uint16_t* Ae = tc.A + (int64_t)e * r * tc.in;
                const uint16_t* b0row = Be + (int64_t)rowA * r;
                const uint16_t* b1row = b0row + 8 * r;
                float acc[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;

                if constexpr (KP == 8) {
                    const int k = 2 * t;
                    const uint32_t a0 = ld_b_pair(b0row, k, r, okA0, r_even);
                    const uint32_t a1 = ld_b_pair(b1row, k, r, okA1, r_even);
                    const uint4 x0 = ld_a_row8(Ae + (int64_t)k * tc.in + colc, k, r, col_ok);
                    const uint4 x1 = ld_a_row8(Ae + (int64_t)(k + 1) * tc.in + colc, k + 1, r, col_ok);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_k8(acc[j], a0, a1, __byte_perm(word_of(x0, j), word_of(x1, j), sel));
                } else {
#pragma unroll
                    for (int k0 = 0; k0 < KP; k0 += 16) {
                        const int k = k0 + 2 * t;
                        uint32_t a[4];
                        a[0] = ld_b_pair(b0row, k, r, okA0, r_even);
                        a[1] = ld_b_pair(b1row, k, r, okA1, r_even);
                        a[2] = ld_b_pair(b0row, k + 8, r, okA0, r_even);
                        a[3] = ld_b_pair(b1row, k + 8, r, okA1, r_even);
                        const uint4 x0 = ld_a_row8(Ae + (int64_t)k * tc.in + colc, k, r, col_ok);
                        const uint4 x1 = ld_a_row8(Ae + (int64_t)(k + 1) * tc.in + colc, k + 1, r, col_ok);
                        const uint4 x2 = ld_a_row8(Ae + (int64_t)(k + 8) * tc.in + colc, k + 8, r, col_ok);
                        const uint4 x3 = ld_a_row8(Ae + (int64_t)(k + 9) * tc.in + colc, k + 9, r, col_ok);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_k16(acc[j], a, __byte_perm(word_of(x0, j), word_of(x1, j), sel),
                                    __byte_perm(word_of(x2, j), word_of(x3, j), sel));
                    }
                }
                const float c = cf.c[ei];
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int q = 0; q < 4; ++q) tot[j][q] = __fmaf_rn(c, acc[j][q], tot[j][q]);
            }

            // W <- rne(float(W) + dW) for the two 16-byte chunks of this group
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = tc.row0 + 16 * warp + g + 8 * hh;
                const int col = tc.col0 + 32 * cg + 8 * t;
                if (row < tc.out && col < tc.in) {
                    const uint4 w = wv[cg][hh];
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = bf2_to_f2(word_of(w, j));
                        o[j] = f2_to_bf2(f.x + tot[j][2 * hh], f.y + tot[j][2 * hh + 1]);
                    }
                    st_stream_16(tc.W + (int64_t)row * tc.in + col, make_uint4(o[0], o[1], o[2], o[3]));
                }
                // this chunk's registers are free: start reading the next tile's
                if (has_next) {
                    const int nrow = tn.row0 + 16 * warp + g + 8 * hh;
                    const int ncol = tn.col0 + 32 * cg + 8 * t;
                    wv[cg][hh] = (nrow < tn.out && ncol < tn.in)
                                     ? ld_stream_16(tn.Wsrc + (int64_t)nrow * tn.in + ncol)
                                     : make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        if (!has_next) break;
        tile = next;
        tc = tn;
    }
}

}  // namespace adafuse

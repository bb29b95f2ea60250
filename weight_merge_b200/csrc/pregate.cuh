// pregate.cuh -- token-level pre-gating kernel (router GEMV + top-2 + gates).
//
// AdaFuse (gist.science technical summary, section 2-ga): a top-2 router in
// the first layer makes one routing decision per token, applied to every
// adapter layer afterwards.
//
// Design: an HBM-bound GEMV over h.  A CTA of 256 threads (8 warps) takes a
// group of TPB tokens; thread i walks the float4 chunks i, i+256, ... of d
// (4 rows of Wr each), keeping TPB x EMAX fp32 partial logits in registers, so
// each Wr value fetched serves TPB tokens.  A fixed xor-shuffle tree and then
// a fixed in-order sum over the 8 warps finish each logit.
//
// Wr comes from one of three places with the same arithmetic:
//   kWrShared  large batches: Wr staged once per (persistent) CTA in shared
//              memory, each 4-row chunk padded to an odd number of 16-byte
//              slots so per-thread float4 reads are bank-conflict free;
//   kWrVector  E == EMAX: a row of Wr is EMAX/4 aligned float4 loads;
//   kWrScalar  E < EMAX: scalar loads, zero for experts past E.
// Every token's logits are therefore bitwise the same whatever batch it is
// gated in, and every expert column goes through exactly the same operation
// sequence, so two equal columns of Wr give bitwise-equal logits and the tie
// rule (lower index first) is exact.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace adafuse {

constexpr int kPregateThreads = 256;
enum : int { kWrShared = 0, kWrVector = 1, kWrScalar = 2 };

// The routing decision of one token from its logits z[0..E): top-k under
// (z descending, index ascending) -- pick j is the largest logit not yet
// picked, the lower index among equals -- and gates = the softmax over all E
// renormalised over the picks, in the closed form g_j = x_j / (1 + x_1 +
// ...), x_j = exp(z_j - z_0) <= 1.  Written as one adafuse_route (slots 2) or
// adafuse_route4 (slots 4) record at index t.
template <int EMAX>
__device__ __forceinline__ void route_tail(const float (&z)[EMAX], int E, int k, int slots,
                                           int32_t* __restrict__ route, int64_t t) {
    int pick[4] = {-1, -1, -1, -1};
    float zp[4] = {0.f, 0.f, 0.f, 0.f};
    uint64_t taken = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (j >= k) break;
        int best = -1;
        float zb = 0.f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e >= E || ((taken >> e) & 1ull)) continue;
            if (best < 0 || z[e] > zb) { best = e; zb = z[e]; }
        }
        if (best < 0) break;
        pick[j] = best;
        zp[j] = zb;
        taken |= 1ull << best;
    }
    float x[4] = {1.f, 0.f, 0.f, 0.f};
    float den = 1.f;
#pragma unroll
    for (int j = 1; j < 4; ++j)
        if (pick[j] >= 0) {
            x[j] = expf(zp[j] - zp[0]);
            den = den + x[j];
        }
    float g[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) g[j] = pick[j] >= 0 ? x[j] / den : 0.f;
    if (slots == 2) {
        reinterpret_cast<int4*>(route)[t] =
            make_int4(pick[0], pick[1], __float_as_int(g[0]), __float_as_int(g[1]));
    } else {
        int4* r4 = reinterpret_cast<int4*>(route) + 2 * t;
        r4[0] = make_int4(pick[0], pick[1], pick[2], pick[3]);
        r4[1] = make_int4(__float_as_int(g[0]), __float_as_int(g[1]), __float_as_int(g[2]),
                          __float_as_int(g[3]));
    }
}

template <int EMAX, int TPB, int WR>
__global__ void __launch_bounds__(kPregateThreads)
pregate_kernel(const float* __restrict__ h, int64_t T, int64_t d, const float* __restrict__ Wr,
               int E, int k, int slots, int32_t* __restrict__ route, float* __restrict__ logits) {
    static_assert(EMAX % 4 == 0, "EMAX");
    constexpr int kWarps = kPregateThreads / 32;
    constexpr int S4 = EMAX + 1;             // float4 slots per chunk in shared memory
    __shared__ float part[kWarps][TPB][EMAX];
    extern __shared__ float4 wr_s[];
    const int64_t nchunk = d >> 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if constexpr (WR == kWrShared) {
        if (E == EMAX && (reinterpret_cast<uintptr_t>(Wr) & 15u) == 0) {
            // a 4-row chunk of Wr is EMAX contiguous float4 in global memory
            const float4* src = reinterpret_cast<const float4*>(Wr);
#pragma unroll 8
            for (int64_t i = threadIdx.x; i < nchunk * EMAX; i += kPregateThreads)
                wr_s[(i / EMAX) * S4 + (i % EMAX)] = __ldg(src + i);
        } else {
            float* wf = reinterpret_cast<float*>(wr_s);
#pragma unroll 8
            for (int64_t i = threadIdx.x; i < nchunk * 4 * EMAX; i += kPregateThreads) {
                const int64_t row = i / EMAX;
                const int e = (int)(i % EMAX);
                wf[(row >> 2) * (4 * S4) + (row & 3) * EMAX + e] = e < E ? __ldg(Wr + row * E + e) : 0.f;
            }
        }
        __syncthreads();
    }

    for (int64_t g = blockIdx.x; g * TPB < T; g += gridDim.x) {
        const int64_t t0 = g * TPB;
        float acc[TPB][EMAX];
#pragma unroll
        for (int tt = 0; tt < TPB; ++tt)
#pragma unroll
            for (int e = 0; e < EMAX; ++e) acc[tt][e] = 0.f;

#pragma unroll 2
        for (int64_t c = threadIdx.x; c < nchunk; c += kPregateThreads) {
            float4 hv[TPB];
#pragma unroll
            for (int tt = 0; tt < TPB; ++tt)
                hv[tt] = (t0 + tt < T) ? __ldcs(reinterpret_cast<const float4*>(h + (t0 + tt) * d) + c)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float w[EMAX];                       // row 4c+q of Wr, experts 0..EMAX-1
                if constexpr (WR == kWrShared) {
#pragma unroll
                    for (int k = 0; k < EMAX / 4; ++k) {
                        const float4 f = wr_s[c * S4 + q * (EMAX / 4) + k];
                        w[4 * k] = f.x; w[4 * k + 1] = f.y; w[4 * k + 2] = f.z; w[4 * k + 3] = f.w;
                    }
                } else if constexpr (WR == kWrVector) {
                    const float4* row = reinterpret_cast<const float4*>(Wr + (4 * c + q) * (int64_t)EMAX);
#pragma unroll
                    for (int k = 0; k < EMAX / 4; ++k) {
                        const float4 f = __ldg(row + k);
                        w[4 * k] = f.x; w[4 * k + 1] = f.y; w[4 * k + 2] = f.z; w[4 * k + 3] = f.w;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < EMAX; ++e) w[e] = e < E ? __ldg(Wr + (4 * c + q) * E + e) : 0.f;
                }
#pragma unroll
                for (int e = 0; e < EMAX; ++e)
#pragma unroll
                    for (int tt = 0; tt < TPB; ++tt) {
                        const float x = q == 0 ? hv[tt].x : q == 1 ? hv[tt].y : q == 2 ? hv[tt].z : hv[tt].w;
                        acc[tt][e] = __fmaf_rn(x, w[e], acc[tt][e]);
                    }
            }
        }

        // warp tree (same shape for every (token, expert)), then warps in order
#pragma unroll
        for (int tt = 0; tt < TPB; ++tt)
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                float v = acc[tt][e];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) part[warp][tt][e] = v;
            }
        __syncthreads();

        if (threadIdx.x < TPB && t0 + threadIdx.x < T) {
            const int tt = threadIdx.x;
            float z[EMAX];
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                float v = part[0][tt][e];
#pragma unroll
                for (int w = 1; w < kWarps; ++w) v += part[w][tt][e];
                z[e] = v;
            }
            if (logits != nullptr) {
#pragma unroll
                for (int e = 0; e < EMAX; ++e)
                    if (e < E) logits[(t0 + tt) * E + e] = z[e];
            } else {
                route_tail<EMAX>(z, E, k, slots, route, t0 + tt);
            }
        }
        __syncthreads();   // part[] is reused by the next token group
    }
}


// ---------------------------------------------------------------------------
// Token-group form of the same router for batches (E <= 8, d <= 4096).  It
// computes every logit with exactly the operation sequence of pregate_kernel
// above -- virtual thread i = 32 * vw + lane of a 256-thread group (vw = 0..7)
// accumulates the float4 chunks i, i + 256, ... in order (one fp32 FMA per
// element and expert), the xor tree at lane distances 16, 8, 4, 2, 1 finishes
// each virtual warp's sum, and the eight virtual-warp sums are added in order
// -- so both kernels give the same bits for the same token, and the launch
// may pick either by batch size without changing any route.
//
// What changes is who does the work.  A pair of warps owns a group of
// kGroupTokens tokens: the even warp walks virtual warps 0..3, the odd warp
// 4..7.  Per virtual warp and chunk index m a warp's lanes load the group's h
// chunks (two such steps ahead of the arithmetic, in a ring of four register
// slots), read Wr's rows from shared memory (staged once per CTA, by TMA
// tile loads with 128-byte swizzle when E == 8, else by the CTA's threads in
// the same layout; shared by the group's tokens) and accumulate; a
// reduce-scatter over the same lane
// pairs as the xor tree (5 rounds, 31 shuffles for 32 (token, expert) sums)
// then leaves lane L with token L / 8, expert L % 8 of that virtual warp.  The
// even warp adds its four sums in order and hands the partial sum to the odd
// warp through shared memory (a 64-thread named barrier per pair, buffers
// alternating by group), which adds its own four in order: the same eight
// additions as one warp walking all eight.  Four lanes of the odd warp then
// run the four tokens' top-k tails side by side.

// bar.sync on barrier `id` for `nthreads` threads (whole warps) of the CTA;
// orders their shared-memory accesses like __syncthreads does for all.
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

constexpr int kGroupTokens = 4;
constexpr int kGroupThreads = 512;                // 8 warp pairs
constexpr int kGroupPairs = kGroupThreads / 64;
constexpr int kGroupMaxChunks = 4;                 // d <= 256 * 4 * 4 = 4096
constexpr int64_t kGroupMinTokens = 64;           // smaller batches: pregate_kernel

constexpr int kGroupWrBoxRows = 256;                // chunks per Wr tile load (32 KB)

// Wr in shared memory: chunk c (rows 4c..4c+3, experts 0..7) is 128 bytes,
// its float4 f stored at slot c * 8 + (f ^ (c % 8)) -- the layout a TMA tile
// load with 128-byte swizzle writes into a 1024-byte-aligned buffer -- so
// lanes reading their own chunks 128 bytes apart hit distinct bank groups.
// Whole 256-chunk boxes (zero past d).
__host__ __device__ constexpr size_t group_wr_bytes(int64_t d) {
    return (size_t)((d / 4 + kGroupWrBoxRows - 1) / kGroupWrBoxRows) * kGroupWrBoxRows * 128;
}
__host__ __device__ constexpr size_t group_smem_bytes(int64_t d) {
    // 1024 bytes of alignment slack, Wr, the pairs' partial sums (two
    // buffers of 32 lanes each) and the staging barrier
    return 1024 + group_wr_bytes(d) + (size_t)kGroupPairs * 2 * 32 * sizeof(float) + 16;
}

// wr_map (used when wr_tma != 0): Wr viewed as [d / 4 chunks][32 floats],
// box 32 x 256, 128-byte swizzle; E must be 8.  status receives
// ADAFUSE_STATUS_TIMEOUT if those loads do not land within the wait limit.
template <int NCH>
__global__ void __launch_bounds__(kGroupThreads, 1)
pregate_group_kernel(const float* __restrict__ h, int64_t T, int64_t d,
                     const float* __restrict__ Wr, int E, int k, int slots,
                     int32_t* __restrict__ route, float* __restrict__ logits,
                     const __grid_constant__ CUtensorMap wr_map, int wr_tma,
                     int32_t* __restrict__ status) {
    extern __shared__ __align__(1024) uint8_t group_smem_raw[];
    float4* wr_s = reinterpret_cast<float4*>(
        (reinterpret_cast<uintptr_t>(group_smem_raw) + 1023) & ~uintptr_t(1023));
    float* zpart_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(wr_s) + group_wr_bytes(d));
    uint64_t* wr_bar = reinterpret_cast<uint64_t*>(zpart_s + kGroupPairs * 2 * 32);
    const int64_t nchunk = d >> 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = warp >> 1, half = warp & 1;
    constexpr int TPB = kGroupTokens;
    constexpr int kSteps = 4 * NCH;   // (virtual warp, chunk index) steps per warp and group
    const int64_t ngroups = (T + TPB - 1) / TPB;
    // groups go round the CTAs first, so every SM gets a share of a batch
    const int64_t g_first = blockIdx.x + (int64_t)pair * gridDim.x;
    const int64_t g_step = (int64_t)gridDim.x * kGroupPairs;
    // step s of this warp in group g: virtual warp 4 * half + s / NCH, chunk
    // index s % NCH; the group's h chunks for it (zero past d or T).  Groups
    // of 4 whole tokens with d = 1024 * NCH (every chunk inside d) take the
    // unchecked loads.  d <= 4096 here, so token offsets fit 32 bits.
    const bool d_full = nchunk == 256 * NCH;
    const int nch32 = (int)nchunk;
    const int lane_c = 128 * half + lane;            // chunk of step 0 (vw = 4 * half)
    auto group_ptr = [&](int64_t g) {
        return reinterpret_cast<const float4*>(h) + g * TPB * nchunk + lane_c;
    };
    auto load_step = [&](const float4* gp, int64_t g, int s, float4 (&hv)[TPB]) {
        const int off = 32 * (s / NCH) + 256 * (s % NCH);
        const int c = lane_c + off;
        const int64_t t0 = g * TPB;
        if (d_full && t0 + TPB <= T) {
#pragma unroll
            for (int tt = 0; tt < TPB; ++tt) hv[tt] = __ldcs(gp + off + tt * nch32);
        } else {
#pragma unroll
            for (int tt = 0; tt < TPB; ++tt)
                hv[tt] = (c < nch32 && t0 + tt < T) ? __ldcs(gp + off + tt * nch32)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    float4 ring[4][TPB];   // step s in slot s % 4 (kSteps is a multiple of 4)
    // the first group's first loads go out before Wr is staged, so the two
    // latencies overlap
    load_step(group_ptr(g_first), g_first, 0, ring[0]);
    load_step(group_ptr(g_first), g_first, 1, ring[1]);

    // ---- Wr into shared memory (the swizzled layout above): by TMA tile
    // loads when the launch encoded a map (E == 8, Wr 16-byte aligned),
    // otherwise by every thread, kStageBatch loads in flight before their
    // stores (experts past E read as zero)
    if (wr_tma) {
        volatile int* no_abort = reinterpret_cast<volatile int*>(wr_bar + 1);   // stays 0
        if (threadIdx.x == 0) {
            *no_abort = 0;
            sm100::mbar_init(wr_bar, 1);
            sm100::fence_mbar_init();
        }
        __syncthreads();
        const int nbox = (int)((nchunk + kGroupWrBoxRows - 1) / kGroupWrBoxRows);
        if (threadIdx.x == 0) {
            sm100::mbar_arrive_expect_tx(wr_bar, (uint32_t)nbox * kGroupWrBoxRows * 128u);
            for (int b = 0; b < nbox; ++b)
                sm100::tma_load_2d(reinterpret_cast<uint8_t*>(wr_s) + (size_t)b * kGroupWrBoxRows * 128,
                                   &wr_map, 0, b * kGroupWrBoxRows, wr_bar);
        }
        const bool landed = sm100::mbar_wait_bounded(wr_bar, 0, no_abort, 1000000000ull);
        // every thread of the CTA leaves together, or none does (the warp
        // pairs meet at named barriers later)
        if (__syncthreads_or(!landed)) {
            if (threadIdx.x == 0) atomicOr(status, ADAFUSE_STATUS_TIMEOUT);
            return;
        }
    } else {
        constexpr int kStageBatch = 8;
        const bool vec = E == 8 && (reinterpret_cast<uintptr_t>(Wr) & 15u) == 0;
        const int64_t total = nchunk * 8;
        for (int64_t i0 = threadIdx.x; i0 < total; i0 += kStageBatch * kGroupThreads) {
            float4 v[kStageBatch];
#pragma unroll
            for (int u = 0; u < kStageBatch; ++u) {
                const int64_t i = i0 + (int64_t)u * kGroupThreads;
                const int64_t c = i >> 3;
                const int f = (int)(i & 7);
                if (i >= total) {
                    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (vec) {
                    v[u] = __ldg(reinterpret_cast<const float4*>(Wr) + i);
                } else {
                    const int64_t row = 4 * c + (f >> 1);
                    const int e0 = (f & 1) * 4;
                    v[u].x = e0 + 0 < E ? __ldg(Wr + row * E + e0 + 0) : 0.f;
                    v[u].y = e0 + 1 < E ? __ldg(Wr + row * E + e0 + 1) : 0.f;
                    v[u].z = e0 + 2 < E ? __ldg(Wr + row * E + e0 + 2) : 0.f;
                    v[u].w = e0 + 3 < E ? __ldg(Wr + row * E + e0 + 3) : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kStageBatch; ++u) {
                const int64_t i = i0 + (int64_t)u * kGroupThreads;
                if (i < total) wr_s[(i >> 3) * 8 + ((i & 7) ^ ((i >> 3) & 7))] = v[u];
            }
        }
        __syncthreads();
    }

    const bool b16 = (lane & 16) != 0, b8 = (lane & 8) != 0, b4 = (lane & 4) != 0,
               b2 = (lane & 2) != 0, b1 = (lane & 1) != 0;
    int parity = 0;
    for (int64_t g = g_first; g < ngroups; g += g_step, parity ^= 1) {
        const float4* gp = group_ptr(g);
        const float4* gp_next = group_ptr(g + g_step);
        float zs[4];   // lane L: this warp's four virtual-warp sums for token L / 8, expert L % 8
        // acc2[tt][p]: experts 2p and 2p + 1 of token tt as a packed fp32
        // pair; fma.rn.f32x2 rounds each lane as fma.rn.f32 does, so every
        // (token, expert) sum takes the FMA sequence of pregate_kernel
        uint64_t acc2[TPB][4];
#pragma unroll
        for (int s = 0; s < kSteps; ++s) {
            const int m = s % NCH;
            const int vw = 4 * half + s / NCH;
            // two steps ahead: this group's step s + 2, or the next group's
            if (s + 2 < kSteps)
                load_step(gp, g, s + 2, ring[(s + 2) & 3]);
            else
                load_step(gp_next, g + g_step, s + 2 - kSteps, ring[(s + 2) & 3]);
            if (m == 0) {
#pragma unroll
                for (int tt = 0; tt < TPB; ++tt)
#pragma unroll
                    for (int pe = 0; pe < 4; ++pe) acc2[tt][pe] = 0ull;
            }
            const int c = 32 * vw + lane + 256 * m;
            if (d_full || c < nch32) {
                const int sw = c & 7;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 wa = wr_s[c * 8 + ((2 * q) ^ sw)], wb = wr_s[c * 8 + ((2 * q + 1) ^ sw)];
                    const uint64_t w2[4] = {sm100::f32x2(wa.x, wa.y), sm100::f32x2(wa.z, wa.w),
                                            sm100::f32x2(wb.x, wb.y), sm100::f32x2(wb.z, wb.w)};
#pragma unroll
                    for (int tt = 0; tt < TPB; ++tt) {
                        const float4 x4 = ring[s & 3][tt];
                        const float x = q == 0 ? x4.x : q == 1 ? x4.y : q == 2 ? x4.z : x4.w;
                        const uint64_t xx = sm100::f32x2(x, x);
#pragma unroll
                        for (int pe = 0; pe < 4; ++pe)
                            acc2[tt][pe] = sm100::fma_f32x2(xx, w2[pe], acc2[tt][pe]);
                    }
                }
            }
            if (m == NCH - 1) {
                float acc[TPB][8];
#pragma unroll
                for (int tt = 0; tt < TPB; ++tt)
#pragma unroll
                    for (int pe = 0; pe < 4; ++pe)
                        sm100::f32x2_split(acc2[tt][pe], acc[tt][2 * pe], acc[tt][2 * pe + 1]);
                // the virtual warp's 32 sums (value index tt * 8 + e) by
                // reduce-scatter: each round a lane keeps the half of its
                // values its lane bit selects and adds its partner's copies of
                // them, the pairs the xor tree adds; lane L ends with value L
                float r16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float lo = acc[i >> 3][i & 7], hi = acc[(16 + i) >> 3][(16 + i) & 7];
                    r16[i] = (b16 ? hi : lo) + __shfl_xor_sync(0xffffffffu, b16 ? lo : hi, 16);
                }
                float r8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    r8[i] = (b8 ? r16[8 + i] : r16[i]) +
                            __shfl_xor_sync(0xffffffffu, b8 ? r16[i] : r16[8 + i], 8);
                float r4[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    r4[i] = (b4 ? r8[4 + i] : r8[i]) +
                            __shfl_xor_sync(0xffffffffu, b4 ? r8[i] : r8[4 + i], 4);
                float r2[2];
#pragma unroll
                for (int i = 0; i < 2; ++i)
                    r2[i] = (b2 ? r4[2 + i] : r4[i]) +
                            __shfl_xor_sync(0xffffffffu, b2 ? r4[i] : r4[2 + i], 2);
                zs[s / NCH] = (b1 ? r2[1] : r2[0]) +
                              __shfl_xor_sync(0xffffffffu, b1 ? r2[0] : r2[1], 1);
            }
        }
        // the eight virtual-warp sums in order: virtual warps 0..3 here (even
        // warp), then 4..7 on top of them (odd warp)
        float* buf = zpart_s + (pair * 2 + parity) * 32;
        float zsum;
        if (half == 0) {
            zsum = zs[0];
#pragma unroll
            for (int i = 1; i < 4; ++i) zsum = zsum + zs[i];
            buf[lane] = zsum;
            named_barrier_sync(1 + pair, 64);
            continue;
        }
        named_barrier_sync(1 + pair, 64);
        zsum = buf[lane];
#pragma unroll
        for (int i = 0; i < 4; ++i) zsum = zsum + zs[i];
        // ---- the group's decisions: lane 8 * tt gathers token tt's logits
        const int tt = lane >> 3, e = lane & 7;
        const int64_t t = g * TPB + tt;
        if (logits != nullptr) {
            if (t < T && e < E) logits[t * E + e] = zsum;
        } else {
            float z[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) z[j] = __shfl_sync(0xffffffffu, zsum, (lane & ~7) + j);
            if (e == 0 && t < T) route_tail<8>(z, E, k, slots, route, t);
        }
    }
}


// ---------------------------------------------------------------------------
// One routing decision for a decode batch: the kernels above, given a logits
// buffer, write each token's fp32 logits z[t][0..E) there instead of its
// route; this kernel (one CTA) then adds them in token order, divides by T
// and applies the token rule (route_tail) to the mean.  With T = 1 the mean
// is the token's own logits, bit for bit, so the batch route of one token is
// its adafuse_pregate route.
constexpr int kMaxBatchTokens = 4096;

template <int EMAX>
__global__ void __launch_bounds__(64)
pregate_batch_reduce_kernel(const float* __restrict__ logits, int64_t T, int E, int k, int slots,
                            int32_t* __restrict__ route) {
    __shared__ float zbar[64];
    const int e = threadIdx.x;
    if (e < E) {
        float v = logits[e];
        for (int64_t t = 1; t < T; ++t) v += logits[t * E + e];
        zbar[e] = v / (float)T;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float z[EMAX];
#pragma unroll
        for (int i = 0; i < EMAX; ++i) z[i] = i < E ? zbar[i] : 0.f;
        route_tail<EMAX>(z, E, k, slots, route, 0);
    }
}

}  // namespace adafuse

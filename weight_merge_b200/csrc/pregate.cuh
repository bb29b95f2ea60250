// pregate.cuh -- token-level pre-gating kernel (router GEMV + top-2 + gates).
//
// AdaFuse (gist.science technical summary, section 2-ga): a top-2 router in
// the first layer makes one routing decision per token, applied to every
// adapter layer afterwards.
//
// Design: HBM-bound GEMV.  One CTA of 256 threads takes TPB tokens; each
// thread walks float4 chunks of d (stride 256 chunks), keeps TPB x EMAX fp32
// partial logits in registers (so each Wr element fetched is used TPB times),
// then a fixed xor-shuffle tree and a fixed in-order sum over the 8 warps
// finish each logit.  Every expert column goes through exactly the same
// operation sequence, so two equal columns of Wr give bitwise-equal logits and
// the tie rule (lower index first) is exact.
#pragma once

#include "common.cuh"

namespace adafuse {

constexpr int kPregateThreads = 256;

template <int EMAX, int TPB>
__global__ void __launch_bounds__(kPregateThreads)
pregate_kernel(const float* __restrict__ h, int64_t T, int64_t d,
               const float* __restrict__ Wr, int E, adafuse_route* __restrict__ route) {
    constexpr int kWarps = kPregateThreads / 32;
    __shared__ float part[kWarps][TPB][EMAX];

    const int64_t t0 = (int64_t)blockIdx.x * TPB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float acc[TPB][EMAX];
#pragma unroll
    for (int tt = 0; tt < TPB; ++tt)
#pragma unroll
        for (int e = 0; e < EMAX; ++e) acc[tt][e] = 0.f;

    const int64_t nchunk = d >> 2;
    for (int64_t c = threadIdx.x; c < nchunk; c += kPregateThreads) {
        float4 hv[TPB];
#pragma unroll
        for (int tt = 0; tt < TPB; ++tt) {
            if (t0 + tt < T)
                hv[tt] = __ldcs(reinterpret_cast<const float4*>(h + (t0 + tt) * d) + c);
            else
                hv[tt] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float* wrow = Wr + (4 * c + q) * (int64_t)E;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                const float w = (e < E) ? __ldg(wrow + e) : 0.f;
#pragma unroll
                for (int tt = 0; tt < TPB; ++tt) {
                    const float x = q == 0 ? hv[tt].x : q == 1 ? hv[tt].y : q == 2 ? hv[tt].z : hv[tt].w;
                    acc[tt][e] = __fmaf_rn(x, w, acc[tt][e]);
                }
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
        // top-2 under (z descending, index ascending)
        int e0 = 0;
        float z0 = z[0];
#pragma unroll
        for (int e = 1; e < EMAX; ++e)
            if (e < E && z[e] > z0) { e0 = e; z0 = z[e]; }
        int e1 = -1;
        float z1 = 0.f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e >= E || e == e0) continue;
            if (e1 < 0 || z[e] > z1) { e1 = e; z1 = z[e]; }
        }
        adafuse_route r;
        r.idx[0] = e0;
        r.idx[1] = e1;
        if (e1 < 0) {
            r.gate[0] = 1.f;
            r.gate[1] = 0.f;
        } else {
            // softmax over all E renormalised over the picks == softmax of
            // the two logits: g0 = 1 / (1 + exp(z1 - z0)), z1 - z0 <= 0.
            const float x = expf(z1 - z0);
            const float den = 1.f + x;
            r.gate[0] = 1.f / den;
            r.gate[1] = x / den;
        }
        reinterpret_cast<int4*>(route)[t0 + tt] =
            make_int4(r.idx[0], r.idx[1], __float_as_int(r.gate[0]), __float_as_int(r.gate[1]));
    }
}

// ---------------------------------------------------------------------------
// Warp-per-token pre-gate for E <= 16 (the common router sizes).
//
// A warp owns TPW tokens at a time; lane l walks the float4 chunks l, l+32,
// ... of d (coalesced 512-byte h reads per warp), keeps TPW x EMAX fp32
// partial logits, and a fixed xor-shuffle tree finishes each logit.  Wr is
// read either from shared memory (large batches: staged once per CTA, rows of
// each 4-row chunk padded to EMAX experts and chunks padded to an odd number
// of 16-byte slots so the per-lane float4 reads are bank-conflict free) or
// straight from global memory through L1 (small batches); the arithmetic
// order is identical either way, so a token's logits -- and hence its route
// -- do not depend on how many tokens were batched with it.  Every expert
// column gets the same operation sequence, so equal columns tie bitwise.
template <int EMAX, int TPW, bool SMEM>
__global__ void __launch_bounds__(512)
pregate_warp_kernel(const float* __restrict__ h, int64_t T, int64_t d,
                    const float* __restrict__ Wr, int E, adafuse_route* __restrict__ route) {
    static_assert(EMAX == 8 || EMAX == 16, "EMAX");
    constexpr int S4 = EMAX + 1;                   // float4 slots per chunk in smem
    extern __shared__ float4 wr_s[];
    const int64_t nchunk = d >> 2;
    if constexpr (SMEM) {
        if (E == EMAX) {
            // a 4-row chunk of Wr is EMAX contiguous float4 in global memory
            const float4* src = reinterpret_cast<const float4*>(Wr);
#pragma unroll 8
            for (int64_t i = threadIdx.x; i < nchunk * EMAX; i += blockDim.x)
                wr_s[(i / EMAX) * S4 + (i % EMAX)] = __ldg(src + i);
        } else {
            float* wf = reinterpret_cast<float*>(wr_s);
#pragma unroll 8
            for (int64_t i = threadIdx.x; i < nchunk * 4 * EMAX; i += blockDim.x) {
                const int64_t row = i / EMAX;
                const int e = (int)(i % EMAX);
                const float v = e < E ? __ldg(Wr + row * E + e) : 0.f;
                wf[(row >> 2) * (4 * S4) + (row & 3) * EMAX + e] = v;
            }
        }
        __syncthreads();
    }
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)(blockDim.x >> 5) * gridDim.x;
    for (int64_t tg = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); tg * TPW < T;
         tg += warps) {
        const int64_t t0 = tg * TPW;
        float acc[TPW][EMAX];
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int e = 0; e < EMAX; ++e) acc[tt][e] = 0.f;
        // unrolled so several chunks' h loads are in flight at once
#pragma unroll 8
        for (int64_t c = lane; c < nchunk; c += 32) {
            float4 hv[TPW];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
                hv[tt] = (t0 + tt < T) ? __ldcs(reinterpret_cast<const float4*>(h + (t0 + tt) * d) + c)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
            float w[4 * EMAX];                     // [row q][expert e] of this chunk
            if constexpr (SMEM) {
#pragma unroll
                for (int k = 0; k < EMAX; ++k) {
                    const float4 f = wr_s[c * S4 + k];
                    w[4 * k] = f.x; w[4 * k + 1] = f.y; w[4 * k + 2] = f.z; w[4 * k + 3] = f.w;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < EMAX; ++e)
                        w[q * EMAX + e] = e < E ? __ldg(Wr + (4 * c + q) * E + e) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < EMAX; ++e)
#pragma unroll
                    for (int tt = 0; tt < TPW; ++tt) {
                        const float x = q == 0 ? hv[tt].x : q == 1 ? hv[tt].y : q == 2 ? hv[tt].z : hv[tt].w;
                        acc[tt][e] = __fmaf_rn(x, w[q * EMAX + e], acc[tt][e]);
                    }
        }
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    acc[tt][e] += __shfl_xor_sync(0xffffffffu, acc[tt][e], off);
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
            if (lane != tt || t0 + tt >= T) continue;
            int e0 = 0;
            float z0 = acc[tt][0];
#pragma unroll
            for (int e = 1; e < EMAX; ++e)
                if (e < E && acc[tt][e] > z0) { e0 = e; z0 = acc[tt][e]; }
            int e1 = -1;
            float z1 = 0.f;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e >= E || e == e0) continue;
                if (e1 < 0 || acc[tt][e] > z1) { e1 = e; z1 = acc[tt][e]; }
            }
            float g0 = 1.f, g1 = 0.f;
            if (e1 >= 0) {
                // softmax over all E renormalised over the picks == softmax of
                // the two logits: g0 = 1 / (1 + exp(z1 - z0)), z1 - z0 <= 0.
                const float x = expf(z1 - z0);
                const float den = 1.f + x;
                g0 = 1.f / den;
                g1 = x / den;
            }
            reinterpret_cast<int4*>(route)[t0 + tt] =
                make_int4(e0, e1, __float_as_int(g0), __float_as_int(g1));
        }
    }
}

}  // namespace adafuse

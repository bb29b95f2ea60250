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

#include "common.cuh"

namespace adafuse {

constexpr int kPregateThreads = 256;
enum : int { kWrShared = 0, kWrVector = 1, kWrScalar = 2 };

template <int EMAX, int TPB, int WR>
__global__ void __launch_bounds__(kPregateThreads)
pregate_kernel(const float* __restrict__ h, int64_t T, int64_t d, const float* __restrict__ Wr,
               int E, adafuse_route* __restrict__ route) {
    static_assert(EMAX % 4 == 0, "EMAX");
    constexpr int kWarps = kPregateThreads / 32;
    constexpr int S4 = EMAX + 1;             // float4 slots per chunk in shared memory
    __shared__ float part[kWarps][TPB][EMAX];
    extern __shared__ float4 wr_s[];
    const int64_t nchunk = d >> 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if constexpr (WR == kWrShared) {
        if (E == EMAX) {
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
        __syncthreads();   // part[] is reused by the next token group
    }
}

}  // namespace adafuse

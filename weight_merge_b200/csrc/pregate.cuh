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
               int E, int k, int slots, int32_t* __restrict__ route) {
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
            // top-k under (z descending, index ascending): pick j is the
            // largest logit not yet picked, the lower index among equals
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
            // softmax over all E renormalised over the picks == softmax of the
            // picked logits: g_j = x_j / (1 + x_1 + ...), x_j = exp(z_j - z_0) <= 1
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
                reinterpret_cast<int4*>(route)[t0 + tt] =
                    make_int4(pick[0], pick[1], __float_as_int(g[0]), __float_as_int(g[1]));
            } else {
                int4* r4 = reinterpret_cast<int4*>(route) + 2 * (t0 + tt);
                r4[0] = make_int4(pick[0], pick[1], pick[2], pick[3]);
                r4[1] = make_int4(__float_as_int(g[0]), __float_as_int(g[1]), __float_as_int(g[2]),
                                  __float_as_int(g[3]));
            }
        }
        __syncthreads();   // part[] is reused by the next token group
    }
}

}  // namespace adafuse

// switch_fold.cuh -- the tensor-core switch for ranks up to 8 with every
// expert's coefficient folded into its adapter operand, so that a tile's whole
// update is one tcgen05.mma chain into ONE fp32 TMEM accumulator.
//
// AdaFuse (gist.science technical summary, section 2-na) concatenates the
// selected adapters and runs one GEMM over the concatenation.  The
// concatenated operand built here carries the coefficients c_e exactly enough
// for fp32 accumulation:
//   c_e A_e = H_e + M_e + L_e      (H, M, L bf16)
// c_e is fp32 and A_e bf16, so their product has at most 32 significant
// bits.  H is the bf16 rounding of it, M that of what H leaves, L that of what
// M leaves (each residual formed exactly, see fold_split); each rounding
// leaves at most 2^-8 of its input, so |c_e A_e - H - M - L| <= ~2^-24
// |c_e A_e|, one fp32 rounding's worth.  Then
//   sum_e c_e B_e A_e = sum_e (B_e H_e + B_e M_e + B_e L_e)
// is three K = 16 MMAs per PAIR of experts: the MMA's A operand is the two
// experts' 128 x 8 B-row blocks side by side along K (the descriptor's K
// stride steps from one block to the other), its B operand the pair's 16
// folded rows of one term.
//
// A fold launch writes the operand for the switch's experts; the switch
// launch that follows on the same stream reads it:
//   Af [col block of 128][pair][half of 64 cols][48 rows][64 cols] bf16,
//   row = term * 16 + slot * 8 + k (rows k >= rank, absent slots and columns
//   past the weight's end are zero), each 128-byte row 128B-swizzled as TMA
//   would place it, so one 12 KB bulk copy brings a pair's operand for a tile.
//
// With one accumulator per tile, TMEM's 512 columns hold four tiles: the MMA
// warp runs up to four tiles ahead of the epilogue instead of waiting for it
// to read four accumulators, and an in-place top-4 switch (up to 8 experts)
// needs no second TMEM batch.  Warp roles, the W ring, the store warp and the
// bounded waits are those of switch_tc_kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "switch_tc.cuh"

namespace adafuse {

constexpr int kFoldMaxPairs = kMaxCoefs / 2;                  // 4 pairs = 8 experts
constexpr int kFoldRows = 48;                                 // 3 terms x 2 slots x 8
constexpr uint32_t kFoldHalfBytes = kFoldRows * 128;          // 48 rows x 64 cols bf16
constexpr uint32_t kFoldPairBytes = 2 * kFoldHalfBytes;       // per (col block, pair)
constexpr uint32_t kFoldBlockBytes = kFoldMaxPairs * kFoldPairBytes;  // per col block
constexpr int kFoldAcc = 4;                                   // TMEM accumulators
constexpr int kFoldThreads = 256;                             // fold launch block

// Bytes of folded operand one weight of `in` columns needs.
__host__ __device__ constexpr size_t fold_bytes_for(int in) {
    return (size_t)((in + kTile - 1) / kTile) * kFoldBlockBytes;
}

struct FoldConfig {
    static constexpr int kWStages = 5;
    static constexpr int kOpStages = 4;
    static constexpr uint32_t kBBlockBytes = 128 * 8 * 2;              // one expert's B rows
    static constexpr uint32_t kOpStageBytes = kFoldPairBytes + 2 * kBBlockBytes;  // 16 KB
    static constexpr uint32_t kOpBytes = kOpStages * kOpStageBytes;
    static constexpr uint32_t kWBytes = kWStages * kWTileBytes;
    static constexpr uint32_t kBarBytes = 8 * (3 * kWStages + 2 * kOpStages + 2 * kFoldAcc) + 16;
    static constexpr uint32_t kSmemBytes = 1024 /*alignment slack*/ + kOpBytes + kWBytes + kBarBytes;
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(kOpStageBytes % 1024 == 0 && kFoldHalfBytes % 1024 == 0, "swizzle atoms stay aligned");
};

// One value's three bf16 terms: hi + mid + lo = c * a up to ~2^-24 |c a|, in
// fp32 with exact steps.  c * a (24 + 8 significant bits) is p + e exactly,
// p = fl(c a) and e = fma(c, a, -p) (the error-free product).  With E the
// exponent of c a, hi = bf16(p) has its bits in [E-7, E+1], so the residual
// c a - hi = (p - hi) + e lies in [E-31, E-8]: 24 bits, an fp32 number; both
// p - hi (<= 16 bits) and the sum are therefore exact.  mid = bf16 of that
// residual, and residual - mid is exact again; lo = bf16 of what is left.
__device__ __forceinline__ void fold_split(float c, float a, uint16_t& hi, uint16_t& mid, uint16_t& lo) {
    const float p = c * a;
    const float e = __fmaf_rn(c, a, -p);
    const __nv_bfloat16 h = __float2bfloat16_rn(p);
    const float r1 = (p - __bfloat162float(h)) + e;
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    const __nv_bfloat16 l = __float2bfloat16_rn(r2);
    hi = __bfloat16_as_ushort(h);
    mid = __bfloat16_as_ushort(m);
    lo = __bfloat16_as_ushort(l);
}

// Fold launch over weights [w0, w0 + nw).  A block's 256 threads are
// (half, slot, k, 16-byte chunk) of one (col block, pair) item; blocks stride
// over a weight's items (x) and over the weights (y).  Each thread folds 8
// values of A_e[k] and writes their three terms to rows term*16 + slot*8 + k
// of the item.
__global__ void __launch_bounds__(kFoldThreads) fold_operands_kernel(
    const PairDesc* __restrict__ pairs, int64_t w0, int64_t nw, int r, const int32_t* prev,
    const int32_t* cur, int slots, int E, float s) {
    // the coefficient list, built once per block (the switch reports bad routes)
    __shared__ Coefs8 s_cf;
    __shared__ int s_status;
    if (threadIdx.x == 0) s_status = build_coefs(prev, cur, slots, E, s, s_cf);
    __syncthreads();
    if (s_status != 0) return;
    const Coefs8 cf = s_cf;
    const int npairs = (cf.n + 1) >> 1;
    if (npairs == 0) return;
    const int tid = threadIdx.x;
    const int chunk = tid & 7, k = (tid >> 3) & 7, slot = (tid >> 6) & 1, half = tid >> 7;
    for (int64_t wi = blockIdx.y; wi < nw; wi += gridDim.y) {
        const PairDesc& pd = pairs[w0 + wi];
        const int in = pd.in;
        const int ncb = (in + kTile - 1) / kTile;
        for (int item = blockIdx.x; item < ncb * npairs; item += gridDim.x) {
            const int cb = item / npairs, pr = item - cb * npairs;
            const int ei = 2 * pr + slot;
            const int col = cb * kTile + half * 64 + chunk * 8;
            uint4 raw = make_uint4(0u, 0u, 0u, 0u);
            float c = 0.f;
            if (ei < cf.n && k < r && col < in) {
                const int e = coef_expert(cf, ei);
                c = coef_value(cf, ei);
                raw = __ldg(reinterpret_cast<const uint4*>(pd.A + ((size_t)e * r + k) * (size_t)in + col));
            }
            const uint32_t a[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t th[4], tm[4], tl[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint16_t h0, m0, l0, h1, m1, l1;
                fold_split(c, __uint_as_float(a[j] << 16), h0, m0, l0);
                fold_split(c, __uint_as_float(a[j] & 0xffff0000u), h1, m1, l1);
                th[j] = (uint32_t)h0 | ((uint32_t)h1 << 16);
                tm[j] = (uint32_t)m0 | ((uint32_t)m1 << 16);
                tl[j] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            uint8_t* base = reinterpret_cast<uint8_t*>(pd.Af) +
                            ((size_t)cb * kFoldMaxPairs + pr) * kFoldPairBytes + (size_t)half * kFoldHalfBytes;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const int row = q * 16 + slot * 8 + k;
                const uint32_t* t = q == 0 ? th : q == 1 ? tm : tl;
                *reinterpret_cast<uint4*>(base + row * 128 + ((chunk ^ (row & 7)) << 4)) =
                    make_uint4(t[0], t[1], t[2], t[3]);
            }
        }
    }
}

__global__ void __launch_bounds__(kTcThreads, 1) switch_fold_kernel(const TcParams p) {
    using C = FoldConfig;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* op_ring = smem;                       // [kOpStages][Af pair (12 KB) | B blocks (2 x 2 KB)]
    uint8_t* w_ring = smem + C::kOpBytes;          // [kWStages][box0 | box1]
    uint64_t* bars = reinterpret_cast<uint64_t*>(w_ring + C::kWBytes);
    uint64_t* w_full = bars;
    uint64_t* w_empty = w_full + C::kWStages;
    uint64_t* op_full = w_empty + C::kWStages;
    uint64_t* op_empty = op_full + C::kOpStages;
    uint64_t* acc_full = op_empty + C::kOpStages;  // [kFoldAcc]
    uint64_t* acc_empty = acc_full + kFoldAcc;     // [kFoldAcc]
    uint64_t* epi_done = acc_empty + kFoldAcc;     // [kWStages]: epilogue wrote the tile
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_done + C::kWStages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    Coefs8 cf;
    const int st = build_coefs(p.prev, p.cur, p.slots, p.E, p.s, cf);
    if (st != 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, st);
        return;
    }
    if (cf.n == 0 && !p.rebase) return;  // identity switch
    const int64_t first = p.t_begin + blockIdx.x;
    if (first >= p.t_end) return;
    // pairs of experts per tile; 0 only for a re-base to an empty route, where
    // every tile is W0 passed through the epilogue with nothing added
    const int npairs = (cf.n + 1) >> 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 1);
            mbar_init(&epi_done[i], kTcEpiThreads);
        }
        for (int i = 0; i < C::kOpStages; ++i) {
            mbar_init(&op_full[i], 1);
            mbar_init(&op_empty[i], 1);
        }
        for (int i = 0; i < kFoldAcc; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], kTcEpiThreads / 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto fail = [&](int where) {
        if (!*abort_flag) {
            *abort_flag = 1;
            atomicOr(p.status, ADAFUSE_STATUS_TIMEOUT);
        }
        (void)where;
    };

    if (warp == 0) {
        // ---------------- W producer: tiles into the W ring ----
        if (lane == 0) {
            int ws = 0;
            uint32_t wph = 0;
            uint32_t last_pair = 0xffffffffu;
            TileEntry te_next = fetch_tile(p.tiles, first, p.t_end);
            for (int64_t t = first; t < p.t_end && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile(te_next);
                te_next = fetch_tile(p.tiles, t + gridDim.x, p.t_end);
                const CUtensorMap* mW = p.rebase ? p.w0_maps + ti.pair : p.maps + kMapsPerPair * (size_t)ti.pair;
                if (ti.pair != last_pair) {
                    tensormap_acquire(mW);
                    last_pair = ti.pair;
                }
                if (!mbar_wait_bounded(&w_empty[ws], wph ^ 1, abort_flag, kWaitLimitNs)) { fail(1); break; }
                uint8_t* wdst = w_ring + (size_t)ws * kWTileBytes;
                mbar_arrive_expect_tx(&w_full[ws], w_tile_bytes(p.blk, ti.wide));
                load_w_tile(wdst, mW, ti.row0, ti.col0, ti.wide, p.blk, &w_full[ws]);
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
                if (t + gridDim.x < p.t_end && (te_next.x & kTilePairMask) != ti.pair) {
                    const uint32_t np = te_next.x & kTilePairMask;
                    tensormap_prefetch(p.rebase ? p.w0_maps + np : p.maps + kMapsPerPair * (size_t)np);
                }
            }
        }
    } else if (warp == 3) {
        // ---------------- operand producer: per tile and expert pair, the
        // pair's folded A columns (one 12 KB bulk copy) and each expert's B rows
        if (lane == 0 && npairs > 0) {
            int os = 0;
            uint32_t oph = 0;
            TileEntry te_next = fetch_tile(p.tiles, first, p.t_end);
            for (int64_t t = first; t < p.t_end && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile(te_next);
                te_next = fetch_tile(p.tiles, t + gridDim.x, p.t_end);
                const PairDesc& pd = p.pairs[ti.pair];
                const int out = pd.out;
                const int out_rows = out - ti.row0 < 128 ? out - ti.row0 : 128;
                // rows past the weight's end are not fetched (their products
                // only reach accumulator rows that are never stored)
                const uint32_t bbytes = (uint32_t)out_rows * 16u;
                const uint8_t* af = reinterpret_cast<const uint8_t*>(pd.Af) +
                                    (size_t)(ti.col0 / kTile) * kFoldBlockBytes;
                bool ok = true;
#pragma unroll 1
                for (int pr = 0; pr < npairs; ++pr) {
                    const bool has_b = 2 * pr + 1 < cf.n;
                    if (!mbar_wait_bounded(&op_empty[os], oph ^ 1, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    uint8_t* a_dst = op_ring + (size_t)os * C::kOpStageBytes;
                    uint8_t* b_dst = a_dst + kFoldPairBytes;
                    mbar_arrive_expect_tx(&op_full[os], kFoldPairBytes + (has_b ? 2u : 1u) * bbytes +
                                                            (pr == 0 && (t - first) / gridDim.x + 1 == p.stall
                                                                 ? kStallBytes : 0u));
                    bulk_load(a_dst, af + (size_t)pr * kFoldPairBytes, kFoldPairBytes, &op_full[os]);
                    const int ea = coef_expert(cf, 2 * pr);
                    bulk_load(b_dst, pd.Bk + ((size_t)ea * out + ti.row0) * 8, bbytes, &op_full[os]);
                    if (has_b) {
                        const int eb = coef_expert(cf, 2 * pr + 1);
                        bulk_load(b_dst + C::kBBlockBytes, pd.Bk + ((size_t)eb * out + ti.row0) * 8, bbytes,
                                  &op_full[os]);
                    }
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) { fail(2); break; }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: per tile, 3 MMAs per expert pair into
        // one of four TMEM accumulators ----------------
        if (lane == 0 && npairs > 0) {
            constexpr uint32_t idesc = instr_desc_bf16(128, 128, /*B MN-major*/ 1);
            int os = 0, ab = 0;
            uint32_t oph = 0, aph = 0;
            bool ok = true;
            for (int64_t t = first; t < p.t_end && ok && !*abort_flag; t += gridDim.x) {
                if (!mbar_wait_bounded(&acc_empty[ab], aph ^ 1, abort_flag, kWaitLimitNs)) { fail(3); break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + 128u * (uint32_t)ab;
#pragma unroll 1
                for (int pr = 0; pr < npairs; ++pr) {
                    // TMA's complete_tx on the mbarrier orders the operand
                    // bytes before the MMA's shared-memory reads
                    if (!mbar_wait_bounded(&op_full[os], oph, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    const uint32_t a_s = smem_u32(op_ring + (size_t)os * C::kOpStageBytes);
                    const uint32_t b_s = a_s + kFoldPairBytes;
                    // MMA A operand: [B_ea | B_eb], 128 x 16, K-major, plain
                    // core-matrix layout; the K-group stride steps to the second
                    // expert's block.  A lone expert re-reads its own block and
                    // meets the zero rows of the absent slot.
                    const uint64_t da =
                        smem_desc(b_s, 2 * pr + 1 < cf.n ? C::kBBlockBytes : 0u, 128, kSwizzleNone);
#pragma unroll
                    for (int q = 0; q < 3; ++q) {
                        // MMA B operand: term q's 16 folded rows, N-major, two
                        // 64-column halves (LBO apart), 8-row K groups SBO apart
                        const uint64_t db = smem_desc(a_s + 2048u * q, kFoldHalfBytes, 1024, kSwizzle128B);
                        tc_mma_f16(d_tmem, da, db, idesc, (pr > 0 || q > 0) ? 1u : 0u);
                    }
                    tc_commit(&op_empty[os]);
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) { fail(4); break; }
                tc_commit(&acc_full[ab]);
                if (++ab == kFoldAcc) { ab = 0; aph ^= 1; }
            }
        }
    } else if (warp == 2) {
        // ---------------- store warp: TMA-stores each finished tile over
        // itself and frees its smem stage once the store has read it ----
        if (lane == 0) {
            int ws = 0;
            uint32_t wph = 0;
            TileEntry te_next = fetch_tile(p.tiles, first, p.t_end);
            for (int64_t t = first; t < p.t_end && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile(te_next);
                te_next = fetch_tile(p.tiles, t + gridDim.x, p.t_end);
                if (!mbar_wait_bounded(&epi_done[ws], wph, abort_flag, kWaitLimitNs)) { fail(7); break; }
                const CUtensorMap* mW = p.maps + kMapsPerPair * (size_t)ti.pair;
                uint8_t* wsrc = w_ring + (size_t)ws * kWTileBytes;
                store_w_tile(mW, wsrc, ti.row0, ti.col0, ti.wide, p.blk);
                bulk_commit();
                bulk_wait_read<0>();
                mbar_arrive(&w_empty[ws]);
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
            }
            bulk_wait<0>();
        }
    } else {
        // ---------------- epilogue: one accumulator read per tile ----------
        // Every decision that can end the loop is warp-uniform, so
        // tcgen05.ld's .sync.aligned form always sees the whole warp.
        const int ew = warp - kTcEpiWarp0;      // 0..15
        const int quarter = warp & 3;           // TMEM lanes this warp may read
        const int cgrp = ew >> 2;               // 32-column group 0..3
        const int half = cgrp >> 1;             // which 64-column TMA box
        const int row = quarter * 32 + lane;
        const uint32_t t_lane = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cgrp * 32);
        int ws = 0, ab = 0;
        uint32_t wph = 0, aph = 0;
        for (int64_t t = first; t < p.t_end; t += gridDim.x) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            float tot[32];
            bool ok = true;
            if (npairs > 0) {
                ok = mbar_wait_bounded(&acc_full[ab], aph, abort_flag, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) { fail(5); break; }
                tc_fence_after();
                tmem_ld32(t_lane + 128u * (uint32_t)ab, tot);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[ab]);
                if (++ab == kFoldAcc) { ab = 0; aph ^= 1; }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) tot[i] = 0.f;
            }
            ok = mbar_wait_bounded(&w_full[ws], wph, abort_flag, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) { fail(6); break; }
            uint8_t* rowp = w_ring + (size_t)ws * kWTileBytes + (size_t)half * kWBoxBytes + row * 128;
            epi_update_row(rowp, cgrp, row, tot);
            fence_async_smem();
            mbar_arrive(&epi_done[ws]);
            if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
        }
    }

    // teardown: after an abort give in-flight TMA copies and MMAs time to land
    __syncwarp();
    __syncthreads();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) { }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace adafuse

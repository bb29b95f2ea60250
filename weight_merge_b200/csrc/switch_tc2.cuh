// switch_tc2.cuh -- the fused adapter switch on CTA pairs: a cluster of two
// CTAs on neighbouring SMs shares one tcgen05.mma with cta_group::2.
//
// Same update as switch_tc.cuh (AdaFuse, gist.science technical summary,
// section 2-na: per W tile W <- bf16_rne(W + sum_e c_e (B_e A_e))), with a
// 256 x 128 block of W per pair and step of the persistent loop:
//   * each CTA owns 128 rows of the block: its W tile, its rows of B_e (the
//     MMA's A operand, M/2 = 128 rows in each CTA) and its 128 x 128 slice of
//     every accumulator in its own TMEM;
//   * the A_e columns (the MMA's B operand, N = 128) are split between the two
//     CTAs, 64 columns each, so each SM stages half of them;
//   * the even CTA issues the MMAs; both CTAs arrive on the even CTA's "full"
//     barrier, and their operand loads complete on it; each MMA batch's
//     completion frees the operand stage in both CTAs;
//   * the even CTA's W producer picks the blocks (a static stride over the
//     table, or tickets from a per-context counter) and publishes each W
//     stage's block entry to both CTAs: its own slot with a plain store, the
//     odd CTA's with an 8-byte st.async that completes on the odd CTA's
//     barrier; it reuses a stage only after both CTAs' store warps released
//     it (the even CTA's "empty" barrier counts both).
// Per selected expert a CTA stages 128 x r B rows + r x 64 A columns instead
// of 128 x r + r x 128: at rank 64 that is 24 KB instead of 32 KB per tile,
// which leaves room for a deeper operand ring next to the W ring.
// Warp roles and bounded waits are those of switch_tc_kernel; an abort in
// either CTA is copied to the other CTA's flag.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "switch_tc.cuh"

namespace adafuse {

// Pair-table entry (x): pair index in bits 0..29; kTileWideBit: the block's
// second 64-column half starts inside the weight; kTileLowerBit: the block's
// second 128-row half starts inside the weight.  y = (row block << 16) | col tile.
constexpr uint32_t kTileLowerBit = 0x40000000u;
constexpr uint32_t kTile2PairMask = 0x3fffffffu;
constexpr int kBlockRows = 2 * kTile;  // rows of W per CTA pair and step

template <int KP>
struct Tc2Config {
    static_assert(KP == 16 || KP == 32 || KP == 64, "KP");
    // stage counts from a sweep at the Llama-2-7B (r = 64) and 13B (r = 16) shapes
    static constexpr int kWStages = KP == 64 ? 3 : KP == 32 ? 4 : 6;
    static constexpr int kOpStages = KP == 64 ? 5 : KP == 32 ? 7 : 5;
    static constexpr uint32_t kAHalfBytes = KP * 128;   // KP rows x 64 columns of A_e
    static constexpr uint32_t kBBytes = 128 * KP * 2;    // 128 rows x KP of B_e
    static constexpr uint32_t kOpStageBytes = kAHalfBytes + kBBytes;
    static constexpr uint32_t kOpBytes = kOpStages * kOpStageBytes;
    static constexpr uint32_t kWBytes = kWStages * kWTileBytes;
    static constexpr uint32_t kBLayout = KP == 16 ? sm100::kSwizzle32B
                                       : KP == 32 ? sm100::kSwizzle64B
                                                  : sm100::kSwizzle128B;
    static constexpr uint32_t kBSbo = 8 * KP * 2;
    // barriers (w_full, w_empty, epi_done, te_full per W stage; op_full,
    // op_empty per operand stage; acc_full, acc_empty), the W stages' tile
    // entries, tmem base + abort flag
    static constexpr uint32_t kBarBytes = 8 * (4 * kWStages + 2 * kOpStages + 2) + 8 * kWStages + 16;
    static constexpr uint32_t kSmemBytes = 1024 + kOpBytes + kWBytes + kBarBytes;
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(kOpStageBytes % 1024 == 0 && kAHalfBytes % 1024 == 0, "swizzle atoms stay aligned");
};

struct PairTile {
    uint32_t pair;
    int row0, col0;  // this CTA's 128 x 128 tile
    bool wide;       // second 64-column half inside the weight
    bool lower;      // the block's second 128-row half inside the weight
    bool rows;       // this CTA's tile has rows inside the weight
};

__device__ __forceinline__ PairTile decode_pair_tile(TileEntry te, uint32_t q) {
    PairTile t;
    t.pair = te.x & kTile2PairMask;
    t.wide = (te.x & kTileWideBit) != 0;
    t.lower = (te.x & kTileLowerBit) != 0;
    t.row0 = (int)(te.y >> 16) * kBlockRows + (int)q * kTile;
    t.col0 = (int)(te.y & 0xffffu) * kTile;
    t.rows = q == 0 || t.lower;
    return t;
}

template <int KP>
__global__ void __launch_bounds__(kTcThreads, 1) switch_tc2_kernel(const TcParams p) {
    using C = Tc2Config<KP>;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // the same offsets in both CTAs: MMA descriptors name one address for both
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* op_ring = smem;                       // [kOpStages][A half | B rows]
    uint8_t* w_ring = smem + C::kOpBytes;          // [kWStages][box0 | box1]
    uint64_t* bars = reinterpret_cast<uint64_t*>(w_ring + C::kWBytes);
    uint64_t* w_full = bars;
    uint64_t* w_empty = w_full + C::kWStages;
    uint64_t* op_full = w_empty + C::kWStages;     // used in the even CTA only
    uint64_t* op_empty = op_full + C::kOpStages;
    uint64_t* acc_full = op_empty + C::kOpStages;
    uint64_t* acc_empty = acc_full + 1;            // used in the even CTA only
    uint64_t* epi_done = acc_empty + 1;            // [kWStages]
    uint64_t* te_full = epi_done + C::kWStages;    // [kWStages]: the stage's block entry is set
    TileEntry* te_slot = reinterpret_cast<TileEntry*>(te_full + C::kWStages);  // [kWStages]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(te_slot + C::kWStages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    Coefs8 cf;
    const int st = build_coefs(p.prev, p.cur, p.slots, p.E, p.s, cf);
    if (st != 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, st);
        return;
    }
    if (cf.n == 0 && !p.rebase) return;  // identity switch (both CTAs agree)
    const int64_t n_clusters = (int64_t)cluster_count_x();
    const int64_t first = p.t_begin + (int64_t)cluster_id_x();
    // (the dynamic schedule needs every pair at teardown to reset its
    // counter; the launch never has more pairs than blocks, so no pair
    // leaves here then)
    if (!p.dyn && first >= p.t_end) return;        // both CTAs agree

    const uint32_t q = cluster_ctarank();  // 0: issues the MMAs
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            // even CTA: its own and the odd CTA's store warp release the stage
            mbar_init(&w_empty[i], 2);
            mbar_init(&epi_done[i], kTcEpiThreads);
            mbar_init(&te_full[i], 1);
        }
        for (int i = 0; i < C::kOpStages; ++i) {
            // one arrival (with its own bytes) from each CTA per use: the even
            // CTA cannot finish a use the odd CTA has not reached, so neither
            // CTA's "empty" barrier can complete two phases ahead of its waiter
            mbar_init(&op_full[i], 2);
            mbar_init(&op_empty[i], 1);   // one MMA completion per use
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * (kTcEpiThreads / 32));  // epilogue warps of both CTAs
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised and the TMEM address written
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t peer_abort = cluster_addr((const void*)abort_flag, q ^ 1u);

    auto fail = [&](int where) {
        if (!*abort_flag) {
            *abort_flag = 1;
            st_cluster_u32(peer_abort, 1u);
            atomicOr(p.status, ADAFUSE_STATUS_TIMEOUT);
        }
        (void)where;
    };

    if (warp == 0) {
        // ---------------- W producer: this CTA's tiles into the W ring ----
        // The even CTA's producer picks the blocks for both CTAs (see the file
        // head); the odd CTA's producer takes them from its tile-entry slots.
        if (lane == 0) {
            int ws = 0;
            uint32_t wph = 0;
            uint32_t last_pair = 0xffffffffu;
            const uint32_t peer_te_full = cluster_addr(te_full, 1);
            const uint32_t peer_te_slot = cluster_addr(te_slot, 1);
            auto next_block = [&](int64_t t) -> int64_t {
                if (t >= p.t_end) return t;
                return p.dyn ? p.t_begin + (int64_t)atomicAdd(p.sched, 1ull) : t + n_clusters;
            };
            int64_t t = 0, tn = 0;
            TileEntry te = make_uint2(0u, 0u), te_n = te;
            if (q == 0) {
                t = p.dyn ? next_block(p.t_begin) : first;
                te = fetch_tile(p.tiles, t, p.t_end);
            }
            while (!*abort_flag) {
                if (q == 0) {
                    tn = next_block(t);
                    te_n = fetch_tile(p.tiles, tn, p.t_end);
                    if (!mbar_wait_bounded(&w_empty[ws], wph ^ 1, abort_flag, kWaitLimitNs)) { fail(1); break; }
                    const TileEntry pub = t >= p.t_end ? make_uint2(kTileEndX, kTileEndX) : te;
                    te_slot[ws] = pub;
                    mbar_arrive(&te_full[ws]);
                    const uint32_t pf = peer_te_full + 8u * (uint32_t)ws;
                    mbar_arrive_expect_tx_cluster(pf, 8u);
                    st_async_v2_cluster(peer_te_slot + 8u * (uint32_t)ws, pub.x, pub.y, pf);
                    if (t >= p.t_end) break;
                } else {
                    if (!mbar_wait_bounded(&te_full[ws], wph, abort_flag, kWaitLimitNs)) { fail(1); break; }
                    te = te_slot[ws];
                    if (te.x == kTileEndX) break;
                }
                const PairTile ti = decode_pair_tile(te, q);
                const CUtensorMap* mW = p.rebase ? p.w0_maps + ti.pair : p.maps + kMapsPerPair * (size_t)ti.pair;
                if (ti.pair != last_pair) {
                    tensormap_acquire(mW);
                    last_pair = ti.pair;
                }
                uint8_t* wdst = w_ring + (size_t)ws * kWTileBytes;
                if (ti.rows) {
                    mbar_arrive_expect_tx(&w_full[ws], w_tile_bytes(p.blk, ti.wide));
                    load_w_tile(wdst, mW, ti.row0, ti.col0, ti.wide, p.blk, &w_full[ws]);
                } else {
                    // no rows of this weight here: the stage is only passed along
                    mbar_arrive(&w_full[ws]);
                }
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
                if (q == 0) {
                    if (tn < p.t_end && (te_n.x & kTile2PairMask) != ti.pair) {
                        const uint32_t np = te_n.x & kTile2PairMask;
                        tensormap_prefetch(p.rebase ? p.w0_maps + np : p.maps + kMapsPerPair * (size_t)np);
                    }
                    t = tn;
                    te = te_n;
                }
            }
        }
    } else if (warp == 3) {
        // ---------------- operand producer (both CTAs): per block and expert,
        // this CTA's B_e rows and its half of the A_e columns, counted on the
        // even CTA's full barrier ----
        if (lane == 0) {
            const uint32_t full0 = cluster_addr(op_full, 0);
            int os = 0, ts = 0;
            uint32_t oph = 0, tph = 0;
            uint32_t last_pair = 0xffffffffu;
            bool ok = true;
            int tile_no = 0;   // blocks this pair has taken (for the stall hook)
            while (!*abort_flag) {
                if (!mbar_wait_bounded(&te_full[ts], tph, abort_flag, kWaitLimitNs)) { ok = false; break; }
                const TileEntry te = te_slot[ts];
                if (++ts == C::kWStages) { ts = 0; tph ^= 1; }
                if (te.x == kTileEndX) break;
                const bool stall_here = ++tile_no == p.stall;
                const PairTile ti = decode_pair_tile(te, q);
                const CUtensorMap* mA = p.maps + kMapsPerPair * (size_t)ti.pair + 1;
                const CUtensorMap* mB = mA + 1;
                if (ti.pair != last_pair) {
                    tensormap_acquire(mA);
                    tensormap_acquire(mB);
                    last_pair = ti.pair;
                }
                const bool load_a = q == 0 || ti.wide;
                const uint32_t bytes = (ti.rows ? C::kBBytes : 0u) + (load_a ? C::kAHalfBytes : 0u);
#pragma unroll 1
                for (int ei = 0; ei < cf.n; ++ei) {
                    const int e = coef_expert(cf, ei);
                    if (!mbar_wait_bounded(&op_empty[os], oph ^ 1, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    uint8_t* a_dst = op_ring + (size_t)os * C::kOpStageBytes;
                    uint8_t* b_dst = a_dst + C::kAHalfBytes;
                    const uint32_t full = full0 + 8u * (uint32_t)os;
                    mbar_arrive_expect_tx_cluster(
                        full, bytes + (q == 0 && ei == 0 && stall_here ? kStallBytes : 0u));
                    if (ti.rows) tma_load_3d_pair(b_dst, mB, 0, ti.row0, e, full);
                    if (load_a) tma_load_3d_pair(a_dst, mA, ti.col0 + 64 * (int)q, 0, e, full);
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) break;
            }
            if (!ok) fail(2);
            // every stage filled here is released by an MMA completion that
            // arrives on this CTA's barrier: see the last ones land
            for (int j = 0; ok && !*abort_flag && j < C::kOpStages; ++j) {
                if (!mbar_wait_bounded(&op_empty[os], oph ^ 1, abort_flag, kWaitLimitNs)) { fail(8); break; }
                if (++os == C::kOpStages) { os = 0; oph ^= 1; }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA) ----------------
        if (lane == 0 && q == 0) {
            constexpr uint32_t idesc = instr_desc_bf16(kBlockRows, 128, /*B MN-major*/ 1);
            int os = 0, ts = 0;
            uint32_t oph = 0, aph = 0, tph = 0;
            const int nb = tmem_batches(cf);
            bool ok = true;
            while (ok && !*abort_flag) {
                if (!mbar_wait_bounded(&te_full[ts], tph, abort_flag, kWaitLimitNs)) { fail(9); break; }
                const bool end = te_slot[ts].x == kTileEndX;
                if (++ts == C::kWStages) { ts = 0; tph ^= 1; }
                if (end) break;
#pragma unroll 1
              for (int b0 = 0; b0 < nb * kTmemBatch && ok; b0 += kTmemBatch) {
                if (!mbar_wait_bounded(acc_empty, aph ^ 1, abort_flag, kWaitLimitNs)) { fail(3); ok = false; break; }
                tc_fence_after();
                const int b1 = cf.n < b0 + kTmemBatch ? cf.n : b0 + kTmemBatch;
#pragma unroll 1
                for (int ei = b0; ei < b1; ++ei) {
                    // TMA's complete_tx on the mbarrier orders the operand
                    // bytes before the MMA's shared-memory reads: no tcgen05 fence
                    if (!mbar_wait_bounded(&op_full[os], oph, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    const uint32_t a_s = smem_u32(op_ring + (size_t)os * C::kOpStageBytes);
                    const uint32_t b_s = a_s + C::kAHalfBytes;
#pragma unroll
                    for (int k = 0; k < KP / 16; ++k) {
                        // MMA A operand: this CTA's 128 B_e rows x KP, K-major, swizzled
                        const uint64_t da = smem_desc(b_s + 32u * k, 16, C::kBSbo, C::kBLayout);
                        // MMA B operand: KP x 64 A_e columns per CTA, N-major,
                        // 8-row K groups 1024 B apart (one swizzle atom wide)
                        const uint64_t db = smem_desc(a_s + 2048u * k, C::kAHalfBytes, 1024, kSwizzle128B);
                        tc_mma_f16_pair(tmem_base + 128u * (ei - b0), da, db, idesc, k > 0 ? 1u : 0u);
                    }
                    tc_commit_pair(&op_empty[os], 0x3);
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) { fail(4); break; }
                tc_commit_pair(acc_full, 0x3);
                aph ^= 1;
              }
            }
        }
    } else if (warp == 2) {
        // ---------------- store warp: this CTA's finished tiles ----
        if (lane == 0) {
            int ws = 0;
            uint32_t wph = 0;
            // the stage is released on the even CTA's "empty" barrier (it
            // counts both CTAs' store warps)
            const uint32_t w_empty0 = cluster_addr(w_empty, 0);
            while (!*abort_flag) {
                if (!mbar_wait_bounded(&te_full[ws], wph, abort_flag, kWaitLimitNs)) { fail(10); break; }
                const TileEntry te = te_slot[ws];
                if (te.x == kTileEndX) break;
                const PairTile ti = decode_pair_tile(te, q);
                if (!mbar_wait_bounded(&epi_done[ws], wph, abort_flag, kWaitLimitNs)) { fail(7); break; }
                if (ti.rows) {
                    const CUtensorMap* mW = p.maps + kMapsPerPair * (size_t)ti.pair;
                    uint8_t* wsrc = w_ring + (size_t)ws * kWTileBytes;
                    store_w_tile(mW, wsrc, ti.row0, ti.col0, ti.wide, p.blk);
                    bulk_commit();
                    bulk_wait_read<0>();
                }
                mbar_arrive_cluster(w_empty0 + 8u * (uint32_t)ws);
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
            }
            bulk_wait<0>();
        }
    } else {
        // ---------------- epilogue (both CTAs, own TMEM lanes) ----------------
        const int ew = warp - kTcEpiWarp0;      // 0..15
        const int quarter = warp & 3;           // TMEM lanes this warp may read
        const int cgrp = ew >> 2;               // 32-column group 0..3
        const int half = cgrp >> 1;             // which 64-column TMA box
        const int row = quarter * 32 + lane;
        const uint32_t t_lane = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cgrp * 32);
        const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
        const int nb = tmem_batches(cf);
        int ws = 0;
        uint32_t wph = 0, aph = 0;
        for (;;) {
            if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
            {
                const bool ok = mbar_wait_bounded(&te_full[ws], wph, abort_flag, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) { fail(11); break; }
                if (te_slot[ws].x == kTileEndX) break;   // the same for every thread
            }
            // one TMEM batch of up to four experts at a time
            float tot[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) tot[i] = 0.f;
            bool ok = true;
#pragma unroll 1
            for (int b0 = 0; b0 < nb * kTmemBatch; b0 += kTmemBatch) {
                ok = mbar_wait_bounded(acc_full, aph, abort_flag, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                aph ^= 1;
                tc_fence_after();
                epi_combine(t_lane, cf, b0, tot);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty0);
            }
            if (!ok) { fail(5); break; }

            ok = mbar_wait_bounded(&w_full[ws], wph, abort_flag, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) { fail(6); break; }
            uint8_t* rowp = w_ring + (size_t)ws * kWTileBytes + (size_t)half * kWBoxBytes + row * 128;
            epi_update_row(rowp, cgrp, row, tot);
            fence_async_smem();
            mbar_arrive(&epi_done[ws]);
            if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
        }
    }

    // teardown: after an abort give in-flight copies and MMAs time to land;
    // neither CTA leaves while the other may still touch its shared memory
    __syncwarp();
    __syncthreads();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) { }
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
    // dynamic schedule: every pair has taken its last ticket by now; the last
    // one to get here leaves the counter at zero for the next launch
    if (p.dyn && q == 0 && threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1ull) == (unsigned long long)n_clusters - 1) {
            atomicExch(p.sched, 0ull);
            atomicExch(p.sched + 1, 0ull);
        }
    }
}

}  // namespace adafuse

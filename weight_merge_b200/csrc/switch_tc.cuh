// switch_tc.cuh -- fused adapter switch on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM), with TMA moving every tile.
//
// AdaFuse (gist.science technical summary, section 2-na): one launch walks the
// segment table and, per 128x128 W tile, applies
//   W <- bf16_rne(W + sum_e c_e (B_e A_e)),  c_e = s (g_cur(e) - g_prev(e)).
// The pages' ingredients map onto Blackwell like this:
//   "segmented"       the tile table; each CTA takes its tiles by ticket in
//                     table order or by a fixed stride (persistent grid, one
//                     CTA per SM);
//   "gather/concat"   per tile and selected expert, TMA fetches the expert's
//                     B rows [row0, row0+128) x [0, r) and A columns
//                     [col0, col0+128) x [0, r) straight from the stacked
//                     [E, ...] tensors (the expert index is the TMA z
//                     coordinate); rank r is padded to KP in {16,32,64} by
//                     TMA's out-of-bounds zero fill;
//   "parallel GEMM"   one tcgen05.mma chain per expert into its own fp32 TMEM
//                     accumulator (4 experts x 128 columns = all 512 columns);
//   "in place"        W tiles go HBM -> smem (TMA, 128B swizzle; one operation
//                     per tile where the weight's in is a multiple of 64) ->
//                     registers, the epilogue adds sum_e c_e acc_e in fp32
//                     (packed fp32 pairs) and rounds once, and TMA stores the
//                     tile back over itself;
//   "prefetch buffer" mbarrier-driven smem rings for W tiles and for operand
//                     slices, filled ahead of use by a producer warp.
// Warp roles: warp 0 W-tile producer (TMA), warp 1 TMEM owner
// + MMA issuer, warp 2 TMA store of finished tiles, warp 3 operand-slice
// producer, warps 4..19 epilogue (row = 32*(warp%4) + lane, 32-column group =
// (warp-4)/4).  The two producers are separate so that W loads run ahead of
// the MMA-paced operand ring.
// Every wait is bounded: on a timeout the CTA raises ADAFUSE_STATUS_TIMEOUT,
// stops issuing work, lets in-flight copies drain, frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace adafuse {

constexpr int kTcThreads = 640;            // 20 warps
constexpr int kTcEpiWarp0 = 4;             // first epilogue warp
constexpr int kTcEpiThreads = 512;         // warps 4..19
constexpr uint32_t kWTileBytes = 128 * 128 * 2;
constexpr uint32_t kWBoxBytes = kWTileBytes / 2;   // 128 rows x 64 cols
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr uint32_t kStallBytes = 16;

// KP: per-expert contraction depth (rank padded to 16, 32 or 64).
// BBULK: rank <= 8.  Its B rows (128 x 8, from B itself at rank 8 or from the
// context's zero-padded copy below) are one contiguous 2 KB block already in
// the plain core-matrix layout, fetched with one bulk copy; its A columns are
// an 8-row TMA box per 64-column half, and the MMA's second 8-deep K group
// reads a shared zero block instead (through the descriptor's K-group stride),
// so each operand stage is 4 KB and the W ring gets a sixth stage.
template <int KP, bool BBULK>
struct TcConfig {
    static_assert(KP == 16 || KP == 32 || KP == 64, "KP");
    static_assert(!BBULK || KP == 16, "the bulk path is rank 8");
    static constexpr int kWStages = BBULK ? 6 : KP == 64 ? 3 : KP == 32 ? 4 : 5;
    static constexpr int kOpStages = KP == 16 ? 6 : 4;
    static constexpr uint32_t kARows = BBULK ? 8 : KP;             // A rows fetched
    static constexpr uint32_t kAHalfBytes = kARows * 128;          // rows x 64 cols bf16
    static constexpr uint32_t kABytes = 2 * kAHalfBytes;
    static constexpr uint32_t kBBytes = BBULK ? 128 * 8 * 2 : 128 * KP * 2;  // 128 x r|KP
    static constexpr uint32_t kOpStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kOpBytes = kOpStages * kOpStageBytes;
    static constexpr uint32_t kZeroBytes = BBULK ? 2048 : 0;      // K rows 8..15 of both halves
    static constexpr uint32_t kWBytes = kWStages * kWTileBytes;
    static constexpr uint32_t kBLayout = KP == 16 ? sm100::kSwizzle32B
                                       : KP == 32 ? sm100::kSwizzle64B
                                                  : sm100::kSwizzle128B;
    static constexpr uint32_t kBSbo = 8 * KP * 2;          // 8 rows of the swizzled B slice
    // barriers (w_full, w_empty, epi_done, te_full per W stage; op_full,
    // op_empty per operand stage; acc_full, acc_empty), the W stages' tile
    // entries, tmem base + abort flag, after the data
    static constexpr uint32_t kBarBytes = 8 * (4 * kWStages + 2 * kOpStages + 2) + 8 * kWStages + 16;
    static constexpr uint32_t kSmemBytes =
        1024 /*alignment slack*/ + kOpBytes + kZeroBytes + kWBytes + kBarBytes;
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(kOpStageBytes % 1024 == 0 && kAHalfBytes % 1024 == 0, "swizzle atoms stay aligned");
};

// Tensor maps per (layer, target): W, A, B, and A as 64-column blocks.
//   plain (some weight's in is not a multiple of 64): W [out, in] with a
//     64 x 128 box (two loads or stores per 128 x 128 tile), A [E, r, in]
//     with a 64 x rows box (two loads per expert and tile);
//   blocked (every in a multiple of 64): W as [in/64 blocks][out][64] with a
//     64 x 128 x 2 box and A as [E][in/64][r][64] with a 64 x rows x 2 x 1
//     box, so one TMA operation moves a whole tile's W or an expert's A
//     columns into the same shared-memory layout (blocks 16 KB / 1 KB apart).
//     The number of TMA operations per tile is a measured cost of these
//     kernels.  Slot 1 keeps the plain A map, which the pair kernel uses.
constexpr int kMapsPerPair = 4;

// One W tile (128 rows x 128 columns at (row0, col0)): the bytes its load
// brings, the load and the store.  A half past the weight's last column is
// zero-filled on load (blocked) or not loaded (plain), and never stored.
__device__ __forceinline__ uint32_t w_tile_bytes(bool blk, bool wide) {
    return (blk || wide) ? kWTileBytes : kWBoxBytes;
}
__device__ __forceinline__ void load_w_tile(void* dst, const CUtensorMap* m, int row0, int col0,
                                            bool wide, bool blk, uint64_t* bar) {
    if (blk) {
        sm100::tma_load_3d(dst, m, 0, row0, col0 >> 6, bar);
    } else {
        sm100::tma_load_2d(dst, m, col0, row0, bar);
        if (wide) sm100::tma_load_2d(static_cast<uint8_t*>(dst) + kWBoxBytes, m, col0 + 64, row0, bar);
    }
}
__device__ __forceinline__ void store_w_tile(const CUtensorMap* m, const void* src, int row0,
                                             int col0, bool wide, bool blk) {
    if (blk) {
        sm100::tma_store_3d(m, src, 0, row0, col0 >> 6);
    } else {
        sm100::tma_store_2d(m, src, col0, row0);
        if (wide) sm100::tma_store_2d(m, static_cast<const uint8_t*>(src) + kWBoxBytes, col0 + 64, row0);
    }
}

struct TcParams {
    const PairDesc* pairs;
    const TileEntry* tiles;
    const CUtensorMap* maps;  // kMapsPerPair per pair: W, A, B, A as 64-column blocks
    int blk;                  // 1: blocked maps (see kMapsPerPair)
    int64_t t_begin, t_end;
    const int32_t* prev;  // routes of `slots` slots (adafuse_route or adafuse_route4)
    const int32_t* cur;
    int slots;
    int E;
    float s;
    int32_t* status;
    // re-base switch: W tiles are read through w0_maps (one map per pair, on
    // the pristine base W0) and written through the W maps, prev is null, and
    // a tile is written even when no expert is selected (it copies W0).
    int rebase;
    const CUtensorMap* w0_maps;
    // test hook (0 = off): the first operand stage of the stall-th tile each
    // CTA (or CTA pair) processes announces kStallBytes more than its loads
    // deliver, so the MMA warp's bounded wait runs out and the launch ends
    // through the timeout path; the CTA's earlier tiles are finished and
    // stored, that tile and later ones are not
    int stall;
    // tile schedule: 0 = static (CTA b takes tiles b, b + grid, ...); 1 =
    // dynamic (the W producers take tickets from sched[0] in table order, so
    // the tiles in flight stay a compact window of the table however the
    // CTAs' speeds drift apart; the last CTA to finish zeroes sched[0..1])
    int dyn;
    unsigned long long* sched;
};

// End-of-schedule marker in a W stage's tile-entry slot.
constexpr uint32_t kTileEndX = 0xffffffffu;

// Tile entries are fetched one iteration ahead (the loops below keep the next
// entry in a register), so no tile waits on a dependent global load.
__device__ __forceinline__ TileEntry fetch_tile(const TileEntry* tiles, int64_t i, int64_t end) {
    return i < end ? __ldg(tiles + i) : make_uint2(0u, 0u);
}

struct TileInfo {
    uint32_t pair;
    int row0, col0;
    bool wide;  // second 64-column half starts inside the weight
};

__device__ __forceinline__ TileInfo decode_tile(TileEntry te) {
    TileInfo ti;
    ti.pair = te.x & kTilePairMask;
    ti.wide = (te.x & kTileWideBit) != 0;
    ti.row0 = (int)(te.y >> 16) * kTile;
    ti.col0 = (int)(te.y & 0xffffu) * kTile;
    return ti;
}

// Epilogue arithmetic shared by both tensor-core kernels, for one thread's row
// and 32-column group.  TMEM holds at most four 128-column accumulators, so
// the experts of a switch come in batches of up to four (kTmemBatch):
//   tot += sum_{e in batch} c_e * acc_e   (experts in order, fp32 FMA)
constexpr int kTmemBatch = 4;

// Batches per tile: at least one, so that a re-base with an empty route still
// passes every tile through the epilogue.
__device__ __forceinline__ int tmem_batches(const Coefs8& cf) {
    return cf.n == 0 ? 1 : (cf.n + kTmemBatch - 1) / kTmemBatch;
}

__device__ __forceinline__ void epi_combine(uint32_t t_lane, const Coefs8& cf, int b0,
                                            float (&tot)[32]) {
#pragma unroll
    for (int ei = 0; ei < kTmemBatch; ++ei) {
        if (b0 + ei < cf.n) {
            const float c = coef_value(cf, b0 + ei);
            const uint64_t cc = sm100::f32x2(c, c);
            float v[32];
            sm100::tmem_ld32(t_lane + 128u * ei, v);
            sm100::tmem_wait_ld();
            // tot[i] = fma(c, v[i], tot[i]), two columns per instruction
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const uint64_t r = sm100::fma_f32x2(cc, sm100::f32x2(v[i], v[i + 1]),
                                                    sm100::f32x2(tot[i], tot[i + 1]));
                sm100::f32x2_split(r, tot[i], tot[i + 1]);
            }
        }
    }
}

//   W <- bf16_rne(W + tot) for this thread's 32 columns of a 128B-swizzled row
//   of 64 columns (4 chunks of 16 bytes, chunk index XOR row % 8)
__device__ __forceinline__ void epi_update_row(uint8_t* rowp, int cgrp, int row, const float (&tot)[32]) {
    uint4 w[4];
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        const int chunk = (cgrp & 1) * 4 + c4;
        w[c4] = sm100::lds128(rowp + ((chunk ^ (row & 7)) << 4));
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t wv[4] = {w[c4].x, w[c4].y, w[c4].z, w[c4].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // (W_lo + tot, W_hi + tot) in one packed fp32 add
            float lo, hi;
            sm100::f32x2_split(
                sm100::add_f32x2(sm100::f32x2(__uint_as_float(wv[j] << 16),
                                              __uint_as_float(wv[j] & 0xffff0000u)),
                                 sm100::f32x2(tot[8 * c4 + 2 * j], tot[8 * c4 + 2 * j + 1])),
                lo, hi);
            const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
            wv[j] = *reinterpret_cast<const uint32_t*>(&b);
        }
        const int chunk = (cgrp & 1) * 4 + c4;
        sm100::sts128(rowp + ((chunk ^ (row & 7)) << 4), make_uint4(wv[0], wv[1], wv[2], wv[3]));
    }
}

template <int KP, bool BBULK>
__global__ void __launch_bounds__(kTcThreads, 1) switch_tc_kernel(const TcParams p) {
    using C = TcConfig<KP, BBULK>;
    using namespace sm100;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* op_ring = smem;                       // [kOpStages][A (rows x 128) | B (128 x r|KP)]
    uint8_t* zero_blk = smem + C::kOpBytes;        // rank 8: zero K rows 8..15
    uint8_t* w_ring = zero_blk + C::kZeroBytes;    // [kWStages][box0 | box1]
    uint64_t* bars = reinterpret_cast<uint64_t*>(w_ring + C::kWBytes);
    uint64_t* w_full = bars;
    uint64_t* w_empty = w_full + C::kWStages;
    uint64_t* op_full = w_empty + C::kWStages;
    uint64_t* op_empty = op_full + C::kOpStages;
    uint64_t* acc_full = op_empty + C::kOpStages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* epi_done = acc_empty + 1;            // [kWStages]: epilogue wrote the tile
    uint64_t* te_full = epi_done + C::kWStages;    // [kWStages]: the stage's tile entry is set
    TileEntry* te_slot = reinterpret_cast<TileEntry*>(te_full + C::kWStages);  // [kWStages]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(te_slot + C::kWStages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    Coefs8 cf;
    const int st = build_coefs(p.prev, p.cur, p.slots, p.E, p.s, cf);
    if (st != 0) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, st);
        return;
    }
    if (cf.n == 0 && !p.rebase) return;  // identity switch
    const int64_t first = p.t_begin + blockIdx.x;
    // (the dynamic schedule needs every CTA at teardown to reset its counter;
    // the launch never has more CTAs than tiles, so no CTA leaves here then)
    if (!p.dyn && first >= p.t_end) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if constexpr (BBULK) {
        // read by the tensor cores (async proxy) through the MMA descriptors
        for (uint32_t i = threadIdx.x; i < C::kZeroBytes / 16; i += blockDim.x)
            reinterpret_cast<uint4*>(zero_blk)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_async_smem();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kWStages; ++i) {
            mbar_init(&w_full[i], 1);
            mbar_init(&w_empty[i], 1);
            mbar_init(&epi_done[i], kTcEpiThreads);
            mbar_init(&te_full[i], 1);
        }
        for (int i = 0; i < C::kOpStages; ++i) {
            mbar_init(&op_full[i], 1);
            mbar_init(&op_empty[i], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kTcEpiThreads / 32);
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
        // Runs ahead of everything else, limited only by free W stages.  It
        // picks the tiles (the next ticket is taken one tile ahead) and
        // publishes each stage's tile entry, or the end marker, to the other
        // roles through te_slot / te_full.
        if (lane == 0) {
            int ws = 0;
            uint32_t wph = 0;
            uint32_t last_pair = 0xffffffffu;
            auto next_tile = [&](int64_t t) -> int64_t {
                if (t >= p.t_end) return t;
                return p.dyn ? p.t_begin + (int64_t)atomicAdd(p.sched, 1ull) : t + gridDim.x;
            };
            int64_t t = p.dyn ? next_tile(p.t_begin) : first;
            TileEntry te = fetch_tile(p.tiles, t, p.t_end);
            while (!*abort_flag) {
                const int64_t tn = next_tile(t);
                const TileEntry te_n = fetch_tile(p.tiles, tn, p.t_end);
                if (!mbar_wait_bounded(&w_empty[ws], wph ^ 1, abort_flag, kWaitLimitNs)) { fail(1); break; }
                if (t >= p.t_end) {
                    te_slot[ws] = make_uint2(kTileEndX, kTileEndX);
                    mbar_arrive(&te_full[ws]);
                    break;
                }
                te_slot[ws] = te;
                mbar_arrive(&te_full[ws]);
                const TileInfo ti = decode_tile(te);
                const CUtensorMap* mW = p.rebase ? p.w0_maps + ti.pair : p.maps + kMapsPerPair * (size_t)ti.pair;
                if (ti.pair != last_pair) {
                    tensormap_acquire(mW);
                    last_pair = ti.pair;
                }
                uint8_t* wdst = w_ring + (size_t)ws * kWTileBytes;
                mbar_arrive_expect_tx(&w_full[ws], w_tile_bytes(p.blk, ti.wide));
                load_w_tile(wdst, mW, ti.row0, ti.col0, ti.wide, p.blk, &w_full[ws]);
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
                if (tn < p.t_end && (te_n.x & kTilePairMask) != ti.pair) {
                    const uint32_t np = te_n.x & kTilePairMask;
                    const CUtensorMap* nm = p.maps + kMapsPerPair * (size_t)np;
                    tensormap_prefetch(p.rebase ? p.w0_maps + np : nm);
                    tensormap_prefetch(nm + (p.blk ? 3 : 1));
                    tensormap_prefetch(nm + 2);
                }
                t = tn;
                te = te_n;
            }
        }
    } else if (warp == 3) {
        // ---------------- operand producer: per tile and expert, the B-row and
        // A-column slices into the operand ring (paced by the MMA warp) ----
        if (lane == 0) {
            int os = 0, ts = 0;
            uint32_t oph = 0, tph = 0;
            uint32_t last_pair = 0xffffffffu;
            int tile_no = 0;   // tiles this CTA has taken (for the stall hook)
            while (!*abort_flag) {
                if (!mbar_wait_bounded(&te_full[ts], tph, abort_flag, kWaitLimitNs)) { fail(8); break; }
                const TileEntry te = te_slot[ts];
                if (++ts == C::kWStages) { ts = 0; tph ^= 1; }
                if (te.x == kTileEndX) break;
                const bool stall_here = ++tile_no == p.stall;
                const TileInfo ti = decode_tile(te);
                const uint32_t pair = ti.pair;
                const int row0 = ti.row0, col0 = ti.col0;
                const CUtensorMap* mA = p.maps + kMapsPerPair * (size_t)pair + (p.blk ? 3 : 1);
                const CUtensorMap* mB = p.maps + kMapsPerPair * (size_t)pair + 2;
                if (pair != last_pair) {
                    tensormap_acquire(mA);
                    tensormap_acquire(mB);
                    last_pair = pair;
                }
                const bool second = ti.wide;
                // A columns of one expert: one blocked load of both 64-column
                // halves, or one plain load per half inside the weight
                const uint32_t a_bytes = (p.blk || second) ? 2 * C::kAHalfBytes : C::kAHalfBytes;
                int out_rows = 128;
                const uint16_t* Bbase = nullptr;
                int out = 0;
                if constexpr (BBULK) {
                    const PairDesc& pd = p.pairs[pair];
                    out = pd.out;
                    Bbase = pd.Bk;
                    out_rows = out - row0 < 128 ? out - row0 : 128;
                }
                bool ok = true;
#pragma unroll 1
                for (int ei = 0; ei < cf.n; ++ei) {
                    const int e = coef_expert(cf, ei);
                    if (!mbar_wait_bounded(&op_empty[os], oph ^ 1, abort_flag, kWaitLimitNs)) { ok = false; break; }
                    uint8_t* a_dst = op_ring + (size_t)os * C::kOpStageBytes;
                    uint8_t* b_dst = a_dst + C::kABytes;
                    if constexpr (BBULK) {
                        // rows past the weight's end are not fetched (their
                        // products only reach accumulator rows never stored)
                        const uint32_t bbytes = (uint32_t)out_rows * 16u;
                        mbar_arrive_expect_tx(&op_full[os], bbytes + a_bytes +
                                                                (stall_here && ei == 0 ? kStallBytes : 0u));
                        bulk_load(b_dst, Bbase + ((size_t)e * out + row0) * 8, bbytes, &op_full[os]);
                    } else {
                        mbar_arrive_expect_tx(&op_full[os], C::kBBytes + a_bytes +
                                                                (stall_here && ei == 0 ? kStallBytes : 0u));
                        tma_load_3d(b_dst, mB, 0, row0, e, &op_full[os]);
                    }
                    if (p.blk) {
                        tma_load_4d(a_dst, mA, 0, 0, col0 >> 6, e, &op_full[os]);
                    } else {
                        tma_load_3d(a_dst, mA, col0, 0, e, &op_full[os]);
                        if (second) tma_load_3d(a_dst + C::kAHalfBytes, mA, col0 + 64, 0, e, &op_full[os]);
                    }
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) { fail(2); break; }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = instr_desc_bf16(128, 128, /*B MN-major*/ 1);
            const uint32_t zero_s = smem_u32(zero_blk);
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
                    const uint32_t b_s = a_s + C::kABytes;
#pragma unroll
                    for (int k = 0; k < KP / 16; ++k) {
                        // MMA A operand: B_e slice, 128 x KP, K-major, rows swizzled
                        // rank 8 (bulk-copied, plain core-matrix layout): the
                        // second 8-deep K chunk re-reads the first (LBO 0) and
                        // meets the zero A rows below, so it adds 0
                        const uint64_t da = BBULK
                            ? smem_desc(b_s, 0, 128, kSwizzleNone)
                            : smem_desc(b_s + 32u * k, 16, C::kBSbo, C::kBLayout);
                        // MMA B operand: A_e slice, KP x 128, N-major, two 64-column
                        // halves (LBO apart), 8-row K groups SBO apart.  Rank 8
                        // holds only K rows 0..7 per half; the K-group stride
                        // points at the zero block (half 1 lands on its second KB).
                        const uint64_t db = BBULK
                            ? smem_desc(a_s, C::kAHalfBytes, zero_s - a_s, kSwizzle128B)
                            : smem_desc(a_s + 2048u * k, C::kAHalfBytes, 1024, kSwizzle128B);
                        tc_mma_f16(tmem_base + 128u * (ei - b0), da, db, idesc, k > 0 ? 1u : 0u);
                    }
                    tc_commit(&op_empty[os]);
                    if (++os == C::kOpStages) { os = 0; oph ^= 1; }
                }
                if (!ok) { fail(4); break; }
                tc_commit(acc_full);
                aph ^= 1;
              }
            }
        }
    } else {
        // ---------------- epilogue ----------------
        // Every decision that can end the loop is made warp-uniform
        // (__all_sync / __any_sync) so tcgen05.ld's .sync.aligned form always
        // sees the whole warp.
        if (warp == 2) {
            // ---- store warp: TMA-stores each finished tile over itself and
            // frees its smem stage as soon as the store has read it.
            if (lane == 0) {
                int ws = 0;
                uint32_t wph = 0;
                while (!*abort_flag) {
                    if (!mbar_wait_bounded(&te_full[ws], wph, abort_flag, kWaitLimitNs)) { fail(10); break; }
                    const TileEntry te = te_slot[ws];
                    if (te.x == kTileEndX) break;
                    const TileInfo ti = decode_tile(te);
                    const int row0 = ti.row0, col0 = ti.col0;
                    if (!mbar_wait_bounded(&epi_done[ws], wph, abort_flag, kWaitLimitNs)) { fail(7); break; }
                    const CUtensorMap* mW = p.maps + kMapsPerPair * (size_t)ti.pair;
                    uint8_t* wsrc = w_ring + (size_t)ws * kWTileBytes;
                    store_w_tile(mW, wsrc, row0, col0, ti.wide, p.blk);
                    bulk_commit();
                    bulk_wait_read<0>();
                    mbar_arrive(&w_empty[ws]);
                    if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
                }
                bulk_wait<0>();
            }
        } else {
            const int ew = warp - kTcEpiWarp0;      // 0..15
            const int quarter = warp & 3;           // TMEM lanes this warp may read
            const int cgrp = ew >> 2;               // 32-column group 0..3
            const int half = cgrp >> 1;             // which 64-column TMA box
            const int row = quarter * 32 + lane;
            const uint32_t t_lane = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(cgrp * 32);
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
                // 1) sum_e c_e * acc_e for this thread's row, 32 columns,
                //    one TMEM batch of up to four experts at a time
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
                    if (lane == 0) mbar_arrive(acc_empty);
                }
                if (!ok) { fail(5); break; }

                // 2) W: smem (128B-swizzled rows of 64 columns) -> +dW -> smem
                ok = mbar_wait_bounded(&w_full[ws], wph, abort_flag, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) { fail(6); break; }
                uint8_t* rowp = w_ring + (size_t)ws * kWTileBytes + (size_t)half * kWBoxBytes + row * 128;
                epi_update_row(rowp, cgrp, row, tot);
                fence_async_smem();
                mbar_arrive(&epi_done[ws]);
                if (++ws == C::kWStages) { ws = 0; wph ^= 1; }
            }
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
    // dynamic schedule: every CTA has taken its last ticket by now; the last
    // one to get here leaves the counter at zero for the next launch
    if (p.dyn && threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1ull) == (unsigned long long)gridDim.x - 1) {
            atomicExch(p.sched, 0ull);
            atomicExch(p.sched + 1, 0ull);
        }
    }
}

}  // namespace adafuse

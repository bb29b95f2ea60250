// adafuse_abi.cu -- C ABI of the adapter switch: context, segment table,
// argument checks and kernel launches.  See include/adafuse.h for the
// contract of each entry point.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "adafuse.h"
#include "common.cuh"
#include "pregate.cuh"
#include "switch_mma.cuh"
#include "switch_tc.cuh"
#include "switch_tc_host.cuh"

using namespace adafuse;

struct adafuse_ctx {
    int device = 0;
    int sm_count = 0;
    int32_t n_layers = 0, n_targets = 0, n_experts = 0, rank = 0;
    float alpha = 0.f, scale = 0.f;
    int64_t n_tiles = 0;
    std::vector<int64_t> layer_tile_begin;  // [n_layers + 1]
    PairDesc* d_pairs = nullptr;
    TileEntry* d_tiles = nullptr;
    int32_t* d_status = nullptr;
    CUtensorMap* d_maps = nullptr;  // kMapsPerPair per pair when the tensor-core kernel can run
    bool blk = false;               // those maps are blocked (every weight's in % 64 == 0)
    int tc_kp = 0;                  // its padded rank (16, 32, 64), 0 = not eligible
    int kernel = ADAFUSE_KERNEL_AUTO;
    std::vector<PairDesc> h_pairs;  // host copy of d_pairs (re-base pointers are patched in)
    CUtensorMap* d_w0_maps = nullptr;  // 1 per pair on the re-base source W0
    bool has_base = false;
    int stall_at = 0;  // test hook: the next tensor-core launch stalls at each CTA's n-th tile
    // pair kernel: 256 x 128 blocks, layer-major like the tile table
    TileEntry* d_blocks = nullptr;
    uint16_t* d_bpad = nullptr;              // rank < 8: B with rows zero-padded to 8
    uint16_t* d_fold = nullptr;              // rank <= 8: folded-coefficient operands
                                             // (allocated on first use, see ensure_fold)
    bool fold_failed = false;                // that allocation failed: the kernel is off
    float* d_logits = nullptr;               // [kMaxBatchTokens, E] batch pre-gate scratch
    unsigned long long* d_sched = nullptr;   // [2] ticket counter of the dynamic tile schedule
    int schedule = ADAFUSE_SCHEDULE_AUTO;
    std::vector<int64_t> layer_block_begin;  // [n_layers + 1]
    int pair_clusters = 0;                   // co-resident CTA pairs (0 = not queried yet)
    int max_ctas = 0;                        // cap on a switch's persistent grid (0 = none)
};

namespace {

thread_local char g_last_error[256] = "";

int cuda_fail(cudaError_t e, const char* what) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
    return ADAFUSE_ERR_CUDA;
}

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    bool ok = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        ok = (prev == dev) || cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// CTAs a switch launch may keep resident: every SM, or the caller's cap
// (adafuse_set_max_ctas) so that other work can run beside the switch.
int switch_ctas(const adafuse_ctx* c) {
    return c->max_ctas > 0 && c->max_ctas < c->sm_count ? c->max_ctas : c->sm_count;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Raise a kernel's dynamic shared-memory limit only when this device has not
// been given at least `bytes` for that kernel yet (the host call is not free,
// and the decode-time pre-gate launches are short).  Keyed by the kernel's
// address and the device: kernels of one signature are different entries.
struct SmemAttrEntry {
    const void* fn;
    int device;
    size_t bytes;
};

template <typename Kernel>
void ensure_smem_attr(Kernel kernel, size_t bytes, int device) {
    static std::mutex mu;
    static std::vector<SmemAttrEntry> done;
    const void* fn = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lk(mu);
    for (const SmemAttrEntry& en : done)
        if (en.fn == fn && en.device == device && en.bytes >= bytes) return;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
        cudaSuccess)
        return;   // the launch reports the error
    for (SmemAttrEntry& en : done)
        if (en.fn == fn && en.device == device) {
            en.bytes = bytes;
            return;
        }
    done.push_back({fn, device, bytes});
}

// Shape and pointer checks shared by create and the host-only table query.
int check_desc(const adafuse_desc* d, bool need_pointers) {
    if (d == nullptr || d->targets == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    if (d->n_layers < 1 || d->n_targets < 1) return ADAFUSE_ERR_INVALID_ARG;
    if (d->n_experts < 1 || d->n_experts > 64) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    if (d->rank < 1 || d->rank > 64) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    if (!std::isfinite(d->alpha)) return ADAFUSE_ERR_INVALID_ARG;
    const int64_t n = (int64_t)d->n_layers * d->n_targets;
    if (n > (int64_t)1 << 30) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;  // pair index < 2^31
    for (int64_t i = 0; i < n; ++i) {
        const adafuse_target& t = d->targets[i];
        if (t.out <= 0 || t.in <= 0) return ADAFUSE_ERR_INVALID_ARG;
        if (t.out % 8 != 0 || t.in % 8 != 0) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
        // tile indices are packed in 16 bits; element offsets in int32 rows
        if (ceil_div(t.out, kTile) > 65535 || ceil_div(t.in, kTile) > 65535)
            return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
        if (t.out > INT32_MAX || t.in > INT32_MAX) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
        if (need_pointers) {
            if (t.W == nullptr || t.A == nullptr || t.B == nullptr) return ADAFUSE_ERR_INVALID_ARG;
            if (!aligned16(t.W) || !aligned16(t.A) || !aligned16(t.B)) return ADAFUSE_ERR_INVALID_ARG;
        }
    }
    return ADAFUSE_OK;
}

// The segment table: every (layer, target) weight cut into 128x128 tiles
// (the last row / column of tiles may be ragged), layer-major, then target,
// then row tile, then column tile.  Each W element lies in exactly one tile.
template <typename Emit>
int64_t walk_tiles(const adafuse_desc* d, Emit&& emit) {
    int64_t n = 0;
    for (int32_t l = 0; l < d->n_layers; ++l)
        for (int32_t k = 0; k < d->n_targets; ++k) {
            const adafuse_target& t = d->targets[(int64_t)l * d->n_targets + k];
            const int64_t rt = ceil_div(t.out, kTile), ct = ceil_div(t.in, kTile);
            for (int64_t i = 0; i < rt; ++i)
                for (int64_t j = 0; j < ct; ++j) emit(l, k, i, j, n++);
        }
    return n;
}

// The pair kernel's table: every (layer, target) weight cut into 256 x 128
// blocks (two 128-row tiles, one per CTA of a pair), in the same order.
template <typename Emit>
int64_t walk_blocks(const adafuse_desc* d, Emit&& emit) {
    int64_t n = 0;
    for (int32_t l = 0; l < d->n_layers; ++l)
        for (int32_t k = 0; k < d->n_targets; ++k) {
            const adafuse_target& t = d->targets[(int64_t)l * d->n_targets + k];
            const int64_t rb = ceil_div(t.out, kBlockRows), ct = ceil_div(t.in, kTile);
            for (int64_t i = 0; i < rb; ++i)
                for (int64_t j = 0; j < ct; ++j) emit(l, k, i, j, n++);
        }
    return n;
}

// The pair kernel takes the tensor-core kernel's ranks except 8 (whose A
// tensor maps fetch exactly 8 rows for the single-CTA kernel's layout).
bool pair_eligible(const adafuse_ctx* c) { return c->tc_kp != 0 && c->rank > 8; }

// The folded kernel takes ranks up to 8 unless its operand buffer could not
// be allocated (it is allocated on first use, see ensure_fold).
bool fold_eligible(const adafuse_ctx* c) {
    return c->tc_kp != 0 && c->rank <= 8 && !c->fold_failed;
}

// The folded kernel's operand buffer, allocated on the first call that needs
// it (adafuse_set_switch_kernel(FOLD), or the first in-place top-k switch that
// AUTO gives to the folded kernel) rather than at create: a context that
// never folds pays nothing for it.  Allocating synchronises the device, so
// the first use may not be captured into a graph (INVALID_ARG then, with
// nothing enqueued).  An allocation failure turns the kernel off for the
// context (OUT_OF_MEMORY).
int ensure_fold(adafuse_ctx* c, cudaStream_t capture_check) {
    if (c->d_fold != nullptr) return ADAFUSE_OK;
    if (!fold_eligible(c)) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(capture_check, &cs);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cs != cudaStreamCaptureStatusNone) return ADAFUSE_ERR_INVALID_ARG;
    size_t total = 0;
    for (const PairDesc& pd : c->h_pairs) total += fold_bytes_for(pd.in);
    std::vector<PairDesc> pairs;
    try {
        pairs = c->h_pairs;
    } catch (...) {
        return ADAFUSE_ERR_OUT_OF_MEMORY;
    }
    uint16_t* buf = nullptr;
    e = cudaMalloc(&buf, total);
    if (e == cudaErrorMemoryAllocation) {
        (void)cudaGetLastError();
        c->fold_failed = true;
        return ADAFUSE_ERR_OUT_OF_MEMORY;
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(folded operands)");
    size_t off = 0;
    for (PairDesc& pd : pairs) {
        pd.Af = buf + off / 2;
        off += fold_bytes_for(pd.in);
    }
    // the descriptors may be read by work still in flight: replace them once
    // the device is idle
    e = cudaDeviceSynchronize();
    if (e == cudaSuccess)
        e = cudaMemcpy(c->d_pairs, pairs.data(), sizeof(PairDesc) * pairs.size(),
                       cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(buf);
        return cuda_fail(e, "folded operand descriptors");
    }
    c->h_pairs.swap(pairs);
    c->d_fold = buf;
    return ADAFUSE_OK;
}

// Rank < 8: copy every B [E, out, r] into its [E, out, 8] zero-padded slot
// (the padding columns are zeroed once, at create).
cudaError_t copy_padded_b(const adafuse_ctx* c, cudaStream_t s) {
    for (const PairDesc& pd : c->h_pairs) {
        const size_t rows = (size_t)c->n_experts * (size_t)pd.out;
        const cudaError_t e = cudaMemcpy2DAsync(const_cast<uint16_t*>(pd.Bk), 16, pd.B,
                                                (size_t)c->rank * 2, (size_t)c->rank * 2, rows,
                                                cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

int kp_class(int r) { return r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

// The parameters of one tensor-core launch over entries [t0, t1) of `tiles`
// (the tile table, or the block table for the pair kernel).  Consumes the
// pending stall-hook request, so it applies to exactly one launch.
TcParams tc_params(adafuse_ctx* c, const TileEntry* tiles, int64_t t0, int64_t t1,
                   const int32_t* prev, const int32_t* cur, int slots, bool rebase, bool dyn) {
    TcParams prm;
    prm.pairs = c->d_pairs;
    prm.tiles = tiles;
    prm.maps = c->d_maps;
    prm.blk = c->blk ? 1 : 0;
    prm.t_begin = t0;
    prm.t_end = t1;
    prm.prev = prev;
    prm.cur = cur;
    prm.slots = slots;
    prm.E = c->n_experts;
    prm.s = c->scale;
    prm.status = c->d_status;
    prm.rebase = rebase ? 1 : 0;
    prm.w0_maps = c->d_w0_maps;
    prm.stall = c->stall_at;
    c->stall_at = 0;
    prm.dyn = dyn ? 1 : 0;
    prm.sched = dyn ? c->d_sched : nullptr;
    return prm;
}

template <int KP, bool BBULK>
cudaError_t launch_tc(adafuse_ctx* c, int64_t t0, int64_t t1, const int32_t* prev,
                      const int32_t* cur, int slots, cudaStream_t s, bool rebase) {
    // AUTO schedule: dynamic for this kernel
    const TcParams prm = tc_params(c, c->d_tiles, t0, t1, prev, cur, slots, rebase,
                                   c->schedule != ADAFUSE_SCHEDULE_STATIC);
    return launch_switch_tc<KP, BBULK>(prm, c->device, switch_ctas(c), s);
}

template <int KP>
cudaError_t launch_tc2(adafuse_ctx* c, int64_t b0, int64_t b1, const int32_t* prev,
                       const int32_t* cur, int slots, cudaStream_t s, bool rebase) {
    if (c->pair_clusters == 0) {
        const cudaError_t e = pair_kernel_clusters<KP>(c->sm_count, &c->pair_clusters);
        if (e != cudaSuccess) {
            c->pair_clusters = 0;
            return e;
        }
    }
    // AUTO schedule: static for the pair kernel
    const TcParams prm = tc_params(c, c->d_blocks, b0, b1, prev, cur, slots, rebase,
                                   c->schedule == ADAFUSE_SCHEDULE_DYNAMIC);
    const int cap = switch_ctas(c) / 2 > 0 ? switch_ctas(c) / 2 : 1;
    return launch_switch_tc2<KP>(prm, c->pair_clusters < cap ? c->pair_clusters : cap, s);
}

}  // namespace

extern "C" {

const char* adafuse_last_error(void) { return g_last_error; }

const char* adafuse_strerror(int code) {
    switch (code) {
        case ADAFUSE_OK: return "ok";
        case ADAFUSE_ERR_INVALID_ARG: return "invalid argument";
        case ADAFUSE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case ADAFUSE_ERR_CUDA: return "CUDA runtime error";
        case ADAFUSE_ERR_DEVICE_FAULT: return "device status word set (bad route)";
        case ADAFUSE_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0";
        case ADAFUSE_ERR_OUT_OF_MEMORY: return "out of memory";
        default: return "unknown error";
    }
}

int adafuse_tile_size(void) { return kTile; }

int adafuse_segment_table(const adafuse_desc* desc, int32_t* entries, int64_t capacity,
                          int64_t* count) {
    if (count == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    const int rc = check_desc(desc, false);
    if (rc != ADAFUSE_OK) return rc;
    const int64_t n = walk_tiles(desc, [](int, int, int64_t, int64_t, int64_t) {});
    *count = n;
    if (entries == nullptr) return ADAFUSE_OK;
    if (capacity < n) return ADAFUSE_ERR_INVALID_ARG;
    walk_tiles(desc, [&](int l, int k, int64_t i, int64_t j, int64_t q) {
        entries[4 * q + 0] = l;
        entries[4 * q + 1] = k;
        entries[4 * q + 2] = (int32_t)(i * kTile);
        entries[4 * q + 3] = (int32_t)(j * kTile);
    });
    return ADAFUSE_OK;
}

int adafuse_create(adafuse_ctx** out, const adafuse_desc* desc, int device) {
    if (out == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = check_desc(desc, true);
    if (rc != ADAFUSE_OK) return rc;

    int ndev = 0;
    cudaError_t e = cudaGetDeviceCount(&ndev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
    if (device < 0 || device >= ndev) return ADAFUSE_ERR_INVALID_ARG;
    DeviceGuard guard(device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0) return ADAFUSE_ERR_UNSUPPORTED_DEVICE;

    adafuse_ctx* c = new (std::nothrow) adafuse_ctx();
    if (c == nullptr) return ADAFUSE_ERR_OUT_OF_MEMORY;
    c->device = device;
    c->sm_count = prop.multiProcessorCount;
    c->n_layers = desc->n_layers;
    c->n_targets = desc->n_targets;
    c->n_experts = desc->n_experts;
    c->rank = desc->rank;
    c->alpha = desc->alpha;
    c->scale = desc->alpha / (float)desc->rank;

    const int64_t npairs = (int64_t)desc->n_layers * desc->n_targets;
    std::vector<PairDesc> pairs((size_t)npairs);
    for (int64_t i = 0; i < npairs; ++i) {
        const adafuse_target& t = desc->targets[i];
        pairs[i].W = static_cast<uint16_t*>(t.W);
        pairs[i].W0 = nullptr;
        pairs[i].A = static_cast<const uint16_t*>(t.A);
        pairs[i].B = static_cast<const uint16_t*>(t.B);
        pairs[i].Bk = pairs[i].B;
        pairs[i].Af = nullptr;
        pairs[i].out = (int32_t)t.out;
        pairs[i].in = (int32_t)t.in;
        pairs[i].layer = (int32_t)(i / desc->n_targets);
        pairs[i].target = (int32_t)(i % desc->n_targets);
    }
    std::vector<TileEntry> tiles;
    c->layer_tile_begin.assign((size_t)desc->n_layers + 1, 0);
    try {
        tiles.reserve((size_t)walk_tiles(desc, [](int, int, int64_t, int64_t, int64_t) {}));
        walk_tiles(desc, [&](int l, int k, int64_t i, int64_t j, int64_t) {
            const adafuse_target& tg = desc->targets[(int64_t)l * desc->n_targets + k];
            TileEntry te;
            te.x = (uint32_t)((int64_t)l * desc->n_targets + k);
            if (j * kTile + 64 < tg.in) te.x |= kTileWideBit;
            te.y = (uint32_t)((i << 16) | j);
            tiles.push_back(te);
            c->layer_tile_begin[(size_t)l + 1] = (int64_t)tiles.size();
        });
    } catch (...) {
        delete c;
        return ADAFUSE_ERR_OUT_OF_MEMORY;
    }
    c->n_tiles = (int64_t)tiles.size();
    try {
        c->h_pairs = pairs;
    } catch (...) {
        delete c;
        return ADAFUSE_ERR_OUT_OF_MEMORY;
    }

    auto fail = [&](cudaError_t err, const char* what) {
        cudaFree(c->d_pairs);
        cudaFree(c->d_tiles);
        cudaFree(c->d_status);
        cudaFree(c->d_maps);
        cudaFree(c->d_blocks);
        cudaFree(c->d_bpad);
        cudaFree(c->d_fold);
        cudaFree(c->d_sched);
        cudaFree(c->d_logits);
        delete c;
        return err == cudaErrorMemoryAllocation ? ADAFUSE_ERR_OUT_OF_MEMORY : cuda_fail(err, what);
    };
    // ranks below 8: the tensor-core path reads B through a copy with 16-byte
    // rows (a legal TMA stride), zero-padded past the rank
    if (desc->rank < 8 && tc_kp_for(desc->rank) != 0) {
        size_t total = 0;
        for (const PairDesc& pd : pairs) total += (size_t)desc->n_experts * (size_t)pd.out * 8;
        if ((e = cudaMalloc(&c->d_bpad, total * 2)) != cudaSuccess)
            return fail(e, "cudaMalloc(padded B)");
        if ((e = cudaMemset(c->d_bpad, 0, total * 2)) != cudaSuccess)
            return fail(e, "cudaMemset(padded B)");
        size_t off = 0;
        for (PairDesc& pd : pairs) {
            pd.Bk = c->d_bpad + off;
            off += (size_t)desc->n_experts * (size_t)pd.out * 8;
        }
        c->h_pairs = pairs;
        if ((e = copy_padded_b(c, nullptr)) != cudaSuccess) return fail(e, "cudaMemcpy2D(padded B)");
        if ((e = cudaDeviceSynchronize()) != cudaSuccess) return fail(e, "padded B");
    }
    if ((e = cudaMalloc(&c->d_pairs, sizeof(PairDesc) * pairs.size())) != cudaSuccess)
        return fail(e, "cudaMalloc(pairs)");
    if ((e = cudaMalloc(&c->d_tiles, sizeof(TileEntry) * tiles.size())) != cudaSuccess)
        return fail(e, "cudaMalloc(tiles)");
    if ((e = cudaMalloc(&c->d_status, sizeof(int32_t))) != cudaSuccess)
        return fail(e, "cudaMalloc(status)");
    if ((e = cudaMalloc(&c->d_logits, sizeof(float) * kMaxBatchTokens * desc->n_experts)) != cudaSuccess)
        return fail(e, "cudaMalloc(batch logits)");
    if ((e = cudaMalloc(&c->d_sched, 2 * sizeof(unsigned long long))) != cudaSuccess)
        return fail(e, "cudaMalloc(schedule)");
    if ((e = cudaMemset(c->d_sched, 0, 2 * sizeof(unsigned long long))) != cudaSuccess)
        return fail(e, "cudaMemset(schedule)");
    if ((e = cudaMemcpy(c->d_pairs, pairs.data(), sizeof(PairDesc) * pairs.size(),
                        cudaMemcpyHostToDevice)) != cudaSuccess)
        return fail(e, "cudaMemcpy(pairs)");
    if ((e = cudaMemcpy(c->d_tiles, tiles.data(), sizeof(TileEntry) * tiles.size(),
                        cudaMemcpyHostToDevice)) != cudaSuccess)
        return fail(e, "cudaMemcpy(tiles)");
    if ((e = cudaMemset(c->d_status, 0, sizeof(int32_t))) != cudaSuccess)
        return fail(e, "cudaMemset(status)");

    // tensor maps for the tensor-core kernel (when the rank allows TMA)
    c->tc_kp = tc_kp_for(desc->rank);
    if (c->tc_kp != 0) {
        EncodeTiledFn enc = encode_tiled_fn();
        std::vector<CUtensorMap> maps;
        bool ok = enc != nullptr;
        if (ok) {
            try {
                maps.resize((size_t)npairs * kMapsPerPair);
            } catch (...) {
                ok = false;
            }
        }
        // blocked maps where every weight allows them; plain ones if the
        // driver refuses a blocked encoding
        c->blk = blocked_maps_ok(pairs.data(), npairs);
        for (int pass = 0; pass < 2; ++pass) {
            bool enc_ok = ok;
            for (int64_t i = 0; enc_ok && i < npairs; ++i)
                enc_ok = encode_pair_maps(enc, pairs[i], desc->n_experts, desc->rank, c->tc_kp,
                                          c->blk, &maps[kMapsPerPair * i]);
            if (enc_ok || !c->blk) {
                ok = ok && enc_ok;
                break;
            }
            c->blk = false;
        }
        if (ok) {
            if ((e = cudaMalloc(&c->d_maps, sizeof(CUtensorMap) * maps.size())) != cudaSuccess)
                return fail(e, "cudaMalloc(maps)");
            if ((e = cudaMemcpy(c->d_maps, maps.data(), sizeof(CUtensorMap) * maps.size(),
                                cudaMemcpyHostToDevice)) != cudaSuccess)
                return fail(e, "cudaMemcpy(maps)");
        } else {
            c->tc_kp = 0;  // fall back to the mma.sync kernel for this context
        }
    }
    if (pair_eligible(c)) {
        std::vector<TileEntry> blocks;
        try {
            c->layer_block_begin.assign((size_t)desc->n_layers + 1, 0);
            blocks.reserve((size_t)walk_blocks(desc, [](int, int, int64_t, int64_t, int64_t) {}));
            walk_blocks(desc, [&](int l, int k, int64_t i, int64_t j, int64_t) {
                const adafuse_target& tg = desc->targets[(int64_t)l * desc->n_targets + k];
                TileEntry te;
                te.x = (uint32_t)((int64_t)l * desc->n_targets + k);
                if (j * kTile + 64 < tg.in) te.x |= kTileWideBit;
                if (i * kBlockRows + kTile < tg.out) te.x |= kTileLowerBit;
                te.y = (uint32_t)((i << 16) | j);
                blocks.push_back(te);
                c->layer_block_begin[(size_t)l + 1] = (int64_t)blocks.size();
            });
        } catch (...) {
            return fail(cudaErrorMemoryAllocation, "block table");
        }
        if ((e = cudaMalloc(&c->d_blocks, sizeof(TileEntry) * blocks.size())) != cudaSuccess)
            return fail(e, "cudaMalloc(blocks)");
        if ((e = cudaMemcpy(c->d_blocks, blocks.data(), sizeof(TileEntry) * blocks.size(),
                            cudaMemcpyHostToDevice)) != cudaSuccess)
            return fail(e, "cudaMemcpy(blocks)");
    }
    *out = c;
    return ADAFUSE_OK;
}

int adafuse_destroy(adafuse_ctx* ctx) {
    if (ctx == nullptr) return ADAFUSE_OK;
    DeviceGuard guard(ctx->device);
    cudaFree(ctx->d_pairs);
    cudaFree(ctx->d_tiles);
    cudaFree(ctx->d_status);
    cudaFree(ctx->d_maps);
    cudaFree(ctx->d_w0_maps);
    cudaFree(ctx->d_blocks);
    cudaFree(ctx->d_bpad);
    cudaFree(ctx->d_fold);
    cudaFree(ctx->d_sched);
    cudaFree(ctx->d_logits);
    delete ctx;
    return ADAFUSE_OK;
}

int adafuse_set_switch_kernel(adafuse_ctx* ctx, int kernel) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    if (kernel != ADAFUSE_KERNEL_AUTO && kernel != ADAFUSE_KERNEL_MMA_SYNC &&
        kernel != ADAFUSE_KERNEL_TCGEN05 && kernel != ADAFUSE_KERNEL_TCGEN05_PAIR &&
        kernel != ADAFUSE_KERNEL_TCGEN05_FOLD)
        return ADAFUSE_ERR_INVALID_ARG;
    if (kernel == ADAFUSE_KERNEL_TCGEN05 && ctx->tc_kp == 0) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    if (kernel == ADAFUSE_KERNEL_TCGEN05_PAIR && !pair_eligible(ctx))
        return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    if (kernel == ADAFUSE_KERNEL_TCGEN05_FOLD) {
        if (!fold_eligible(ctx)) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
        DeviceGuard guard(ctx->device);
        if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
        const int rc = ensure_fold(ctx, nullptr);
        if (rc != ADAFUSE_OK) return rc;
    }
    ctx->kernel = kernel;
    return ADAFUSE_OK;
}

int adafuse_get_topk_switch_kernel(adafuse_ctx* ctx) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    // measured on B200 at the Llama-2-7B shape, top-4 in place: the folded
    // kernel's single accumulator holds up to 8 experts (79% of peak), where
    // the four-accumulator kernel needs two TMEM passes per tile (58%)
    if (ctx->kernel == ADAFUSE_KERNEL_AUTO && fold_eligible(ctx)) return ADAFUSE_KERNEL_TCGEN05_FOLD;
    return adafuse_get_switch_kernel(ctx);
}

int adafuse_set_tile_schedule(adafuse_ctx* ctx, int schedule) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    if (schedule != ADAFUSE_SCHEDULE_STATIC && schedule != ADAFUSE_SCHEDULE_DYNAMIC &&
        schedule != ADAFUSE_SCHEDULE_AUTO)
        return ADAFUSE_ERR_INVALID_ARG;
    ctx->schedule = schedule;
    return ADAFUSE_OK;
}

int adafuse_set_max_ctas(adafuse_ctx* ctx, int32_t max_ctas) {
    if (ctx == nullptr || max_ctas < 0) return ADAFUSE_ERR_INVALID_ARG;
    ctx->max_ctas = max_ctas;
    return ADAFUSE_OK;
}

int adafuse_get_tensor_map_layout(const adafuse_ctx* ctx) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    return ctx->tc_kp == 0 ? ADAFUSE_MAPS_NONE : ctx->blk ? ADAFUSE_MAPS_BLOCKED : ADAFUSE_MAPS_PLAIN;
}

int adafuse_get_switch_kernel(adafuse_ctx* ctx) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    if (ctx->kernel == ADAFUSE_KERNEL_AUTO) {
        // measured on B200 at the Llama shapes: the pair kernel is level at
        // rank 64 and ahead at rank 16; rank 8 keeps the single-CTA kernel's
        // bulk-copied B rows and deeper W ring
        if (pair_eligible(ctx)) return ADAFUSE_KERNEL_TCGEN05_PAIR;
        return ctx->tc_kp != 0 ? ADAFUSE_KERNEL_TCGEN05 : ADAFUSE_KERNEL_MMA_SYNC;
    }
    return ctx->kernel;
}

}  // extern "C"

namespace {

// Top-k pre-gating into routes of `slots` slots (2: adafuse_route, 4:
// adafuse_route4).  The same kernels and arithmetic for every k and batch.
int pregate_launch(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d, const float* Wr,
                   int k, int slots, void* route_out, void* stream, float* logits = nullptr) {
    int32_t* route = static_cast<int32_t*>(route_out);
    if (ctx == nullptr || T < 0 || d < 1 || (d & 3) != 0) return ADAFUSE_ERR_INVALID_ARG;
    if (T == 0) return ADAFUSE_OK;
    if (h == nullptr || Wr == nullptr || (route == nullptr && logits == nullptr))
        return ADAFUSE_ERR_INVALID_ARG;
    if (!aligned16(h) || !aligned16(route) || (reinterpret_cast<uintptr_t>(Wr) & 3u))
        return ADAFUSE_ERR_INVALID_ARG;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int E = ctx->n_experts;
    // Batches of 64+ tokens with up to 8 experts and d <= 4096: the
    // token-group kernel (a warp pair per 4 tokens).  It computes the same
    // bits as pregate_kernel, which takes every other case, so a token's
    // route does not depend on which one ran.
    const int64_t nch = ceil_div(d >> 2, 256);
    if (E <= 8 && nch <= kGroupMaxChunks && T >= kGroupMinTokens) {
        const size_t smem = group_smem_bytes(d);
        const int64_t ngroups = ceil_div(T, kGroupTokens);
        const unsigned grid = (unsigned)std::min<int64_t>(ngroups, (int64_t)ctx->sm_count);
        // Wr staged by TMA tile loads when it is [d/4][32] floats (E == 8)
        // at a 16-byte-aligned address; by the CTA's threads otherwise
        CUtensorMap wr_map;
        std::memset(&wr_map, 0, sizeof(wr_map));
        int wr_tma = 0;
        if (E == 8 && aligned16(Wr)) {
            EncodeTiledFn enc = encode_tiled_fn();
            const cuuint64_t dims[2] = {32, (cuuint64_t)(d >> 2)};
            const cuuint64_t strides[1] = {128};
            const cuuint32_t box[2] = {32, (cuuint32_t)kGroupWrBoxRows};
            const cuuint32_t ones[2] = {1, 1};
            wr_tma = enc != nullptr &&
                     enc(&wr_map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(Wr), dims,
                         strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
        auto go = [&](auto kernel) {
            ensure_smem_attr(kernel, smem, ctx->device);
            kernel<<<grid, kGroupThreads, smem, s>>>(h, T, d, Wr, E, k, slots, route, logits, wr_map,
                                                     wr_tma, ctx->d_status);
        };
        switch (nch) {
            case 1: go(pregate_group_kernel<1>); break;
            case 2: go(pregate_group_kernel<2>); break;
            case 3: go(pregate_group_kernel<3>); break;
            default: go(pregate_group_kernel<4>); break;
        }
        const cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "pregate launch");
    }
    const int emax = E <= 8 ? 8 : E <= 16 ? 16 : E <= 32 ? 32 : 64;
    const int tpb = 64 / emax;   // tokens per CTA group: TPB x EMAX partial logits per thread
    const int64_t groups = ceil_div(T, tpb);
    // Wr in shared memory for batches that amortise staging it (persistent
    // CTAs); otherwise read from global memory.  Same arithmetic either way.
    // Rows of Wr are read as float4 only when Wr is 16-byte aligned (the ABI
    // asks for 4-byte alignment); otherwise element by element.
    const bool wr16 = (reinterpret_cast<uintptr_t>(Wr) & 15u) == 0;
    const size_t wr_smem = (size_t)d * (emax + 1) * 4;
    const bool shared = T >= 256 && wr_smem <= 160 * 1024;
    const unsigned grid = (unsigned)(shared ? std::min<int64_t>(groups, (int64_t)ctx->sm_count) : groups);
    auto go = [&](auto kernel, size_t smem) {
        if (smem > 0) ensure_smem_attr(kernel, smem, ctx->device);
        kernel<<<grid, kPregateThreads, smem, s>>>(h, T, d, Wr, E, k, slots, route, logits);
    };
    if (shared) {
        switch (emax) {
            case 8: go(pregate_kernel<8, 8, kWrShared>, wr_smem); break;
            case 16: go(pregate_kernel<16, 4, kWrShared>, wr_smem); break;
            case 32: go(pregate_kernel<32, 2, kWrShared>, wr_smem); break;
            default: go(pregate_kernel<64, 1, kWrShared>, wr_smem); break;
        }
    } else if (E == emax && wr16) {
        switch (emax) {
            case 8: go(pregate_kernel<8, 8, kWrVector>, 0); break;
            case 16: go(pregate_kernel<16, 4, kWrVector>, 0); break;
            case 32: go(pregate_kernel<32, 2, kWrVector>, 0); break;
            default: go(pregate_kernel<64, 1, kWrVector>, 0); break;
        }
    } else {
        switch (emax) {
            case 8: go(pregate_kernel<8, 8, kWrScalar>, 0); break;
            case 16: go(pregate_kernel<16, 4, kWrScalar>, 0); break;
            case 32: go(pregate_kernel<32, 2, kWrScalar>, 0); break;
            default: go(pregate_kernel<64, 1, kWrScalar>, 0); break;
        }
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "pregate launch");
}

}  // namespace

extern "C" {

int adafuse_pregate(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d, const float* Wr,
                    adafuse_route* route, void* stream) {
    return pregate_launch(ctx, h, T, d, Wr, 2, 2, route, stream);
}

int adafuse_pregate_topk(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                         const float* Wr, int32_t k, adafuse_route4* route, void* stream) {
    if (k < 1 || k > ADAFUSE_MAX_TOP_K) return ADAFUSE_ERR_INVALID_ARG;
    return pregate_launch(ctx, h, T, d, Wr, k, 4, route, stream);
}

}  // extern "C"

namespace {

// One routing decision for the whole batch: the tokens' logits into the
// context's scratch (the per-token kernels, same arithmetic), then their
// mean and the token rule in one more launch.
int pregate_batch_launch(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d, const float* Wr,
                         int k, int slots, void* route_out, void* stream) {
    if (ctx == nullptr || T < 0 || T > kMaxBatchTokens) return ADAFUSE_ERR_INVALID_ARG;
    if (T == 0) return ADAFUSE_OK;
    if (route_out == nullptr || !aligned16(route_out)) return ADAFUSE_ERR_INVALID_ARG;
    const int rc = pregate_launch(ctx, h, T, d, Wr, k, slots, nullptr, stream, ctx->d_logits);
    if (rc != ADAFUSE_OK) return rc;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* route = static_cast<int32_t*>(route_out);
    const int E = ctx->n_experts;
    switch (E <= 8 ? 8 : E <= 16 ? 16 : E <= 32 ? 32 : 64) {
        case 8: pregate_batch_reduce_kernel<8><<<1, 64, 0, s>>>(ctx->d_logits, T, E, k, slots, route); break;
        case 16: pregate_batch_reduce_kernel<16><<<1, 64, 0, s>>>(ctx->d_logits, T, E, k, slots, route); break;
        case 32: pregate_batch_reduce_kernel<32><<<1, 64, 0, s>>>(ctx->d_logits, T, E, k, slots, route); break;
        default: pregate_batch_reduce_kernel<64><<<1, 64, 0, s>>>(ctx->d_logits, T, E, k, slots, route); break;
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "batch pregate launch");
}

}  // namespace

extern "C" {

int adafuse_pregate_batch(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                          const float* Wr, adafuse_route* route, void* stream) {
    return pregate_batch_launch(ctx, h, T, d, Wr, 2, 2, route, stream);
}

int adafuse_pregate_batch_topk(adafuse_ctx* ctx, const float* h, int64_t T, int64_t d,
                               const float* Wr, int32_t k, adafuse_route4* route,
                               void* stream) {
    if (k < 1 || k > ADAFUSE_MAX_TOP_K) return ADAFUSE_ERR_INVALID_ARG;
    return pregate_batch_launch(ctx, h, T, d, Wr, k, 4, route, stream);
}

}  // extern "C"

namespace {

// One switch launch over layers [layer_begin, layer_begin + n_layers): in
// place (prev, cur) or, with rebase, W <- rne(W0 + dW_cur).
int launch_switch(adafuse_ctx* ctx, int32_t layer_begin, int32_t n_layers,
                  const void* prev_route, const void* cur_route, int slots, void* stream,
                  bool rebase) {
    const int32_t* prev = static_cast<const int32_t*>(prev_route);
    const int32_t* cur = static_cast<const int32_t*>(cur_route);
    if (ctx == nullptr || n_layers < 0 || layer_begin < 0) return ADAFUSE_ERR_INVALID_ARG;
    if ((int64_t)layer_begin + n_layers > ctx->n_layers) return ADAFUSE_ERR_INVALID_ARG;
    if (!aligned16(prev) || !aligned16(cur)) return ADAFUSE_ERR_INVALID_ARG;
    if (n_layers == 0) return ADAFUSE_OK;
    const int64_t t0 = ctx->layer_tile_begin[(size_t)layer_begin];
    const int64_t t1 = ctx->layer_tile_begin[(size_t)layer_begin + n_layers];
    if (t1 <= t0) return ADAFUSE_OK;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int kind = slots == 4 && !rebase ? adafuse_get_topk_switch_kernel(ctx)
                                     : adafuse_get_switch_kernel(ctx);
    if (kind == ADAFUSE_KERNEL_TCGEN05_FOLD && ctx->d_fold == nullptr) {
        const int rc = ensure_fold(ctx, s);
        if (rc == ADAFUSE_ERR_OUT_OF_MEMORY && ctx->kernel == ADAFUSE_KERNEL_AUTO)
            kind = slots == 4 && !rebase ? adafuse_get_topk_switch_kernel(ctx)
                                         : adafuse_get_switch_kernel(ctx);  // AUTO falls back
        else if (rc != ADAFUSE_OK)
            return rc;
    }
    if (kind == ADAFUSE_KERNEL_TCGEN05_PAIR) {
        const int64_t b0 = ctx->layer_block_begin[(size_t)layer_begin];
        const int64_t b1 = ctx->layer_block_begin[(size_t)layer_begin + n_layers];
        cudaError_t e = cudaSuccess;
        if (ctx->tc_kp == 16)
            e = launch_tc2<16>(ctx, b0, b1, prev, cur, slots, s, rebase);
        else if (ctx->tc_kp == 32)
            e = launch_tc2<32>(ctx, b0, b1, prev, cur, slots, s, rebase);
        else
            e = launch_tc2<64>(ctx, b0, b1, prev, cur, slots, s, rebase);
        return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "switch launch");
    }
    if (kind == ADAFUSE_KERNEL_TCGEN05_FOLD) {
        // the folded kernel walks its tiles by a static stride
        const TcParams prm =
            tc_params(ctx, ctx->d_tiles, t0, t1, prev, cur, slots, rebase, false);
        const int64_t w0 = (int64_t)layer_begin * ctx->n_targets;
        const int64_t nw = (int64_t)n_layers * ctx->n_targets;
        const cudaError_t e =
            launch_switch_fold(prm, w0, nw, ctx->rank, ctx->device, switch_ctas(ctx), s);
        return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "switch launch");
    }
    if (kind == ADAFUSE_KERNEL_TCGEN05) {
        cudaError_t e = cudaSuccess;
        if (ctx->rank <= 8)
            e = launch_tc<16, true>(ctx, t0, t1, prev, cur, slots, s, rebase);
        else if (ctx->tc_kp == 16)
            e = launch_tc<16, false>(ctx, t0, t1, prev, cur, slots, s, rebase);
        else if (ctx->tc_kp == 32)
            e = launch_tc<32, false>(ctx, t0, t1, prev, cur, slots, s, rebase);
        else
            e = launch_tc<64, false>(ctx, t0, t1, prev, cur, slots, s, rebase);
        return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "switch launch");
    }
    const int64_t want = (int64_t)switch_ctas(ctx) * 2;
    const unsigned grid = (unsigned)(t1 - t0 < want ? t1 - t0 : want);
    const int E = ctx->n_experts, r = ctx->rank;
    const float sc = ctx->scale;
    const int rb = rebase ? 1 : 0;
    auto go = [&](auto kernel) {
        kernel<<<grid, kSwitchThreads, 0, s>>>(ctx->d_pairs, ctx->d_tiles, t0, t1, prev, cur, E, r,
                                               sc, ctx->d_status, rb);
    };
    const bool four = slots == 4;
    switch (kp_class(r)) {
        case 8: four ? go(switch_mma_kernel<8, 4>) : go(switch_mma_kernel<8, 2>); break;
        case 16: four ? go(switch_mma_kernel<16, 4>) : go(switch_mma_kernel<16, 2>); break;
        case 32: four ? go(switch_mma_kernel<32, 4>) : go(switch_mma_kernel<32, 2>); break;
        default: four ? go(switch_mma_kernel<64, 4>) : go(switch_mma_kernel<64, 2>); break;
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "switch launch");
}

}  // namespace

extern "C" {

int adafuse_switch_batch_layers(adafuse_ctx* ctx, int32_t layer_begin, int32_t n_layers,
                                const adafuse_route* prev, const adafuse_route* cur,
                                void* stream) {
    return launch_switch(ctx, layer_begin, n_layers, prev, cur, 2, stream, false);
}

int adafuse_set_base(adafuse_ctx* ctx, const void* const* W0) {
    if (ctx == nullptr || W0 == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    const size_t n = ctx->h_pairs.size();
    for (size_t i = 0; i < n; ++i)
        if (W0[i] == nullptr || !aligned16(W0[i]) || W0[i] == ctx->h_pairs[i].W)
            return ADAFUSE_ERR_INVALID_ARG;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    std::vector<PairDesc> pairs;
    std::vector<CUtensorMap> maps;
    try {
        pairs = ctx->h_pairs;
        if (ctx->tc_kp != 0) maps.resize(n);
    } catch (...) {
        return ADAFUSE_ERR_OUT_OF_MEMORY;
    }
    for (size_t i = 0; i < n; ++i) pairs[i].W0 = static_cast<const uint16_t*>(W0[i]);
    if (ctx->tc_kp != 0) {
        EncodeTiledFn enc = encode_tiled_fn();
        if (enc == nullptr) return ADAFUSE_ERR_CUDA;
        for (size_t i = 0; i < n; ++i) {
            if (!encode_w_map(enc, pairs[i].W0, pairs[i].out, pairs[i].in, ctx->blk, &maps[i]))
                return ADAFUSE_ERR_CUDA;
        }
    }
    // everything the kernels may still be reading is replaced only after the
    // device is idle with respect to this context's stream-ordered work
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    if (ctx->tc_kp != 0 && ctx->d_w0_maps == nullptr) {
        e = cudaMalloc(&ctx->d_w0_maps, sizeof(CUtensorMap) * n);
        if (e != cudaSuccess)
            return e == cudaErrorMemoryAllocation ? ADAFUSE_ERR_OUT_OF_MEMORY : cuda_fail(e, "cudaMalloc(w0 maps)");
    }
    if (ctx->tc_kp != 0) {
        e = cudaMemcpy(ctx->d_w0_maps, maps.data(), sizeof(CUtensorMap) * n, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(w0 maps)");
    }
    e = cudaMemcpy(ctx->d_pairs, pairs.data(), sizeof(PairDesc) * n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(pairs)");
    ctx->h_pairs.swap(pairs);
    ctx->has_base = true;
    return ADAFUSE_OK;
}

int adafuse_rebase_layers(adafuse_ctx* ctx, int32_t layer_begin, int32_t n_layers,
                          const adafuse_route* cur, void* stream) {
    if (ctx == nullptr || !ctx->has_base) return ADAFUSE_ERR_INVALID_ARG;
    return launch_switch(ctx, layer_begin, n_layers, nullptr, cur, 2, stream, true);
}

int adafuse_rebase(adafuse_ctx* ctx, const adafuse_route* cur, void* stream) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    return adafuse_rebase_layers(ctx, 0, ctx->n_layers, cur, stream);
}

int adafuse_switch(adafuse_ctx* ctx, const adafuse_route* prev, const adafuse_route* cur,
                   void* stream) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    return adafuse_switch_batch_layers(ctx, 0, ctx->n_layers, prev, cur, stream);
}

int adafuse_switch_topk_layers(adafuse_ctx* ctx, int32_t layer_begin, int32_t n_layers,
                               const adafuse_route4* prev, const adafuse_route4* cur,
                               void* stream) {
    return launch_switch(ctx, layer_begin, n_layers, prev, cur, 4, stream, false);
}

int adafuse_switch_topk(adafuse_ctx* ctx, const adafuse_route4* prev, const adafuse_route4* cur,
                        void* stream) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    return adafuse_switch_topk_layers(ctx, 0, ctx->n_layers, prev, cur, stream);
}

int adafuse_rebase_topk(adafuse_ctx* ctx, const adafuse_route4* cur, void* stream) {
    if (ctx == nullptr || !ctx->has_base) return ADAFUSE_ERR_INVALID_ARG;
    return launch_switch(ctx, 0, ctx->n_layers, nullptr, cur, 4, stream, true);
}

int adafuse_refresh_adapters(adafuse_ctx* ctx, void* stream) {
    if (ctx == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    if (ctx->d_bpad == nullptr) return ADAFUSE_OK;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    const cudaError_t e = copy_padded_b(ctx, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ADAFUSE_OK : cuda_fail(e, "cudaMemcpy2D(padded B)");
}

int adafuse_debug_stall_next_switch_at(adafuse_ctx* ctx, int32_t tile) {
    if (ctx == nullptr || tile < 1) return ADAFUSE_ERR_INVALID_ARG;
    if (adafuse_get_switch_kernel(ctx) == ADAFUSE_KERNEL_MMA_SYNC) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    ctx->stall_at = tile;
    return ADAFUSE_OK;
}

int adafuse_debug_stall_next_switch(adafuse_ctx* ctx) {
    return adafuse_debug_stall_next_switch_at(ctx, 1);
}

int adafuse_get_device_status(adafuse_ctx* ctx, void* stream, int32_t* status) {
    if (ctx == nullptr || status == nullptr) return ADAFUSE_ERR_INVALID_ARG;
    DeviceGuard guard(ctx->device);
    if (!guard.ok) return cuda_fail(cudaGetLastError(), "cudaSetDevice");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ctx->d_status, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->d_status, 0, sizeof v, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "device status read");
    *status = v;
    return v == 0 ? ADAFUSE_OK : ADAFUSE_ERR_DEVICE_FAULT;
}

}  // extern "C"

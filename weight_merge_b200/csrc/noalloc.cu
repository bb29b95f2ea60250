// noalloc.cu -- adafuse_switch_noalloc: the fused switch for callers that
// cannot allocate device memory.
//
// Why it exists: adafuse_create allocates (cudaMalloc) its segment table,
// weight descriptors and status word.  Some callers cannot do that -- for
// example a serving engine that has handed all free HBM to its own memory
// pool at start-up (a later cudaMalloc fails or fragments the pool), or a
// decode loop that must never hit cudaMalloc's implicit device
// synchronisation.  This entry point switches a model without a context and
// without any allocation: the only device memory it uses beyond the caller's
// buffers is one file-scope static array (kScratchBytes, below), which every
// GPU that loads the library holds until the process exits.
//
// Each call writes the per-weight table into that array through a few small
// launches that carry the entries as kernel arguments (no host staging
// buffer, no host-to-device copy), so every call shares the array: calls
// whose work overlaps on the GPU (different streams, or different host
// threads without ordering) race on it.  Calls on one stream are ordered and
// safe.  The first call on a device looks up the array's device address
// (cudaGetSymbolAddress) once for that device.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "adafuse.h"
#include "common.cuh"
#include "switch_mma.cuh"

namespace adafuse {
namespace noalloc {

// One (layer, target) weight plus where its tiles start in the tile index
// space (prefix sum of ceil(out/128) * ceil(in/128) over earlier weights).
struct Entry {
    uint16_t* W;
    const uint16_t* A;
    const uint16_t* B;
    int32_t out;
    int32_t in;
    int64_t tile_begin;
};

constexpr size_t kScratchBytes = 64 * 1024;                    // 64 KiB per GPU
constexpr int kMaxWeights = (int)(kScratchBytes / sizeof(Entry));  // 1638 weights
constexpr int kMaxDevices = 64;

// The scratch: a table of kMaxWeights entries.  Host code must not pass this
// symbol to a kernel (on the host it names a stand-in, not device memory);
// the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Binary search: the weight whose tile range holds global tile `t`.
__device__ __forceinline__ int find_weight(const Entry* tab, int n, int64_t t) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ TileCoord tile_of(const Entry* tab, int w, int64_t t) {
    const Entry& en = tab[w];
    const int64_t local = t - en.tile_begin;
    const int64_t ct = (en.in + kTile - 1) / kTile;
    TileCoord tc;
    tc.W = en.W;
    tc.Wsrc = en.W;
    tc.A = en.A;
    tc.B = en.B;
    tc.out = en.out;
    tc.in = en.in;
    tc.row0 = (int)(local / ct) * kTile;
    tc.col0 = (int)(local % ct) * kTile;
    return tc;
}

// The register-streaming mma.sync switch (see switch_mma.cuh for the layout
// and the A-column permutation), with tiles decoded from the scratch table
// instead of a per-context tile list.
template <int KP>
__global__ void __launch_bounds__(kSwitchThreads, 2)
switch_noalloc_kernel(const Entry* __restrict__ tab, int n_weights, int64_t n_tiles,
                      const adafuse_route* prev, const adafuse_route* cur, int E, int r, float s,
                      int32_t* status) {
    Coefs cf;
    const int st = build_coefs(prev, cur, E, s, cf);
    if (st != 0) {
        if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, st);
        return;
    }
    if (cf.n == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sel = (g & 1) ? 0x7632u : 0x5410u;
    const bool r_even = (r & 1) == 0;

    int64_t tile = blockIdx.x;
    if (tile >= n_tiles) return;
    int wi = find_weight(tab, n_weights, tile);
    TileCoord tc = tile_of(tab, wi, tile);

    uint4 wv[4][2];
#pragma unroll
    for (int cg = 0; cg < 4; ++cg)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int row = tc.row0 + 16 * warp + g + 8 * hh;
            const int col = tc.col0 + 32 * cg + 8 * t;
            wv[cg][hh] = (row < tc.out && col < tc.in)
                             ? ld_stream_16(tc.W + (int64_t)row * tc.in + col)
                             : make_uint4(0u, 0u, 0u, 0u);
        }

    for (;;) {
        const int64_t next = tile + gridDim.x;
        const bool has_next = next < n_tiles;
        TileCoord tn = tc;
        if (has_next) {
            while (wi + 1 < n_weights && tab[wi + 1].tile_begin <= next) ++wi;
            tn = tile_of(tab, wi, next);
        }

        const int rowA = tc.row0 + 16 * warp + g;
        const bool okA0 = rowA < tc.out, okA1 = rowA + 8 < tc.out;

#pragma unroll
        for (int cg = 0; cg < 4; ++cg) {
            const int colc = tc.col0 + 32 * cg + 8 * (g >> 1);
            const bool col_ok = colc < tc.in;
            float tot[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) tot[j][q] = 0.f;

#pragma unroll
            for (int ei = 0; ei < 4; ++ei) {
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
                if (has_next) {
                    const int nrow = tn.row0 + 16 * warp + g + 8 * hh;
                    const int ncol = tn.col0 + 32 * cg + 8 * t;
                    wv[cg][hh] = (nrow < tn.out && ncol < tn.in)
                                     ? ld_stream_16(tn.W + (int64_t)nrow * tn.in + ncol)
                                     : make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        if (!has_next) break;
        tile = next;
        tc = tn;
    }
}

// The table is written on the device by small launches whose arguments carry
// up to kFillChunk entries each (3.8 KB of a launch's 4 KB argument space).
constexpr int kFillChunk = 96;
struct EntryChunk {
    Entry e[kFillChunk];
};
static_assert(sizeof(EntryChunk) + 16 <= 4096, "kernel argument space");

__global__ void fill_table_kernel(Entry* tab, const EntryChunk chunk, int first, int count) {
    const int i = threadIdx.x;
    if (i < count) tab[first + i] = chunk.e[i];
}

// Per-device set-up (the scratch's device address), guarded by g_mu; the
// mutex is held only while a device is set up, never across GPU work.
std::mutex g_mu;
void* g_scratch_dev[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

// Once per device, with that device current: the scratch's device address.
int setup_device(int dev, void** scratch, int* sms) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_scratch_dev[dev] == nullptr) {
        int major = 0, minor = 0, count = 0;
        cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
        if (major != 10 || minor != 0) return ADAFUSE_ERR_UNSUPPORTED_DEVICE;
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
        g_sm_count[dev] = count;
        g_scratch_dev[dev] = p;
    }
    *scratch = g_scratch_dev[dev];
    *sms = g_sm_count[dev];
    return ADAFUSE_OK;
}

}  // namespace noalloc
}  // namespace adafuse

using namespace adafuse;
using namespace adafuse::noalloc;

extern "C" int adafuse_switch_noalloc(const adafuse_desc* desc, const adafuse_route* prev,
                                      const adafuse_route* cur, int32_t* status, void* stream) {
    if (desc == nullptr || desc->targets == nullptr || desc->n_layers < 1 || desc->n_targets < 1)
        return ADAFUSE_ERR_INVALID_ARG;
    if (desc->n_experts < 1 || desc->n_experts > 64 || desc->rank < 1 || desc->rank > 64)
        return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
    if (!std::isfinite(desc->alpha)) return ADAFUSE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(prev) & 15u) || (reinterpret_cast<uintptr_t>(cur) & 15u) ||
        (reinterpret_cast<uintptr_t>(status) & 3u))
        return ADAFUSE_ERR_INVALID_ARG;
    const int64_t n = (int64_t)desc->n_layers * desc->n_targets;
    static_assert(kMaxWeights == ADAFUSE_NOALLOC_MAX_WEIGHTS, "header limit");
    static_assert(kScratchBytes == ADAFUSE_NOALLOC_SCRATCH_BYTES, "header size");
    if (n > kMaxWeights) return ADAFUSE_ERR_UNSUPPORTED_SHAPE;  // more than the scratch holds
    // every argument is checked before anything is enqueued
    int64_t tiles = 0;
    for (int64_t i = 0; i < n; ++i) {
        const adafuse_target& t = desc->targets[i];
        if (t.out <= 0 || t.in <= 0) return ADAFUSE_ERR_INVALID_ARG;
        if (t.out % 8 != 0 || t.in % 8 != 0 || t.out > INT32_MAX || t.in > INT32_MAX)
            return ADAFUSE_ERR_UNSUPPORTED_SHAPE;
        if (t.W == nullptr || t.A == nullptr || t.B == nullptr) return ADAFUSE_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(t.W) | reinterpret_cast<uintptr_t>(t.A) |
             reinterpret_cast<uintptr_t>(t.B)) & 15u)
            return ADAFUSE_ERR_INVALID_ARG;
        tiles += ((t.out + kTile - 1) / kTile) * ((t.in + kTile - 1) / kTile);
    }

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ADAFUSE_ERR_UNSUPPORTED_DEVICE;
    void* scratch = nullptr;
    int sms = 0;
    int rc = setup_device(dev, &scratch, &sms);
    if (rc != ADAFUSE_OK) return rc;
    Entry* tab = static_cast<Entry*>(scratch);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the table is rewritten in full by every call, in stream order before
    // the switch launch; the status output starts at zero
    EntryChunk chunk;
    int64_t begin = 0;
    for (int64_t i0 = 0; i0 < n; i0 += kFillChunk) {
        const int cnt = (int)(n - i0 < kFillChunk ? n - i0 : kFillChunk);
        for (int j = 0; j < cnt; ++j) {
            const adafuse_target& t = desc->targets[i0 + j];
            Entry& en = chunk.e[j];
            en.W = static_cast<uint16_t*>(t.W);
            en.A = static_cast<const uint16_t*>(t.A);
            en.B = static_cast<const uint16_t*>(t.B);
            en.out = (int32_t)t.out;
            en.in = (int32_t)t.in;
            en.tile_begin = begin;
            begin += ((t.out + kTile - 1) / kTile) * ((t.in + kTile - 1) / kTile);
        }
        fill_table_kernel<<<1, kFillChunk, 0, s>>>(tab, chunk, (int)i0, cnt);
        e = cudaGetLastError();
        if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
    }
    if (status != nullptr) {
        e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
        if (e != cudaSuccess) return ADAFUSE_ERR_CUDA;
    }
    if (tiles == 0) return ADAFUSE_OK;
    const int64_t want = (int64_t)sms * 2;
    const unsigned grid = (unsigned)(tiles < want ? tiles : want);
    const int E = desc->n_experts, r = desc->rank;
    const float sc = desc->alpha / (float)desc->rank;
    const int nw = (int)n;
    if (r <= 8)
        switch_noalloc_kernel<8><<<grid, kSwitchThreads, 0, s>>>(tab, nw, tiles, prev, cur, E, r, sc, status);
    else if (r <= 16)
        switch_noalloc_kernel<16><<<grid, kSwitchThreads, 0, s>>>(tab, nw, tiles, prev, cur, E, r, sc, status);
    else if (r <= 32)
        switch_noalloc_kernel<32><<<grid, kSwitchThreads, 0, s>>>(tab, nw, tiles, prev, cur, E, r, sc, status);
    else
        switch_noalloc_kernel<64><<<grid, kSwitchThreads, 0, s>>>(tab, nw, tiles, prev, cur, E, r, sc, status);
    e = cudaGetLastError();
    return e == cudaSuccess ? ADAFUSE_OK : ADAFUSE_ERR_CUDA;
}

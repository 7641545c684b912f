// fp8bq_api.cu -- the C ABI of the blockwise FP8 weight quantizer: argument
// checks, the choice of kernel variant per tensor, grouping into launches,
// tensor-map encoding for the TMA variant, and status reporting.
//
// The entry points follow scaled_fp8_blockwise(data_hp, weight_block_size)
// (verl docs "fp8_kernel.py -- FP8 量化内核", section 1 "统一入口") and the
// per-layer quant_weights stream ("vllm_fp8_utils.py" docs, section 3
// "权重量化").  The pages launch one kernel per tensor; here a whole list of
// tensors becomes one persistent launch per kernel variant.
#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/fp8bq.h"
#include "fp8bq_internal.h"

using namespace fp8bq;

namespace {

std::atomic<int> g_path{FP8BQ_PATH_AUTO};
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<uint32_t> g_inject{0};
std::atomic<int> g_pdl{1};

int esize_of(int32_t dtype) { return dtype == FP8BQ_BF16 ? 2 : 4; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

// ------------------------------------------------------------------ checks

fp8bq_status check_desc(const fp8bq_desc &D, bool *empty) {
    if (D.dtype_in != FP8BQ_BF16 && D.dtype_in != FP8BQ_F32) return FP8BQ_ERR_DTYPE;
    if (D.block_m < 1 || D.block_n < 1 || (int64_t)D.block_m * D.block_n > 65536)
        return FP8BQ_ERR_BLOCK;
    if (D.M < 0 || D.N < 0 || D.batch < 0 || D.ld < D.N || D.ld < 0) return FP8BQ_ERR_SHAPE;
    if (D.M >= (1ll << 31) || D.N >= (1ll << 31)) return FP8BQ_ERR_SHAPE;
    *empty = D.M == 0 || D.N == 0 || D.batch == 0;
    if (*empty) return FP8BQ_OK;
    if (D.batch > 1 && (D.x_batch_stride < 0 || D.y_batch_stride < 0 || D.s_batch_stride < 0))
        return FP8BQ_ERR_SHAPE;
    const int64_t tiles = D.batch * cdiv(D.M, D.block_m) * cdiv(D.N, D.block_n);
    if (tiles >= (1ll << 31)) return FP8BQ_ERR_SHAPE;
    if (D.x == nullptr || D.y_u8 == nullptr || D.descale_f32 == nullptr) return FP8BQ_ERR_NULL;
    const int es = esize_of(D.dtype_in);
    if (((uintptr_t)D.x % es) != 0 || ((uintptr_t)D.descale_f32 % 4) != 0) return FP8BQ_ERR_ALIGN;
    // every byte offset the kernels form must fit comfortably in 64 bits
    const int64_t gm = cdiv(D.M, D.block_m), gn = cdiv(D.N, D.block_n);
    const __int128 b1 = D.batch - 1, lim = (__int128)1 << 62;
    const bool multi = D.batch > 1;
    if ((b1 * (multi ? D.x_batch_stride : 0) + (__int128)(D.M - 1) * D.ld + D.N) * es > lim ||
        b1 * (multi ? D.y_batch_stride : 0) + (__int128)D.M * D.N > lim ||
        (b1 * (multi ? D.s_batch_stride : 0) + (__int128)gm * gn) * 4 > lim)
        return FP8BQ_ERR_SHAPE;
    if (multi && (D.y_batch_stride < D.M * D.N || D.s_batch_stride < gm * gn))
        return FP8BQ_ERR_OVERLAP;
    return FP8BQ_OK;
}

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
    bool out;
};

// Byte ranges each argument spans.  Outputs may overlap nothing; inputs may
// overlap each other.
fp8bq_status check_overlap(const fp8bq_desc *t, int n, const std::vector<char> &empty) {
    std::vector<Span> sp;
    sp.reserve((size_t)n * 3);
    for (int i = 0; i < n; ++i) {
        if (empty[i]) continue;
        const fp8bq_desc &D = t[i];
        const int64_t es = esize_of(D.dtype_in);
        const int64_t b1 = D.batch - 1;
        const int64_t gm = cdiv(D.M, D.block_m), gn = cdiv(D.N, D.block_n);
        const int64_t xe = (b1 * (D.batch > 1 ? D.x_batch_stride : 0) + (D.M - 1) * D.ld + D.N) * es;
        const int64_t ye = b1 * (D.batch > 1 ? D.y_batch_stride : 0) + D.M * D.N;
        const int64_t se = (b1 * (D.batch > 1 ? D.s_batch_stride : 0) + gm * gn) * 4;
        sp.push_back({(uintptr_t)D.x, (uintptr_t)D.x + (uintptr_t)xe, false});
        sp.push_back({(uintptr_t)D.y_u8, (uintptr_t)D.y_u8 + (uintptr_t)ye, true});
        sp.push_back({(uintptr_t)D.descale_f32, (uintptr_t)D.descale_f32 + (uintptr_t)se, true});
    }
    std::sort(sp.begin(), sp.end(), [](const Span &a, const Span &b) { return a.lo < b.lo; });
    // Sweep: track the furthest end of any output and of any input seen so far.
    uintptr_t out_end = 0, in_end = 0;
    for (const Span &s : sp) {
        if (s.out) {
            if (s.lo < out_end || s.lo < in_end) return FP8BQ_ERR_OVERLAP;
            out_end = std::max(out_end, s.hi);
        } else {
            if (s.lo < out_end) return FP8BQ_ERR_OVERLAP;
            in_end = std::max(in_end, s.hi);
        }
    }
    return FP8BQ_OK;
}

// ------------------------------------------------------------------ device

fp8bq_status check_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return FP8BQ_ERR_DEVICE;
    }
    static std::atomic<int> ok_cache[64];  // 0 unknown, 1 ok, 2 not usable
    if (dev < 64) {
        const int c = ok_cache[dev].load();
        if (c) return c == 1 ? FP8BQ_OK : FP8BQ_ERR_DEVICE;
    }
    int major = 0, minor = 0;
    bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
              cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
              major == 10 && minor == 0;
    if (!ok) cudaGetLastError();
    if (dev < 64) ok_cache[dev].store(ok ? 1 : 2);
    return ok ? FP8BQ_OK : FP8BQ_ERR_DEVICE;
}

// ------------------------------------------------------------------ variants

bool vector_fits(const fp8bq_desc &D, Variant v) {
    const int es = esize_of(D.dtype_in), vec = 16 / es;
    const int team = kVecTeamThreads(v, es), slots = kVecSlots(v);
    if (D.block_n % vec) return false;
    const int vpr = D.block_n / vec;
    if (!is_pow2(vpr) || vpr > team) return false;
    if (v == Variant::VecT16 || v == Variant::VecT32)
        return (int64_t)D.block_m * vpr == team;  // one row-step per block
    return cdiv(D.block_m, team / vpr) <= slots;
}

// Alignment that lets whole 16-byte input vectors and whole output vectors
// (vec bytes of e4m3 codes) be moved without straddling a row end.
bool vector_aligned(const fp8bq_desc &D) {
    const int es = esize_of(D.dtype_in), vec = 16 / es;
    if ((uintptr_t)D.x % 16 || (D.ld * es) % 16 || D.N % vec) return false;
    if ((uintptr_t)D.y_u8 % vec) return false;
    if (D.batch > 1 && ((D.x_batch_stride * es) % 16 || D.y_batch_stride % vec)) return false;
    return true;
}

// The weaker alignment of the vector kernel's HALVES mode: 8-byte input rows
// and output pieces of half a vector (4 codes for bf16, 2 for fp32), so every
// row holds a whole number of 8-byte input halves (bf16 rows of 4100
// elements, say).
bool halves_aligned(const fp8bq_desc &D) {
    const int es = esize_of(D.dtype_in), half = 8 / es;
    if ((uintptr_t)D.x % 8 || (D.ld * es) % 8 || D.N % half) return false;
    if ((uintptr_t)D.y_u8 % half) return false;
    if (D.batch > 1 && ((D.x_batch_stride * es) % 8 || D.y_batch_stride % half)) return false;
    return true;
}

Variant vector_variant(const fp8bq_desc &D) {
    for (Variant v : {Variant::VecT16, Variant::VecT32, Variant::VecT64, Variant::VecT128,
                      Variant::VecTBig})
        if (vector_fits(D, v)) return v;
    return Variant::Generic;
}

// Geometry of the TMA kernel for a tensor: a ring slot (one tile) holds
// `group` vertically stacked blocks, at most 256 rows and 128x128 elements;
// consumer thread ct holds rows ct / vpr + i * rs (rs = 256 / vpr).  Either
// a block is a whole number of row-steps (reduced across the CTA) or it is
// a power-of-two group of at most 32 lanes within one row-step (reduced with
// shuffles, `subwarp`).  Returns false if neither holds.
bool tma_geom(const fp8bq_desc &D, int *group, bool *subwarp) {
    const int es = esize_of(D.dtype_in), vec = 16 / es;
    if (D.block_n > 256 || (D.block_n * es) % 16) return false;
    const int vpr = D.block_n / vec;
    if (!is_pow2(vpr) || vpr > kTmaConsumerThreads) return false;
    const int rs = kTmaConsumerThreads / vpr;
    const int slots = 128 * 128 * es / 16 / kTmaConsumerThreads;
    const int max_rows = std::min(256, 128 * 128 / D.block_n);
    if (D.block_m > max_rows) return false;
    if (D.batch > 1 && D.x_batch_stride == 0) return false;
    if (!vector_aligned(D)) return false;
    if (D.block_m % rs == 0) {
        const int spb = D.block_m / rs;
        if (spb > slots) return false;
        *group = std::min(max_rows / D.block_m, slots / spb);
        *subwarp = false;
        return *group >= 1;
    }
    const int64_t lanes = (int64_t)D.block_m * vpr;
    if (lanes <= 32 && is_pow2(lanes) && rs % D.block_m == 0) {
        *group = max_rows / D.block_m;
        *subwarp = true;
        return *group >= 1;
    }
    return false;
}

// AUTO: the TMA ring when one block fills a ring slot of at least 16 KB
// (measured: with stacked small blocks the ring's 8 consumer warps spend too
// long per tile, and the team-per-tile vector kernel is 2-2.5x faster), the
// vector kernel for other 16- or 8-byte-aligned tensors, the generic kernel
// otherwise.
constexpr int64_t kTmaMinSlotBytes = 16384;

// A call whose TMA tensors hold less input than this runs them on the vector
// kernel instead.  Measured on B200, one bf16 tensor with 128x128 blocks per
// call (TMA / vector): 4096x4096 (33 MB of input) 0.783 / 0.848 of the copy
// peak, 4096x12288 and 12345x4096 (101 MB) 0.890-0.893 / 0.954-0.961,
// 24576x4096 (201 MB) 0.946 / 0.915, 49152x4096 (403 MB) 0.978 / 0.865; one
// Qwen3-8B-shaped layer (7 tensors, 386 MB) 0.987 / 0.879.
constexpr uint64_t kTmaMinCallBytes = 128ull << 20;

Variant choose(const fp8bq_desc &D, int path) {
    if (path == FP8BQ_PATH_GENERIC) return Variant::Generic;
    int g;
    bool sub;
    const bool tma = tma_geom(D, &g, &sub);
    if (path == FP8BQ_PATH_TMA && tma) return Variant::Tma;
    if (path == FP8BQ_PATH_AUTO && tma && g == 1 &&
        (int64_t)D.block_m * D.block_n * esize_of(D.dtype_in) >= kTmaMinSlotBytes)
        return Variant::Tma;
    if (!vector_aligned(D) && !halves_aligned(D)) return Variant::Generic;
    return vector_variant(D);
}

// Two horizontally adjacent 128x128 bf16 blocks per TMA ring slot (each tile
// row is then 512 contiguous bytes).  Measured on the whole Qwen3-8B-shaped
// weight set: 6.44-6.47 TB/s with 2 slots of 64 KB, against 6.08-6.17 TB/s
// for one block per 32 KB slot (4 slots) and 5.66 TB/s for 3 paired slots.
#ifndef FP8BQ_TMA_PAIR
#define FP8BQ_TMA_PAIR 1
#endif

bool tma_paired(const fp8bq_desc &D) {
    return FP8BQ_TMA_PAIR && D.dtype_in == FP8BQ_BF16 && D.block_m == 128 && D.block_n == 128;
}

// ------------------------------------------------------------------ tensor maps

// L2 promotion of the TMA tile loads (CUtensorMapL2promotion: 0 none, 1 64 B,
// 2 128 B, 3 256 B); a block row is 256 bytes of bf16 (512 in a paired tile).
#ifndef FP8BQ_TMA_L2_PROMOTION
#define FP8BQ_TMA_L2_PROMOTION 3
#endif

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

struct MapKey {
    uintptr_t x;
    int64_t M, N, ld, batch, xbs;
    int32_t dtype, bm, bn;
    bool operator==(const MapKey &o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
    size_t operator()(const MapKey &k) const {
        const uint64_t *w = reinterpret_cast<const uint64_t *>(&k);
        uint64_t h = 1469598103934665603ull;
        for (size_t i = 0; i < sizeof(MapKey) / 8; ++i) h = (h ^ w[i]) * 1099511628211ull;
        return (size_t)h;
    }
};

// Encoded maps are cached by (pointer, shape, strides, block): a trainer's
// weight buffers are the same on every sync step, so steady state encodes
// nothing.
bool encode_map(const fp8bq_desc &D, CUtensorMap *out) {
    static std::mutex mu;
    static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
    MapKey key;
    std::memset(&key, 0, sizeof key);
    key.x = (uintptr_t)D.x;
    key.M = D.M;
    key.N = D.N;
    key.ld = D.ld;
    key.batch = D.batch;
    key.xbs = D.batch > 1 ? D.x_batch_stride : D.M * D.ld;
    key.dtype = D.dtype_in;
    key.bm = D.block_m;
    key.bn = D.block_n;
    {
        std::lock_guard<std::mutex> g(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *out = it->second;
            return true;
        }
    }
    auto fn = encode_fn();
    if (!fn) return false;
    const int es = esize_of(D.dtype_in);
    cuuint64_t dims[3] = {(cuuint64_t)D.N, (cuuint64_t)D.M, (cuuint64_t)D.batch};
    cuuint64_t strides[2] = {(cuuint64_t)(D.ld * es), (cuuint64_t)(key.xbs * es)};
    int group = 1;
    bool sub = false;
    if (!tma_geom(D, &group, &sub)) return false;
    const int pair = tma_paired(D) ? 2 : 1;
    cuuint32_t box[3] = {(cuuint32_t)(pair * D.block_n), (cuuint32_t)(group * D.block_m), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap m;
    CUresult r = fn(&m,
                    D.dtype_in == FP8BQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    3, const_cast<void *>(D.x), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    (CUtensorMapL2promotion)FP8BQ_TMA_L2_PROMOTION, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> g(mu);
    if (cache.size() > 8192) cache.clear();
    cache.emplace(key, m);
    *out = m;
    return true;
}

// ------------------------------------------------------------------ launches

// Blocks stacked along M in one tile of variant v.
int tile_group(const fp8bq_desc &D, Variant v) {
    if (v == Variant::Tma) {
        int g = 1;
        bool sub = false;
        tma_geom(D, &g, &sub);
        return g;
    }
    return kTileBlocksM(v);
}

uint64_t tiles_of(const fp8bq_desc &D, Variant v) {
    const int64_t h = v == Variant::Tma && tma_paired(D) ? 2 : 1;  // blocks side by side
    return (uint64_t)D.batch * cdiv(cdiv(D.M, D.block_m), tile_group(D, v)) *
           cdiv(cdiv(D.N, D.block_n), h);
}

// The extent the bounds checks of a checked build take for an output of
// `bytes` bytes: one byte short under FP8BQ_INJECT_TRIM_OUTPUTS.
[[maybe_unused]] uint64_t checked_out_extent(uint64_t bytes) {
    return (g_inject.load() & FP8BQ_INJECT_TRIM_OUTPUTS) && bytes ? bytes - 1 : bytes;
}

void fill_tile_desc(const fp8bq_desc &D, Variant v, uint32_t begin, TileDesc *o) {
    o->x = D.x;
    o->y = D.y_u8;
    o->s = D.descale_f32;
    o->ld = D.ld;
    o->xbs = D.batch > 1 ? D.x_batch_stride : 0;
    o->ybs = D.batch > 1 ? D.y_batch_stride : 0;
    o->sbs = D.batch > 1 ? D.s_batch_stride : 0;
    o->M = (int32_t)D.M;
    o->N = (int32_t)D.N;
    o->bm = D.block_m;
    o->bn = D.block_n;
    o->gm = (int32_t)cdiv(D.M, D.block_m);
    o->gn = (int32_t)cdiv(D.N, D.block_n);
    o->tile_begin = begin;
    o->tiles = (uint32_t)tiles_of(D, v);
#if FP8BQ_CHECKED
    const int64_t b1 = D.batch - 1;
    o->x_bytes = (uint64_t)((b1 * o->xbs + (D.M - 1) * D.ld + D.N) * esize_of(D.dtype_in));
    o->y_bytes = checked_out_extent((uint64_t)(b1 * o->ybs + D.M * D.N));
    o->s_bytes = checked_out_extent((uint64_t)((b1 * o->sbs + (int64_t)o->gm * o->gn) * 4));
#endif
}

template <int MAXD>
void pack_header(DescPack<MAXD> &p) {
    p.n = 0;
    p.total_tiles = 0;
    p.inject = g_inject.load();
    p.group = 1;
    p.wait_limit_ns = g_wait_limit_ns.load();
}

// Launch one group (same variant, dtype and, for vector/TMA, block shape) in
// chunks that fit the parameter pack and keep the tile count below 2^31.
template <int MAXD>
cudaError_t launch_group(Variant v, int es, bool halves, const fp8bq_desc *t,
                         const std::vector<int> &idx, cudaStream_t st) {
    static thread_local DescPack<MAXD> p;  // large: keep it off the stack
    size_t i = 0;
    while (i < idx.size()) {
        pack_header(p);
        while (i < idx.size() && p.n < MAXD) {
            const fp8bq_desc &D = t[idx[i]];
            const uint64_t tiles = tiles_of(D, v);
            if (p.n > 0 && (uint64_t)p.total_tiles + tiles >= (1ull << 31)) break;
            fill_tile_desc(D, v, p.total_tiles, &p.d[p.n]);
            p.total_tiles += (uint32_t)tiles;
            ++p.n;
            ++i;
        }
        const cudaError_t e = v == Variant::Generic ? launch_generic<MAXD>(es, p, st)
                                                    : launch_vector<MAXD>(v, es, halves, p, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int MAXD>
cudaError_t launch_tma_group(int es, const fp8bq_desc *t, const std::vector<int> &idx,
                             const std::vector<CUtensorMap> &maps, cudaStream_t st) {
    static thread_local TmaPack<MAXD> P;  // large: keep it off the stack
    size_t i = 0;
    while (i < idx.size()) {
        pack_header(P.p);
        P.evict_first = 0;
        while (i < idx.size() && P.p.n < MAXD) {
            const fp8bq_desc &D = t[idx[i]];
            const uint64_t tiles = tiles_of(D, Variant::Tma);
            if (P.p.n > 0 && (uint64_t)P.p.total_tiles + tiles >= (1ull << 31)) break;
            fill_tile_desc(D, Variant::Tma, P.p.total_tiles, &P.p.d[P.p.n]);
            P.maps[P.p.n] = maps[i];
            const uint64_t in_bytes = (uint64_t)D.batch * (uint64_t)D.M * (uint64_t)D.N * es;
            if (in_bytes >= kEvictFirstMinBytes) P.evict_first = 1;
            P.p.total_tiles += (uint32_t)tiles;
            ++P.p.n;
            ++i;
        }
        int group = 1;
        bool sub = false;
        tma_geom(t[idx[0]], &group, &sub);  // the same for every tensor of the group
        P.p.group = group;
        const cudaError_t e = tma_paired(t[idx[0]]) ? launch_tma_pair<MAXD>(P, st)
                                                    : launch_tma<MAXD>(es, sub, P, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// ------------------------------------------------------------------ concurrent groups
//
// The launch groups of one call (one per kernel variant, dtype and block
// shape) touch disjoint outputs and only read their inputs, so they may run
// side by side: the first group runs on the caller's stream, the others on
// library streams that wait for the caller's stream first, and the caller's
// stream waits for all of them before anything it enqueues later.  Then one
// variant's ramp-up and last partial wave overlap another's work instead of
// adding up.  The streams and events are made once per device and kept (they
// are not device memory); the fork and join are events, so the call behaves
// like any sequence of launches on the caller's stream.  A call on a stream
// that is capturing a CUDA graph launches all its groups on that stream (a
// library stream forked into one caller's capture would take in another
// thread's launches until that capture ends).
#ifndef FP8BQ_GROUP_STREAMS
#define FP8BQ_GROUP_STREAMS 1
#endif
constexpr int kForkStreams = 4;

struct Fork {
    std::mutex mu;                          // one fork/join at a time per device
    bool ok = false;
    cudaStream_t s[kForkStreams] = {};
    cudaEvent_t start = nullptr, done[kForkStreams] = {};
};

Fork *fork_of_device() {
    static PerDevice<Fork *> forks;
    return forks.get([] {
        Fork *f = new Fork;
        f->ok = cudaEventCreateWithFlags(&f->start, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; f->ok && i < kForkStreams; ++i)
            f->ok = cudaStreamCreateWithFlags(&f->s[i], cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&f->done[i], cudaEventDisableTiming) == cudaSuccess;
        if (!f->ok) cudaGetLastError();
        return f;
    });
}

// Launch groups 0..n-1 (launch(g, stream)); several groups run concurrently.
template <typename L>
fp8bq_status run_groups(size_t n, L &&launch, cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (n > 1 && cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        cudaGetLastError();
        cs = cudaStreamCaptureStatusActive;  // unknown: do not fork
    }
    Fork *f = FP8BQ_GROUP_STREAMS && n > 1 && cs == cudaStreamCaptureStatusNone
                  ? fork_of_device()
                  : nullptr;
    if (f == nullptr || !f->ok) {
        for (size_t g = 0; g < n; ++g)
            if (launch(g, stream) != cudaSuccess) return FP8BQ_ERR_DEVICE;
        return FP8BQ_OK;
    }
    std::lock_guard<std::mutex> lock(f->mu);
    bool ok = cudaEventRecord(f->start, stream) == cudaSuccess;
    const int aux = (int)std::min<size_t>(n - 1, kForkStreams);
    for (int i = 0; ok && i < aux; ++i) ok = cudaStreamWaitEvent(f->s[i], f->start, 0) == cudaSuccess;
    if (!ok) {  // nothing forked: run everything on the caller's stream
        cudaGetLastError();
        for (size_t g = 0; g < n; ++g)
            if (launch(g, stream) != cudaSuccess) return FP8BQ_ERR_DEVICE;
        return FP8BQ_OK;
    }
    for (size_t g = 0; g < n; ++g)  // group g on stream g % (aux + 1); 0 = the caller's
        if (launch(g, g % (aux + 1) == 0 ? stream : f->s[g % (aux + 1) - 1]) != cudaSuccess)
            ok = false;
    // join every forked stream, whatever happened above
    for (int i = 0; i < aux; ++i)
        if (cudaEventRecord(f->done[i], f->s[i]) != cudaSuccess ||
            cudaStreamWaitEvent(stream, f->done[i], 0) != cudaSuccess)
            ok = false;
    if (!ok) cudaGetLastError();
    return ok ? FP8BQ_OK : FP8BQ_ERR_DEVICE;
}

struct GroupKey {
    Variant v;
    int es, bm, bn;
    bool halves;
    bool operator==(const GroupKey &o) const {
        return v == o.v && es == o.es && bm == o.bm && bn == o.bn && halves == o.halves;
    }
};

// The launches of one call: its tensors grouped by kernel variant (the
// caller's order kept inside a group), with the TMA groups' tensor maps.
// The same quantization on a geometry the kernels run better, for tensors of
// at least kReshapeMinBytes of input with few rows (the result is identical
// byte for byte; only the kernel's view changes):
//  * a tensor of one block row (M <= block_m / 4) takes blocks of M rows: a
//    block's absmax already covers only its M valid rows, and the descale
//    grid (1 x gn) and code layout are unchanged;
//  * row-wise blocks (block_m == 1) on fewer than kFoldRows contiguous rows
//    (ld == N, N a multiple of block_n, one matrix) are refolded as k times
//    more rows of N / k elements: every block keeps its elements, and both
//    the codes and the descales keep their row-major order (block (r, j)
//    becomes block (r k + j / (gn / k), j % (gn / k)), the same linear index).
// Measured on B200 before this (bf16, one 2^27-element row): 1 x 128 blocks
// 1.1 TB/s on the vector kernel (seven of the eight rows of its stacked tile
// empty), 128 x 128 blocks 0.09 TB/s (one valid row in 128).
constexpr uint64_t kReshapeMinBytes = 4ull << 20;
constexpr int64_t kFoldRows = 256;

fp8bq_desc reshaped(const fp8bq_desc &D) {
    fp8bq_desc o = D;
    if ((uint64_t)D.batch * (uint64_t)D.M * (uint64_t)D.N * esize_of(D.dtype_in) < kReshapeMinBytes)
        return o;
    if (o.M <= o.block_m / 4) o.block_m = (int32_t)o.M;
    if (o.block_m == 1 && o.batch == 1 && o.ld == o.N && o.M < kFoldRows && o.N % o.block_n == 0) {
        const int64_t gn = o.N / o.block_n;
        const int64_t es = esize_of(o.dtype_in);
        int64_t k = 1;
        // folded rows stay a whole number of 16-byte vectors if the rows were
        while (o.M * k < kFoldRows && gn % (2 * k) == 0 &&
               ((o.N * es) % 16 != 0 || (o.N / (2 * k) * es) % 16 == 0))
            k *= 2;
        o.M *= k;
        o.N /= k;
        o.ld = o.N;
    }
    return o;
}

struct Plan {
    std::vector<fp8bq_desc> descs;  // reshaped() of each tensor of the call
    std::vector<GroupKey> keys;
    std::vector<std::vector<int>> members;
    std::vector<std::vector<CUtensorMap>> maps;
};

// Check every descriptor, then group them.  FP8BQ_OK with an empty plan when
// there is nothing to do.
fp8bq_status make_plan(const fp8bq_desc *table, int n, Plan &plan) {
    if (n < 0) return FP8BQ_ERR_ARG;
    if (n > 0 && table == nullptr) return FP8BQ_ERR_NULL;
    std::vector<char> empty((size_t)n, 0);
    bool any = false;
    for (int i = 0; i < n; ++i) {
        bool e = false;
        const fp8bq_status s = check_desc(table[i], &e);
        if (s != FP8BQ_OK) return s;
        empty[i] = e;
        any |= !e;
    }
    if (!any) return FP8BQ_OK;
    const fp8bq_status so = check_overlap(table, n, empty);
    if (so != FP8BQ_OK) return so;
    const fp8bq_status sd = check_device();
    if (sd != FP8BQ_OK) return sd;
    plan.descs.resize((size_t)n);
    for (int i = 0; i < n; ++i) plan.descs[i] = empty[i] ? table[i] : reshaped(table[i]);

    // The kernel variant of each tensor.  AUTO sends a call's TMA tensors to
    // the vector kernel when together they hold less than kTmaMinCallBytes of
    // input: short launches start sooner on the vector kernel's two CTAs per
    // SM than on the TMA ring of one CTA per SM.
    const int path = g_path.load();
    std::vector<Variant> var((size_t)n, Variant::Generic);
    uint64_t tma_bytes = 0;
    for (int i = 0; i < n; ++i) {
        if (empty[i]) continue;
        const fp8bq_desc &D = plan.descs[i];
        var[i] = choose(D, path);
        if (var[i] == Variant::Tma)
            tma_bytes += (uint64_t)D.batch * (uint64_t)D.M * (uint64_t)D.N * esize_of(D.dtype_in);
    }
    const bool small_call = path == FP8BQ_PATH_AUTO && tma_bytes < kTmaMinCallBytes;

    std::vector<GroupKey> &keys = plan.keys;
    std::vector<std::vector<int>> &members = plan.members;
    std::vector<std::vector<CUtensorMap>> &maps = plan.maps;
    for (int i = 0; i < n; ++i) {
        if (empty[i]) continue;
        const fp8bq_desc &D = plan.descs[i];
        Variant v = var[i];
        CUtensorMap m;
        if (v == Variant::Tma && (small_call || !encode_map(D, &m)))
            v = choose(D, FP8BQ_PATH_VECTOR);
        // vector / TMA launches need one block shape; generic ones only one
        // size class (CTA per block for >= 2048 elements, else warp per block)
        const bool big = (int64_t)D.block_m * D.block_n >= 2048;
        const bool halves = v != Variant::Generic && v != Variant::Tma && !vector_aligned(D);
        GroupKey k{v, esize_of(D.dtype_in), v == Variant::Generic ? (int)big : D.block_m,
                   v == Variant::Generic ? 0 : D.block_n, halves};
        size_t g = 0;
        while (g < keys.size() && !(keys[g] == k)) ++g;
        if (g == keys.size()) {
            keys.push_back(k);
            members.emplace_back();
            maps.emplace_back();
        }
        members[g].push_back(i);
        if (v == Variant::Tma) maps[g].push_back(m);
    }
    return FP8BQ_OK;
}

// Launches of one group: packs of at most MAXD descriptors and fewer than
// 2^31 tiles (the chunking of launch_group / launch_tma_group).
template <int MAXD>
int packs_of(const fp8bq_desc *t, const std::vector<int> &idx, Variant v) {
    int packs = 0;
    size_t i = 0;
    while (i < idx.size()) {
        ++packs;
        int nd = 0;
        uint64_t total = 0;
        while (i < idx.size() && nd < MAXD) {
            const uint64_t tiles = tiles_of(t[idx[i]], v);
            if (nd > 0 && total + tiles >= (1ull << 31)) break;
            total += tiles;
            ++nd;
            ++i;
        }
    }
    return packs;
}

int launches_of(const Plan &plan) {
    const fp8bq_desc *table = plan.descs.data();
    int total = 0;
    for (size_t g = 0; g < plan.keys.size(); ++g) {
        const std::vector<int> &idx = plan.members[g];
        const bool small = idx.size() <= (size_t)kMaxDescSmall;
        const Variant v = plan.keys[g].v;
        if (v == Variant::Tma)
            total += small ? packs_of<kMaxDescSmall>(table, idx, v) : packs_of<kMaxDescTma>(table, idx, v);
        else
            total += small ? packs_of<kMaxDescSmall>(table, idx, v)
                           : packs_of<kMaxDescLarge>(table, idx, v);
    }
    return total;
}

fp8bq_status run(const fp8bq_desc *caller_table, int n, cudaStream_t stream) {
    Plan plan;
    const fp8bq_status sp = make_plan(caller_table, n, plan);
    if (sp != FP8BQ_OK || plan.keys.empty()) return sp;
    const fp8bq_desc *table = plan.descs.data();
    const std::vector<GroupKey> &keys = plan.keys;
    const std::vector<std::vector<int>> &members = plan.members;
    const std::vector<std::vector<CUtensorMap>> &maps = plan.maps;
    auto launch = [&](size_t g, cudaStream_t st) -> cudaError_t {
        if (keys[g].v == Variant::Tma)
            return members[g].size() <= (size_t)kMaxDescSmall
                       ? launch_tma_group<kMaxDescSmall>(keys[g].es, table, members[g], maps[g], st)
                       : launch_tma_group<kMaxDescTma>(keys[g].es, table, members[g], maps[g], st);
        if (members[g].size() <= (size_t)kMaxDescSmall)
            return launch_group<kMaxDescSmall>(keys[g].v, keys[g].es, keys[g].halves, table,
                                               members[g], st);
        return launch_group<kMaxDescLarge>(keys[g].v, keys[g].es, keys[g].halves, table,
                                           members[g], st);
    };
    return run_groups(keys.size(), launch, stream);
}

// ------------------------------------------------------------------ dequantization

fp8bq_status check_dequant_desc(const fp8bq_dequant_desc &D, bool *empty) {
    if (D.dtype_out != FP8BQ_BF16 && D.dtype_out != FP8BQ_F32) return FP8BQ_ERR_DTYPE;
    if (D.block_m < 1 || D.block_n < 1 || (int64_t)D.block_m * D.block_n > 65536)
        return FP8BQ_ERR_BLOCK;
    if (D.batch < 0 || D.M < 0 || D.N < 0 || D.ld_out < D.N || D.M >= (1ll << 31) ||
        D.N >= (1ll << 31))
        return FP8BQ_ERR_SHAPE;
    *empty = D.batch == 0 || D.M == 0 || D.N == 0;
    if (*empty) return FP8BQ_OK;
    if (D.batch > 1 && D.out_batch_stride < 0) return FP8BQ_ERR_SHAPE;
    if (D.batch > 1 && D.out_batch_stride < (D.M - 1) * D.ld_out + D.N) return FP8BQ_ERR_OVERLAP;
    if (D.y_u8 == nullptr || D.descale_f32 == nullptr || D.out == nullptr) return FP8BQ_ERR_NULL;
    if ((uintptr_t)D.descale_f32 % 4 || (uintptr_t)D.out % esize_of(D.dtype_out))
        return FP8BQ_ERR_ALIGN;
    const __int128 b1 = D.batch - 1, lim = (__int128)1 << 62;
    if ((b1 * (D.batch > 1 ? D.out_batch_stride : 0) + (__int128)(D.M - 1) * D.ld_out + D.N) *
                esize_of(D.dtype_out) > lim ||
        (__int128)D.batch * D.M * D.N > lim)
        return FP8BQ_ERR_SHAPE;
    return FP8BQ_OK;
}

bool dequant_vector_ok(const fp8bq_dequant_desc &D) {
    const int oes = esize_of(D.dtype_out);
    const int64_t obs = D.batch > 1 ? D.out_batch_stride : 0;
    return D.N % 16 == 0 && D.block_n % 16 == 0 && (uintptr_t)D.y_u8 % 16 == 0 &&
           (uintptr_t)D.out % 16 == 0 && (D.ld_out * oes) % 16 == 0 && (obs * oes) % 16 == 0;
}

template <int MAXD>
cudaError_t launch_dequant_group(const fp8bq_dequant_desc *t, const std::vector<int> &idx,
                                 bool vector, int oes, cudaStream_t st) {
    static thread_local DequantPack<MAXD> p;
    size_t i = 0;
    while (i < idx.size()) {
        p.n = 0;
        p.pad_ = 0;
        p.total = 0;
        while (i < idx.size() && p.n < MAXD) {
            const fp8bq_dequant_desc &D = t[idx[i]];
            DequantDesc &o = p.d[p.n];
            o.y = D.y_u8;
            o.s = D.descale_f32;
            o.out = D.out;
            o.M = D.M;
            o.N = D.N;
            o.ldo = D.ld_out;
            o.obs = D.batch > 1 ? D.out_batch_stride : 0;
            o.bm = D.block_m;
            o.bn = D.block_n;
            o.gm = (int32_t)cdiv(D.M, D.block_m);
            o.gn = (int32_t)cdiv(D.N, D.block_n);
            o.begin = p.total;
            // vector: warp items of 32 x U x 16 codes per row; generic: one element
            o.items = vector ? (uint64_t)(D.batch * D.M) *
                                   (uint64_t)cdiv(D.N / 16, 32 * dequant_unroll())
                             : (uint64_t)(D.batch * D.M * D.N);
#if FP8BQ_CHECKED
            o.y_bytes = (uint64_t)(D.batch * D.M * D.N);
            o.s_bytes = (uint64_t)(D.batch * o.gm * (int64_t)o.gn * 4);
            o.out_bytes = checked_out_extent(
                (uint64_t)(((D.batch - 1) * o.obs + (D.M - 1) * D.ld_out + D.N) * oes));
#endif
            p.total += o.items;
            ++p.n;
            ++i;
        }
        const cudaError_t e = launch_dequant<MAXD>(p, oes, vector, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

fp8bq_status run_dequant(const fp8bq_dequant_desc *t, int n, cudaStream_t stream) {
    if (n < 0) return FP8BQ_ERR_ARG;
    if (n > 0 && t == nullptr) return FP8BQ_ERR_NULL;
    std::vector<char> empty((size_t)n, 0);
    bool any = false;
    for (int i = 0; i < n; ++i) {
        bool e = false;
        const fp8bq_status st = check_dequant_desc(t[i], &e);
        if (st != FP8BQ_OK) return st;
        empty[i] = e;
        any |= !e;
    }
    if (!any) return FP8BQ_OK;
    // Outputs may overlap nothing; codes and descales are inputs.
    std::vector<Span> sp;
    for (int i = 0; i < n; ++i) {
        if (empty[i]) continue;
        const fp8bq_dequant_desc &D = t[i];
        const int64_t oes = esize_of(D.dtype_out), b1 = D.batch - 1;
        const int64_t gm = cdiv(D.M, D.block_m), gn = cdiv(D.N, D.block_n);
        const int64_t obs = D.batch > 1 ? D.out_batch_stride : 0;
        const uintptr_t o = (uintptr_t)D.out, y = (uintptr_t)D.y_u8, s = (uintptr_t)D.descale_f32;
        sp.push_back({o, o + (uintptr_t)((b1 * obs + (D.M - 1) * D.ld_out + D.N) * oes), true});
        sp.push_back({y, y + (uintptr_t)(D.batch * D.M * D.N), false});
        sp.push_back({s, s + (uintptr_t)(D.batch * gm * gn * 4), false});
    }
    std::sort(sp.begin(), sp.end(), [](const Span &a, const Span &b) { return a.lo < b.lo; });
    uintptr_t out_end = 0, in_end = 0;
    for (const Span &x : sp) {
        if (x.out) {
            if (x.lo < out_end || x.lo < in_end) return FP8BQ_ERR_OVERLAP;
            out_end = std::max(out_end, x.hi);
        } else {
            if (x.lo < out_end) return FP8BQ_ERR_OVERLAP;
            in_end = std::max(in_end, x.hi);
        }
    }
    const fp8bq_status sd = check_device();
    if (sd != FP8BQ_OK) return sd;
    const bool generic_only = g_path.load() == FP8BQ_PATH_GENERIC;
    std::vector<int> groups[2][2];  // [vector][output is bf16]
    for (int i = 0; i < n; ++i) {
        if (empty[i]) continue;
        const bool v = !generic_only && dequant_vector_ok(t[i]);
        groups[v][t[i].dtype_out == FP8BQ_BF16].push_back(i);
    }
    std::vector<std::pair<int, int>> used;  // (vector, bf16 output) of each non-empty group
    for (int v = 0; v < 2; ++v)
        for (int b = 0; b < 2; ++b)
            if (!groups[v][b].empty()) used.emplace_back(v, b);
    auto launch = [&](size_t k, cudaStream_t st) -> cudaError_t {
        const int v = used[k].first, b = used[k].second;
        const std::vector<int> &g = groups[v][b];
        return g.size() <= (size_t)kMaxDescSmall
                   ? launch_dequant_group<kMaxDescSmall>(t, g, v, b ? 2 : 4, st)
                   : launch_dequant_group<kMaxDescLarge>(t, g, v, b ? 2 : 4, st);
    };
    return run_groups(used.size(), launch, stream);
}

// ------------------------------------------------------------------ per-tensor scales

template <int MAXD>
cudaError_t launch_scale_group(const fp8bq_scale_desc *t, const std::vector<int> &idx, int es,
                               float *scale_out, uint64_t out_bytes, cudaStream_t st) {
    static thread_local ScalePack<MAXD> p;
    size_t i = 0;
    while (i < idx.size()) {
        p.n = 0;
        p.pad_ = 0;
        p.total = 0;
        p.acc = reinterpret_cast<uint32_t *>(scale_out);
        p.acc_bytes = out_bytes;
        while (i < idx.size() && p.n < MAXD) {
            const fp8bq_scale_desc &D = t[idx[i]];
            ScaleDesc &o = p.d[p.n];
            o.x = D.x;
            o.numel = D.numel;
            o.begin = p.total;
            o.items = (uint64_t)cdiv(D.numel, kScaleItem);
            o.out = idx[i];
            o.pad_ = 0;
            p.total += o.items;
            ++p.n;
            ++i;
        }
        if (p.total == 0) continue;
        const cudaError_t e = launch_scale_amax<MAXD>(p, es, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

fp8bq_status run_tensor_scale(const fp8bq_scale_desc *t, int n, float *scale_out,
                              cudaStream_t stream) {
    if (n < 0) return FP8BQ_ERR_ARG;
    if (n == 0) return FP8BQ_OK;
    if (t == nullptr || scale_out == nullptr) return FP8BQ_ERR_NULL;
    if ((uintptr_t)scale_out % 4) return FP8BQ_ERR_ALIGN;
    const uintptr_t o_lo = (uintptr_t)scale_out, o_hi = o_lo + (uintptr_t)n * 4;
    for (int i = 0; i < n; ++i) {
        const fp8bq_scale_desc &D = t[i];
        if (D.dtype_in != FP8BQ_BF16 && D.dtype_in != FP8BQ_F32) return FP8BQ_ERR_DTYPE;
        if (D.numel < 0 || D.numel > ((int64_t)1 << 60)) return FP8BQ_ERR_SHAPE;
        if (D.numel == 0) continue;
        if (D.x == nullptr) return FP8BQ_ERR_NULL;
        const int es = esize_of(D.dtype_in);
        if ((uintptr_t)D.x % es) return FP8BQ_ERR_ALIGN;
        const uintptr_t lo = (uintptr_t)D.x, hi = lo + (uintptr_t)(D.numel * es);
        if (lo < o_hi && o_lo < hi) return FP8BQ_ERR_OVERLAP;
    }
    const fp8bq_status sd = check_device();
    if (sd != FP8BQ_OK) return sd;
    const uint64_t out_bytes = checked_out_extent((uint64_t)n * 4);
    if (launch_scale_zero(scale_out, n, out_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return FP8BQ_ERR_DEVICE;
    }
    std::vector<int> groups[2];  // [is fp32]
    for (int i = 0; i < n; ++i)
        if (t[i].numel > 0) groups[t[i].dtype_in == FP8BQ_F32].push_back(i);
    for (int g = 0; g < 2; ++g) {
        if (groups[g].empty()) continue;
        const int es = g ? 4 : 2;
        const cudaError_t e =
            groups[g].size() <= (size_t)kMaxDescSmall
                ? launch_scale_group<kMaxDescSmall>(t, groups[g], es, scale_out, out_bytes, stream)
                : launch_scale_group<kMaxDescLarge>(t, groups[g], es, scale_out, out_bytes, stream);
        if (e != cudaSuccess) return FP8BQ_ERR_DEVICE;
    }
    return launch_scale_finalize(scale_out, n, out_bytes, stream) == cudaSuccess
               ? FP8BQ_OK
               : FP8BQ_ERR_DEVICE;
}

// The bounds records of every kernel source file, summed (checked builds;
// zeros without any CUDA call in a default build).
cudaError_t bounds_records(uint64_t *count, uint64_t *first, bool clear) {
    cudaError_t (*const fns[])(uint64_t *, uint64_t *, bool) = {
        bounds_record_kernels, bounds_record_tma, bounds_record_dequant, bounds_record_scale};
    *count = 0;
    *first = 0;
    for (auto fn : fns) {
        uint64_t c = 0, f = 0;
        const cudaError_t e = fn(&c, &f, clear);
        if (e != cudaSuccess) return e;
        *count += c;
        if (*first == 0) *first = f;
    }
    return cudaSuccess;
}

}  // namespace

bool fp8bq::pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

extern "C" {

fp8bq_status fp8bq_tensor_scale(const fp8bq_scale_desc *desc_table, int n_tensors,
                                float *scale_out, cudaStream_t stream) {
    return run_tensor_scale(desc_table, n_tensors, scale_out, stream);
}

fp8bq_status fp8bq_quantize(const void *x, fp8bq_dtype dtype_in, int64_t M, int64_t N, int64_t ld,
                            int block_m, int block_n, uint8_t *y_u8, float *descale_f32,
                            cudaStream_t stream) {
    fp8bq_desc D;
    std::memset(&D, 0, sizeof D);
    D.x = x;
    D.y_u8 = y_u8;
    D.descale_f32 = descale_f32;
    D.M = M;
    D.N = N;
    D.ld = ld;
    D.batch = 1;
    D.dtype_in = (int32_t)dtype_in;
    D.block_m = block_m;
    D.block_n = block_n;
    return run(&D, 1, stream);
}

fp8bq_status fp8bq_quantize_batched(const fp8bq_desc *desc_table, int n_tensors,
                                    cudaStream_t stream) {
    return run(desc_table, n_tensors, stream);
}

fp8bq_status fp8bq_dequantize(const uint8_t *y_u8, const float *descale_f32, int64_t batch,
                              int64_t M, int64_t N, int block_m, int block_n, void *out,
                              fp8bq_dtype dtype_out, int64_t ld_out, int64_t out_batch_stride,
                              cudaStream_t stream) {
    fp8bq_dequant_desc D;
    std::memset(&D, 0, sizeof D);
    D.y_u8 = y_u8;
    D.descale_f32 = descale_f32;
    D.out = out;
    D.batch = batch;
    D.M = M;
    D.N = N;
    D.ld_out = ld_out;
    D.out_batch_stride = out_batch_stride;
    D.dtype_out = (int32_t)dtype_out;
    D.block_m = block_m;
    D.block_n = block_n;
    return run_dequant(&D, 1, stream);
}

fp8bq_status fp8bq_dequantize_batched(const fp8bq_dequant_desc *desc_table, int n_tensors,
                                      cudaStream_t stream) {
    return run_dequant(desc_table, n_tensors, stream);
}

const char *fp8bq_status_string(fp8bq_status s) {
    switch (s) {
        case FP8BQ_OK: return "FP8BQ_OK";
        case FP8BQ_ERR_NULL: return "FP8BQ_ERR_NULL: a required pointer is NULL";
        case FP8BQ_ERR_SHAPE: return "FP8BQ_ERR_SHAPE: invalid shape, stride or batch";
        case FP8BQ_ERR_BLOCK: return "FP8BQ_ERR_BLOCK: invalid block shape";
        case FP8BQ_ERR_DTYPE: return "FP8BQ_ERR_DTYPE: unknown input dtype";
        case FP8BQ_ERR_OVERLAP: return "FP8BQ_ERR_OVERLAP: an output overlaps an input or output";
        case FP8BQ_ERR_DEVICE: return "FP8BQ_ERR_DEVICE: no usable sm_100 device or CUDA error";
        case FP8BQ_ERR_DEVICE_TIMEOUT:
            return "FP8BQ_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
        case FP8BQ_ERR_ALIGN: return "FP8BQ_ERR_ALIGN: misaligned input or descale pointer";
        case FP8BQ_ERR_ARG: return "FP8BQ_ERR_ARG: invalid argument";
        case FP8BQ_ERR_DEVICE_UNSAFE:
            return "FP8BQ_ERR_DEVICE_UNSAFE: a kernel returned with a tile copy in flight; "
                   "stop using the GPU";
        case FP8BQ_ERR_DEVICE_BOUNDS:
            return "FP8BQ_ERR_DEVICE_BOUNDS: a checked kernel skipped an access outside its "
                   "tensor";
    }
    return "FP8BQ_?: unknown status";
}

fp8bq_status fp8bq_sync_status(cudaStream_t stream) {
    if (check_device() != FP8BQ_OK) return FP8BQ_ERR_DEVICE;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return FP8BQ_ERR_DEVICE;
    }
    uint32_t w = 0;
    if (read_and_clear_error_word(&w) != cudaSuccess) {
        cudaGetLastError();
        return FP8BQ_ERR_DEVICE;
    }
    if (w & 2u) return FP8BQ_ERR_DEVICE_UNSAFE;
    if (w) return FP8BQ_ERR_DEVICE_TIMEOUT;
    uint64_t count = 0, first = 0;
    if (bounds_records(&count, &first, false) != cudaSuccess) {
        cudaGetLastError();
        return FP8BQ_ERR_DEVICE;
    }
    return count ? FP8BQ_ERR_DEVICE_BOUNDS : FP8BQ_OK;
}

int fp8bq_version(void) { return FP8BQ_VERSION; }

fp8bq_status fp8bq_set_path(fp8bq_path path) {
    if (path < FP8BQ_PATH_AUTO || path > FP8BQ_PATH_GENERIC) return FP8BQ_ERR_ARG;
    g_path.store((int)path);
    return FP8BQ_OK;
}

fp8bq_path fp8bq_get_path(void) { return (fp8bq_path)g_path.load(); }

fp8bq_status fp8bq_set_pdl(int enable) {
    g_pdl.store(enable ? 1 : 0);
    return FP8BQ_OK;
}

int fp8bq_get_pdl(void) { return g_pdl.load(); }

int fp8bq_path_for(const fp8bq_desc *desc) {
    if (desc == nullptr) return -1;
    bool e = false;
    if (check_desc(*desc, &e) != FP8BQ_OK) return -1;
    switch (choose(reshaped(*desc), g_path.load())) {
        case Variant::Tma: return FP8BQ_PATH_TMA;
        case Variant::Generic: return FP8BQ_PATH_GENERIC;
        default: return FP8BQ_PATH_VECTOR;
    }
}

int fp8bq_launch_count(const fp8bq_desc *desc_table, int n_tensors) {
    Plan plan;
    if (make_plan(desc_table, n_tensors, plan) != FP8BQ_OK) return -1;
    return launches_of(plan);
}

fp8bq_status fp8bq_debug_set_wait_limit_ns(uint64_t ns) {
    g_wait_limit_ns.store(ns ? ns : 2000000000ull);
    return FP8BQ_OK;
}

fp8bq_status fp8bq_debug_set_inject(uint32_t flags) {
    const uint32_t known =
        FP8BQ_INJECT_DROP_FIRST_LOAD | (FP8BQ_CHECKED ? FP8BQ_INJECT_TRIM_OUTPUTS : 0u);
    if (flags & ~known) return FP8BQ_ERR_ARG;
    g_inject.store(flags);
    return FP8BQ_OK;
}

int fp8bq_checked_build(void) { return FP8BQ_CHECKED ? 1 : 0; }

fp8bq_status fp8bq_debug_take_bounds(uint64_t *count, uint64_t *first_address) {
    uint64_t c = 0, f = 0;
    if (FP8BQ_CHECKED) {
        if (check_device() != FP8BQ_OK) return FP8BQ_ERR_DEVICE;
        if (cudaDeviceSynchronize() != cudaSuccess || bounds_records(&c, &f, true) != cudaSuccess) {
            cudaGetLastError();
            return FP8BQ_ERR_DEVICE;
        }
    }
    if (count) *count = c;
    if (first_address) *first_address = f;
    return FP8BQ_OK;
}

}  // extern "C"

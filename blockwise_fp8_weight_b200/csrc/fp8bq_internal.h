// fp8bq_internal.h -- what the host side of the library and its kernels share.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver entry point is fetched at run time)
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#ifndef FP8BQ_CHECKED
#define FP8BQ_CHECKED 0  // 1: the bounds-checked build (see fp8bq_device.cuh)
#endif

namespace fp8bq {

// ------------------------------------------------------------------ per-device host state
//
// Kernel attributes (the dynamic shared-memory limit), resident CTAs per SM
// and the SM count are properties of a device: each is computed once per
// device, with that device current, so one process may drive several GPUs.
constexpr int kMaxDevices = 64;

inline int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        dev = 0;
    }
    return dev;
}

// A value made once per device (devices beyond kMaxDevices: made on every call).
template <typename T>
class PerDevice {
  public:
    template <typename F>
    T get(F &&make) {
        const int dev = current_device();
        if (dev < 0 || dev >= kMaxDevices) return make();
        std::call_once(once_[dev], [&] { val_[dev] = make(); });
        return val_[dev];
    }

  private:
    std::once_flag once_[kMaxDevices];
    T val_[kMaxDevices];
};

// Streaming multiprocessors of the current device.
inline int sm_count() {
    static PerDevice<int> n;
    return n.get([] {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, current_device()) !=
                cudaSuccess ||
            v <= 0) {
            cudaGetLastError();
            v = 148;
        }
        return v;
    });
}

// The eps floor of the block absmax.  The pages print the floor (absmax =
// max(max|x|, eps)) but not its value; 1e-10 is this library's reading.
constexpr float kEps = 1e-10f;
// Largest finite float8_e4m3fn value: the fp8_max / -fp8_min of the scale step.
constexpr float kFp8Max = 448.0f;

// One weight tensor as the kernels see it (kernel-parameter space).
struct TileDesc {
    const void *x;      // input base
    uint8_t *y;         // e4m3fn output base
    float *s;           // descale base
    int64_t ld;         // input row stride, elements
    int64_t xbs;        // input batch stride, elements
    int64_t ybs;        // output batch stride, bytes
    int64_t sbs;        // descale batch stride, floats
    int32_t M, N;       // matrix shape
    int32_t bm, bn;     // block shape
    int32_t gm, gn;     // block grid of one matrix
    uint32_t tile_begin;// first tile id of this tensor within the launch
    uint32_t tiles;     // batch * gm * gn
#if FP8BQ_CHECKED
    uint64_t x_bytes, y_bytes, s_bytes;  // extents of x, y and s (the bounds checks)
#endif
};
static_assert(sizeof(TileDesc) == (FP8BQ_CHECKED ? 112 : 88), "TileDesc layout");

// Grouped-launch parameters.  MAXD bounds the descriptors per launch so the
// whole pack stays inside the 32 KB kernel-parameter limit.
template <int MAXD>
struct DescPack {
    int32_t n;              // descriptors used
    uint32_t total_tiles;   // sum of tiles
    uint32_t inject;        // FP8BQ_INJECT_* flags (TMA kernel)
    int32_t group;          // blocks stacked along M per TMA tile (TMA kernel)
    uint64_t wait_limit_ns; // bound of every device wait (TMA kernel)
    TileDesc d[MAXD];
};

template <int MAXD>
struct alignas(64) TmaPack {
    CUtensorMap maps[MAXD];  // one 3-D map per descriptor: {N, M, batch}, box {bn, bm, 1}
    DescPack<MAXD> p;
    uint32_t evict_first;  // 1: load every tile with an L2 evict-first policy
};

// A TMA launch whose largest tensor has at least this many input bytes loads
// all its tiles with an L2 evict-first policy.  Measured on B200 (the same
// DRAM bytes either way; the policy changes how well they are scheduled):
// single tensors and expert stacks of 0.4-1.9 GB quantize 4-9 % faster with
// it, the 8-200 MB tensors of a dense model 2-5 % slower; and mixing the two
// policies in one launch loses most of the gain (lines loaded with the
// default priority outlive every evict-first line and hold L2 capacity).
constexpr uint64_t kEvictFirstMinBytes = 256ull << 20;

constexpr int kMaxDescSmall = 8;
// 320 * 88 B + header = 28.2 KB; checked builds 256 * 112 B + header = 28.7 KB
constexpr int kMaxDescLarge = FP8BQ_CHECKED ? 256 : 320;
constexpr int kMaxDescTma = 128;    // 128 * (128 + 88) B + header = 27.7 KB
static_assert(sizeof(DescPack<kMaxDescLarge>) < 32000, "kernel parameter limit");
static_assert(sizeof(TmaPack<kMaxDescTma>) < 32000, "kernel parameter limit");

// Programmatic dependent launch (on unless fp8bq_set_pdl(0)): every kernel of
// the library is launched with programmatic stream serialization, so it may
// be scheduled while the previous kernel of the stream drains; it lets the
// next kernel launch at once and waits for the previous one (griddepcontrol)
// before its first global-memory access.  Stream order of memory effects is
// unchanged: only launch latency and the kernel prologue overlap.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Kernel variants, by input element size and team shape.
enum class Variant : int {
    Generic = 0,
    VecT16 = 1,   // a team of 16 threads per 8 stacked blocks of one row-step each
    VecT64 = 2,   // a team of 64 threads per block (<= 512 vectors)
    VecTBig = 3,  // one team per CTA (<= 2048 vectors)
    Tma = 4,
    VecT32 = 5,   // a team of 32 threads (a warp) per 8 stacked blocks of one row-step each
    VecT128 = 6,  // a team of 128 threads per block (<= 1024 vectors)
};

// Launchers (vector and generic: fp8bq_kernels.cu; TMA: fp8bq_tma.cu).  Each
// returns cudaSuccess or the launch error.
// halves: rows only 8-byte aligned (each 16-byte vector moved as two halves)
template <int MAXD>
cudaError_t launch_vector(Variant v, int esize, bool halves, const DescPack<MAXD> &p,
                          cudaStream_t st);
template <int MAXD>
cudaError_t launch_generic(int esize, const DescPack<MAXD> &p, cudaStream_t st);
template <int MAXD>
cudaError_t launch_tma(int esize, bool subwarp, const TmaPack<MAXD> &p, cudaStream_t st);
template <int MAXD>
cudaError_t launch_tma_pair(const TmaPack<MAXD> &p, cudaStream_t st);

// Dequantization (fp8bq_dequant.cu): one matrix stack per descriptor, a
// grouped launch walks the concatenated work items (a warp-wide row segment
// of 32 x U x 16 codes for the vector kernel, U = dequant_unroll(); one
// element for the generic one) of all descriptors of a pack.
struct DequantDesc {
    const uint8_t *y;   // [batch, M, N] codes
    const float *s;     // [batch, gm, gn] descales
    void *out;          // matrix b at out + b * obs elements, row stride ldo
    int64_t M, N, ldo, obs;
    int32_t bm, bn, gm, gn;
    uint64_t begin;     // first work item of this descriptor
    uint64_t items;     // work items of this descriptor
#if FP8BQ_CHECKED
    uint64_t y_bytes, s_bytes, out_bytes;  // extents (the bounds checks)
#endif
};
static_assert(sizeof(DequantDesc) == (FP8BQ_CHECKED ? 112 : 88), "DequantDesc layout");

template <int MAXD>
struct DequantPack {
    int32_t n;
    int32_t pad_;
    uint64_t total;
    DequantDesc d[MAXD];
};
static_assert(sizeof(DequantPack<kMaxDescLarge>) < 32000, "kernel parameter limit");

template <int MAXD>
cudaError_t launch_dequant(const DequantPack<MAXD> &p, int out_esize, bool vector, cudaStream_t st);
// U: a work item of the vector dequant kernel holds U x 16 codes per lane
int dequant_unroll();

// Per-tensor scales (fp8bq_scale.cu): the tensors of a pack are cut into
// work items of kScaleItem elements; every warp folds its items' absmax into
// acc[out] (the caller's output, zeroed first, as fp32 bit patterns).
constexpr int64_t kScaleItem = 8192;
struct ScaleDesc {
    const void *x;
    int64_t numel;
    uint64_t begin;   // first work item
    uint64_t items;   // ceil(numel / kScaleItem)
    int32_t out;      // index into the output
    int32_t pad_;
};
template <int MAXD>
struct ScalePack {
    int32_t n;
    int32_t pad_;
    uint64_t total;
    uint32_t *acc;
    uint64_t acc_bytes;  // extent of acc (the bounds checks of checked builds)
    ScaleDesc d[MAXD];
};
static_assert(sizeof(ScalePack<kMaxDescLarge>) < 32000, "kernel parameter limit");
template <int MAXD>
cudaError_t launch_scale_amax(const ScalePack<MAXD> &p, int esize, cudaStream_t st);
// out_bytes: the extent of scale_out that the bounds checks of checked builds take
cudaError_t launch_scale_zero(float *scale_out, int n, uint64_t out_bytes, cudaStream_t st);
cudaError_t launch_scale_finalize(float *scale_out, int n, uint64_t out_bytes, cudaStream_t st);

// Device error word access (fp8bq_tma.cu).
cudaError_t read_and_clear_error_word(uint32_t *out);

// Bounds records of checked builds, one per kernel source file (count of
// skipped accesses, one of their addresses; both 0 in a default build).
cudaError_t bounds_record_kernels(uint64_t *count, uint64_t *first, bool clear);
cudaError_t bounds_record_tma(uint64_t *count, uint64_t *first, bool clear);
cudaError_t bounds_record_dequant(uint64_t *count, uint64_t *first, bool clear);
cudaError_t bounds_record_scale(uint64_t *count, uint64_t *first, bool clear);

// Team geometry used by the vector kernels (host eligibility must agree).
constexpr int kVecTeamThreads(Variant v, int esize) {
    return v == Variant::VecT16    ? 16
           : v == Variant::VecT32  ? 32
           : v == Variant::VecT64  ? 64
           : v == Variant::VecT128 ? 128
                                   : (esize == 2 ? 256 : 512);
}
constexpr int kVecSlots(Variant v) { return 8; }
// Blocks per tile along M: the small-block kernel stacks 8 blocks per tile.
constexpr int kTileBlocksM(Variant v) {
    return v == Variant::VecT16 || v == Variant::VecT32 ? 8 : 1;
}

constexpr int kTmaConsumerThreads = 256;
constexpr int kTmaStageBytes = 32768;

}  // namespace fp8bq

// fp8bq_dequant.cu -- dequantization kernels: out = decode(y) * descale.
//
// The descale written by the quantizer is the dequantization multiplier
// ("vllm_fp8_utils.py" docs, section 3: it is loaded as "<name>_scale_inv"),
// so the reverse map is one fp32 multiply per element, rounded to nearest
// even, then (for bf16 output) rounded to bf16.  The pass is HBM-bound:
// 1 byte read and 2 (bf16) or 4 (fp32) bytes written per element.
//
// decode() is exact in two steps: cvt.rn.f16x2.e4m3x2 (every e4m3fn value,
// subnormals included, is a normal fp16 value) and fp16 -> fp32.
#include "fp8bq_device.cuh"
#include "fp8bq_internal.h"

namespace fp8bq {
namespace {

// Two e4m3fn codes (low byte first) -> their fp32 values.
__device__ __forceinline__ void decode2(uint16_t codes, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
    asm("{\n\t.reg .f16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\t"
        "cvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
}

// {lo, hi} * {s, s}, each lane one IEEE round-to-nearest multiply.
__device__ __forceinline__ void mul2(float &lo, float &hi, uint64_t ss) {
    uint64_t a, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(lo), "f"(hi));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(ss));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// Byte ranges of a descriptor's codes, descales and output (the bounds checks
// of checked builds; only ever expanded inside FP8BQ_IN).
#define DQ_SPAN_Y(a) (dev::Span{(uint64_t)(a).y, (uint64_t)(a).y + (a).y_bytes})
#define DQ_SPAN_S(a) (dev::Span{(uint64_t)(a).s, (uint64_t)(a).s + (a).s_bytes})
#define DQ_SPAN_O(a) (dev::Span{(uint64_t)(a).out, (uint64_t)(a).out + (a).out_bytes})

// Descriptor of work item k (items grow along each thread's grid-stride walk,
// so the cursor only moves forward).
template <int MAXD>
__device__ __forceinline__ const DequantDesc &find(const DequantPack<MAXD> &p, uint64_t k, int &d) {
    while (k >= p.d[d].begin + p.d[d].items) ++d;
    return p.d[d];
}

// The descriptor holding work item k (< p.total), by bisection over the
// descriptors' first items: where a walk starts, so that short walks (a
// grid of many CTAs) do not scan the table from its first entry.
template <int MAXD>
__device__ __forceinline__ int first_desc(const DequantPack<MAXD> &p, uint64_t k) {
    int lo = 0, hi = p.n - 1;  // the answer lies in [lo, hi]
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.d[mid].begin <= k) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Vector kernel: a work item is a warp-wide row segment of 32 x U x 16 codes,
// numbered row-major over (matrix, row, segment) and walked grid-stride by
// warps, so index arithmetic is paid once per segment.  A lane loads
// 16 / OES codes at a time (8 for bf16 output, 4 for fp32), so each load
// feeds exactly one 16-byte store and a warp store writes 512 contiguous
// bytes, filling every sector it touches; all of a lane's loads of an item
// are issued before any is used.  N and block_n are multiples of 16, so the
// codes of one load share a descale.
#ifndef FP8BQ_DQ_UNROLL
#define FP8BQ_DQ_UNROLL 4  // measured, fraction of the copy peak on one layer / the whole
                           // weight set: grid of 8 CTAs per SM: 1 -> 0.62 / 0.62, 2 -> 0.82 /
                           // 0.86, 4 -> 0.92-0.94 / 0.89-0.91, 8 -> 0.82 / 0.86; grid of 32
                           // per SM: 2 -> 0.86 / 0.83, 4 -> 0.96 / 0.97, 8 -> 0.81 / 0.82
#endif
// Measured and dropped: a lane loading 16 codes and writing them with two
// 16-byte stores 32 bytes apart (each warp store half-fills 32 sectors; 0.84
// of the copy peak on one layer and on the whole set); the same, software-
// pipelined, with the next item's loads in flight while the current one is
// decoded (0.71-0.75: more registers, fewer warps); 64 x 128 output tiles
// written into shared memory and handed to TMA tile stores (0.69-0.72: two
// CTA barriers per tile and one issuing thread serialise the tiles);
// numbering the items in 32 bits with shifts for power-of-two blocks (with
// the index arithmetic gone, nothing hides the load latency); one warp per
// whole row (4,199 / 3,889 GB/s against 5,499 for the two-store form).
constexpr int kDqUnroll = FP8BQ_DQ_UNROLL;

template <int OES, int MAXD>
__global__ void __launch_bounds__(256) k_dequant_vec(const __grid_constant__ DequantPack<MAXD> p) {
    dev::pdl_entry();
    constexpr int CPL = 16 / OES;              // codes per lane load
    constexpr int L = kDqUnroll * 16 / CPL;    // loads per lane per item
    const int lane = threadIdx.x & 31;
    const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x >> 5);
    const uint64_t k0 = (uint64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    int d = k0 < p.total ? first_desc(p, k0) : 0;
    for (uint64_t k = k0; k < p.total; k += warps) {
        const DequantDesc &a = find(p, k, d);
        const int64_t nc = a.N / CPL;
        const int64_t segs = (nc + 32 * L - 1) / (32 * L);
        const int64_t local = (int64_t)(k - a.begin);
        const int64_t row_all = local / segs;            // b * M + r
        const int64_t chunk0 = (local - row_all * segs) * 32 * L + lane;
        if (chunk0 >= nc) continue;
        const int64_t b = row_all / a.M;
        const int64_t r = row_all - b * a.M;
        const uint8_t *src = a.y + row_all * a.N;
        uint32_t q[L][CPL / 4];
#pragma unroll
        for (int u = 0; u < L; ++u) {
            const int64_t chunk = chunk0 + 32 * u;
            if (chunk < nc) {
                if (!FP8BQ_IN(DQ_SPAN_Y(a), src + chunk * CPL, CPL)) {
#pragma unroll
                    for (int j = 0; j < CPL / 4; ++j) q[u][j] = 0;
                } else if constexpr (CPL == 8) {
                    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                                 : "=r"(q[u][0]), "=r"(q[u][1])
                                 : "l"(src + chunk * 8));
                } else {
                    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];"
                                 : "=r"(q[u][0])
                                 : "l"(src + chunk * 4));
                }
            }
        }
        const float *srow = a.s + (b * a.gm + r / a.bm) * a.gn;
        char *orow = (char *)a.out + ((b * a.obs) + r * a.ldo) * OES;
#pragma unroll
        for (int u = 0; u < L; ++u) {
            const int64_t chunk = chunk0 + 32 * u;
            if (chunk >= nc) break;
            const int64_t c = chunk * CPL;
            const float *sp = srow + c / a.bn;
            const float s = FP8BQ_IN(DQ_SPAN_S(a), sp, 4) ? __ldg(sp) : 0.0f;
            uint64_t ss;
            asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
            float v[CPL];
#pragma unroll
            for (int j = 0; j < CPL / 4; ++j) {
                decode2((uint16_t)(q[u][j] & 0xffffu), v[4 * j + 0], v[4 * j + 1]);
                decode2((uint16_t)(q[u][j] >> 16), v[4 * j + 2], v[4 * j + 3]);
            }
#pragma unroll
            for (int j = 0; j < CPL / 2; ++j) mul2(v[2 * j], v[2 * j + 1], ss);
            char *dst = orow + c * OES;
            if (!FP8BQ_IN(DQ_SPAN_O(a), dst, 16)) continue;
            if constexpr (OES == 2) {
                uint32_t o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(o[0]),
                             "r"(o[1]), "r"(o[2]), "r"(o[3])
                             : "memory");
            } else {
                asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v[0]),
                             "f"(v[1]), "f"(v[2]), "f"(v[3])
                             : "memory");
            }
        }
    }
}

// One element per work item: any N, block shape, alignment or stride.
template <int OES, int MAXD>
__global__ void __launch_bounds__(256)
    k_dequant_generic(const __grid_constant__ DequantPack<MAXD> p) {
    dev::pdl_entry();
    const uint64_t k0 = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int d = k0 < p.total ? first_desc(p, k0) : 0;
    for (uint64_t k = k0; k < p.total; k += (uint64_t)gridDim.x * blockDim.x) {
        const DequantDesc &a = find(p, k, d);
        const int64_t per_b = a.M * a.N;
        const int64_t local = (int64_t)(k - a.begin);
        const int64_t b = local / per_b;
        const int64_t rem = local - b * per_b;
        const int64_t r = rem / a.N;
        const int64_t c = rem - r * a.N;
        const float *sp = a.s + (b * a.gm + r / a.bm) * a.gn + c / a.bn;
        const float s = FP8BQ_IN(DQ_SPAN_S(a), sp, 4) ? __ldg(sp) : 0.0f;
        float v, unused;
        const uint8_t code = FP8BQ_IN(DQ_SPAN_Y(a), a.y + local, 1) ? __ldg(a.y + local) : 0;
        decode2((uint16_t)code, v, unused);
        v = __fmul_rn(v, s);
        char *dst = (char *)a.out + (b * a.obs + r * a.ldo + c) * OES;
        if (!FP8BQ_IN(DQ_SPAN_O(a), dst, OES)) continue;
        if constexpr (OES == 2)
            *(uint16_t *)dst = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xffffu);
        else
            *(float *)dst = v;
    }
}

// Grid cap, in CTAs per SM.  Four 256-thread CTAs are resident per SM (64
// registers a thread), so the cap sets how many waves of short-lived CTAs a
// launch runs; late waves fill the SMs whose CTAs finished early.  Measured on
// B200 (whole weight set / one layer / [64,64] blocks, fraction of the copy
// peak): 2 -> 0.76 / 0.74 / 0.67, 4 -> 0.90 / 0.91 / 0.87, 8 -> 0.91 / 0.94 /
// 0.88, 16 -> 0.92 / 0.96 / 0.91, 32 -> 0.965 / 0.955 / 0.90, 64 -> 0.974 /
// 0.948 / 0.90, no cap -> 0.94 / 0.94 / 0.90 (0.27 on the whole set before the
// walks started with a bisection instead of a scan of the descriptor table).
#ifndef FP8BQ_DQ_CTAS_PER_SM
#define FP8BQ_DQ_CTAS_PER_SM 32
#endif
unsigned dq_grid(uint64_t work) {
    const uint64_t need = (work + 255) / 256;
    const uint64_t cap = (uint64_t)sm_count() * FP8BQ_DQ_CTAS_PER_SM;
    return (unsigned)(need < 1 ? 1 : need < cap ? need : cap);
}

}  // namespace

int dequant_unroll() { return kDqUnroll; }

template <int MAXD>
cudaError_t launch_dequant(const DequantPack<MAXD> &p, int out_esize, bool vector, cudaStream_t st) {
    const unsigned grid = dq_grid(vector ? p.total * 32 : p.total);  // vector: a warp per item
    if (vector)
        return out_esize == 2 ? launch_kernel(k_dequant_vec<2, MAXD>, grid, 256, 0, st, p)
                              : launch_kernel(k_dequant_vec<4, MAXD>, grid, 256, 0, st, p);
    return out_esize == 2 ? launch_kernel(k_dequant_generic<2, MAXD>, grid, 256, 0, st, p)
                          : launch_kernel(k_dequant_generic<4, MAXD>, grid, 256, 0, st, p);
}

template cudaError_t launch_dequant<kMaxDescSmall>(const DequantPack<kMaxDescSmall> &, int, bool,
                                                   cudaStream_t);
template cudaError_t launch_dequant<kMaxDescLarge>(const DequantPack<kMaxDescLarge> &, int, bool,
                                                   cudaStream_t);

FP8BQ_DEFINE_BOUNDS_RECORD(bounds_record_dequant)

}  // namespace fp8bq

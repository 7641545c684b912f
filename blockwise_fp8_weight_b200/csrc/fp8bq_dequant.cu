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

// Descriptor of work item k (items grow along each thread's grid-stride walk,
// so the cursor only moves forward).
template <int MAXD>
__device__ __forceinline__ const DequantDesc &find(const DequantPack<MAXD> &p, uint64_t k, int &d) {
    while (k >= p.d[d].begin + p.d[d].items) ++d;
    return p.d[d];
}

// Vector kernel: a work item is a warp-wide row segment of 32 x U x 16 codes
// (U 16-byte loads per lane, all issued before any is used; N and block_n are
// multiples of 16, so the 16 codes of a load share one descale).  Items are
// numbered row-major over (matrix, row, segment) and walked grid-stride by
// warps, so index arithmetic is paid once per segment.
#ifndef FP8BQ_DQ_UNROLL
#define FP8BQ_DQ_UNROLL 2  // measured: 1 -> 4.36, 2 -> 5.41, 4 -> 5.61 TB/s on one layer,
                           // 4.64 / 5.58 / 5.48 TB/s on the whole weight set
#endif
// Measured and dropped: 64 x 128 output tiles written into shared memory and
// handed to TMA tile stores (72.9 M instructions on one layer, about the
// same as here, and 121 us instead of 108 us cold; 0.69-0.72 of the copy
// peak live against 0.84: two CTA barriers per tile and one issuing thread
// serialise the tiles); numbering the items in 32 bits with shifts for
// power-of-two blocks (43.9 M instead of 75.2 M instructions on one layer,
// yet 142 us instead of 108 us: with the index arithmetic gone, nothing
// hides the load latency -- long-scoreboard stalls 21 per issue against
// 3.4), and one warp per whole row (4,199 / 3,889 GB/s against 5,499).
constexpr int kDqUnroll = FP8BQ_DQ_UNROLL;

template <int OES, int MAXD>
__global__ void __launch_bounds__(256) k_dequant_vec(const __grid_constant__ DequantPack<MAXD> p) {
    dev::pdl_entry();
    constexpr int U = kDqUnroll;
    const int lane = threadIdx.x & 31;
    const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x >> 5);
    int d = 0;
    for (uint64_t k = (uint64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < p.total;
         k += warps) {
        const DequantDesc &a = find(p, k, d);
        const int64_t n16 = a.N / 16;
        const int64_t segs = (n16 + 32 * U - 1) / (32 * U);
        const int64_t local = (int64_t)(k - a.begin);
        const int64_t row_all = local / segs;            // b * M + r
        const int64_t chunk0 = (local - row_all * segs) * 32 * U + lane;
        if (chunk0 >= n16) continue;
        const int64_t b = row_all / a.M;
        const int64_t r = row_all - b * a.M;
        const uint8_t *src = a.y + row_all * a.N;
        uint4 q[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t chunk = chunk0 + 32 * u;
            if (chunk < n16)
                asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(q[u].x), "=r"(q[u].y), "=r"(q[u].z), "=r"(q[u].w)
                             : "l"(src + chunk * 16));
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t chunk = chunk0 + 32 * u;
            if (chunk >= n16) break;
            const int64_t c = chunk * 16;
            const float s = __ldg(a.s + (b * a.gm + r / a.bm) * a.gn + c / a.bn);
            uint64_t ss;
            asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
            float v[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                decode2((uint16_t)(w[j] & 0xffffu), v[4 * j + 0], v[4 * j + 1]);
                decode2((uint16_t)(w[j] >> 16), v[4 * j + 2], v[4 * j + 3]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) mul2(v[2 * j], v[2 * j + 1], ss);
            char *dst = (char *)a.out + ((b * a.obs) + r * a.ldo + c) * OES;
            if constexpr (OES == 2) {
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "r"(o[0]),
                             "r"(o[1]), "r"(o[2]), "r"(o[3])
                             : "memory");
                asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 16),
                             "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                             : "memory");
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + 16 * j),
                                 "f"(v[4 * j]), "f"(v[4 * j + 1]), "f"(v[4 * j + 2]),
                                 "f"(v[4 * j + 3])
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
    int d = 0;
    for (uint64_t k = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; k < p.total;
         k += (uint64_t)gridDim.x * blockDim.x) {
        const DequantDesc &a = find(p, k, d);
        const int64_t per_b = a.M * a.N;
        const int64_t local = (int64_t)(k - a.begin);
        const int64_t b = local / per_b;
        const int64_t rem = local - b * per_b;
        const int64_t r = rem / a.N;
        const int64_t c = rem - r * a.N;
        const float s = __ldg(a.s + (b * a.gm + r / a.bm) * a.gn + c / a.bn);
        float v, unused;
        decode2((uint16_t)__ldg(a.y + local), v, unused);
        v = __fmul_rn(v, s);
        const int64_t o = b * a.obs + r * a.ldo + c;
        if constexpr (OES == 2)
            ((uint16_t *)a.out)[o] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xffffu);
        else
            ((float *)a.out)[o] = v;
    }
}

unsigned dq_grid(uint64_t work) {
    const uint64_t need = (work + 255) / 256;
    const uint64_t cap = (uint64_t)sm_count() * 8;
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

}  // namespace fp8bq

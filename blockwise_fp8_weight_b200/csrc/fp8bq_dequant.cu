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

// Vector kernel: a work item is a warp-wide segment of one matrix row, 32
// lanes x U x 16 codes (U 16-byte loads per lane, all issued before any is
// used; N and block_n are multiples of 16, so the 16 codes of a load share
// one descale).  Items are numbered (matrix, row, segment) over the
// descriptors of a launch (fewer than 2^32 per launch, host-checked) and
// walked grid-stride by warps; an item costs one or two 32-bit divisions,
// and the column block of a chunk a shift (power-of-two block_n).
#ifndef FP8BQ_DQ_UNROLL
#define FP8BQ_DQ_UNROLL 2
#endif
constexpr int kDqUnroll = FP8BQ_DQ_UNROLL;

__device__ __forceinline__ uint32_t div_p2(uint32_t v, uint32_t d, int log2d) {
    return log2d >= 0 ? v >> log2d : v / d;
}

template <int OES, int MAXD>
__global__ void __launch_bounds__(256) k_dequant_vec(const __grid_constant__ DequantPack<MAXD> p) {
    dev::pdl_entry();
    constexpr int U = kDqUnroll;
    const int lane = threadIdx.x & 31;
    const uint32_t warps = gridDim.x * (blockDim.x >> 5);
    const uint32_t total = (uint32_t)p.total;
    int d = 0;
    for (uint32_t k = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); k < total; k += warps) {
        const DequantDesc &a = find(p, k, d);
        const uint32_t n16 = (uint32_t)(a.N / 16);
        const uint32_t segs = (n16 + 32 * U - 1) / (32 * U);
        const uint32_t local = k - (uint32_t)a.begin;
        const uint32_t row_all = local / segs;  // b * M + r
        const uint32_t c0 = (local - row_all * segs) * 32 * U + lane;
        if (c0 >= n16) continue;
        uint32_t b = 0, r = row_all;
        if (row_all >= (uint32_t)a.M) {
            b = row_all / (uint32_t)a.M;
            r = row_all - b * (uint32_t)a.M;
        }
        const uint8_t *src = a.y + (uint64_t)row_all * (uint64_t)a.N;
        const float *srow =
            a.s + ((int64_t)b * a.gm + div_p2(r, (uint32_t)a.bm, a.bm_log2)) * a.gn;
        char *dst = (char *)a.out + ((int64_t)b * a.obs + (int64_t)r * a.ldo) * OES;
        {
            uint4 q[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t c = c0 + 32 * u;
                if (c < n16)
                    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(q[u].x), "=r"(q[u].y), "=r"(q[u].z), "=r"(q[u].w)
                                 : "l"(src + (uint64_t)c * 16));
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t c = c0 + 32 * u;
                if (c >= n16) break;
                const float s = __ldg(srow + div_p2(c * 16, (uint32_t)a.bn, a.bn_log2));
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
                char *o = dst + (uint64_t)c * 16 * OES;
                if constexpr (OES == 2) {
                    uint32_t h[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) h[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(o), "r"(h[0]),
                                 "r"(h[1]), "r"(h[2]), "r"(h[3])
                                 : "memory");
                    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(o + 16),
                                 "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                                 : "memory");
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(o + 16 * j),
                                     "f"(v[4 * j]), "f"(v[4 * j + 1]), "f"(v[4 * j + 2]),
                                     "f"(v[4 * j + 3])
                                     : "memory");
                }
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

}  // namespace

int dequant_unroll() { return kDqUnroll; }

namespace {

unsigned dq_grid(uint64_t work) {
    const uint64_t need = (work + 255) / 256;
    const uint64_t cap = (uint64_t)sm_count() * 8;
    return (unsigned)(need < 1 ? 1 : need < cap ? need : cap);
}

}  // namespace

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

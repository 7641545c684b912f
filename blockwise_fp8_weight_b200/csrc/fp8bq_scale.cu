// fp8bq_scale.cu -- per-tensor FP8 scales: scale = max(max|x|, eps) / 448.
//
// The FP8-RL report recalibrates the Q/K/V scales of its FP8 KV cache every
// RL step (abstract).  This is the block recipe of the weight quantizer
// applied to a whole tensor: a read-only pass (HBM-bound, numel * esize bytes)
// then one division pair per tensor.
//
// Pass 1 (k_scale_amax): the tensors of a launch are cut into items of
// kScaleItem elements; each CTA walks items grid-stride and its threads fold
// them into a running max of bit patterns; when the CTA moves on to another
// tensor (and at the end) it reduces and does one atomicMax into that
// tensor's output slot, which holds fp32 bit patterns meanwhile (the output
// was zeroed first; for non-negative floats the integer order of the bits is
// the numeric order).  Pass 2 (k_scale_finalize) turns the bits into the
// scale in place.
#include "fp8bq_device.cuh"
#include "fp8bq_internal.h"

namespace fp8bq {
namespace {

template <int ESIZE>
__device__ __forceinline__ uint32_t elem_abs(const char *base, int64_t i, const dev::Span &xs) {
    if (!FP8BQ_IN(xs, base + i * ESIZE, ESIZE)) return 0;
    if constexpr (ESIZE == 2)
        return ((uint32_t)__ldg((const unsigned short *)base + i) & 0x7fffu) << 16;
    else
        return __float_as_uint(__ldg((const float *)base + i)) & 0x7fffffffu;
}

// Fold a running max into the output slot of tensor `out`: CTA-wide reduce,
// then one atomicMax (called when a CTA moves to another tensor and at the
// end, so a tensor sees about one atomic per CTA).
__device__ __forceinline__ void flush_max(uint32_t m, uint32_t *acc, int out, uint32_t *red,
                                          const dev::Span &accs) {
    m = __reduce_max_sync(0xffffffffu, m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = red[0];
        for (int w = 1; w < 8; ++w) t = max(t, red[w]);
        if (t && FP8BQ_IN(accs, acc + out, 4)) atomicMax(acc + out, t);
    }
    __syncthreads();
}

template <int ESIZE, int MAXD>
__global__ void __launch_bounds__(256) k_scale_amax(const __grid_constant__ ScalePack<MAXD> p) {
    dev::pdl_entry();
    constexpr int VEC = 16 / ESIZE;            // elements per 16-byte load
    constexpr int LOADS = kScaleItem / 256 / VEC;
    __shared__ uint32_t red[8];
    int d = 0, cur = -1;
    if (blockIdx.x < p.total) {  // the descriptor of this CTA's first item, by bisection
        int hi = p.n - 1;
        while (d < hi) {
            const int mid = (d + hi + 1) >> 1;
            if (p.d[mid].begin <= blockIdx.x) d = mid;
            else hi = mid - 1;
        }
    }
    uint32_t m = 0;
    const dev::Span accs{(uint64_t)p.acc, (uint64_t)p.acc + p.acc_bytes};
    for (uint64_t it = blockIdx.x; it < p.total; it += gridDim.x) {
        while (it >= p.d[d].begin + p.d[d].items) ++d;
        if (d != cur) {  // uniform across the CTA: `it` is per CTA
            if (cur >= 0) flush_max(m, p.acc, p.d[cur].out, red, accs);
            m = 0;
            cur = d;
        }
        const ScaleDesc &D = p.d[d];
        const int64_t e0 = (int64_t)(it - D.begin) * kScaleItem;
        const int64_t len = min((int64_t)kScaleItem, D.numel - e0);
        const char *base = (const char *)D.x + e0 * ESIZE;
        const dev::Span xs{(uint64_t)D.x, (uint64_t)D.x + (uint64_t)D.numel * ESIZE};
        if (len == kScaleItem && ((uintptr_t)base & 15) == 0) {
            uint4 v[LOADS];
#pragma unroll
            for (int j = 0; j < LOADS; ++j) {
                const char *a = base + ((int64_t)j * 256 + threadIdx.x) * 16;
                v[j] = FP8BQ_IN(xs, a, 16) ? dev::ldg_stream_v4(a) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int j = 0; j < LOADS; ++j) {
                if constexpr (ESIZE == 2) {
                    const uint32_t a = dev::absmax_bf16x2(v[j].x & 0x7fff7fffu, v[j].y);
                    const uint32_t b = dev::absmax_bf16x2(v[j].z & 0x7fff7fffu, v[j].w);
                    m = max(m, dev::absmax_bits_bf16x2(dev::absmax_bf16x2(a, b)));
                } else {
                    const uint32_t a = dev::absmax_f32(v[j].x & 0x7fffffffu, v[j].y);
                    const uint32_t b = dev::absmax_f32(v[j].z & 0x7fffffffu, v[j].w);
                    m = max(m, dev::absmax_bits_f32(dev::absmax_f32(a, b)));
                }
            }
        } else {
            for (int64_t i = threadIdx.x; i < len; i += 256) m = max(m, elem_abs<ESIZE>(base, i, xs));
        }
    }
    if (cur >= 0) flush_max(m, p.acc, p.d[cur].out, red, accs);
}

// Zero the accumulators (a kernel rather than a memset, so that the next
// kernel of the chain can overlap its launch with this one).
__global__ void k_scale_zero(float *scale_out, int n, uint64_t out_bytes) {
    dev::pdl_entry();
    [[maybe_unused]] const dev::Span os{(uint64_t)scale_out, (uint64_t)scale_out + out_bytes};
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        if (FP8BQ_IN(os, scale_out + i, 4)) scale_out[i] = 0.0f;
}

__global__ void k_scale_finalize(float *scale_out, int n, uint64_t out_bytes) {
    dev::pdl_entry();
    [[maybe_unused]] const dev::Span os{(uint64_t)scale_out, (uint64_t)scale_out + out_bytes};
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (!FP8BQ_IN(os, scale_out + i, 4)) continue;
        const uint32_t bits = reinterpret_cast<const uint32_t *>(scale_out)[i];
        const float a = fmaxf(__uint_as_float(bits), kEps);
        scale_out[i] = __fdiv_rn(a, kFp8Max);
    }
}

}  // namespace

// Grid cap, in CTAs per SM (8 of these 256-thread CTAs are resident per SM):
// many short-lived CTAs, each starting at its descriptor by bisection, even
// out the SMs' finishing times.  Measured on B200 (Q/K/V activations, 201 MB
// / the whole weight set, 13.9 GB; fraction of the copy peak, a read-only
// pass may exceed it): 4 -> 0.92 / 1.07, 8 -> 0.955 / 1.07, 16 -> 0.95 /
// 1.07, 32 -> 0.98 / 1.05, 64 -> 0.97-0.98 / 1.10-1.11, 128 -> 0.972 /
// 1.130, 256 -> 0.972 / 1.108.
#ifndef FP8BQ_SCALE_CTAS_PER_SM
#define FP8BQ_SCALE_CTAS_PER_SM 128
#endif
template <int MAXD>
cudaError_t launch_scale_amax(const ScalePack<MAXD> &p, int esize, cudaStream_t st) {
    const uint64_t cap = (uint64_t)sm_count() * FP8BQ_SCALE_CTAS_PER_SM;
    const unsigned grid = (unsigned)(p.total < cap ? (p.total ? p.total : 1) : cap);
    return esize == 2 ? launch_kernel(k_scale_amax<2, MAXD>, grid, 256, 0, st, p)
                      : launch_kernel(k_scale_amax<4, MAXD>, grid, 256, 0, st, p);
}

cudaError_t launch_scale_zero(float *scale_out, int n, uint64_t out_bytes, cudaStream_t st) {
    const int blocks = (n + 255) / 256;
    return launch_kernel(k_scale_zero, blocks < 1 ? 1 : blocks, 256, 0, st, scale_out, n,
                         out_bytes);
}

cudaError_t launch_scale_finalize(float *scale_out, int n, uint64_t out_bytes, cudaStream_t st) {
    const int blocks = (n + 255) / 256;
    return launch_kernel(k_scale_finalize, blocks < 1 ? 1 : blocks, 256, 0, st, scale_out, n,
                         out_bytes);
}

template cudaError_t launch_scale_amax<kMaxDescSmall>(const ScalePack<kMaxDescSmall> &, int,
                                                      cudaStream_t);
template cudaError_t launch_scale_amax<kMaxDescLarge>(const ScalePack<kMaxDescLarge> &, int,
                                                      cudaStream_t);

FP8BQ_DEFINE_BOUNDS_RECORD(bounds_record_scale)

}  // namespace fp8bq

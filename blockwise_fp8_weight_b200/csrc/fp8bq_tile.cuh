// fp8bq_tile.cuh -- what the quantize kernels share: the tile of a grouped
// launch (a block, or G stacked blocks, of one tensor of the descriptor table),
// the block absmax on bit patterns, the scale of stacked blocks, the
// quantize-and-store of a 16-byte vector, and the host-side grid sizing.
#pragma once

#include "fp8bq_device.cuh"
#include "fp8bq_internal.h"

namespace fp8bq {

// Tile geometry shared by all kernels.
struct Tile {
    const char *src;  // first element of the block
    uint8_t *dst;     // first output byte of the block
    float *sdst;      // descale slot
    int64_t ld;       // input row stride, elements
    int64_t ldy;      // output row stride (= N)
    int rows, cols;   // valid extent
    int b, bi, bj;    // coordinates (TMA)
    int gn;           // descale row length (blocks per matrix row)
#if FP8BQ_CHECKED
    dev::Span xs, ys, ss;  // byte ranges of the tensor's x, y and s
#endif
};

// The tile whose first block is (bi, bj) of matrix b of descriptor D: grp
// vertically stacked blocks (H side by side); rows / cols count the valid
// extent of all of them and sdst points at the first block's descale.
template <int ESIZE, int H = 1>
__device__ __forceinline__ Tile tile_at(const TileDesc &D, uint32_t b, uint32_t bi, uint32_t bj,
                                        uint32_t grp) {
    const int64_t r0 = (int64_t)bi * D.bm, c0 = (int64_t)bj * D.bn;
    Tile T;
    T.src = (const char *)D.x + ((int64_t)b * D.xbs + r0 * D.ld + c0) * ESIZE;
    T.dst = D.y + (int64_t)b * D.ybs + r0 * D.N + c0;
    T.sdst = D.s + (int64_t)b * D.sbs + (int64_t)bi * D.gn + bj;
    T.ld = D.ld;
    T.ldy = D.N;
    T.rows = (int)min((int64_t)grp * D.bm, (int64_t)D.M - r0);
    T.cols = (int)min((int64_t)H * D.bn, (int64_t)D.N - c0);
    T.b = (int)b;
    T.bi = (int)bi;
    T.bj = (int)bj;
    T.gn = D.gn;
#if FP8BQ_CHECKED
    T.xs = {(uint64_t)D.x, (uint64_t)D.x + D.x_bytes};
    T.ys = {(uint64_t)D.y, (uint64_t)D.y + D.y_bytes};
    T.ss = {(uint64_t)D.s, (uint64_t)D.s + D.s_bytes};
#endif
    return T;
}

// Tile t of a launch.  A tile is G vertically adjacent blocks of one matrix
// (G = 1 except for the small-block kernels); d is a cursor into the
// descriptor table that only moves forward (tile ids grow along every walk).
template <int ESIZE, int G = 1, int MAXD, int H = 1>
__device__ __forceinline__ Tile make_tile(const DescPack<MAXD> &p, uint32_t t, int &d,
                                          int g_rt = 1) {
    while (t >= p.d[d].tile_begin + p.d[d].tiles) ++d;
    const TileDesc &D = p.d[d];
    const uint32_t local = t - D.tile_begin;
    // G is the compile-time group; g_rt a run-time one (used when G == 0);
    // H blocks side by side along N (the paired TMA kernel)
    const uint32_t grp = G == 0 ? (uint32_t)g_rt : (uint32_t)G;
    const uint32_t gmu = grp == 1 ? (uint32_t)D.gm : ((uint32_t)D.gm + grp - 1) / grp;
    const uint32_t gnu = H == 1 ? (uint32_t)D.gn : ((uint32_t)D.gn + H - 1) / H;
    const uint32_t per = gmu * gnu;
    const uint32_t b = local / per;
    const uint32_t rem = local - b * per;
    const uint32_t bgi = rem / gnu;
    return tile_at<ESIZE, H>(D, b, bgi * grp, (rem - bgi * gnu) * H, grp);
}

// The tiles t0, t0 + stride, t0 + 2 stride, ... of one team, visited in
// order.  make_tile pays two integer divisions per tile; here the position
// (matrix b, block-group row, block column) advances by the stride written in
// the mixed radix of the current descriptor (two compares, a few adds), and
// divisions are paid only when the walk enters another descriptor.
template <int ESIZE, int G, int MAXD>
struct TileCursor {
    const DescPack<MAXD> &p;
    const uint32_t stride;
    int d = 0;
    bool started = false;
    uint32_t local = 0, b = 0, bgi = 0, bj = 0;  // position within descriptor d
    uint32_t gmu = 1, gnu = 1;                     // its block-group rows and block columns
    uint32_t sa = 0, sb = 0, sc = 0;               // the stride in that radix

    __device__ __forceinline__ TileCursor(const DescPack<MAXD> &pk, uint32_t s) : p(pk), stride(s) {}

    __device__ __forceinline__ void seek(uint32_t t) {
        while (t >= p.d[d].tile_begin + p.d[d].tiles) ++d;
        const TileDesc &D = p.d[d];
        gmu = G == 1 ? (uint32_t)D.gm : ((uint32_t)D.gm + G - 1) / G;
        gnu = (uint32_t)D.gn;
        const uint32_t per = gmu * gnu;
        local = t - D.tile_begin;
        b = local / per;
        uint32_t rem = local - b * per;
        bgi = rem / gnu;
        bj = rem - bgi * gnu;
        sa = stride / per;
        rem = stride - sa * per;
        sb = rem / gnu;
        sc = rem - sb * gnu;
    }

    // The tile t (< total): the first call seeks, later ones must pass the
    // previous t + stride.
    __device__ __forceinline__ Tile next(uint32_t t) {
        if (!started) {
            started = true;
            seek(t);
        } else {
            local += stride;
            if (local >= p.d[d].tiles) {
                seek(t);
            } else {
                bj += sc;
                uint32_t c = bj >= gnu ? 1u : 0u;
                bj -= c * gnu;
                bgi += sb + c;
                c = bgi >= gmu ? 1u : 0u;
                bgi -= c * gmu;
                b += sa + c;
            }
        }
        return tile_at<ESIZE>(p.d[d], b, bgi * G, bj, G);
    }
};

// absmax bits of V 16-byte vectors: four independent running maxima (one per
// 32-bit lane of the vectors) so the max chains overlap, merged at the end.
template <int ESIZE, int V>
__device__ __forceinline__ uint32_t tile_absmax(const uint4 (&R)[V]) {
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        if constexpr (ESIZE == 2) {
            m0 = dev::absmax_bf16x2(m0, R[i].x);
            m1 = dev::absmax_bf16x2(m1, R[i].y);
            m2 = dev::absmax_bf16x2(m2, R[i].z);
            m3 = dev::absmax_bf16x2(m3, R[i].w);
        } else {
            m0 = dev::absmax_f32(m0, R[i].x);
            m1 = dev::absmax_f32(m1, R[i].y);
            m2 = dev::absmax_f32(m2, R[i].z);
            m3 = dev::absmax_f32(m3, R[i].w);
        }
    }
    if constexpr (ESIZE == 2)
        return dev::absmax_bf16x2(dev::absmax_bf16x2(m0, m1), dev::absmax_bf16x2(m2, m3));
    else
        return dev::absmax_f32(dev::absmax_f32(m0, m1), dev::absmax_f32(m2, m3));
}

// fp32 bit pattern of the absmax accumulated by tile_absmax
template <int ESIZE>
__device__ __forceinline__ uint32_t absmax_to_f32_bits(uint32_t m) {
    if constexpr (ESIZE == 2)
        return dev::absmax_bits_bf16x2(m);
    else
        return dev::absmax_bits_f32(m);
}

// Scales of V blocks whose absmax bits m[0..V-1] every lane of an aligned
// group of L >= V lanes already holds: lane q of the group computes block q
// (one division pair per lane instead of V), then every lane fetches the V
// reciprocals by shuffle.  Returns the scale of block (lane % L) (valid for
// lanes with lane % L < V, which write the descales).
template <int V>
__device__ __forceinline__ float group_scales(const uint32_t (&m)[V], int L, uint32_t mask,
                                              float (&r)[V]) {
    const int lane = threadIdx.x & 31;
    const int q = lane & (L - 1);
    uint32_t mq = m[0];
#pragma unroll
    for (int i = 1; i < V; ++i) mq = (q == i) ? m[i] : mq;
    float sq, rq;
    dev::block_scale(mq, kEps, sq, rq);
    const int base = lane & ~(L - 1);
#pragma unroll
    for (int i = 0; i < V; ++i) r[i] = __shfl_sync(mask, rq, base + i);
    return sq;
}

// Quantize one 16-byte vector with rr = {r, r} and store its codes (8 bytes
// for bf16, 4 for fp32).
template <int ESIZE>
__device__ __forceinline__ void vec_quant_store(const uint4 &v, uint64_t rr, uint8_t *dst) {
    if constexpr (ESIZE == 2) {
        uint2 o;
        o.x = dev::quant_bf16x4(v.x, v.y, rr);
        o.y = dev::quant_bf16x4(v.z, v.w, rr);
        dev::stg_stream_v2(dst, o);
    } else {
        dev::stg_stream_u32(dst, dev::quant_f32x4(v.x, v.y, v.z, v.w, rr));
    }
}

// The output stores of a tile (T: a Tile, or a kernel's own record of one
// with the same fields): the codes of one 16-byte vector, and one descale.
// In a checked build each is made only inside the tensor's byte range.
template <int ESIZE, typename TT>
__device__ __forceinline__ void store_codes(const TT &T, const uint4 &v, uint64_t rr, uint8_t *dst) {
    if (FP8BQ_IN(T.ys, dst, 16 / ESIZE)) vec_quant_store<ESIZE>(v, rr, dst);
}
template <typename TT>
__device__ __forceinline__ void store_descale(const TT &T, float *dst, float s) {
    if (FP8BQ_IN(T.ss, dst, 4)) *dst = s;
}

// ------------------------------------------------------------------ grid sizing (host)

template <typename K>
inline int resident_ctas(K kernel, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
        n < 1)
        n = 1;
    return n;
}

// Set-up of one kernel on one device: the dynamic shared-memory limit (when
// above the 48 KB default) and the resident CTAs per SM it allows.
struct KernelSetup {
    cudaError_t attr;
    int occ;
};

template <typename K>
inline KernelSetup setup_kernel(K kernel, int threads, size_t smem) {
    KernelSetup s{cudaSuccess, 1};
    if (smem > 48 * 1024)
        s.attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (s.attr == cudaSuccess) s.occ = resident_ctas(kernel, threads, smem);
    return s;
}

inline unsigned grid_for(uint32_t work_units, int units_per_cta, int ctas_per_sm) {
    const uint64_t need = (work_units + (uint32_t)units_per_cta - 1) / (uint32_t)units_per_cta;
    const uint64_t cap = (uint64_t)sm_count() * (uint64_t)ctas_per_sm;
    return (unsigned)(need < cap ? (need ? need : 1) : cap);
}

}  // namespace fp8bq

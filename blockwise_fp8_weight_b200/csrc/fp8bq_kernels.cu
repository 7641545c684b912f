// fp8bq_kernels.cu -- sm_100a kernels of the blockwise FP8 weight quantizer.
//
// Every kernel computes, for each [bm, bn] block of each tensor of a grouped
// launch (verl docs "fp8_kernel.py -- FP8 量化内核", section 2 "Triton 实现"):
//   a = max(max |x| over the block's valid elements, eps)
//   s = a / 448, r = 1 / s                (IEEE fp32 divisions)
//   y = e4m3fn(clamp(x * r, -448, 448))   (single-rounded multiply, RNE, satfinite)
//   descale = s
// The block absmax is taken on bit patterns: for a non-negative IEEE value the
// unsigned integer order of the bits equals the numeric order, so max over
// (bits & 0x7fff...) is exactly the fp32 absmax (bf16 is the top half of fp32).
//
// The pages' kernel runs one Triton program per block on a 2-D grid per tensor
// and one launch per tensor.  Here one persistent launch walks the tiles of
// all tensors of a group (the descriptor table travels in the kernel
// parameters); three variants share the arithmetic:
//   k_vector   16-byte coalesced global loads into registers, next tile
//              prefetched while the current one is reduced and stored;
//   k_tma      a producer warp streams 2-D TMA tiles into a shared-memory
//              ring, consumer warps reduce and quantize (bounded waits);
//   k_generic  element-wise loads, one warp per block: any alignment,
//              stride or block shape.
#include "fp8bq_device.cuh"
#include "fp8bq_internal.h"

namespace fp8bq {

// Bit 0: a consumer or producer wait ran out.  Bit 1: the end-of-kernel drain
// of in-flight TMA copies ran out.
__device__ uint32_t g_error_word;

constexpr uint64_t kDrainLimitNs = 2000000000ull;

// Tuning constants (compile-time; the defaults are the measured best on B200).
#ifndef FP8BQ_VEC_CTAS_PER_SM
#define FP8BQ_VEC_CTAS_PER_SM 2   // resident 256-thread vector CTAs per SM
#endif
// Depth of the vector kernel's cp.async ring (16-byte aligned rows), by team.
// Measured on B200 (stages 0 = register ping-pong / 2 / 3 / 4): [1,128] blocks
// 4.95 / 5.37 / 5.47 / 4.46 TB/s; [64,64] blocks 5.57 / 6.21 / 6.03 / 5.39;
// 128x128 blocks 5.63 / 6.22 / 6.20 / 5.23 (4 stages leave one CTA per SM).
#ifndef FP8BQ_VEC_STAGES_T16
#define FP8BQ_VEC_STAGES_T16 3
#endif
#ifndef FP8BQ_VEC_STAGES
#define FP8BQ_VEC_STAGES 2
#endif
#ifndef FP8BQ_TMA_STAGES_BF16
#define FP8BQ_TMA_STAGES_BF16 4   // 32 KB ring slots per TMA CTA (bf16 tiles)
#endif
#ifndef FP8BQ_TMA_STAGES_F32
#define FP8BQ_TMA_STAGES_F32 3    // 64 KB ring slots per TMA CTA (fp32 tiles)
#endif
#ifndef FP8BQ_TMA_CTAS_PER_SM
#define FP8BQ_TMA_CTAS_PER_SM 1   // resident TMA CTAs per SM
#endif

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
};

// Tile t of a launch.  A tile is G vertically adjacent blocks of one matrix
// (G = 1 except for the small-block vector kernel); rows counts the valid
// rows of all G blocks and sdst points at the first block's descale.
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
    const uint32_t bi = bgi * grp;
    const uint32_t bj = (rem - bgi * gnu) * H;
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
    return T;
}

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
            m0 = max(m0, R[i].x & 0x7fffffffu);
            m1 = max(m1, R[i].y & 0x7fffffffu);
            m2 = max(m2, R[i].z & 0x7fffffffu);
            m3 = max(m3, R[i].w & 0x7fffffffu);
        }
    }
    if constexpr (ESIZE == 2)
        return dev::absmax_bf16x2(dev::absmax_bf16x2(m0, m1), dev::absmax_bf16x2(m2, m3));
    else
        return max(max(m0, m1), max(m2, m3));
}

// fp32 bit pattern of the absmax accumulated by vec_absmax / tile_absmax
template <int ESIZE>
__device__ __forceinline__ uint32_t absmax_to_f32_bits(uint32_t m) {
    if constexpr (ESIZE == 2)
        return max(m & 0xffffu, m >> 16) << 16;
    else
        return m;
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

// Reduce-scatter of 8 per-lane maxima over an aligned team of 16 lanes:
// three halving exchange steps (xor 8, 4, 2) and one full step (xor 1).
// Afterwards team lane q holds the team-wide max of slot 4*b3 + 2*b2 + b1
// (b_k = bit k of q), i.e. slot q / 2; 8 shuffles instead of 32.
__device__ __forceinline__ uint32_t reduce_scatter8x16(const uint32_t (&m)[8], uint32_t mask,
                                                      int q) {
    const bool h3 = q & 8, h2 = q & 4, h1 = q & 2;
    uint32_t a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t send = h3 ? m[j] : m[j + 4];
        const uint32_t keep = h3 ? m[j + 4] : m[j];
        a[j] = max(keep, __shfl_xor_sync(mask, send, 8));
    }
    uint32_t b[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t send = h2 ? a[j] : a[j + 2];
        const uint32_t keep = h2 ? a[j + 2] : a[j];
        b[j] = max(keep, __shfl_xor_sync(mask, send, 4));
    }
    const uint32_t send = h1 ? b[0] : b[1];
    uint32_t c = max(h1 ? b[1] : b[0], __shfl_xor_sync(mask, send, 2));
    return max(c, __shfl_xor_sync(mask, c, 1));
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

// The same for a lane's 16 bytes held as two 8-byte halves (rows that are
// only 8-byte aligned): each half is quantized and stored on its own, the
// upper one only when hi_ok (it lies inside the row).  Codes: 4 bytes per
// bf16 half, 2 per fp32 half.
template <int ESIZE>
__device__ __forceinline__ void vec_quant_store_halves(const uint4 &v, uint64_t rr, uint8_t *dst,
                                                       bool hi_ok) {
    if constexpr (ESIZE == 2) {
        dev::stg_stream_u32(dst, dev::quant_bf16x4(v.x, v.y, rr));
        if (hi_ok) dev::stg_stream_u32(dst + 4, dev::quant_bf16x4(v.z, v.w, rr));
    } else {
        dev::stg_stream_u16(dst, dev::quant_pair_bits(v.x, v.y, rr));
        if (hi_ok) dev::stg_stream_u16(dst + 2, dev::quant_pair_bits(v.z, v.w, rr));
    }
}

// ============================================================== vector kernel
//
// A team of TEAM threads owns one block at a time; a block of bm x bn
// elements is bm rows of vpr = bn / VEC 16-byte vectors.  Thread `lane` of the
// team holds the vectors (row0 + i * rstep, cv), i < V, with cv = lane % vpr,
// row0 = lane / vpr, rstep = TEAM / vpr: consecutive lanes read consecutive
// 16-byte pieces of a row, so each warp load covers whole 256-byte row
// segments.  bm and bn are the same for every tensor of a launch.  The tile's
// vectors reach the registers through a per-thread cp.async ring in shared
// memory (S stages).

//
// G > 1 (small blocks): a tile is G vertically adjacent blocks and slot i of
// every thread holds a vector of block i (one block is exactly one row-step
// of the team, bm * vpr == TEAM), so each slot is reduced on its own.
//
// HALVES (rows only 8-byte aligned; N a multiple of VEC / 2): the same
// geometry, each 16-byte vector moved as two 8-byte halves; a half beyond
// the row end reads as zeros (no effect on the absmax) and is not stored.
//
// S > 0: the loads go through a private ring of S stages per thread in shared
// memory (cp.async; two 8-byte copies per vector in HALVES mode), S - 1 tiles
// in flight while one is reduced and stored.  S == 0: two register sets, the
// next tile loaded while the current one is processed.
template <int ESIZE, int TEAM, int V, int CTA, int G, int MAXD, bool HALVES, int S>
__global__ void __launch_bounds__(CTA, (CTA <= 256 ? FP8BQ_VEC_CTAS_PER_SM : 1))
    k_vector(const __grid_constant__ DescPack<MAXD> p) {
    dev::pdl_entry();
    static_assert(G == 1 || (G == 8 && V == 8 && TEAM == 16), "stacked blocks: 8 over 16 lanes");
    constexpr int VEC = 16 / ESIZE;
    constexpr int TEAMS = CTA / TEAM;
    constexpr int WPT = TEAM >= 32 ? TEAM / 32 : 1;
    __shared__ uint32_t red[2][TEAMS][WPT];

    const int team = threadIdx.x / TEAM;
    const int lane = threadIdx.x % TEAM;
    const uint32_t stride = gridDim.x * TEAMS;
    uint32_t t = blockIdx.x * TEAMS + team;
    if (t >= p.total_tiles) return;

    const int vpr = p.d[0].bn / VEC;  // power of two, <= TEAM (host-checked)
    const int cv = lane & (vpr - 1);
    const int row0 = lane / vpr;
    const int rstep = TEAM / vpr;
    const int colv = cv * VEC;
    const uint32_t shfl_mask =
        TEAM >= 32 ? 0xffffffffu : (((1u << TEAM) - 1u) << ((threadIdx.x & 31) & ~(TEAM - 1)));
    int d = 0;  // current descriptor; advances monotonically with the tile id

    // upper 8-byte half of this lane's vector inside the row (HALVES only)
    auto hi_ok = [&](const Tile &T) { return colv + VEC / 2 < T.cols; };
    auto store = [&](const uint4 &v, uint64_t rr, uint8_t *dst, const Tile &T) {
        if constexpr (HALVES)
            vec_quant_store_halves<ESIZE>(v, rr, dst, hi_ok(T));
        else
            vec_quant_store<ESIZE>(v, rr, dst);
    };

    auto load = [&](uint4 (&R)[V], const Tile &T) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int r = row0 + i * rstep;
            if (r < T.rows && colv < T.cols) {
                const char *a = T.src + ((int64_t)r * T.ld + colv) * ESIZE;
                if constexpr (HALVES) {
                    const uint2 lo = dev::ldg_v2(a);
                    const uint2 hi = hi_ok(T) ? dev::ldg_v2(a + 8) : make_uint2(0u, 0u);
                    R[i] = make_uint4(lo.x, lo.y, hi.x, hi.y);
                } else {
                    R[i] = dev::ldg_stream_v4(a);
                }
            } else {
                R[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };

    auto process_slots = [&](const uint4 (&R)[V], const Tile &T) {
      if constexpr (TEAM == 16 && V == 8) {  // the only stacked-block instantiation
        const int bm = p.d[0].bm;
        uint32_t m[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const uint4 one[1] = {R[i]};
            m[i] = absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE, 1>(one));
        }
        // lane q ends with the max of slot q / 2, computes its scale, and the
        // reciprocal of slot i is fetched from lane 2 i of the team
        const uint32_t mq = reduce_scatter8x16(m, shfl_mask, lane);
        float s_mine, r_mine;
        dev::block_scale(mq, kEps, s_mine, r_mine);
        const int base = (threadIdx.x & 31) & ~(TEAM - 1);
        float r[V];
#pragma unroll
        for (int i = 0; i < V; ++i) r[i] = __shfl_sync(shfl_mask, r_mine, base + 2 * i);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            if (i * bm >= T.rows) break;  // blocks below the matrix
            const int rr = row0 + i * rstep;
            if (rr < T.rows && colv < T.cols)
                store(R[i], dev::splat2(r[i]), T.dst + (int64_t)rr * T.ldy + colv, T);
        }
        const int slot = lane >> 1;
        if ((lane & 1) == 0 && slot * bm < T.rows) T.sdst[(int64_t)slot * T.gn] = s_mine;
      }
    };

    auto process = [&](const uint4 (&R)[V], const Tile &T, uint32_t it) {
        if constexpr (G > 1) {
            process_slots(R, T);
            return;
        }
        uint32_t m = absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE>(R));
        if constexpr (TEAM <= 32) {
#pragma unroll
            for (int o = TEAM / 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(shfl_mask, m, o));
        } else {
            m = __reduce_max_sync(0xffffffffu, m);
            if ((lane & 31) == 0) red[it & 1][team][lane >> 5] = m;
            dev::named_bar_sync(1 + team, TEAM);
            m = red[it & 1][team][0];
#pragma unroll
            for (int w = 1; w < WPT; ++w) m = max(m, red[it & 1][team][w]);
        }
        float s, r;
        dev::block_scale(m, kEps, s, r);
        const uint64_t r2 = dev::splat2(r);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int rr = row0 + i * rstep;
            if (rr < T.rows && colv < T.cols)
                store(R[i], r2, T.dst + (int64_t)rr * T.ldy + colv, T);
        }
        if (lane == 0) *T.sdst = s;
    };

    if constexpr (S > 0) {
        extern __shared__ __align__(1024) uint8_t ring[];  // dynamic shared memory
        uint4 *const stage = reinterpret_cast<uint4 *>(ring);  // [S][V][CTA] 16-byte vectors
        auto issue = [&](int s, const Tile &T) {
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int r = row0 + i * rstep;
                const bool ok = r < T.rows && colv < T.cols;
                const char *src = ok ? T.src + ((int64_t)r * T.ld + colv) * ESIZE : T.src;
                uint4 *dst = &stage[(s * V + i) * CTA + threadIdx.x];
                if constexpr (HALVES) {
                    const bool ok_hi = ok && hi_ok(T);
                    dev::cp_async_8(dst, src, ok);
                    dev::cp_async_8(reinterpret_cast<char *>(dst) + 8, ok_hi ? src + 8 : src,
                                    ok_hi);
                } else {
                    dev::cp_async_16(dst, src, ok);
                }
            }
            dev::cp_async_commit();
        };
        Tile Ts[S];
        uint32_t tn = t;  // next tile to issue; t: next tile to process
#pragma unroll
        for (int s = 0; s < S; ++s) {
            if (tn < p.total_tiles) {
                Ts[s] = make_tile<ESIZE, G>(p, tn, d);
                issue(s, Ts[s]);
            } else {
                dev::cp_async_commit();  // empty group: keeps the wait count uniform
            }
            tn += stride;
        }
        uint32_t it = 0;
        bool more = true;
        while (more) {
#pragma unroll
            for (int s = 0; s < S; ++s) {
                if (t >= p.total_tiles) {
                    more = false;
                    break;
                }
                dev::cp_async_wait<S - 1>();  // this thread's copies of stage s have landed
                uint4 R[V];
#pragma unroll
                for (int i = 0; i < V; ++i) R[i] = stage[(s * V + i) * CTA + threadIdx.x];
                process(R, Ts[s], it++);  // consumes R: the stage is free again
                if (tn < p.total_tiles) {
                    Ts[s] = make_tile<ESIZE, G>(p, tn, d);
                    issue(s, Ts[s]);
                } else {
                    dev::cp_async_commit();
                }
                tn += stride;
                t += stride;
            }
        }
        dev::cp_async_wait<0>();
        return;
    }

    uint4 A[V], B[V];
    Tile ta = make_tile<ESIZE, G>(p, t, d);
    load(A, ta);
    uint32_t it = 0;
    while (true) {
        const uint32_t t1 = t + stride;
        const bool h1 = t1 < p.total_tiles;
        Tile tb;
        if (h1) {
            tb = make_tile<ESIZE, G>(p, t1, d);
            load(B, tb);
        }
        process(A, ta, it++);
        if (!h1) break;
        const uint32_t t2 = t1 + stride;
        const bool h2 = t2 < p.total_tiles;
        if (h2) {
            ta = make_tile<ESIZE, G>(p, t2, d);
            load(A, ta);
        }
        process(B, tb, it++);
        if (!h2) break;
        t = t2;
    }
}

// ============================================================== generic kernel
//
// One warp per block, element-wise loads and byte stores: any row stride,
// alignment and block shape.  Two passes over the block (absmax, then
// quantize); the second pass reads the block again, mostly from L1/L2.

template <int ESIZE>
__device__ __forceinline__ uint32_t elem_abs_bits(const char *p) {
    if constexpr (ESIZE == 2)
        return ((uint32_t)__ldg((const unsigned short *)p) & 0x7fffu) << 16;
    else
        return __float_as_uint(__ldg((const float *)p)) & 0x7fffffffu;
}

template <int ESIZE>
__device__ __forceinline__ float elem_f32(const char *p) {
    if constexpr (ESIZE == 2)
        return __uint_as_float((uint32_t)__ldg((const unsigned short *)p) << 16);
    else
        return __ldg((const float *)p);
}

template <int ESIZE, int MAXD>
__global__ void __launch_bounds__(256) k_generic(const __grid_constant__ DescPack<MAXD> p) {
    dev::pdl_entry();
    const int lane = threadIdx.x & 31;
    const uint32_t stride = gridDim.x * 8;
    int d = 0;
    for (uint32_t t = blockIdx.x * 8 + (threadIdx.x >> 5); t < p.total_tiles; t += stride) {
        const Tile T = make_tile<ESIZE>(p, t, d);
        uint32_t m = 0;
        for (int r = 0; r < T.rows; ++r) {
            const char *row = T.src + (int64_t)r * T.ld * ESIZE;
#pragma unroll 4
            for (int c = lane; c < T.cols; c += 32) m = max(m, elem_abs_bits<ESIZE>(row + c * ESIZE));
        }
        m = __reduce_max_sync(0xffffffffu, m);
        float s, rc;
        dev::block_scale(m, kEps, s, rc);
        for (int r = 0; r < T.rows; ++r) {
            const char *row = T.src + (int64_t)r * T.ld * ESIZE;
            uint8_t *out = T.dst + (int64_t)r * T.ldy;
#pragma unroll 4
            for (int c = lane; c < T.cols; c += 32) {
                const float v = __fmul_rn(elem_f32<ESIZE>(row + c * ESIZE), rc);
                out[c] = (uint8_t)(dev::cvt_e4m3x2(v, 0.0f) & 0xffu);
            }
        }
        if (lane == 0) *T.sdst = s;
    }
}

// The same with the whole CTA on one block (blocks of >= 2048 elements): the
// 8 warps take alternate rows, so a block's loads are spread over 256
// threads instead of 32.
template <int ESIZE, int MAXD>
__global__ void __launch_bounds__(256) k_generic_cta(const __grid_constant__ DescPack<MAXD> p) {
    dev::pdl_entry();
    __shared__ uint32_t red[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int d = 0;
    for (uint32_t t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
        const Tile T = make_tile<ESIZE>(p, t, d);
        uint32_t m = 0;
        for (int r = warp; r < T.rows; r += 8) {
            const char *row = T.src + (int64_t)r * T.ld * ESIZE;
#pragma unroll 4
            for (int c = lane; c < T.cols; c += 32) m = max(m, elem_abs_bits<ESIZE>(row + c * ESIZE));
        }
        m = __reduce_max_sync(0xffffffffu, m);
        if (lane == 0) red[warp] = m;
        __syncthreads();
        m = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = max(m, red[w]);
        __syncthreads();  // red is rewritten by the next tile
        float s, rc;
        dev::block_scale(m, kEps, s, rc);
        for (int r = warp; r < T.rows; r += 8) {
            const char *row = T.src + (int64_t)r * T.ld * ESIZE;
            uint8_t *out = T.dst + (int64_t)r * T.ldy;
#pragma unroll 4
            for (int c = lane; c < T.cols; c += 32) {
                const float v = __fmul_rn(elem_f32<ESIZE>(row + c * ESIZE), rc);
                out[c] = (uint8_t)(dev::cvt_e4m3x2(v, 0.0f) & 0xffu);
            }
        }
        if (threadIdx.x == 0) *T.sdst = s;
    }
}

// The tiles one TMA CTA processes: every gridDim.x-th tile, starting at its
// own index (a contiguous run of tiles per CTA measured no better).
struct TileWalk {
    uint32_t t, end, step;
    __device__ __forceinline__ explicit TileWalk(uint32_t total)
        : t(blockIdx.x), end(total), step(gridDim.x) {}
};

// ============================================================== TMA kernel
//
// Warp 0 (one elected lane) is the producer: for each tile of this CTA it
// waits until the ring slot is free, arms the slot's "full" barrier with the
// tile's byte count and issues one 3-D tensor-map load (no multicast).  Warps
// 1..8 are consumers: they wait for "full", copy the tile from shared memory
// into registers, release the slot ("empty"), reduce the absmax, and quantize
// + store from registers.  Every wait is bounded; a wait that runs out sets
// the device error word, all consumers leave together (a barrier that also
// ORs a failure flag), and the producer waits (bounded) for each copy it
// issued before it returns.
//
// A tile is G vertically stacked blocks (one ring slot of up to 32 KB of bf16
// / 64 KB of fp32; G = 1 for 128x128 blocks).  Consumer thread ct holds the
// 16-byte vectors (row0 + i * RS, cv), i < V, of the tile, RS = 256 / vpr.
//   MODE_ONE  (G = 1): the tile is one block, reduced across the 8 consumer
//             warps (the 128x128 case).
//   MODE_CTA  (bm a multiple of RS, G > 1): slot i belongs to block
//             i / (bm / RS); each block is reduced across the 8 warps.
//   MODE_SUB  (a block is L = bm * vpr <= 32 lanes of one slot): each slot is
//             reduced within its group of L lanes with shuffles.
enum { MODE_ONE = 0, MODE_SUB = 1, MODE_CTA = 2 };

template <int ESIZE, int STAGES, int MODE, int MAXD, bool EF>
__global__ void __launch_bounds__(32 + kTmaConsumerThreads, FP8BQ_TMA_CTAS_PER_SM)
    k_tma(const __grid_constant__ TmaPack<MAXD> P) {
    dev::pdl_entry();
    constexpr int VEC = 16 / ESIZE;
    constexpr int STAGE_BYTES = 128 * 128 * ESIZE;
    constexpr int V = STAGE_BYTES / 16 / kTmaConsumerThreads;
    constexpr int NW = kTmaConsumerThreads / 32;
    extern __shared__ __align__(1024) uint8_t ring[];
    // Where each slot's tile goes: written by the producer before it arms the
    // slot's barrier, read by the consumers after the barrier completes.
    struct SlotInfo {
        uint8_t *dst;
        float *sdst;
        int64_t ldy;
        int32_t rows, cols, gn, pad;
    };
    __shared__ SlotInfo info[STAGES];
    __shared__ __align__(8) uint64_t full[STAGES];
    __shared__ __align__(8) uint64_t empty[STAGES];
    __shared__ uint32_t red[2][V][NW];
    __shared__ volatile int abort_flag;

    const DescPack<MAXD> &p = P.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            dev::mbar_init(&full[s], 1);
            dev::mbar_init(&empty[s], NW);
        }
        abort_flag = 0;
        dev::fence_mbar_init();
    }
    __syncthreads();

    const int bm = p.d[0].bm, bn = p.d[0].bn, grp = p.group;
    const uint32_t tile_bytes = (uint32_t)(grp * bm * bn * ESIZE);

    if (warp == 0) {
        if (lane != 0) return;
        int d = 0;
        uint32_t k = 0;
        bool dropped0 = false;
        for (TileWalk w(p.total_tiles); w.t < w.end; w.t += w.step, ++k) {
            const int st = (int)(k % STAGES);
            const uint32_t round = k / STAGES;
            if (round > 0 &&
                !dev::mbar_wait_bounded(&empty[st], (round - 1) & 1u, p.wait_limit_ns, &abort_flag)) {
                if (!abort_flag) {
                    atomicOr(&g_error_word, 1u);
                    abort_flag = 1;
                }
                break;
            }
            const Tile T = make_tile<ESIZE, 0>(p, w.t, d, grp);
            info[st].dst = T.dst;
            info[st].sdst = T.sdst;
            info[st].ldy = T.ldy;
            info[st].rows = T.rows;
            info[st].cols = T.cols;
            info[st].gn = p.d[d].gn;
            dev::mbar_arrive_expect_tx(&full[st], tile_bytes);
            if ((p.inject & 1u) && blockIdx.x == 0 && k == 0)
                dropped0 = true;  // fault injection: this slot's barrier can never complete
            else
                dev::tma_load_3d(ring + (size_t)st * STAGE_BYTES, &P.maps[d], &full[st],
                                 T.bj * bn, T.bi * bm, T.b, EF);
        }
        // Drain: each slot's last issued copy must land before the CTA exits.
        const uint32_t issued = k;
        for (int st = 0; st < STAGES && (uint32_t)st < issued; ++st) {
            const uint32_t fills = (issued - (uint32_t)st + STAGES - 1) / STAGES;
            if (dropped0 && st == 0 && fills == 1) continue;
            if (!dev::mbar_wait_bounded(&full[st], (fills - 1) & 1u, kDrainLimitNs, nullptr))
                atomicOr(&g_error_word, 2u);
        }
        return;
    }

    // consumers
    const int ct = threadIdx.x - 32;
    const int cw = ct >> 5;
    const int vpr = bn / VEC;
    const int cv = ct & (vpr - 1);
    const int row0 = ct / vpr;
    const int rstep = kTmaConsumerThreads / vpr;
    const int colv = cv * VEC;
    const int box_rows = grp * bm;
    // MODE_CTA: slots per block; MODE_SUB: lanes per block
    const int spb = MODE == MODE_SUB ? 1 : bm / rstep;
    const int L = MODE == MODE_SUB ? bm * vpr : 32;
    const uint32_t sub_mask =
        L >= 32 ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    uint32_t k = 0;
    for (TileWalk w(p.total_tiles); w.t < w.end; w.t += w.step, ++k) {
        const int st = (int)(k % STAGES);
        const bool ok = dev::mbar_wait_bounded(&full[st], (k / STAGES) & 1u, p.wait_limit_ns,
                                               &abort_flag);
        SlotInfo T = {nullptr, nullptr, 0, 0, 0, 0, 0};
        if (ok) T = info[st];
        uint4 R[V];
        const uint8_t *stage = ring + (size_t)st * STAGE_BYTES;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int r = row0 + i * rstep;
            if (ok && r < box_rows)
                R[i] = *reinterpret_cast<const uint4 *>(stage + ((size_t)r * bn + colv) * ESIZE);
            else
                R[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        if (lane == 0 && ok) dev::mbar_arrive(&empty[st]);

        if constexpr (MODE != MODE_SUB) {
            if (MODE == MODE_ONE) {  // one block per tile: one CTA-wide reduction
                uint32_t m = __reduce_max_sync(0xffffffffu,
                                               absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE>(R)));
                if (lane == 0) red[k & 1][0][cw] = m;
            } else {  // per-slot warp maxima; a block's slots are combined below
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const uint4 one[1] = {R[i]};
                    const uint32_t m = __reduce_max_sync(
                        0xffffffffu, absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE, 1>(one)));
                    if (lane == 0) red[k & 1][i][cw] = m;
                }
            }
            if (dev::named_bar_or(1, kTmaConsumerThreads, !ok)) {
                if (ct == 0) {
                    atomicOr(&g_error_word, 1u);
                    abort_flag = 1;
                }
                break;
            }
            if (MODE == MODE_ONE) {
                uint32_t m = red[k & 1][0][0];
#pragma unroll
                for (int ww = 1; ww < NW; ++ww) m = max(m, red[k & 1][0][ww]);
                float s, r;
                dev::block_scale(m, kEps, s, r);
                const uint64_t r2 = dev::splat2(r);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int rr = row0 + i * rstep;
                    if (rr < T.rows && colv < T.cols)
                        vec_quant_store<ESIZE>(R[i], r2, T.dst + (int64_t)rr * T.ldy + colv);
                }
                if (ct == 0) *T.sdst = s;
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int j = i / spb;  // block of slot i
                    if (j >= grp || j * bm >= T.rows) continue;
                    uint32_t m = 0;
                    for (int i2 = j * spb; i2 < (j + 1) * spb; ++i2)
                        for (int ww = 0; ww < NW; ++ww) m = max(m, red[k & 1][i2][ww]);
                    float s, r;
                    dev::block_scale(m, kEps, s, r);
                    const int rr = row0 + i * rstep;
                    if (rr < T.rows && colv < T.cols)
                        vec_quant_store<ESIZE>(R[i], dev::splat2(r),
                                               T.dst + (int64_t)rr * T.ldy + colv);
                    if (ct == 0 && i == j * spb) T.sdst[(int64_t)j * T.gn] = s;
                }
            }
        } else {
            if (dev::named_bar_or(1, kTmaConsumerThreads, !ok)) {
                if (ct == 0) {
                    atomicOr(&g_error_word, 1u);
                    abort_flag = 1;
                }
                break;
            }
            uint32_t m[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const uint4 one[1] = {R[i]};
                m[i] = absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE, 1>(one));
                for (int o = L / 2; o > 0; o >>= 1)
                    m[i] = max(m[i], __shfl_xor_sync(sub_mask, m[i], o));
            }
            if (L >= V) {  // one division pair per lane, reciprocals by shuffle
                float r[V];
                const float s_mine = group_scales<V>(m, L, sub_mask, r);
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int rr = row0 + i * rstep;
                    if (rr < T.rows && colv < T.cols)
                        vec_quant_store<ESIZE>(R[i], dev::splat2(r[i]),
                                               T.dst + (int64_t)rr * T.ldy + colv);
                }
                const int q = ct & (L - 1);  // this lane's block: slot q of its group
                if (q < V) {
                    const int blk = (row0 + q * rstep) / bm;
                    if (blk * bm < T.rows) T.sdst[(int64_t)blk * T.gn] = s_mine;
                }
            } else {
#pragma unroll
                for (int i = 0; i < V; ++i) {
                    const int rr = row0 + i * rstep;
                    const int blk = rr / bm;
                    if (blk * bm >= T.rows) continue;  // block below the matrix
                    float s, r;
                    dev::block_scale(m[i], kEps, s, r);
                    if (rr < T.rows && colv < T.cols)
                        vec_quant_store<ESIZE>(R[i], dev::splat2(r),
                                               T.dst + (int64_t)rr * T.ldy + colv);
                    if ((ct & (L - 1)) == 0) T.sdst[(int64_t)blk * T.gn] = s;
                }
            }
        }
    }
}

// ============================================================== paired TMA kernel
//
// The 128x128 bf16 case with two horizontally adjacent blocks per ring slot
// (box {256, 128}: each row of the tile is 512 contiguous bytes, half the TMA
// issues and barrier round trips per byte).  Consumer lane l of a warp holds
// columns of block (l / 16); each block is reduced over its 16 lanes of all 8
// warps.  Same bounded waits, failure handling and drain as k_tma.
#ifndef FP8BQ_TMA_PAIR_STAGES
#define FP8BQ_TMA_PAIR_STAGES 2   // 64 KB ring slots (3 measured 12 % slower)
#endif

template <int STAGES, int MAXD, bool EF>
__global__ void __launch_bounds__(32 + kTmaConsumerThreads, 1)
    k_tma_pair(const __grid_constant__ TmaPack<MAXD> P) {
    dev::pdl_entry();
    constexpr int ESIZE = 2, VEC = 8, BN = 128, BM = 128;
    constexpr int COLS = 2 * BN;                           // tile columns
    constexpr int STAGE_BYTES = BM * COLS * ESIZE;         // 64 KB
    constexpr int VPR = COLS / VEC;                        // 32 vectors per row
    constexpr int RSTEP = kTmaConsumerThreads / VPR;       // 8 rows per step
    constexpr int V = BM / RSTEP;                          // 16 vectors per thread
    constexpr int NW = kTmaConsumerThreads / 32;
    extern __shared__ __align__(1024) uint8_t ring[];
    struct SlotInfo {
        uint8_t *dst;
        float *sdst;
        int64_t ldy;
        int32_t rows, cols;
    };
    __shared__ SlotInfo info[STAGES];
    __shared__ __align__(8) uint64_t full[STAGES];
    __shared__ __align__(8) uint64_t empty[STAGES];
    __shared__ uint32_t red[2][2][NW];
    __shared__ volatile int abort_flag;

    const DescPack<MAXD> &p = P.p;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            dev::mbar_init(&full[s], 1);
            dev::mbar_init(&empty[s], NW);
        }
        abort_flag = 0;
        dev::fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        if (lane != 0) return;
        int d = 0;
        uint32_t k = 0;
        bool dropped0 = false;
        for (TileWalk w(p.total_tiles); w.t < w.end; w.t += w.step, ++k) {
            const int st = (int)(k % STAGES);
            const uint32_t round = k / STAGES;
            if (round > 0 &&
                !dev::mbar_wait_bounded(&empty[st], (round - 1) & 1u, p.wait_limit_ns, &abort_flag)) {
                if (!abort_flag) {
                    atomicOr(&g_error_word, 1u);
                    abort_flag = 1;
                }
                break;
            }
            const Tile T = make_tile<ESIZE, 1, MAXD, 2>(p, w.t, d);
            info[st].dst = T.dst;
            info[st].sdst = T.sdst;
            info[st].ldy = T.ldy;
            info[st].rows = T.rows;
            info[st].cols = T.cols;
            dev::mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
            if ((p.inject & 1u) && blockIdx.x == 0 && k == 0)
                dropped0 = true;
            else
                dev::tma_load_3d(ring + (size_t)st * STAGE_BYTES, &P.maps[d], &full[st],
                                 T.bj * BN, T.bi * BM, T.b, EF);
        }
        const uint32_t issued = k;
        for (int st = 0; st < STAGES && (uint32_t)st < issued; ++st) {
            const uint32_t fills = (issued - (uint32_t)st + STAGES - 1) / STAGES;
            if (dropped0 && st == 0 && fills == 1) continue;
            if (!dev::mbar_wait_bounded(&full[st], (fills - 1) & 1u, kDrainLimitNs, nullptr))
                atomicOr(&g_error_word, 2u);
        }
        return;
    }

    const int ct = threadIdx.x - 32;
    const int cw = ct >> 5;
    const int cv = ct & (VPR - 1);      // = lane
    const int half = cv >> 4;           // block of this lane's columns
    const int row0 = ct / VPR;          // = consumer warp index
    const int colv = cv * VEC;          // column within the tile
    const uint32_t hmask = half ? 0xffff0000u : 0x0000ffffu;
    uint32_t k = 0;
    for (TileWalk w(p.total_tiles); w.t < w.end; w.t += w.step, ++k) {
        const int st = (int)(k % STAGES);
        const bool ok = dev::mbar_wait_bounded(&full[st], (k / STAGES) & 1u, p.wait_limit_ns,
                                               &abort_flag);
        SlotInfo T = {nullptr, nullptr, 0, 0, 0};
        if (ok) T = info[st];
        uint4 R[V];
        const uint8_t *stage = ring + (size_t)st * STAGE_BYTES;
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int r = row0 + i * RSTEP;
            R[i] = ok ? *reinterpret_cast<const uint4 *>(stage + ((size_t)r * COLS + colv) * ESIZE)
                      : make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        if (lane == 0 && ok) dev::mbar_arrive(&empty[st]);

        uint32_t m = absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE>(R));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(hmask, m, o));
        if ((lane & 15) == 0) red[k & 1][half][cw] = m;
        if (dev::named_bar_or(1, kTmaConsumerThreads, !ok)) {
            if (ct == 0) {
                atomicOr(&g_error_word, 1u);
                abort_flag = 1;
            }
            break;
        }
        m = red[k & 1][half][0];
#pragma unroll
        for (int ww = 1; ww < NW; ++ww) m = max(m, red[k & 1][half][ww]);
        if (half * BN >= T.cols) continue;  // second block beyond the matrix
        float s, r;
        dev::block_scale(m, kEps, s, r);
        const uint64_t r2 = dev::splat2(r);
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int rr = row0 + i * RSTEP;
            if (rr < T.rows && colv < T.cols)
                vec_quant_store<ESIZE>(R[i], r2, T.dst + (int64_t)rr * T.ldy + colv);
        }
        if ((ct & 15) == 0 && ct < 32) T.sdst[half] = s;
    }
}

// ============================================================== launchers

namespace {

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <typename K>
int resident_ctas(K kernel, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
        n < 1)
        n = 1;
    return n;
}

unsigned grid_for(uint32_t work_units, int units_per_cta, int ctas_per_sm) {
    const uint64_t need = (work_units + (uint32_t)units_per_cta - 1) / (uint32_t)units_per_cta;
    const uint64_t cap = (uint64_t)sm_count() * (uint64_t)ctas_per_sm;
    return (unsigned)(need < cap ? (need ? need : 1) : cap);
}

template <int ESIZE, int TEAM, int V, int CTA, int G, int MAXD, bool HALVES>
cudaError_t launch_vector_h(const DescPack<MAXD> &p, cudaStream_t st) {
    constexpr int S = TEAM == 16 ? FP8BQ_VEC_STAGES_T16 : FP8BQ_VEC_STAGES;
    constexpr size_t smem = (size_t)S * V * CTA * 16;
    auto kern = k_vector<ESIZE, TEAM, V, CTA, G, MAXD, HALVES, S>;
    if constexpr (smem > 48 * 1024) {
        static cudaError_t attr =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (attr != cudaSuccess) return attr;
    }
    static int occ = resident_ctas(kern, CTA, smem);
    const unsigned grid = grid_for(p.total_tiles, CTA / TEAM, occ);
    return launch_kernel(kern, grid, CTA, smem, st, p);
}

template <int ESIZE, int TEAM, int V, int CTA, int G, int MAXD>
cudaError_t launch_vector_t(bool halves, const DescPack<MAXD> &p, cudaStream_t st) {
    return halves ? launch_vector_h<ESIZE, TEAM, V, CTA, G, MAXD, true>(p, st)
                  : launch_vector_h<ESIZE, TEAM, V, CTA, G, MAXD, false>(p, st);
}

}  // namespace

template <int MAXD>
cudaError_t launch_vector(Variant v, int esize, bool halves, const DescPack<MAXD> &p,
                          cudaStream_t st) {
    if (esize == 2) {
        switch (v) {
            case Variant::VecT16: return launch_vector_t<2, 16, 8, 256, 8, MAXD>(halves, p, st);
            case Variant::VecT64: return launch_vector_t<2, 64, 8, 256, 1, MAXD>(halves, p, st);
            case Variant::VecTBig: return launch_vector_t<2, 256, 8, 256, 1, MAXD>(halves, p, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (v) {
        case Variant::VecT16: return launch_vector_t<4, 16, 8, 256, 8, MAXD>(halves, p, st);
        case Variant::VecT64: return launch_vector_t<4, 64, 8, 256, 1, MAXD>(halves, p, st);
        case Variant::VecTBig: return launch_vector_t<4, 512, 8, 512, 1, MAXD>(halves, p, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int MAXD>
cudaError_t launch_generic(int esize, const DescPack<MAXD> &p, cudaStream_t st) {
    // blocks of >= 2048 elements take one CTA each (the host groups generic
    // tensors by this size class, so it is uniform per launch)
    const bool cta = (int64_t)p.d[0].bm * p.d[0].bn >= 2048;
    cudaError_t e;
    if (esize == 2) {
        if (cta) {
            static int occ = resident_ctas(k_generic_cta<2, MAXD>, 256, 0);
            e = launch_kernel(k_generic_cta<2, MAXD>, grid_for(p.total_tiles, 1, occ), 256, 0, st,
                              p);
        } else {
            static int occ = resident_ctas(k_generic<2, MAXD>, 256, 0);
            e = launch_kernel(k_generic<2, MAXD>, grid_for(p.total_tiles, 8, occ), 256, 0, st, p);
        }
    } else {
        if (cta) {
            static int occ = resident_ctas(k_generic_cta<4, MAXD>, 256, 0);
            e = launch_kernel(k_generic_cta<4, MAXD>, grid_for(p.total_tiles, 1, occ), 256, 0, st,
                              p);
        } else {
            static int occ = resident_ctas(k_generic<4, MAXD>, 256, 0);
            e = launch_kernel(k_generic<4, MAXD>, grid_for(p.total_tiles, 8, occ), 256, 0, st, p);
        }
    }
    return e;
}

namespace {
template <int ESIZE, int STAGES, int MODE, int MAXD, bool EF>
cudaError_t launch_tma_e(const TmaPack<MAXD> &p, cudaStream_t st) {
    constexpr size_t smem = (size_t)STAGES * 128 * 128 * ESIZE;
    auto kern = k_tma<ESIZE, STAGES, MODE, MAXD, EF>;
    static cudaError_t attr =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    static int occ = resident_ctas(kern, 32 + kTmaConsumerThreads, smem);
    return launch_kernel(kern, grid_for(p.p.total_tiles, 1, occ), 32 + kTmaConsumerThreads, smem,
                         st, p);
}

// The L2 policy of the tile loads is a template parameter, so the default
// kernels carry no trace of the other policy.
template <int ESIZE, int STAGES, int MODE, int MAXD>
cudaError_t launch_tma_t(const TmaPack<MAXD> &p, cudaStream_t st) {
    return p.evict_first ? launch_tma_e<ESIZE, STAGES, MODE, MAXD, true>(p, st)
                         : launch_tma_e<ESIZE, STAGES, MODE, MAXD, false>(p, st);
}

template <int MAXD, bool EF>
cudaError_t launch_tma_pair_e(const TmaPack<MAXD> &p, cudaStream_t st) {
    constexpr int S = FP8BQ_TMA_PAIR_STAGES;
    constexpr size_t smem = (size_t)S * 128 * 256 * 2;
    auto kern = k_tma_pair<S, MAXD, EF>;
    static cudaError_t attr =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    static int occ = resident_ctas(kern, 32 + kTmaConsumerThreads, smem);
    return launch_kernel(kern, grid_for(p.p.total_tiles, 1, occ), 32 + kTmaConsumerThreads, smem,
                         st, p);
}
}  // namespace

template <int MAXD>
cudaError_t launch_tma_pair(const TmaPack<MAXD> &p, cudaStream_t st) {
    return p.evict_first ? launch_tma_pair_e<MAXD, true>(p, st)
                         : launch_tma_pair_e<MAXD, false>(p, st);
}

template <int MAXD>
cudaError_t launch_tma(int esize, bool subwarp, const TmaPack<MAXD> &p, cudaStream_t st) {
    const int mode = subwarp ? MODE_SUB : p.p.group == 1 ? MODE_ONE : MODE_CTA;
    if (esize == 2) {
        constexpr int S = FP8BQ_TMA_STAGES_BF16;
        return mode == MODE_ONE   ? launch_tma_t<2, S, MODE_ONE, MAXD>(p, st)
               : mode == MODE_SUB ? launch_tma_t<2, S, MODE_SUB, MAXD>(p, st)
                                  : launch_tma_t<2, S, MODE_CTA, MAXD>(p, st);
    }
    constexpr int S = FP8BQ_TMA_STAGES_F32;
    return mode == MODE_ONE   ? launch_tma_t<4, S, MODE_ONE, MAXD>(p, st)
           : mode == MODE_SUB ? launch_tma_t<4, S, MODE_SUB, MAXD>(p, st)
                              : launch_tma_t<4, S, MODE_CTA, MAXD>(p, st);
}

template cudaError_t launch_tma<kMaxDescSmall>(int, bool, const TmaPack<kMaxDescSmall> &,
                                               cudaStream_t);
template cudaError_t launch_tma<kMaxDescTma>(int, bool, const TmaPack<kMaxDescTma> &, cudaStream_t);
template cudaError_t launch_tma_pair<kMaxDescSmall>(const TmaPack<kMaxDescSmall> &, cudaStream_t);
template cudaError_t launch_tma_pair<kMaxDescTma>(const TmaPack<kMaxDescTma> &, cudaStream_t);

cudaError_t read_and_clear_error_word(uint32_t *out) {
    uint32_t zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_error_word, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (*out) e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t));
    return e;
}

template cudaError_t launch_vector<kMaxDescSmall>(Variant, int, bool,
                                                  const DescPack<kMaxDescSmall> &,
                                                  cudaStream_t);
template cudaError_t launch_vector<kMaxDescLarge>(Variant, int, bool,
                                                  const DescPack<kMaxDescLarge> &,
                                                  cudaStream_t);
template cudaError_t launch_generic<kMaxDescSmall>(int, const DescPack<kMaxDescSmall> &,
                                                   cudaStream_t);
template cudaError_t launch_generic<kMaxDescLarge>(int, const DescPack<kMaxDescLarge> &,
                                                   cudaStream_t);

}  // namespace fp8bq

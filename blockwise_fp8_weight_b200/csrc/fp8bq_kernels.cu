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
//   k_vector   16-byte coalesced vectors staged through a per-thread cp.async
//              ring (rows only 8-byte aligned: two 8-byte loads per vector
//              straight into registers) (this file);
//   k_tma      a producer warp streams 3-D TMA tiles into a shared-memory
//              ring, consumer warps reduce and quantize (fp8bq_tma.cu);
//   k_generic  element-wise loads, one warp per block: any alignment,
//              stride or block shape (this file).
#include "fp8bq_tile.cuh"

namespace fp8bq {

// Tuning constants (compile-time; the defaults are the measured best on B200).
// Grid cap of the vector kernel in waves of resident CTAs: the team-of-16
// kernel (stacked small blocks) runs two, the others one.  Measured on B200
// (same box, one wave / two / three, fraction of the copy peak): [1,128]
// blocks 0.86-0.88 / 0.93-0.94 / 0.90; [64,64] blocks 0.95 / 0.95 / 0.93;
// bf16 4096x4096 0.94 / 0.96-0.97 / 0.84; bf16 4000x4100 0.80 / 0.83 / 0.75,
// sixteen of them in one call 0.86 / 0.81 / 0.83; the per-tensor loop over
// the Qwen3-8B-shaped weight set 0.830 / 0.816 / 0.79 -- a second wave of
// short-lived CTAs evens out the SMs' finishing times of some launches and
// costs others their ring's warm-up, so only the 1 x 128 case, which gains
// most, takes it.
#ifndef FP8BQ_VEC_WAVES
#define FP8BQ_VEC_WAVES 1
#endif
#ifndef FP8BQ_VEC_WAVES_T16
#define FP8BQ_VEC_WAVES_T16 2
#endif
// Short launches of the other vector kernels (fewer than 8 tiles per
// resident team) take two waves as well: measured on B200 (same box, one
// wave / two), bf16 4096x4096 0.93 / 0.95-0.97, the edge set 0.88 / 0.89-0.90,
// bf16 4000x4100 0.79-0.80 / 0.77-0.82; the long launches keep one wave
// (sixteen 4000x4100, [64,64] blocks and the per-tensor loop unchanged).
#ifndef FP8BQ_VEC_WAVES_SHORT
#define FP8BQ_VEC_WAVES_SHORT 2
#endif
#ifndef FP8BQ_VEC_SHORT_TILES
#define FP8BQ_VEC_SHORT_TILES 8
#endif
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

// The same over the 32 lanes of a warp: three halving steps (xor 16, 8, 4)
// and two full ones (xor 2, 1); lane q ends with the team-wide max of slot
// 4*b4 + 2*b3 + b2, i.e. slot q / 4.
__device__ __forceinline__ uint32_t reduce_scatter8x32(const uint32_t (&m)[8], int q) {
    const bool h4 = q & 16, h3 = q & 8, h2 = q & 4;
    uint32_t a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t send = h4 ? m[j] : m[j + 4];
        const uint32_t keep = h4 ? m[j + 4] : m[j];
        a[j] = max(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
    uint32_t b[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t send = h3 ? a[j] : a[j + 2];
        const uint32_t keep = h3 ? a[j + 2] : a[j];
        b[j] = max(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
    const uint32_t send = h2 ? b[0] : b[1];
    uint32_t c = max(h2 ? b[1] : b[0], __shfl_xor_sync(0xffffffffu, send, 4));
    c = max(c, __shfl_xor_sync(0xffffffffu, c, 2));
    return max(c, __shfl_xor_sync(0xffffffffu, c, 1));
}

// vec_quant_store for a lane's 16 bytes held as two 8-byte halves (rows that
// are only 8-byte aligned): each half is quantized and stored on its own, the
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
// segments.  bm and bn are the same for every tensor of a launch.

//
// G > 1 (small blocks): a tile is G vertically adjacent blocks and slot i of
// every thread holds a vector of block i (one block is exactly one row-step
// of the team, bm * vpr == TEAM), so each slot is reduced on its own.
//
// HALVES (rows only 8-byte aligned; N a multiple of VEC / 2): the same
// geometry, each 16-byte vector moved as two 8-byte halves; a half beyond
// the row end reads as zeros (no effect on the absmax) and is not stored.
//
// S > 0 (16-byte aligned rows): the loads go through a private ring of S
// stages per thread in shared memory (cp.async), S - 1 tiles in flight while
// one is reduced and stored.  S == 0 (HALVES): two register sets, the next
// tile loaded while the current one is processed.  Measured and dropped for
// HALVES: a ring of 8-byte cp.async copies (4.10 against 4.38-4.65 TB/s), and
// a ring of 16-byte copies from the aligned addresses of rows that start 8
// bytes past a 16-byte boundary, reassembled in shared memory or by shuffle
// (2971-3505 against 5016-5293 GB/s on bf16 4000x4100: divergent even/odd
// rows within a warp, 40 % bank conflicts or a shuffle pair per vector); and
// warps that take rows of one 16-byte alignment (rows w, w + 8, ... of a
// row-step), so that the aligned rows' warps load whole 16-byte vectors and
// store whole 8-byte code runs (0.79-0.80 / 0.81 against 0.81 / 0.86 of the
// copy peak on one / sixteen bf16 4000x4100, same box).
template <int ESIZE, int TEAM, int V, int CTA, int G, int MAXD, bool HALVES, int S>
__global__ void __launch_bounds__(CTA, (CTA <= 256 ? FP8BQ_VEC_CTAS_PER_SM : 1))
    k_vector(const __grid_constant__ DescPack<MAXD> p) {
    dev::pdl_entry();
    static_assert(G == 1 || (G == 8 && V == 8 && (TEAM == 16 || TEAM == 32)),
                  "stacked blocks: 8 over 16 or 32 lanes");
    static_assert(!(HALVES && S > 0), "the cp.async ring takes 16-byte vectors only");
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
    TileCursor<ESIZE, G, MAXD> walk(p, stride);  // the tiles this team loads, in order

    // upper 8-byte half of this lane's vector inside the row (HALVES only)
    auto hi_ok = [&](const Tile &T) { return colv + VEC / 2 < T.cols; };
    auto store = [&](const Tile &T, const uint4 &v, uint64_t rr, uint8_t *dst, bool hi) {
        if constexpr (HALVES) {
            if (FP8BQ_IN(T.ys, dst, hi ? VEC : VEC / 2))
                vec_quant_store_halves<ESIZE>(v, rr, dst, hi);
        } else {
            store_codes<ESIZE>(T, v, rr, dst);
        }
    };
    // Every slot of every lane of the team lies inside the tile (the same for
    // the whole team): the interior tiles skip the per-vector bounds checks.
    auto is_full = [&](const Tile &T) { return T.rows >= V * rstep && T.cols >= vpr * VEC; };
    // Quantize and store slot i of every lane for i < nb (the slots of blocks
    // inside the matrix), with the reciprocal rr(i).
    auto store_all = [&](const uint4 (&R)[V], const Tile &T, int nb, auto rr_of) {
        uint8_t *dst = T.dst + (int64_t)row0 * T.ldy + colv;
        const int64_t ystep = (int64_t)rstep * T.ldy;
        if (is_full(T)) {
#pragma unroll
            for (int i = 0; i < V; ++i) store(T, R[i], rr_of(i), dst + i * ystep, true);
        } else {
            const bool hi = hi_ok(T);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                if (i >= nb) break;
                if (row0 + i * rstep < T.rows && colv < T.cols)
                    store(T, R[i], rr_of(i), dst + i * ystep, hi);
            }
        }
    };

    auto load = [&](uint4 (&R)[V], const Tile &T) {
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const int r = row0 + i * rstep;
            if (r < T.rows && colv < T.cols) {
                const char *a = T.src + ((int64_t)r * T.ld + colv) * ESIZE;
                if constexpr (HALVES) {
                    const uint2 lo = FP8BQ_IN(T.xs, a, 8) ? dev::ldg_v2(a) : make_uint2(0u, 0u);
                    const uint2 hi = hi_ok(T) && FP8BQ_IN(T.xs, a + 8, 8) ? dev::ldg_v2(a + 8)
                                                                          : make_uint2(0u, 0u);
                    R[i] = make_uint4(lo.x, lo.y, hi.x, hi.y);
                } else {
                    R[i] = FP8BQ_IN(T.xs, a, 16) ? dev::ldg_stream_v4(a) : make_uint4(0u, 0u, 0u, 0u);
                }
            } else {
                R[i] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };

    auto process_slots = [&](const uint4 (&R)[V], const Tile &T) {
      if constexpr ((TEAM == 16 || TEAM == 32) && V == 8) {  // the stacked-block instantiations
        const int bm = p.d[0].bm;
        // each slot's maximum as fp32 bits, then integer maxima through the
        // reduce-scatter.  Measured and dropped: keeping the maxima packed as
        // bf16 pairs merged with the bf16 max there, a three-max absmax per
        // vector, and no per-tile block count -- 0.87-0.88 of the copy peak
        // together against 0.90 for this form (same box, A/B); each alone
        // moved little, the generated code at the 128-register bound did.
        uint32_t m[V];
#pragma unroll
        for (int i = 0; i < V; ++i) {
            const uint4 one[1] = {R[i]};
            m[i] = absmax_to_f32_bits<ESIZE>(tile_absmax<ESIZE, 1>(one));
        }
        // lane q ends with the max of slot q / (TEAM / 8), computes its scale,
        // and the reciprocal of slot i is fetched from lane (TEAM / 8) i
        constexpr int LPS = TEAM / 8;  // lanes per slot after the reduce-scatter
        const uint32_t mq = TEAM == 16 ? reduce_scatter8x16(m, shfl_mask, lane)
                                       : reduce_scatter8x32(m, lane);
        float s_mine, r_mine;
        dev::block_scale(mq, kEps, s_mine, r_mine);
        const int base = (threadIdx.x & 31) & ~(TEAM - 1);
        float r[V];
#pragma unroll
        for (int i = 0; i < V; ++i) r[i] = __shfl_sync(shfl_mask, r_mine, base + LPS * i);
        // slots of blocks below the matrix are neither quantized nor stored
        store_all(R, T, (T.rows + bm - 1) / bm, [&](int i) { return dev::splat2(r[i]); });
        const int slot = lane / LPS;
        if (lane % LPS == 0 && slot * bm < T.rows) store_descale(T, T.sdst + (int64_t)slot * T.gn, s_mine);
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
        store_all(R, T, V, [&](int) { return r2; });
        if (lane == 0) store_descale(T, T.sdst, s);
    };

    if constexpr (S > 0) {
        extern __shared__ __align__(1024) uint8_t ring[];  // dynamic shared memory
        uint4 *const stage = reinterpret_cast<uint4 *>(ring);  // [S][V][CTA] 16-byte vectors
        auto issue = [&](int s, const Tile &T) {
            const bool full = is_full(T);
            const char *src0 = T.src + ((int64_t)row0 * T.ld + colv) * ESIZE;
            const int64_t xstep = (int64_t)rstep * T.ld * ESIZE;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const char *src = src0 + i * xstep;
                const bool ok = (full || (row0 + i * rstep < T.rows && colv < T.cols)) &&
                                FP8BQ_IN(T.xs, src, 16);
                dev::cp_async_16(&stage[(s * V + i) * CTA + threadIdx.x], ok ? src : T.src, ok);
            }
            dev::cp_async_commit();
        };
        Tile Ts[S];
        uint32_t tn = t;  // next tile to issue; t: next tile to process
#pragma unroll
        for (int s = 0; s < S; ++s) {
            if (tn < p.total_tiles) {
                Ts[s] = walk.next(tn);
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
                    Ts[s] = walk.next(tn);
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
    Tile ta = walk.next(t);
    load(A, ta);
    uint32_t it = 0;
    while (true) {
        const uint32_t t1 = t + stride;
        const bool h1 = t1 < p.total_tiles;
        Tile tb;
        if (h1) {
            tb = walk.next(t1);
            load(B, tb);
        }
        process(A, ta, it++);
        if (!h1) break;
        const uint32_t t2 = t1 + stride;
        const bool h2 = t2 < p.total_tiles;
        if (h2) {
            ta = walk.next(t2);
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
            for (int c = lane; c < T.cols; c += 32)
                if (FP8BQ_IN(T.xs, row + c * ESIZE, ESIZE))
                    m = max(m, elem_abs_bits<ESIZE>(row + c * ESIZE));
        }
        m = __reduce_max_sync(0xffffffffu, m);
        float s, rc;
        dev::block_scale(m, kEps, s, rc);
        for (int r = 0; r < T.rows; ++r) {
            const char *row = T.src + (int64_t)r * T.ld * ESIZE;
            uint8_t *out = T.dst + (int64_t)r * T.ldy;
#pragma unroll 4
            for (int c = lane; c < T.cols; c += 32) {
                const float x = FP8BQ_IN(T.xs, row + c * ESIZE, ESIZE) ? elem_f32<ESIZE>(row + c * ESIZE)
                                                                      : 0.0f;
                const float v = __fmul_rn(x, rc);
                if (FP8BQ_IN(T.ys, out + c, 1)) out[c] = (uint8_t)(dev::cvt_e4m3x2(v, 0.0f) & 0xffu);
            }
        }
        if (lane == 0) store_descale(T, T.sdst, s);
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
            for (int c = lane; c < T.cols; c += 32)
                if (FP8BQ_IN(T.xs, row + c * ESIZE, ESIZE))
                    m = max(m, elem_abs_bits<ESIZE>(row + c * ESIZE));
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
                const float x = FP8BQ_IN(T.xs, row + c * ESIZE, ESIZE) ? elem_f32<ESIZE>(row + c * ESIZE)
                                                                      : 0.0f;
                const float v = __fmul_rn(x, rc);
                if (FP8BQ_IN(T.ys, out + c, 1)) out[c] = (uint8_t)(dev::cvt_e4m3x2(v, 0.0f) & 0xffu);
            }
        }
        if (threadIdx.x == 0) store_descale(T, T.sdst, s);
    }
}

// ============================================================== launchers

namespace {

template <int ESIZE, int TEAM, int V, int CTA, int G, int MAXD, bool HALVES>
cudaError_t launch_vector_h(const DescPack<MAXD> &p, cudaStream_t st) {
    constexpr int S = HALVES ? 0 : TEAM <= 32 ? FP8BQ_VEC_STAGES_T16 : FP8BQ_VEC_STAGES;
    constexpr size_t smem = (size_t)S * V * CTA * 16;
    auto kern = k_vector<ESIZE, TEAM, V, CTA, G, MAXD, HALVES, S>;
    static PerDevice<KernelSetup> setup;
    const KernelSetup ks = setup.get([&] { return setup_kernel(kern, CTA, smem); });
    if (ks.attr != cudaSuccess) return ks.attr;
    // short launches (fewer than FP8BQ_VEC_SHORT_TILES tiles per resident
    // team) take FP8BQ_VEC_WAVES_SHORT waves
    const uint64_t resident_teams = (uint64_t)sm_count() * ks.occ * (CTA / TEAM);
    const int waves = TEAM <= 32 ? FP8BQ_VEC_WAVES_T16
                      : p.total_tiles < (uint64_t)FP8BQ_VEC_SHORT_TILES * resident_teams
                          ? FP8BQ_VEC_WAVES_SHORT
                          : FP8BQ_VEC_WAVES;
    const unsigned grid = grid_for(p.total_tiles, CTA / TEAM, ks.occ * waves);
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
            case Variant::VecT32: return launch_vector_t<2, 32, 8, 256, 8, MAXD>(halves, p, st);
            case Variant::VecT64: return launch_vector_t<2, 64, 8, 256, 1, MAXD>(halves, p, st);
            case Variant::VecT128: return launch_vector_t<2, 128, 8, 256, 1, MAXD>(halves, p, st);
            case Variant::VecTBig: return launch_vector_t<2, 256, 8, 256, 1, MAXD>(halves, p, st);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (v) {
        case Variant::VecT16: return launch_vector_t<4, 16, 8, 256, 8, MAXD>(halves, p, st);
        case Variant::VecT32: return launch_vector_t<4, 32, 8, 256, 8, MAXD>(halves, p, st);
        case Variant::VecT64: return launch_vector_t<4, 64, 8, 256, 1, MAXD>(halves, p, st);
        case Variant::VecT128: return launch_vector_t<4, 128, 8, 256, 1, MAXD>(halves, p, st);
        case Variant::VecTBig: return launch_vector_t<4, 512, 8, 512, 1, MAXD>(halves, p, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int MAXD>
cudaError_t launch_generic(int esize, const DescPack<MAXD> &p, cudaStream_t st) {
    // blocks of >= 2048 elements take one CTA each (the host groups generic
    // tensors by this size class, so it is uniform per launch)
    const bool cta = (int64_t)p.d[0].bm * p.d[0].bn >= 2048;
    // one occupancy record per kernel (the four kernels share a type, so a
    // static inside a shared helper would be shared too)
    static PerDevice<int> occ_cta2, occ_warp2, occ_cta4, occ_warp4;
    auto go = [&](auto kern, PerDevice<int> &occ, int tiles_per_cta) {
        const int o = occ.get([&] { return resident_ctas(kern, 256, 0); });
        return launch_kernel(kern, grid_for(p.total_tiles, tiles_per_cta, o), 256, 0, st, p);
    };
    cudaError_t e;
    if (esize == 2)
        e = cta ? go(k_generic_cta<2, MAXD>, occ_cta2, 1) : go(k_generic<2, MAXD>, occ_warp2, 8);
    else
        e = cta ? go(k_generic_cta<4, MAXD>, occ_cta4, 1) : go(k_generic<4, MAXD>, occ_warp4, 8);
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

FP8BQ_DEFINE_BOUNDS_RECORD(bounds_record_kernels)

}  // namespace fp8bq

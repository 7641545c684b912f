// fp8bq_tma.cu -- the TMA quantize kernels (sm_100a): a producer warp streams
// 3-D tensor-map tiles (no multicast) into a shared-memory ring, 8 consumer
// warps reduce each block's absmax, compute s = max(a, eps) / 448 and
// r = 1 / s with IEEE divisions, and store e4m3fn(clamp(x * r)) and s (verl
// docs "fp8_kernel.py -- FP8 量化内核", section 2 "Triton 实现").  Every wait
// on an mbarrier is bounded; a wait that runs out sets the device error word.
#include "fp8bq_tile.cuh"

// Grid cap of the TMA kernels in waves of resident CTAs.  Measured on B200
// (same box), two / four waves against one: the whole weight set +0.5 / +1.2 %,
// one layer -0.5 / -3.5 %, the MoE layer -1.5 / -1.2 %: one wave, a
// persistent walk.
#ifndef FP8BQ_TMA_WAVES
#define FP8BQ_TMA_WAVES 1
#endif
// Resident CTAs per SM of the paired kernel (its register budget follows).
// Measured on B200 (same box): two CTAs of one 64 KB slot each (96
// registers) against one CTA of two slots: one layer 0.935-0.939 / 0.984-0.994,
// the whole weight set 0.959 / 0.988-0.989, the MoE layer 0.966-0.974 /
// 1.002-1.006 of the copy peak -- a CTA that overlaps its own next load with
// its current tile beats two that each wait for theirs.
#ifndef FP8BQ_TMA_PAIR_CTAS_PER_SM
#define FP8BQ_TMA_PAIR_CTAS_PER_SM 1
#endif

namespace fp8bq {

// Bit 0: a consumer or producer wait ran out (that launch's outputs are
// incomplete).  Bit 1: the end-of-kernel drain of in-flight TMA copies ran
// out, so a copy may land in shared memory after the CTA has exited
// (reported as FP8BQ_ERR_DEVICE_UNSAFE: nothing run since can be trusted).
__device__ uint32_t g_error_word;

constexpr uint64_t kDrainLimitNs = 2000000000ull;

// Tuning constants of the TMA kernels (compile-time; the defaults are the
// measured best on B200).
#ifndef FP8BQ_TMA_STAGES_BF16
#define FP8BQ_TMA_STAGES_BF16 4   // 32 KB ring slots per TMA CTA (bf16 tiles)
#endif
// 64 KB ring slots per TMA CTA (fp32 tiles).  Measured on B200 (one fp32
// Qwen3-8B-shaped layer / four in one call, fraction of the copy peak):
// 3 slots 0.937-0.944 / 0.954-0.957, 2 slots 1.028-1.030 / 1.048-1.049; as
// for the paired bf16 kernel, a third 64 KB slot per SM slows the stream.
#ifndef FP8BQ_TMA_STAGES_F32
#define FP8BQ_TMA_STAGES_F32 2
#endif
#ifndef FP8BQ_TMA_CTAS_PER_SM
#define FP8BQ_TMA_CTAS_PER_SM 1   // resident TMA CTAs per SM
#endif

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
    dev::pdl_launch_dependents();
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
#if FP8BQ_CHECKED
        dev::Span ys, ss;
#endif
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
        // the map of this CTA's first tile, fetched while the previous kernel
        // of the stream may still be running (the maps are kernel parameters)
        int d0 = 0;
        while (d0 + 1 < p.n && blockIdx.x >= p.d[d0].tile_begin + p.d[d0].tiles) ++d0;
        dev::prefetch_tensormap(&P.maps[d0]);
    }
    dev::pdl_wait();  // the previous kernel has completed; its writes are visible
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
#if FP8BQ_CHECKED
            info[st].ys = T.ys;
            info[st].ss = T.ss;
#endif
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
                        store_codes<ESIZE>(T, R[i], r2, T.dst + (int64_t)rr * T.ldy + colv);
                }
                if (ct == 0) store_descale(T, T.sdst, s);
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
                        store_codes<ESIZE>(T, R[i], dev::splat2(r),
                                           T.dst + (int64_t)rr * T.ldy + colv);
                    if (ct == 0 && i == j * spb) store_descale(T, T.sdst + (int64_t)j * T.gn, s);
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
                        store_codes<ESIZE>(T, R[i], dev::splat2(r[i]),
                                           T.dst + (int64_t)rr * T.ldy + colv);
                }
                const int q = ct & (L - 1);  // this lane's block: slot q of its group
                if (q < V) {
                    const int blk = (row0 + q * rstep) / bm;
                    if (blk * bm < T.rows) store_descale(T, T.sdst + (int64_t)blk * T.gn, s_mine);
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
                        store_codes<ESIZE>(T, R[i], dev::splat2(r),
                                           T.dst + (int64_t)rr * T.ldy + colv);
                    if ((ct & (L - 1)) == 0) store_descale(T, T.sdst + (int64_t)blk * T.gn, s);
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
__global__ void __launch_bounds__(32 + kTmaConsumerThreads, FP8BQ_TMA_PAIR_CTAS_PER_SM)
    k_tma_pair(const __grid_constant__ TmaPack<MAXD> P) {
    dev::pdl_launch_dependents();
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
#if FP8BQ_CHECKED
        dev::Span ys, ss;
#endif
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
        // the map of this CTA's first tile, fetched while the previous kernel
        // of the stream may still be running (the maps are kernel parameters)
        int d0 = 0;
        while (d0 + 1 < p.n && blockIdx.x >= p.d[d0].tile_begin + p.d[d0].tiles) ++d0;
        dev::prefetch_tensormap(&P.maps[d0]);
    }
    dev::pdl_wait();  // the previous kernel has completed; its writes are visible
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
#if FP8BQ_CHECKED
            info[st].ys = T.ys;
            info[st].ss = T.ss;
#endif
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
                store_codes<ESIZE>(T, R[i], r2, T.dst + (int64_t)rr * T.ldy + colv);
        }
        if ((ct & 15) == 0 && ct < 32) store_descale(T, T.sdst + half, s);
    }
}

// ============================================================== launchers

namespace {
template <int ESIZE, int STAGES, int MODE, int MAXD, bool EF>
cudaError_t launch_tma_e(const TmaPack<MAXD> &p, cudaStream_t st) {
    constexpr size_t smem = (size_t)STAGES * 128 * 128 * ESIZE;
    auto kern = k_tma<ESIZE, STAGES, MODE, MAXD, EF>;
    static PerDevice<KernelSetup> setup;
    const KernelSetup ks =
        setup.get([&] { return setup_kernel(kern, 32 + kTmaConsumerThreads, smem); });
    if (ks.attr != cudaSuccess) return ks.attr;
    const unsigned grid = grid_for(p.p.total_tiles, 1, ks.occ * FP8BQ_TMA_WAVES);
    return launch_kernel(kern, grid, 32 + kTmaConsumerThreads, smem, st, p);
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
    static PerDevice<KernelSetup> setup;
    const KernelSetup ks =
        setup.get([&] { return setup_kernel(kern, 32 + kTmaConsumerThreads, smem); });
    if (ks.attr != cudaSuccess) return ks.attr;
    const unsigned grid = grid_for(p.p.total_tiles, 1, ks.occ * FP8BQ_TMA_WAVES);
    return launch_kernel(kern, grid, 32 + kTmaConsumerThreads, smem, st, p);
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

FP8BQ_DEFINE_BOUNDS_RECORD(bounds_record_tma)

}  // namespace fp8bq

// fp8bq_device.cuh -- small sm_100a device helpers (inline PTX) used by the
// quantizer kernels: cache-hinted global loads and stores, the packed
// fp32 -> e4m3fn conversion, mbarriers, TMA tensor loads and named barriers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fp8bq {
namespace dev {

// ---------------------------------------------------------------- launch order

// First statement of every kernel: allow the next kernel of the stream to
// launch (its own wait keeps it from touching memory before this grid has
// finished), then wait until the previous grid has completed and its writes
// are visible.  Both are no-ops without programmatic dependent launch.
__device__ __forceinline__ void pdl_entry() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// The two halves of pdl_entry, for kernels that do work touching no global
// memory the previous kernel may write (shared-memory set-up, prefetching
// their own kernel-parameter tensor maps) between them.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Bring a TMA tensor map (in kernel-parameter space) into the descriptor
// cache ahead of its first use.
__device__ __forceinline__ void prefetch_tensormap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------- checked builds
//
// With FP8BQ_CHECKED=1 every plain global load, store and atomic of the
// kernels is first tested against the byte range of the tensor it belongs to
// (FP8BQ_IN(span, address, bytes)); an access outside it is not made and is
// recorded: a count and one address per translation unit and device.  The
// default build compiles FP8BQ_IN to `true`, so its kernels are unchanged.
#ifndef FP8BQ_CHECKED
#define FP8BQ_CHECKED 0
#endif

// Byte range [lo, hi) of one tensor argument of a kernel.
struct Span {
    uint64_t lo, hi;
};

#if FP8BQ_CHECKED
static __device__ unsigned long long g_bounds_count;
static __device__ unsigned long long g_bounds_first;

static __device__ __noinline__ void bounds_record(const void *p) {
    atomicAdd(&g_bounds_count, 1ull);
    atomicCAS(&g_bounds_first, 0ull, (unsigned long long)(uintptr_t)p);
}

__device__ __forceinline__ bool in_span(const Span &s, const void *p, uint64_t bytes) {
    const uint64_t a = (uint64_t)(uintptr_t)p;
    if (a >= s.lo && a <= s.hi && bytes <= s.hi - a) return true;
    bounds_record(p);
    return false;
}
#define FP8BQ_IN(span, p, bytes) (::fp8bq::dev::in_span((span), (p), (bytes)))
#else
#define FP8BQ_IN(span, p, bytes) true
#endif

// ---------------------------------------------------------------- global memory

// 16-byte streaming load: read-only path, no L1 allocation, 256-byte L2
// prefetch (a tile row is 256 bytes of bf16).
__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 8-byte load on the read-only path for rows that are only 8-byte aligned.
// It allocates in L1: the two 8-byte halves of a lane's 16 bytes are read by
// two loads, and the second one finds the sectors of the first in L1.
__device__ __forceinline__ uint2 ldg_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

// Streaming (evict-first) stores of the e4m3fn codes.
__device__ __forceinline__ void stg_stream_v2(void *p, uint2 v) {
    asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
__device__ __forceinline__ void stg_stream_u32(void *p, uint32_t v) {
    asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void stg_stream_u16(void *p, uint16_t v) {
    asm volatile("st.global.cs.u16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

// ---------------------------------------------------------------- arithmetic
//
// The clamp of the method, clamp(x * r, -448, 448), is not issued as separate
// min/max instructions: cvt.rn.satfinite maps every finite value beyond the
// e4m3fn range to +-448 and rounds every value inside it to nearest even, so
// e4m3(clamp(v)) == cvt.rn.satfinite(v) for every finite v (and v = x * r is
// always finite: |x| <= absmax and r ~ 448 / absmax).

// Two fp32 values -> two e4m3fn codes (round to nearest even, saturating);
// `lo` lands in the low byte (the lower address).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

// A register pair {r, r} for the packed multiplies of one block.
__device__ __forceinline__ uint64_t splat2(float r) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %1};" : "=l"(d) : "f"(r));
    return d;
}

// Codes of the two fp32 values whose bit patterns are a0, a1: one packed
// single-rounded multiply (each lane IEEE round-to-nearest, no FMA, no
// flush-to-zero) and one conversion.  a0 lands in the low byte.
__device__ __forceinline__ uint16_t quant_pair_bits(uint32_t a0, uint32_t a1, uint64_t rr) {
    uint64_t a, d;
    uint16_t h;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "r"(a0), "r"(a1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(rr));
    asm("{\n\t.reg .f32 v0, v1;\n\t"
        "mov.b64 {v0, v1}, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 %0, v1, v0;\n\t}"
        : "=h"(h)
        : "l"(d));
    return h;
}

// Four bf16 (two 32-bit words, element order w0.lo, w0.hi, w1.lo, w1.hi) ->
// four codes in one 32-bit word, element 0 in the low byte.
__device__ __forceinline__ uint32_t quant_bf16x4(uint32_t w0, uint32_t w1, uint64_t rr) {
    const uint16_t c0 = quant_pair_bits(w0 << 16, w0 & 0xffff0000u, rr);
    const uint16_t c1 = quant_pair_bits(w1 << 16, w1 & 0xffff0000u, rr);
    uint32_t o;
    asm("mov.b32 %0, {%1, %2};" : "=r"(o) : "h"(c0), "h"(c1));
    return o;
}

// Four fp32 (bit patterns) -> four codes in one 32-bit word.
__device__ __forceinline__ uint32_t quant_f32x4(uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                uint64_t rr) {
    const uint16_t c0 = quant_pair_bits(a, b, rr);
    const uint16_t c1 = quant_pair_bits(c, d, rr);
    uint32_t o;
    asm("mov.b32 %0, {%1, %2};" : "=r"(o) : "h"(c0), "h"(c1));
    return o;
}

// Running maxima of magnitudes.  Two forms, equal for every non-NaN input:
//   FP8BQ_ABSMAX_FMAX 1: one max.xorsign.abs per pair of bf16 (or per fp32):
//     the magnitude of the result is max(|m|, |w|) exactly (max does not
//     round); its sign bit carries no meaning and is cleared when the
//     maximum is read out (absmax_bits_*).
//   FP8BQ_ABSMAX_FMAX 0: unsigned integer max of the sign-cleared bit
//     patterns (for non-negative IEEE values the integer order of the bits is
//     the numeric order); the running maximum m must have clear sign bits,
//     as every maximum these functions return has.
// Measured on B200 (same box, A/B): 1x128 blocks 5765 -> 5972 GB/s, the whole
// weight set 6421 -> 6456, bf16 4000x4100 5016 -> 5166; 64x64 blocks and
// one layer unchanged.
#ifndef FP8BQ_ABSMAX_FMAX
#define FP8BQ_ABSMAX_FMAX 1
#endif
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t m, uint32_t w) {
    uint32_t d;
#if FP8BQ_ABSMAX_FMAX
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(w));
#else
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(w & 0x7fff7fffu));
#endif
    return d;
}
__device__ __forceinline__ uint32_t absmax_f32(uint32_t m, uint32_t w) {
#if FP8BQ_ABSMAX_FMAX
    uint32_t d;
    asm("max.xorsign.abs.f32 %0, %1, %2;" : "=r"(d) : "r"(m), "r"(w));
    return d;
#else
    return max(m, w & 0x7fffffffu);
#endif
}
// fp32 bit pattern of the larger magnitude of a running bf16x2 maximum, and
// of a running fp32 maximum.
__device__ __forceinline__ uint32_t absmax_bits_bf16x2(uint32_t m) {
    m &= 0x7fff7fffu;
    return max(m & 0xffffu, m >> 16) << 16;
}
__device__ __forceinline__ uint32_t absmax_bits_f32(uint32_t m) { return m & 0x7fffffffu; }

// bf16 halves of a 32-bit word, widened to fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Scale and reciprocal of a block from the bit pattern of its fp32 absmax:
// s = a / 448 and r = 1 / s, both correctly rounded (IEEE round to nearest).
//
// FP8BQ_DIV448_FMA 1: the division by the constant 448 as a multiply by
// z = RN(1/448) and one FMA correction, q0 = RN(a z), s = RN(q0 + RN(a - 448 q0) z)
// (the remainder a - 448 q0 is exact under the FMA): the division by a divisor
// known in advance of Brisebarre, Muller and Raina ("Accelerating correctly
// rounded floating-point division when the divisor is known in advance",
// IEEE Trans. Computers 53(8), 2004), which is correctly rounded for every
// dividend only for some divisors.  For 448 it has been checked against IEEE
// division for every float a >= 1e-10 (the eps floor; tests/c/div448_check.c,
// 1.35e9 values, no difference).  The reciprocal is __frcp_rn, itself
// correctly rounded.  Measured on B200 against two IEEE divisions: 1.6 % fewer
// instructions for 1 x 128 blocks, +0.3-1.5 % on the small-block and ragged
// lines, one layer 0.997 against 0.991-0.995 of the copy peak.
#ifndef FP8BQ_DIV448_FMA
#define FP8BQ_DIV448_FMA 1
#endif
__device__ __forceinline__ void block_scale(uint32_t amax_bits, float eps, float &s, float &r) {
    float a = fmaxf(__uint_as_float(amax_bits), eps);
#if FP8BQ_DIV448_FMA
    constexpr float z = 1.0f / 448.0f;
    const float q0 = __fmul_rn(a, z);
    s = __fmaf_rn(__fmaf_rn(-q0, 448.0f, a), z, q0);
    r = __frcp_rn(s);
#else
    s = __fdiv_rn(a, 448.0f);
    r = __fdiv_rn(1.0f, s);
#endif
}

// ---------------------------------------------------------------- timers, barriers

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Asynchronous 16-byte global -> shared copies (L2 only, 256-byte L2
// prefetch); ok == false copies nothing and zero-fills the 16 bytes.
__device__ __forceinline__ void cp_async_16(void *smem_dst, const void *src, bool ok) {
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)),
                 "l"(src), "r"(ok ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's copy groups are still pending
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// One probe of the phase with parity `parity`; true once that phase completed.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for a phase, giving up after `limit_ns` of global time or as soon as
// *abort becomes nonzero.  Returns true if the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns,
                                                  const volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (abort != nullptr && *abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// 3-D TMA tile load into shared memory, completing on `bar` (no multicast).
// evict_first: the tile's lines get an L2 evict-first policy (every input
// byte is read once); otherwise the default priority.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, uint64_t *bar,
                                            int c0, int c1, int c2, bool evict_first) {
    if (evict_first) {  // a compile-time constant at every call
        asm volatile(
            "{\n\t.reg .b64 pol;\n\t"
            "createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n\t"
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], pol;\n\t}" ::"r"(
                smem_addr(smem_dst)),
            "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
            : "memory");
    } else {
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(smem_dst)),
            "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
            : "memory");
    }
}

// Named barrier over `count` threads.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return out != 0;
}

}  // namespace dev
}  // namespace fp8bq

// Host side of the bounds record: defines `cudaError_t fn(uint64_t *count,
// uint64_t *first, bool clear)` reading (and, with clear, zeroing) this
// translation unit's record on the current device; both are 0 in a default
// build.  One use per kernel source file.
#if FP8BQ_CHECKED
#define FP8BQ_DEFINE_BOUNDS_RECORD(fn)                                                        \
    cudaError_t fn(uint64_t *count, uint64_t *first, bool clear) {                             \
        unsigned long long c = 0, f = 0;                                                       \
        cudaError_t e = cudaMemcpyFromSymbol(&c, ::fp8bq::dev::g_bounds_count, sizeof(c));     \
        if (e == cudaSuccess)                                                                  \
            e = cudaMemcpyFromSymbol(&f, ::fp8bq::dev::g_bounds_first, sizeof(f));             \
        if (e == cudaSuccess && clear && (c || f)) {                                           \
            const unsigned long long zero = 0;                                                 \
            e = cudaMemcpyToSymbol(::fp8bq::dev::g_bounds_count, &zero, sizeof(zero));         \
            if (e == cudaSuccess)                                                              \
                e = cudaMemcpyToSymbol(::fp8bq::dev::g_bounds_first, &zero, sizeof(zero));     \
        }                                                                                      \
        *count = c;                                                                            \
        *first = f;                                                                            \
        return e;                                                                              \
    }
#else
#define FP8BQ_DEFINE_BOUNDS_RECORD(fn)                                                        \
    cudaError_t fn(uint64_t *count, uint64_t *first, bool) {                                   \
        *count = 0;                                                                            \
        *first = 0;                                                                            \
        return cudaSuccess;                                                                    \
    }
#endif

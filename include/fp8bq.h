/*
 * fp8bq.h -- blockwise FP8 (float8_e4m3fn) weight quantizer for NVIDIA B200
 * (sm_100a).  C ABI.
 *
 * The operation (verl documentation page "fp8_kernel.py -- FP8 量化内核",
 * section 1 "统一入口" and section 2 "Triton 实现"): a high-precision [M, N]
 * matrix is cut into [block_m, block_n] blocks (edge blocks are clipped to the
 * matrix).  For each block
 *
 *     a        = max(max |x| over the block's valid elements, eps)
 *     s        = a / 448                      (IEEE fp32 division)
 *     r        = 1 / s                        (IEEE fp32 division)
 *     y[i, j]  = e4m3fn(clamp(x[i, j] * r, -448, 448))
 *     descale  = s
 *
 * where e4m3fn() rounds to nearest, ties to even, saturating, and keeps the
 * sign of a result that rounds to zero; eps = 1e-10f.  (The kernels reach the
 * two correctly rounded quotients without division instructions; the values
 * are those of IEEE division.)  The pages print the
 * eps floor but not its value; 1e-10f is this library's reading.  The result
 * is unique bit for bit: there is no summation, and max is order independent.
 *
 * The descale is the dequantization multiplier, x ~= decode(y) * descale,
 * which the rollout engine loads as "<weight name>_scale_inv" ("vllm_fp8_utils.py"
 * docs, section 3 "权重量化"; verl PR #4415 review, where it is a 2-D tensor
 * after squeeze(-1)).
 *
 * Layouts (all row-major):
 *   x        [M, N] bf16 or fp32 elements, row stride ld >= N (elements).
 *   y        [M, N] bytes (e4m3fn bit patterns), contiguous (row stride N).
 *   descale  [ceil(M/block_m), ceil(N/block_n)] fp32, contiguous.
 *
 * Ownership: the caller allocates and owns x, y and descale (device memory of
 * the current device).  The library writes only y and descale, allocates no
 * device memory per call, and keeps no pointer after a call returns.
 *
 * Devices: a call runs on the current CUDA device, whose memory its pointers
 * must name.  Everything the library sets up for a device (the kernels'
 * dynamic shared-memory limits, resident CTAs per SM, the SM count, its own
 * streams for concurrent launch groups) is made once per device with that
 * device current, so one process may use several GPUs, in turn or at once.
 *
 * Threads: every entry point may be called from several host threads at
 * once, on the same or different streams and devices.  The process-wide
 * settings (fp8bq_set_path, fp8bq_set_pdl and the debug knobs) are shared by
 * all threads; change them while no call is being made.
 *
 * Execution: calls are asynchronous on `stream`, like a kernel launch.  All
 * arguments are checked before anything is launched: a call that returns an
 * argument error (anything but FP8BQ_ERR_DEVICE) launched nothing.  A call may
 * enqueue several launches (one per kernel variant in a grouped call); if the
 * CUDA runtime rejects one of them the call returns FP8BQ_ERR_DEVICE and the
 * launches before it stay enqueued.  Inputs must not overlap outputs, and
 * outputs must not overlap each other (checked on the address ranges each
 * argument spans).
 * NaN and infinite inputs are outside the contract (no error, unspecified
 * codes).
 */
#ifndef FP8BQ_H
#define FP8BQ_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define FP8BQ_API __attribute__((visibility("default")))
#else
#define FP8BQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define FP8BQ_VERSION 10000 /* 1.0.0 */

typedef enum fp8bq_dtype {
    FP8BQ_BF16 = 0, /* bfloat16 input */
    FP8BQ_F32 = 1   /* float32 input */
} fp8bq_dtype;

typedef enum fp8bq_status {
    FP8BQ_OK = 0,
    FP8BQ_ERR_NULL = 1,           /* a required pointer is NULL */
    FP8BQ_ERR_SHAPE = 2,          /* M, N, batch or a stride negative; ld < N; M or N >= 2^31;
                                     too many blocks in one tensor (>= 2^31); an argument's
                                     byte extent beyond 2^62 */
    FP8BQ_ERR_BLOCK = 3,          /* block_m or block_n < 1, or block_m * block_n > 65536 */
    FP8BQ_ERR_DTYPE = 4,          /* dtype_in not an fp8bq_dtype */
    FP8BQ_ERR_OVERLAP = 5,        /* an output overlaps an input or another output */
    FP8BQ_ERR_DEVICE = 6,         /* no usable CUDA device, device is not sm_100, or a CUDA
                                     call failed */
    FP8BQ_ERR_DEVICE_TIMEOUT = 7, /* a bounded wait inside a kernel ran out (reported by
                                     fp8bq_sync_status) */
    FP8BQ_ERR_ALIGN = 8,          /* x not aligned to its element size, or descale not 4-byte
                                     aligned */
    FP8BQ_ERR_ARG = 9,            /* other invalid argument (n_tensors < 0, unknown path) */
    FP8BQ_ERR_DEVICE_UNSAFE = 10, /* a kernel returned with a tile copy still in flight
                                     (reported by fp8bq_sync_status): stop using the GPU */
    FP8BQ_ERR_DEVICE_BOUNDS = 11  /* checked builds only: a kernel skipped a global access
                                     outside its tensor (reported by fp8bq_sync_status) */
} fp8bq_status;

/*
 * Quantize one matrix: scaled_fp8_blockwise(data_hp, weight_block_size) of the
 * "fp8_kernel.py" docs, section 1.
 *
 *   x            device pointer, [M, N] of dtype_in, row stride ld elements.
 *   M, N         rows and columns (0 is allowed: nothing is done).
 *   ld           row stride of x in elements, ld >= N.
 *   block_m/n    block shape; the pages' default weight_block_size is
 *                [128, 128].  1 <= block_m, block_n and block_m*block_n <= 65536.
 *   y_u8         device pointer, M*N bytes, written.
 *   descale_f32  device pointer, ceil(M/block_m)*ceil(N/block_n) floats,
 *                written.
 *   stream       CUDA stream (0 = legacy default stream).
 */
FP8BQ_API fp8bq_status fp8bq_quantize(const void *x, fp8bq_dtype dtype_in, int64_t M, int64_t N,
                            int64_t ld, int block_m, int block_n, uint8_t *y_u8,
                            float *descale_f32, cudaStream_t stream);

/*
 * One tensor of a grouped call.  batch > 1 describes a stack of `batch`
 * matrices (e.g. the experts of a fused-MoE weight [E, M, N]); each gets its
 * own descale grid.  Matrix b starts at
 *   x + b * x_batch_stride   (elements of dtype_in)
 *   y + b * y_batch_stride   (bytes)
 *   descale + b * s_batch_stride (floats).
 * For batch == 1 the three strides are ignored.  For batch > 1 the output
 * strides must keep the matrices apart: y_batch_stride >= M*N and
 * s_batch_stride >= ceil(M/block_m)*ceil(N/block_n).
 */
typedef struct fp8bq_desc {
    const void *x;            /* device, input */
    uint8_t *y_u8;            /* device, e4m3fn output */
    float *descale_f32;       /* device, fp32 descales */
    int64_t M, N, ld;         /* rows, columns, input row stride (elements) */
    int64_t batch;            /* number of matrices, >= 0 (1 for a plain matrix) */
    int64_t x_batch_stride;   /* elements */
    int64_t y_batch_stride;   /* bytes */
    int64_t s_batch_stride;   /* floats */
    int32_t dtype_in;         /* fp8bq_dtype */
    int32_t block_m, block_n; /* block shape */
    int32_t reserved;         /* set to 0 */
} fp8bq_desc;

/*
 * Quantize a list of tensors in as few launches as possible: the
 * quant_weights stream of the "vllm_fp8_utils.py" docs, section 3 (every
 * linear and fused-MoE weight of a layer or a model, each emitting the fp8
 * weight and its "_scale_inv" descale), done as one grouped launch per kernel
 * variant instead of one launch per tensor.
 *
 *   desc_table   HOST memory, n_tensors entries; read during the call only.
 *   n_tensors    >= 0.
 *
 * Every tensor is checked before the first launch; an argument error in any
 * descriptor rejects the whole list and nothing is launched.
 */
FP8BQ_API fp8bq_status fp8bq_quantize_batched(const fp8bq_desc *desc_table, int n_tensors,
                                    cudaStream_t stream);

/*
 * Dequantize: the consumer side of the descale ("_scale_inv") tensor
 * ("vllm_fp8_utils.py" docs, section 3): for every matrix b of a stack,
 *
 *     out[b, r, c] = decode(y[b, r, c]) * descale[b, r / block_m, c / block_n]
 *
 * with one fp32 multiply rounded to nearest even; for bf16 output that fp32
 * product is then rounded to bf16 (nearest even).  The pages print no
 * dequantization code; this is the plain reading of the descale's meaning.
 *
 *   y_u8         device, [batch, M, N] contiguous e4m3fn codes (the layout
 *                fp8bq_quantize writes).
 *   descale_f32  device, [batch, ceil(M/block_m), ceil(N/block_n)] contiguous.
 *   out          device, matrix b at out + b * out_batch_stride (elements),
 *                rows ld_out >= N elements apart, dtype_out bf16 or fp32.
 *
 * Codes 0x7F / 0xFF (NaN) are never written by the quantizer and dequantize
 * to NaN.  Same checks, status codes and stream semantics as fp8bq_quantize.
 */
FP8BQ_API fp8bq_status fp8bq_dequantize(const uint8_t *y_u8, const float *descale_f32,
                                        int64_t batch, int64_t M, int64_t N, int block_m,
                                        int block_n, void *out, fp8bq_dtype dtype_out,
                                        int64_t ld_out, int64_t out_batch_stride,
                                        cudaStream_t stream);

/* One matrix stack of a grouped dequantization (fields as in fp8bq_dequantize). */
typedef struct fp8bq_dequant_desc {
    const uint8_t *y_u8;       /* device, [batch, M, N] contiguous codes */
    const float *descale_f32;  /* device, [batch, ceil(M/bm), ceil(N/bn)] contiguous */
    void *out;                 /* device, dtype_out elements */
    int64_t batch, M, N;
    int64_t ld_out;            /* output row stride, elements, >= N */
    int64_t out_batch_stride;  /* elements; ignored for batch == 1 */
    int32_t dtype_out;         /* fp8bq_dtype */
    int32_t block_m, block_n;
    int32_t reserved;          /* set to 0 */
} fp8bq_dequant_desc;

/*
 * Dequantize a list of matrix stacks in as few launches as possible (one per
 * kernel variant and output dtype), e.g. every weight of a layer or a model.
 * desc_table is HOST memory, read during the call only.  All descriptors are
 * checked before anything is launched.
 */
FP8BQ_API fp8bq_status fp8bq_dequantize_batched(const fp8bq_dequant_desc *desc_table,
                                                int n_tensors, cudaStream_t stream);

/*
 * Per-tensor FP8 scales, e.g. the Q/K/V scales of an FP8 KV cache, which the
 * FP8-RL report recalibrates every RL step (its abstract; the pages print no
 * formula).  Reading: the weight recipe applied to a whole tensor as one
 * block,
 *
 *     scale_out[i] = max(max |x_i|, eps) / 448      (fp32, eps = 1e-10f)
 *
 * so x_i / scale_out[i] fits e4m3fn and scale_out[i] is its dequantization
 * multiplier.  One grouped launch covers all n tensors.
 *
 *   desc_table  HOST memory, n_tensors entries: contiguous device tensors of
 *               numel >= 0 elements (numel 0 gives eps / 448).
 *   scale_out   device, n_tensors floats, written (used as the accumulator
 *               while the call runs; it must not overlap any input).
 */
typedef struct fp8bq_scale_desc {
    const void *x;      /* device, numel contiguous elements */
    int64_t numel;
    int32_t dtype_in;   /* fp8bq_dtype */
    int32_t reserved;   /* set to 0 */
} fp8bq_scale_desc;

FP8BQ_API fp8bq_status fp8bq_tensor_scale(const fp8bq_scale_desc *desc_table, int n_tensors,
                                          float *scale_out, cudaStream_t stream);

/* Human-readable name of a status code (static string, never NULL). */
FP8BQ_API const char *fp8bq_status_string(fp8bq_status status);

/*
 * Synchronize `stream`, then read and clear the library's device error word
 * on the current device.  Returns FP8BQ_ERR_DEVICE_TIMEOUT if a kernel of this
 * library gave up a bounded wait since the last check (its outputs are then
 * incomplete), FP8BQ_ERR_DEVICE if the synchronization failed, else FP8BQ_OK.
 *
 * FP8BQ_ERR_DEVICE_UNSAFE (it takes precedence over the timeout) if a kernel
 * returned while one of its tile copies was still in flight: its end-of-kernel
 * wait for the copies it issued ran out (2 s, which no healthy GPU needs), so
 * the copy may still land in shared memory that a later kernel of any process
 * uses; neither the outputs nor any kernel run since can be trusted, and the
 * process should stop using the GPU.
 *
 * The error word is one per device, shared by every stream of the process:
 * a call reports (and clears) a timeout raised by a kernel on any stream of
 * the device, not only on `stream`, and whichever call reads it first takes
 * it.
 *
 * In a checked build (fp8bq_checked_build() == 1) it returns
 * FP8BQ_ERR_DEVICE_BOUNDS, after the two statuses above, while the bounds
 * record of the current device is not empty (see fp8bq_debug_take_bounds;
 * this call does not clear it).
 */
FP8BQ_API fp8bq_status fp8bq_sync_status(cudaStream_t stream);

/* Library version, FP8BQ_VERSION of the build. */
FP8BQ_API int fp8bq_version(void);

/*
 * Kernel variant selection.  AUTO picks per tensor; the others force one
 * variant for every tensor it can serve (tensors it cannot serve still take
 * the generic kernel).  Process-wide; meant for tests and benchmarks.
 *   VECTOR   16-byte vectorised global loads into registers, persistent
 *            grouped tile walk.
 *   TMA      2-D tensor-map (TMA) tile loads into a shared-memory ring,
 *            one producer warp, consumer warps, bounded mbarrier waits.
 *   GENERIC  element-wise loads; any alignment, stride and block shape.
 */
typedef enum fp8bq_path {
    FP8BQ_PATH_AUTO = 0,
    FP8BQ_PATH_VECTOR = 1,
    FP8BQ_PATH_TMA = 2,
    FP8BQ_PATH_GENERIC = 3
} fp8bq_path;

FP8BQ_API fp8bq_status fp8bq_set_path(fp8bq_path path);
FP8BQ_API fp8bq_path fp8bq_get_path(void);

/*
 * Which variant a tensor would take under the current selection (host only,
 * launches nothing).  Returns FP8BQ_PATH_VECTOR, _TMA or _GENERIC, or -1 if
 * the descriptor is invalid.  This is the tensor's own choice; under AUTO a
 * call whose TMA tensors hold less than 128 MiB of input in all runs them on
 * the vector kernel (short launches start sooner there), which
 * fp8bq_launch_count accounts for.  A tensor of at least 4 MiB of input with
 * few rows is planned on an equivalent geometry with the same codes and
 * descales (a single block row as blocks of its M rows; 1 x bn blocks on
 * fewer than 256 contiguous rows folded into more, shorter rows), and the
 * choice reported is the one for that geometry.
 */
FP8BQ_API int fp8bq_path_for(const fp8bq_desc *desc);

/*
 * Number of kernel launches fp8bq_quantize_batched(desc_table, n_tensors, .)
 * would enqueue under the current selection (host only, launches nothing;
 * needs a usable device, like the call itself).  Returns -1 if the call would
 * return an error.
 */
FP8BQ_API int fp8bq_launch_count(const fp8bq_desc *desc_table, int n_tensors);

/*
 * Programmatic dependent launch (process-wide; on by default).  When on,
 * every kernel of the library is launched so that it may be scheduled while
 * the previous kernel of its stream is still finishing; each of its threads
 * first waits (griddepcontrol.wait) until that kernel has completed and its
 * writes are visible, so stream order of all memory effects is unchanged and
 * only launch latency and the kernel prologue overlap.  The library's kernels
 * also let the next kernel of the stream launch early; a kernel launched by
 * the caller with programmatic stream serialization after one of ours must
 * wait in the same way before it reads our outputs (as CUDA requires of any
 * such kernel).  fp8bq_set_pdl(0) launches plainly; any other value turns it
 * back on.  fp8bq_get_pdl returns 1 or 0.
 */
FP8BQ_API fp8bq_status fp8bq_set_pdl(int enable);
FP8BQ_API int fp8bq_get_pdl(void);

/*
 * Fault-injection and wait-limit knobs for tests (host side; process-wide).
 * fp8bq_debug_set_wait_limit_ns bounds every device-side wait of the TMA
 * kernel (default 2e9 ns; 0 restores the default).
 * fp8bq_debug_set_inject(FP8BQ_INJECT_DROP_FIRST_LOAD) makes the first CTA of
 * the next TMA launches arm its first tile's barrier without issuing the
 * copy, so the consumers' wait can only run out; the kernel then reports
 * FP8BQ_ERR_DEVICE_TIMEOUT through fp8bq_sync_status.  0 turns it off.
 *
 * fp8bq_debug_set_inject(FP8BQ_INJECT_TRIM_OUTPUTS), in a checked build only
 * (elsewhere FP8BQ_ERR_ARG), makes the bounds checks of the next launches
 * take every output (codes, descales, dequantized values, per-tensor scales)
 * as one byte shorter than its true extent, so the kernels' last, legitimate
 * store to each output is reported and skipped: a test of the checks that
 * touches no memory outside any buffer.  Flags combine with |.
 */
#define FP8BQ_INJECT_DROP_FIRST_LOAD 1u
#define FP8BQ_INJECT_TRIM_OUTPUTS 2u
FP8BQ_API fp8bq_status fp8bq_debug_set_wait_limit_ns(uint64_t ns);
FP8BQ_API fp8bq_status fp8bq_debug_set_inject(uint32_t flags);

/*
 * Checked builds (library libfp8bq_checked.so, compiled with FP8BQ_CHECKED=1:
 * a memory-safety aid for runs without a device sanitizer).  Every plain
 * global load, store and atomic of every kernel is first tested against the
 * byte range of the tensor it belongs to, taken from the call's descriptors:
 * the input [x, x + ((batch - 1) x_batch_stride + (M - 1) ld + N) elements),
 * the codes [y, y + (batch - 1) y_batch_stride + M N), the descales
 * [s, s + ((batch - 1) s_batch_stride + gm gn) floats), and the like for the
 * dequantizer and the per-tensor scales.  An access outside its range is not
 * made (a load reads zeros) and is recorded per device: the number of such
 * accesses and the address of one of them.  TMA tile loads are bounded by
 * their tensor maps in hardware and are not checked.  Outputs are otherwise
 * identical to the default build's; the checks cost speed, and the
 * descriptor chunks per launch are smaller (256 instead of 320).
 *
 * fp8bq_checked_build returns 1 in a checked build, else 0.
 * fp8bq_debug_take_bounds synchronizes the current device, stores the record
 * (count of skipped accesses since the last take, and the address of one of
 * them, 0 if none) and clears it; in a default build both are 0.  Either
 * pointer may be NULL.  FP8BQ_ERR_DEVICE if the device cannot be read.
 */
FP8BQ_API int fp8bq_checked_build(void);
FP8BQ_API fp8bq_status fp8bq_debug_take_bounds(uint64_t *count, uint64_t *first_address);

#ifdef __cplusplus
}
#endif

#endif /* FP8BQ_H */

/*
 * far.h -- C ABI of libfar.so: the fused "all-reduce + residual-add +
 * RMSNorm (+FP8-e4m3)" epilogue of a row-parallel linear layer, on one
 * B200 (sm_100a).
 *
 * What one call computes, for every row t of a (T, H) problem (row-major,
 * contiguous, row stride H):
 *
 *   y[t,h]  = sum_{r<W} partials[r][t,h] + residual[t,h]          (fp32)
 *   rinv[t] = 1 / sqrt( (1/H) sum_h y[t,h]^2 + eps )
 *   o[t,h]  = y[t,h] * rinv[t] * (gamma[h] + weight_bias)
 *
 *   residual_out[t,h] = round_to_dtype(y[t,h])
 *   norm_out[t,h]     = round_to_dtype(o[t,h])
 *   static FP8:    quant_out[t,h] = e4m3_satfinite(o[t,h] / scale_in[0])
 *   per-token FP8: scale_out[t] = max_h |o[t,h]| / 448,
 *                  quant_out[t,h] = e4m3_satfinite(o[t,h] / scale_out[t])
 *
 * Sources (web pages, by title and section):
 *  - vllm.models.common.ops.fused_allreduce_rms_norm, docstring of
 *    fused_allreduce_rms_norm: the partials are the ranks' outputs of a
 *    row-parallel linear run without its reduction; the result is
 *    (normed_output, new_residual) = norm(all_reduce(hidden_states), residual);
 *    the fused call passes fp32_acc=True, weight_bias=0.0 for standard
 *    RMSNorm (1.0 for Gemma), and with one rank the op is the plain
 *    norm(hidden_states, residual).
 *  - PR #45307 report, call_trtllm_fused_allreduce_norm: norm_out,
 *    quant_out, scale_out and scale_factor (here scale_in) are optional
 *    outputs/inputs of one call; 3-D [batch, tokens, hidden] inputs are
 *    flattened to (tokens, hidden) before the call.
 *  - vllm.compilation.fusion, FusedAddRMSNormStaticQuantPattern and
 *    FusedAddRMSNormDynamicQuantPattern: static per-tensor and dynamic
 *    per-token symmetric FP8 after the fused add + RMSNorm; the dynamic one
 *    returns one fp32 scale per token.
 *  - vllm.compilation.sequence_parallelism, SequenceParallelismPass
 *    docstring: AllReduce -> RMSNorm rewritten as ReduceScatter -> local
 *    RMSNorm -> AllGather; far_fused_rows() is the local step on a block of
 *    rows, writing at the rows' own offsets (the gather is the layout).
 *  - vllm.distributed.device_communicators.aiter_custom_all_reduce,
 *    use_1stage_fused_ar_rms: rows made of 16-byte packs and a token cap of
 *    80 for the one-kernel path.  Here: H must be a multiple of 8 (16-byte
 *    packs of 2-byte elements), and calls of at most decode_max_rows rows
 *    (default 80) whose rows are long (one CTA would need 4 or more packs
 *    per thread: H >= 8192 at 256 threads) take the cluster-per-row decode
 *    kernel; shorter rows run faster with one CTA per row (measured).
 *
 * Ownership: the caller owns every buffer.  The library allocates and frees
 * nothing per call and never synchronises the stream; a call only enqueues
 * one kernel on `stream` (for per-tensor FP8 a one-CTA kernel that zeroes
 * the workspace's counters, then one or two passes; copies and one kernel
 * per chunk for far_fused_host) and returns.  Results are ready when the stream
 * reaches that point.  The W partials live in the same GPU's memory (the
 * tensor-parallel ranks' outputs gathered on one device); they are read only.
 *
 * Errors: every argument is checked on the host before anything is
 * enqueued.  A bad argument returns an error code and enqueues nothing;
 * nothing is ever skipped silently.  A launch failure returns FAR_ERR_CUDA
 * and far_last_error() gives the CUDA message (per thread).
 */
#ifndef FAR_H_
#define FAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FAR_VERSION 1
#define FAR_MAX_W 16      /* most partial buffers per call            */
#define FAR_MAX_H 16384   /* longest row (elements) the kernels hold  */
#define FAR_E4M3_MAX 448.0f

typedef enum {
    FAR_OK = 0,
    FAR_ERR_INVALID_ARG = 1, /* NULL where a buffer is required, W/T/rows out of range, overlap */
    FAR_ERR_UNSUPPORTED = 2, /* H not a multiple of 8 or above FAR_MAX_H; device not sm_100 */
    FAR_ERR_ALIGNMENT = 3,   /* a tensor pointer not 16-byte aligned (scales: 4-byte) */
    FAR_ERR_CUDA = 4,        /* a CUDA runtime call or the launch failed */
    FAR_ERR_TIMEOUT = 5,     /* reserved for bounded device-side waits */
    FAR_ERR_INTERNAL = 6
} far_status;

typedef enum { FAR_BF16 = 0, FAR_FP16 = 1 } far_dtype;

typedef enum {
    /* writes residual_out (when there is one) and norm_out (required) */
    FAR_AR_RESIDUAL_RMSNORM = 0,
    /* + quant_out, reading the fp32 scalar scale_in[0]; norm_out optional */
    FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC = 1,
    /* + quant_out and scale_out[T] (one fp32 scale per row); norm_out optional */
    FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN = 2,
    /* + quant_out and scale_out[0] (one fp32 scale for all rows of the call);
     * only through far_fused_fp8_tensor, which takes a workspace */
    FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR = 3,
    /* + quant_out and scale_out[T][H / group] (one fp32 scale per row and
     * group of consecutive elements); only through far_fused_fp8_group */
    FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP = 4
} far_pattern;

typedef enum {
    FAR_REGIME_AUTO = 0,    /* decode for <= decode_max_rows long rows, else prefill */
    FAR_REGIME_DECODE = 1,  /* one thread-block cluster per row            */
    FAR_REGIME_PREFILL = 2  /* one CTA per row (or several rows per CTA)  */
} far_regime;

/* Opaque per-device context: caches the SM count, the compute capability
 * and the tuning knobs (read once from the environment in far_create:
 * FAR_DECODE_MAX_ROWS, FAR_FORCE_REGIME=decode|prefill, FAR_DECODE_CLUSTER
 * (CTAs per row; default by rule),
 * FAR_PREFILL_THREADS, FAR_PREFILL_KERNEL=1 ring | 0 direct,
 * FAR_RING_CTAS_PER_SM=1..8, FAR_RING_THREADS: consumer threads per ring
 * CTA, at most 256, FAR_RING_SLOTS: row-segment slots per ring CTA (2..32),
 * FAR_RING_GAMMA_SMEM=1|0: gamma staged in shared memory or read through
 * L1, FAR_RING_WIDE=1|0: the 384-consumer build for rows of 1025-1536
 * packs, FAR_RING_WIDE2=1|0: the 448-consumer build for rows of 513-896
 * packs, FAR_RING_WIDE1=1|0: the one-CTA 512-consumer build for rows of
 * 1537-2048 packs, where the rules take them (each replaces its part of
 * the default
 * geometry, which follows rules
 * measured on B200 by row length, segments per row and whether norm_out is
 * written: plan_ring in reduce_residual_add_b200/csrc/far_abi.cu),
 * FAR_PDL=1|0: launch with programmatic dependent launch, default 1,
 * FAR_RING_MIN_ROWS: fewest rows for the ring kernel, default by rule,
 * FAR_TENSOR_REVERSE=1|0: the second pass of per-tensor FP8 takes the rows
 * from the last one down, default 1, FAR_TENSOR_FUSED=1|0: per-tensor FP8
 * on the ring kernel with a residual_out or norm_out to read back runs both
 * passes in one launch with a bounded wait on rows done between them,
 * default 1). */
/*
 * Programmatic dependent launch: every kernel of this library first waits
 * (griddepcontrol.wait) until the grid it depends on has completed, then
 * lets its own dependents be scheduled.  The next kernel in the stream may
 * therefore start its launch while this one runs, but reads nothing before
 * this one has finished; a preceding kernel that triggers early likewise
 * overlaps its tail with this call's launch. */
/*
 * Threads: calls on one context may come from several host threads at once
 * (its cache of launch shapes and far_fused_host's streams are guarded by
 * locks); far_set_regime and far_test_stall change the context and must not
 * run while other calls on it do.  The device error word far_check reads
 * and clears is one per device, shared by every context on that device.
 */
typedef struct far_ctx far_ctx;

/* How one call would be launched (see far_describe_launch). */
typedef struct {
    int regime;           /* FAR_REGIME_DECODE or FAR_REGIME_PREFILL */
    int ctas_per_row;     /* cluster size for decode, 1 for prefill */
    int rows_per_cta;     /* prefill: rows handled by one CTA        */
    int threads_per_cta;
    int packs_per_thread; /* 16-byte packs of one row held by one thread */
    int64_t grid_ctas;    /* CTAs of the launch                       */
    int kernel;           /* prefill: 1 = TMA bulk-copy ring, 0 = direct loads */
    int ring_slots;       /* ring: shared-memory slots of one row segment */
    int ring_gamma_smem;  /* ring: 1 = gamma staged in shared memory, 0 = read through L1 */
} far_launch_info;

/* Create a context for CUDA device `device` (its ordinal).  Fails with
 * FAR_ERR_UNSUPPORTED on a device other than compute capability 10.0 and
 * with FAR_ERR_CUDA when the device cannot be queried. */
far_status far_create(far_ctx **ctx, int device);

/* Destroy a context (NULL is accepted).  Waits for nothing; the copy
 * streams and events of far_fused_host are released once their work is
 * done. */
far_status far_destroy(far_ctx *ctx);

/*
 * The fused epilogue on all T rows.
 *
 *  partials      host array of W device pointers (1 <= W <= FAR_MAX_W), each
 *                to a (T, H) tensor of `dtype`; read only.
 *  residual      (T, H) `dtype`, or NULL for no residual input (the
 *                sequence-parallel "First" pattern: y is the reduced sum).
 *  residual_out  (T, H) `dtype` receiving round(y).  NULL with a residual
 *                means in place: round(y) overwrites `residual`.  NULL with
 *                no residual means no residual output.  It may equal
 *                `residual`; it may overlap no other buffer.
 *  gamma         (H,) `dtype`, the RMSNorm weight.
 *  T, H          rows (tokens) and hidden size: T >= 0, 8 <= H <= FAR_MAX_H,
 *                H % 8 == 0.  T == 0 is a valid no-op (buffer pointers are
 *                then not checked: nothing is read or written).
 *  eps           added to the mean square inside the root; finite, >= 0.
 *  weight_bias   added to gamma in fp32 (0 standard, 1 Gemma-style); finite.
 *  norm_out      (T, H) `dtype`; required by FAR_AR_RESIDUAL_RMSNORM,
 *                optional (NULL) for the FP8 patterns.
 *  quant_out     (T, H) uint8 e4m3fn codes; required by the FP8 patterns.
 *  scale_in      device pointer to one fp32 (static FP8 only).
 *  scale_out     device array of T fp32 (per-token FP8 only).
 *  pattern       FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR and _FP8_GROUP are
 *                refused here (FAR_ERR_INVALID_ARG): use far_fused_fp8_tensor
 *                and far_fused_fp8_group.
 *  stream        a cudaStream_t (NULL: the legacy default stream).
 *
 * Tensor pointers must be 16-byte aligned, scale pointers 4-byte aligned.
 */
far_status far_fused(far_ctx *ctx,
                     const void *const *partials, int W,
                     const void *residual, void *residual_out,
                     const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                     float eps, float weight_bias, far_pattern pattern,
                     void *norm_out, void *quant_out,
                     const float *scale_in, float *scale_out, void *stream);

/*
 * The same on rows [row_begin, row_end) of a T-row problem: the local-norm
 * step of ReduceScatter -> RMSNorm -> AllGather.  All pointers address the
 * full T-row tensors; rows outside the range are neither read nor written
 * (scale_out included).  0 <= row_begin <= row_end <= T, else
 * FAR_ERR_INVALID_ARG; an empty range is a no-op.  Disjoint row ranges
 * together give exactly (bit for bit) the far_fused result whenever the
 * calls run with the same packs per thread and threads per row
 * (far_describe_launch): the one-CTA and ring kernels reduce a row in the
 * same order then, and the one-CTA kernel's geometry does not depend on the
 * number of rows.  Otherwise (a cluster per row against one CTA per row, or
 * a ring geometry other than the one-CTA kernel's) the fp32 sum of squares
 * is reduced in another order and the outputs agree within the parity
 * tolerances (1 ulp, 1 FP8 step).
 */
far_status far_fused_rows(far_ctx *ctx, int64_t row_begin, int64_t row_end,
                          const void *const *partials, int W,
                          const void *residual, void *residual_out,
                          const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                          float eps, float weight_bias, far_pattern pattern,
                          void *norm_out, void *quant_out,
                          const float *scale_in, float *scale_out, void *stream);

/* Bytes of workspace far_fused_fp8_tensor needs for `rows` rows:
 * 256 + 4*rows, rounded up to 256. */
size_t far_fp8_tensor_workspace_bytes(int64_t rows);

/*
 * Dynamic per-tensor FP8 (vllm.compilation.fusion, the kFp8DynamicTensorSym
 * quantisation key: symmetric, dynamic, one scale per tensor; the page has
 * no fused op for it): the epilogue on rows [row_begin, row_end) of a T-row
 * problem, with ONE fp32 scale = max |o| over all those rows / 448, written
 * to scale_out[0], and quant_out = e4m3_satfinite(o / scale).  Other
 * arguments as far_fused_rows; residual_out, norm_out as there.
 *
 * The scale needs every row before any code, so the call enqueues a
 * one-CTA kernel that zeroes the workspace's first four words, and two
 * passes.  The first reads the
 * inputs and keeps each row's 1/rms and the running amax in `workspace`.
 * With norm_out, the first pass also writes norm_out and the new residual,
 * and the second forms the codes from norm_out -- round(o), o in the 2-byte
 * format -- so the inputs are read once.  Without norm_out and with a new
 * residual to write (a residual_out, or a residual updated in place), the
 * first pass also writes the new residual and the second forms o from it
 * -- o = round(y) * rinv * (gamma + weight_bias), round(y) being the new
 * residual in the 2-byte format -- and writes only the codes.  Either way
 * each code is within one step of the code of o itself, and the scale is
 * the same (it comes from the unrounded o).  Rows whose sum of squares
 * could hide an element that overflows the format, rows with an inf or NaN
 * input, and (with norm_out) rows whose amax reaches the format's largest
 * finite value are rebuilt from the inputs by the second pass instead.  When the persistent kernel serves
 * the call, both passes run in ONE launch: its CTAs take the first pass's
 * rows one at a time from a counter in the workspace, wait (bounded) until
 * every row is done -- a wait on rows, not on CTAs, so the grid need not be
 * co-resident -- then write the codes, the rows done last first, about
 * three quarters of them in fixed rounds and the rest in small chunks from
 * a second counter (FAR_TENSOR_FUSED=0 in the
 * environment at far_create splits them into two kernels); otherwise two
 * kernels run.
 * With neither norm_out nor a new residual to write, the second pass reads
 * the inputs again.
 * `workspace`: device memory of at least
 * far_fp8_tensor_workspace_bytes(row_end - row_begin) bytes, 256-byte
 * aligned, overlapping no argument; its contents are scratch, and two calls
 * that share a workspace must not overlap on the GPU.
 */
far_status far_fused_fp8_tensor(far_ctx *ctx, int64_t row_begin, int64_t row_end,
                                const void *const *partials, int W,
                                const void *residual, void *residual_out,
                                const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                                float eps, float weight_bias,
                                void *norm_out, void *quant_out, float *scale_out,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Per-group FP8 (vllm.distributed.device_communicators.aiter_custom_all_reduce,
 * build_supports_per_group_quant: a fused all-reduce + RMSNorm + per-group
 * quantisation, whose group shape the page does not give): the epilogue on
 * rows [row_begin, row_end) with one fp32 scale per row and per group of
 * `group_size` consecutive hidden elements, scale = max |o| over the group
 * / 448, written to scale_out[t * (H / group_size) + h / group_size], and
 * quant_out = e4m3_satfinite(o / that scale).  group_size: a power of two
 * from 8 to 256 dividing H (else FAR_ERR_UNSUPPORTED).  scale_out holds
 * T * (H / group_size) floats and overlaps no other buffer.  Other
 * arguments as far_fused_rows.
 */
far_status far_fused_fp8_group(far_ctx *ctx, int64_t row_begin, int64_t row_end,
                               const void *const *partials, int W,
                               const void *residual, void *residual_out,
                               const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                               float eps, float weight_bias, int group_size,
                               void *norm_out, void *quant_out, float *scale_out,
                               void *stream);

/* Rows one far_fused_fp8_tensor_noalloc call can take. */
#define FAR_FP8_TENSOR_NOALLOC_MAX_ROWS 65536

/*
 * far_fused_fp8_tensor for callers that cannot allocate device memory: the
 * same operation and arguments, minus the workspace.  The paper has no
 * counterpart; it exists for callers that must not or cannot call
 * cudaMalloc -- servers that hand all free device memory to a fixed pool
 * (a KV cache) at start-up, plain-C callers with no device allocator of
 * their own, and loops that cannot take the device-wide synchronisation
 * cudaMalloc / cudaFree imply.
 *
 * Its scratch (256 KiB + 256 bytes) is a fixed array inside the library:
 * every GPU that loads the library holds it until the process exits, and
 * the call allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).  At most FAR_FP8_TENSOR_NOALLOC_MAX_ROWS rows
 * (row_end - row_begin) per call; more returns FAR_ERR_UNSUPPORTED with
 * the limit in far_last_error().  Every call on a GPU shares the one
 * scratch array, which keeps the last call's contents (the call clears the
 * word that must start at zero itself): calls that overlap on the GPU --
 * on different streams without ordering between them -- race and give
 * wrong results.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  The address is kept for the life
 * of the process: no call may follow a cudaDeviceReset (or any other
 * teardown of the device's primary context) in the same process.  Device
 * ordinals from 256 up are refused (FAR_ERR_UNSUPPORTED).
 */
far_status far_fused_fp8_tensor_noalloc(far_ctx *ctx, int64_t row_begin, int64_t row_end,
                                        const void *const *partials, int W,
                                        const void *residual, void *residual_out,
                                        const void *gamma, int64_t T, int64_t H,
                                        far_dtype dtype, float eps, float weight_bias,
                                        void *norm_out, void *quant_out, float *scale_out,
                                        void *stream);

/* Bytes of device staging far_fused_host needs for W partials of rows of H
 * elements in chunks of `chunk_rows` rows (0: the library's default chunk,
 * about 64 MiB of inputs); 0 for a W or H out of range.  It does not depend
 * on T, the dtype, the pattern or which outputs are wanted. */
size_t far_host_staging_bytes(int W, int64_t H, int64_t chunk_rows);

/*
 * The fused epilogue on HOST buffers: the operation and the arguments of
 * far_fused (and of far_fused_fp8_group for FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP,
 * whose group size is `group_size`; ignored otherwise), except that every
 * tensor -- partials, residual, residual_out, gamma, norm_out, quant_out,
 * scale_in, scale_out -- is in host memory.  The library has no counterpart
 * on the pages, whose inputs are already on the GPU; it serves callers whose
 * activations live in host memory and measures the path end to end.
 *
 * The rows go through `staging` (device memory of at least
 * far_host_staging_bytes(W, H, chunk_rows) bytes, 256-byte aligned) in
 * chunks of `chunk_rows` rows (0: the default): chunk c is copied in on one
 * of the context's two copy streams, reduced and normalised on `stream`,
 * and copied out on the other copy stream, each step ordered by events, so
 * the copy in of chunk c+1 and the copy out of chunk c-1 overlap chunk c.
 * Gamma (and the static scale) are copied once per call.  The results are in
 * the host buffers once `stream` reaches the end of the call (the call
 * itself does not wait); each chunk's kernel is the one far_fused would
 * launch for that many rows, so every row's outputs are those of a device
 * call on the chunk.
 *
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister);
 * pageable memory works, but the driver then copies synchronously and
 * nothing overlaps.  Tensor pointers must be 16-byte aligned, as for
 * far_fused, and the same overlap rules apply.  Per-tensor FP8 is refused
 * (FAR_ERR_UNSUPPORTED): its scale needs every row before any code.
 * chunk_rows < 0 or a staging area that is NULL or too small gives
 * FAR_ERR_INVALID_ARG, a misaligned one FAR_ERR_ALIGNMENT.  The staging
 * area is scratch; calls that share one must not overlap on the GPU (calls
 * on one context are ordered through its events; the enqueueing is
 * serialised by a lock of the context).  That ordering is per context, not
 * per staging area: each call's copies in wait for the previous call's
 * kernels even when the two calls use different staging areas, so calls
 * meant to overlap need contexts of their own.  A CUDA error part-way through the
 * enqueueing returns FAR_ERR_CUDA, and the work already enqueued still runs.
 * The first call on a context creates its two copy streams and seven
 * events, released by far_destroy; make that first call before any stream
 * capture.
 */
far_status far_fused_host(far_ctx *ctx,
                          const void *const *partials, int W,
                          const void *residual, void *residual_out,
                          const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                          float eps, float weight_bias, far_pattern pattern, int group_size,
                          void *norm_out, void *quant_out,
                          const float *scale_in, float *scale_out,
                          int64_t chunk_rows, void *staging, size_t staging_bytes,
                          void *stream);

/* Host-only: the status far_fused_rows would return for these arguments
 * before launching (it touches no GPU and needs no context).  With pattern
 * FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR it checks far_fused_fp8_tensor's
 * arguments other than the workspace; with FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP
 * those of far_fused_fp8_group other than the group size and the extent of
 * scale_out (a scale_out of T floats is assumed for the overlap checks). */
far_status far_validate(int64_t row_begin, int64_t row_end,
                        const void *const *partials, int W,
                        const void *residual, const void *residual_out,
                        const void *gamma, int64_t T, int64_t H, far_dtype dtype,
                        float eps, float weight_bias, far_pattern pattern,
                        const void *norm_out, const void *quant_out,
                        const float *scale_in, const float *scale_out);

/* Override the regime choice and the decode row threshold of a context
 * (decode_max_rows < 0 keeps the current threshold). */
far_status far_set_regime(far_ctx *ctx, far_regime regime, int decode_max_rows);

/* Test hook for the bounded waits.  The TMA ring kernel's producer skips
 * the bulk copy of row segment `segment` (counted from 0 in each CTA's
 * order) in every later launch on this context, so the consumers' wait for
 * it has nothing to end it; every bounded wait then gives up after
 * wait_limit_us microseconds instead of 2 s (0: back to 2 s), the kernel
 * ends, and far_check returns FAR_ERR_TIMEOUT.  segment < 0 switches the
 * hook off.  Outputs of a stalled call are not valid. */
far_status far_test_stall(far_ctx *ctx, int64_t segment, uint32_t wait_limit_us);

/* Fill `info` with the launch geometry a far_fused / far_fused_rows call on
 * `rows` rows of W partials (and a residual when has_residual != 0, writing
 * norm_out when has_norm_out != 0) would use: far_describe_launch_pattern
 * with FAR_AR_RESIDUAL_RMSNORM (patterns 0-2 share one plan). */
far_status far_describe_launch(const far_ctx *ctx, int64_t rows, int64_t H,
                               far_dtype dtype, int W, int has_residual, int has_norm_out,
                               far_launch_info *info);

/* The same for a call of `pattern`.  FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP: the
 * one launch of far_fused_fp8_group (any group size); _FP8_TENSOR: the
 * first launch of far_fused_fp8_tensor, which on the ring kernel with a
 * residual_out or norm_out to read back (kernel 1) also runs the second
 * pass.  Both plan the ring kernel's CTAs per SM and slots by rules of
 * their own and never take the cluster kernel (regime 1 falls back to the
 * one-CTA kernel).  A pattern outside 0-4 gives FAR_ERR_INVALID_ARG. */
far_status far_describe_launch_pattern(const far_ctx *ctx, int64_t rows, int64_t H,
                                       far_dtype dtype, int W, int has_residual,
                                       int has_norm_out, far_pattern pattern,
                                       far_launch_info *info);

/* Wait for `stream`, then read and clear the device-side error word of
 * ctx's device.  FAR_ERR_TIMEOUT: a bounded wait inside a kernel launched
 * since the last far_check gave up (after 2 s), and the outputs of those
 * calls are not valid; the kernel still ended and the CUDA context stays
 * usable.  FAR_OK otherwise.  Synchronises `stream`; not for use during
 * stream capture. */
far_status far_check(far_ctx *ctx, void *stream);

/* Static text for a status code. */
const char *far_status_string(far_status s);

/* The CUDA error text of the calling thread's last FAR_ERR_CUDA ("" if none). */
const char *far_last_error(void);

/* FAR_VERSION of the built library. */
int far_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FAR_H_ */

/*
 * rrf.h -- C ABI of the fused "R-way bf16 sum + residual + RMSNorm + per-row
 * FP8 (e4m3fn) quantisation" library for NVIDIA B200 (sm_100a).
 *
 * The operation is the epilogue of an all-reduce, run on one GPU whose HBM
 * already holds the R rank-partial buffers:
 *
 *   Modular docs, Mojo function `allreduce_rmsnorm_fp8` (module
 *   nn/allreduce_residual_rmsnorm_fp8): a fused allreduce + RMSNorm + FP8
 *   dynamic quantisation in one kernel launch that skips the HBM round trip
 *   between the reduced buffer and the norm.  Its "Args" section fixes the
 *   argument set used here: R input buffers (last dim = cols), an FP8 output
 *   of the input's shape, gamma of length cols, epsilon, weight_offset (an
 *   additive offset for gamma), scale_ub (upper bound for the FP8 scale) and
 *   a float32 scale per row.  Its peer-to-peer transport and signal buffers
 *   have no counterpart on one GPU.
 *
 *   local-inference-lab/b12x PR #283 "PCIeTwoShotBF16": the partials are
 *   accumulated in fp32 in a fixed rank order and rounded to bf16 once, which
 *   makes the result deterministic and within one bf16 rounding of the exact
 *   sum.
 *
 * What one row i computes (x_r are the inputs; every operation is fp32 and
 * rounded once unless stated; RN_bf16 is round-to-nearest-even to bf16):
 *   s_j   = RN_bf16(((x_0 + x_1) + x_2) + ... + x_{R-1})      (rank order)
 *   h_j   = RN_bf16(s_j + residual_in_j), stored to residual_out   (or s_j)
 *   r     = 1 / sqrt(sum_j h_j^2 / cols + eps)
 *   y_j   = (h_j * r) * (gamma_j + weight_offset)
 *   scale = max(min(max_j |y_j|, scale_ub), 1e-12) / 448
 *   q_j   = e4m3fn(y_j / scale), nearest even, saturating at +-448
 *   scales[i] = scale            (dequantise as y ~ e4m3fn_value(q) * scale)
 * The bf16 outputs (s, residual_out) are exact.  The kernels reduce the sum
 * of squares as a fixed-order fp32 tree and take max_j |y_j| as
 * r * max_j |h_j * (gamma_j + weight_offset)| (the same products rounded in
 * the other order), so scales agree with the definition to about 1e-6
 * relative, and a code may differ by one step only where y / scale sits at
 * an e4m3 rounding midpoint.
 *
 * Conventions for every entry point
 *  - Layout: every 2-D array is contiguous row-major [rows, cols] (row stride
 *    cols elements).  bf16 arrays hold IEEE bfloat16, fp8 arrays hold
 *    e4m3fn codes (one byte each), scales are float32.
 *  - Pointers: all data pointers are DEVICE pointers (or managed / host-
 *    mapped memory the device can read).  The array `inputs` itself is a
 *    HOST array of R device pointers; it is copied into the launch's
 *    parameters, so it may be freed as soon as the call returns.
 *  - Ownership: the caller owns every buffer.  The library allocates no
 *    device memory and keeps no state between calls apart from a per-device
 *    cache of the SM count.
 *  - Asynchrony: work is enqueued on `stream` (NULL = the legacy default
 *    stream) and the call returns without synchronising.  Outputs are valid
 *    in stream order only.
 *  - Validation: every argument is checked on the host before any CUDA call.
 *    On an error the call returns a non-zero rrf_status and enqueues
 *    nothing.  rows == 0 is a valid empty call: it returns RRF_OK without
 *    looking at any pointer (empty torch tensors have null data pointers).
 *  - Aliasing: inputs may alias one another.  No output may overlap an
 *    input or another output, except residual_out == residual_in exactly
 *    (the in-place residual update).
 *  - Thread safety: calls from several host threads are safe; calls that
 *    overlap on the GPU and share an output race like any two kernels.
 */
#ifndef RRF_H
#define RRF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The same type as cudaStream_t; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st* rrf_stream_t;

typedef enum rrf_status {
    RRF_OK = 0,
    RRF_ERR_NULL = 1,        /* a required pointer is NULL                           */
    RRF_ERR_RANKS = 2,       /* num_inputs outside [1, RRF_MAX_INPUTS]               */
    RRF_ERR_SHAPE = 3,       /* rows < 0, cols <= 0, cols % 8 != 0, or too large     */
    RRF_ERR_ALIGN = 4,       /* a data pointer is not 16-byte aligned (scales: 4)    */
    RRF_ERR_ALIAS = 5,       /* an output overlaps an input or another output        */
    RRF_ERR_VALUE = 6,       /* eps < 0 or not finite, scale_ub <= 0 or NaN,
                                weight_offset not finite                              */
    RRF_ERR_UNSUPPORTED = 7, /* a forced variant / cluster size / block size that
                                cannot run this shape                                */
    RRF_ERR_CUDA = 8         /* a CUDA call failed: see rrf_last_cuda_error()        */
} rrf_status;

/* At most this many input buffers (the pages' systems use 2, 4 or 8 ranks;
 * the Ascend page allows up to 16). */
#define RRF_MAX_INPUTS 16

/* Largest cols the fused entry points accept (262144): a row is held in
 * registers across up to 16 cooperating blocks of 256 threads, each thread
 * holding 8 vectors of 8 elements. */
#define RRF_MAX_COLS (16 * 256 * 8 * 8)

/* rrf_sum -- the bf16 sum alone.
 *   out[i, j] = RN_bf16(x_0[i, j] + x_1[i, j] + ... + x_{R-1}[i, j]), fp32
 *   accumulation in rank order 0..R-1 (b12x PR #283, opening description).
 * inputs     host array of num_inputs device pointers, each bf16 [rows, cols],
 *            16-byte aligned
 * num_inputs R, 1..RRF_MAX_INPUTS
 * rows, cols rows >= 0; cols > 0 and a multiple of 8 (16-byte rows)
 * out        device pointer, bf16 [rows, cols], 16-byte aligned, must not
 *            overlap any input
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS, RRF_ERR_SHAPE, RRF_ERR_ALIGN,
 *         RRF_ERR_ALIAS, RRF_ERR_CUDA. */
rrf_status rrf_sum(const void* const* inputs, int num_inputs, int64_t rows,
                   int64_t cols, void* out, rrf_stream_t stream);

/* rrf_sum_rmsnorm_fp8 -- the fused operation (Modular docs,
 * `allreduce_rmsnorm_fp8`, "Args"; the residual form is the module name's
 * "residual" and TensorRT-LLM PR #19836's RESIDUAL_RMS_NORM epilogue).
 * inputs        host array of num_inputs device pointers, bf16 [rows, cols]
 * num_inputs    R, 1..RRF_MAX_INPUTS
 * rows, cols    rows >= 0; cols > 0, a multiple of 8, at most RRF_MAX_COLS
 * residual_in   bf16 [rows, cols] or NULL; residual_out bf16 [rows, cols] or
 *               NULL; both NULL (no residual) or both set; they may be equal
 * gamma         bf16 [cols]
 * eps           >= 0, finite (the pages type it as the input dtype; it is
 *               used here as the fp32 value given)
 * weight_offset finite, added to gamma in fp32 (1.0 for unit-offset gamma)
 * scale_ub      > 0 (may be +inf: no clamp)
 * q_out         fp8 e4m3fn codes [rows, cols], 16-byte aligned
 * scales_out    float32 [rows], 4-byte aligned
 * Every bf16 / fp8 pointer must be 16-byte aligned.
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS, RRF_ERR_SHAPE, RRF_ERR_ALIGN,
 *         RRF_ERR_ALIAS, RRF_ERR_VALUE, RRF_ERR_CUDA. */
rrf_status rrf_sum_rmsnorm_fp8(const void* const* inputs, int num_inputs,
                               int64_t rows, int64_t cols, const void* residual_in,
                               void* residual_out, const void* gamma, float eps,
                               float weight_offset, float scale_ub, void* q_out,
                               float* scales_out, rrf_stream_t stream);

/* Launch variants of the fused kernel. */
#define RRF_VARIANT_AUTO 0    /* the built-in choice (rrf_plan_fused)              */
#define RRF_VARIANT_ROW 1     /* one block per row                                 */
#define RRF_VARIANT_CLUSTER 2 /* each row split across a thread-block cluster of
                                 cluster_size blocks whose row statistics meet in
                                 distributed shared memory (TensorRT-LLM PR
                                 #19836: cluster.sync() before remote writes, one
                                 arrive / wait per thread per barrier phase)      */

/* Launch flags of rrf_sum_rmsnorm_fp8_ex. */
#define RRF_FLAG_NO_PDL 1            /* launch without programmatic dependent launch */
#define RRF_FLAG_BARRIER_EXCHANGE 2  /* clusters meet at a cluster barrier phase
                                        instead of the transaction-counted exchange */
#define RRF_FLAG_NO_PREFETCH 4       /* no L2 prefetch before the wait for the
                                        previous kernel (see below)              */
#define RRF_FLAG_PREFETCH 8          /* the L2 prefetch whatever the planner says */
#define RRF_FLAG_DEBUG_STARVE_EXCHANGE 0x100 /* test hook: every block of a cluster
                                        waits for one value more than its peers
                                        send, so its bounded wait runs out (about
                                        2 ms), the kernel sets
                                        RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT and
                                        finishes with meaningless codes and
                                        scales; selects the transaction-counted
                                        exchange and needs a cluster launch     */

/* rrf_sum_rmsnorm_fp8_ex -- rrf_sum_rmsnorm_fp8 with the launch forced, for
 * tests and benchmarks.  variant is one of RRF_VARIANT_*; cluster_size is
 * 2..16 for RRF_VARIANT_CLUSTER (0 = automatic; sizes above 8 are the
 * non-portable cluster sizes B200 allows) and ignored otherwise; block_threads is a multiple of 32 in [32, 1024] or 0
 * (automatic); flags combines RRF_FLAG_*.  Results are bit-identical across
 * variants for the bf16 outputs and agree within the stated tolerance for
 * scales and codes.
 *
 * Cluster exchange: the blocks of a row's cluster share their statistics
 * through st.async stores into each other's shared memory, counted on an
 * mbarrier that each block waits on (the default), or, with
 * RRF_FLAG_BARRIER_EXCHANGE, at a cluster barrier phase following the rules
 * of the TensorRT-LLM PR #19836 write-up: a completed phase before any
 * remote write, one arrive and one wait per thread per phase.  The mbarrier waits are bounded (about 2 ms):
 * a wait that runs out sets RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT in the device
 * error word (rrf_device_error) instead of hanging the GPU.
 *
 * Programmatic dependent launch: by default every kernel of this library is
 * launched so that it may start while the previous kernel in the stream is
 * still finishing; each kernel waits for that kernel (its completion and the
 * visibility of its writes) before it touches global memory, so stream order
 * is kept for every producer.  RRF_FLAG_NO_PDL launches the plain way.
 *
 * L2 prefetch: where the planner expects the grid to be resident at once
 * (decode-sized batches), each block first asks L2 for its slice of the
 * inputs, the residual and gamma (cp.async.bulk.prefetch.L2), then waits for
 * the previous kernel: the HBM fetch overlaps that kernel's tail.  A
 * prefetch returns no data and changes no value the kernel reads after the
 * wait (L2 is the point of coherence of the GPU's own memory), so this is
 * safe whatever the previous kernel writes; it gains nothing for data that
 * kernel has not yet written.  RRF_FLAG_NO_PREFETCH and RRF_FLAG_PREFETCH
 * override the planner.
 * Errors: those of rrf_sum_rmsnorm_fp8, and RRF_ERR_UNSUPPORTED when the
 * forced launch cannot cover the row or flags holds an unknown bit. */
rrf_status rrf_sum_rmsnorm_fp8_ex(const void* const* inputs, int num_inputs,
                                  int64_t rows, int64_t cols, const void* residual_in,
                                  void* residual_out, const void* gamma, float eps,
                                  float weight_offset, float scale_ub, void* q_out,
                                  float* scales_out, int variant, int cluster_size,
                                  int block_threads, int flags, rrf_stream_t stream);

/* ------------------------------------------------------------------------
 * MX output: per-block instead of per-row scales.
 *
 * Ascend CANN docs, aclnnAlltoAllQuantMatmul, mx scenario: the activations'
 * x1Scale has shape (BS, ceil(H/64), 2), one scale per 32 elements of a row.
 * OCP Microscaling Formats (MX) v1.0, conversion to MX: a block of 32
 * elements shares X = 2^(floor(log2(max |V|)) - 8) (8 being the exponent of
 * e4m3's largest normal, 448 = 1.75 * 2^8), stored as an E8M0 code (the
 * exponent biased by 127); each element becomes e4m3fn(V / X), nearest even,
 * saturating.
 *
 * rrf_sum_rmsnorm_mxfp8 -- the sum, the residual and the norm as in
 * rrf_sum_rmsnorm_fp8, then per block of 32 columns of y the E8M0 code of the
 * block's scale and the codes of y / X (no scale_ub: the scale follows the
 * block).  An all-zero block takes code 0.
 * inputs, num_inputs, rows, residual_in, residual_out, gamma, eps,
 * weight_offset   as for rrf_sum_rmsnorm_fp8
 * cols            a multiple of 32
 * q_out           fp8 e4m3fn codes [rows, cols], 16-byte aligned
 * scales_mx_out   E8M0 codes [rows, cols / 32] (one byte each)
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS, RRF_ERR_SHAPE, RRF_ERR_ALIGN,
 *         RRF_ERR_ALIAS, RRF_ERR_VALUE, RRF_ERR_CUDA. */
rrf_status rrf_sum_rmsnorm_mxfp8(const void* const* inputs, int num_inputs, int64_t rows,
                                 int64_t cols, const void* residual_in, void* residual_out,
                                 const void* gamma, float eps, float weight_offset, void* q_out,
                                 void* scales_mx_out, rrf_stream_t stream);

/* The blocked order of MX scale codes, the order the tensor cores'
 * block-scaled MMA reads them in (512-byte atoms of 128 rows x 4 blocks of
 * 32 columns): the code of row r, block j (of cols / 32) lives at byte
 *   ((r / 128) * (cols / 128) + j / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4
 * of a buffer of RRF_MX_BLOCKED_BYTES(rows, cols) bytes (rows rounded up to
 * 128; cols a multiple of 128).  Bytes of the rounded-up rows are not
 * written. */
#define RRF_MX_BLOCKED_BYTES(rows, cols) ((((rows) + 127) / 128) * 128 * ((cols) / 32))

/* rrf_sum_rmsnorm_mxfp8_blocked -- rrf_sum_rmsnorm_mxfp8 with the scale
 * codes in the blocked order (cols a multiple of 128; scales_mx_out holds
 * RRF_MX_BLOCKED_BYTES(rows, cols) bytes), ready for rrf_scaled_mm_mxfp8.
 * Errors: as rrf_sum_rmsnorm_mxfp8. */
rrf_status rrf_sum_rmsnorm_mxfp8_blocked(const void* const* inputs, int num_inputs,
                                         int64_t rows, int64_t cols, const void* residual_in,
                                         void* residual_out, const void* gamma, float eps,
                                         float weight_offset, void* q_out, void* scales_mx_out,
                                         rrf_stream_t stream);

/* The host validation of rrf_sum_rmsnorm_mxfp8 alone (no GPU needed). */
rrf_status rrf_check_mxfp8_args(const void* const* inputs, int num_inputs, int64_t rows,
                                int64_t cols, const void* residual_in, const void* residual_out,
                                const void* gamma, float eps, float weight_offset,
                                const void* q_out, const void* scales_mx_out);

/* ------------------------------------------------------------------------
 * The sharded form: a row's hidden dimension split across devices.
 *
 * Tenstorrent rmsnorm_2d.py (RMSNorm2D, decode_forward / prefill_forward)
 * splits the norm into a pre-all-gather pass that computes per-device row
 * statistics, an all-gather of those statistics, and a post-all-gather pass
 * that normalises each device's shard.  Here the statistics are the pair
 * (sum_j h_j^2, max_j |h_j * (gamma_j + weight_offset)|) over the shard's
 * columns, so the one exchange also carries what the FP8 scale needs: the
 * post pass combines the pairs of every shard in a fixed order (every shard
 * derives the same scale) and quantises its own columns.  The exchange itself
 * (an all-gather of rows * 8 bytes per shard) is the caller's (e.g. NCCL);
 * the result equals rrf_sum_rmsnorm_fp8 on the whole rows up to the order of
 * the fp32 sum of squares.
 * ---------------------------------------------------------------------- */

/* At most this many shards of a row. */
#define RRF_MAX_SHARDS 64

/* rrf_sum_rmsnorm_fp8_pre -- phase 1 on this device's column shard
 * [rows, cols]: the bf16 sum of the inputs, the optional residual (written
 * back), and per row the shard statistics.
 * inputs, num_inputs, rows, cols, residual_in, residual_out  as for
 *               rrf_sum_rmsnorm_fp8 (cols: this shard's columns)
 * h_out         bf16 [rows, cols], 16-byte aligned: receives the norm input
 *               h when there is no residual; must be NULL with a residual
 *               (residual_out then holds h)
 * gamma         bf16 [cols], this shard's gamma
 * weight_offset added to gamma (as for rrf_sum_rmsnorm_fp8)
 * stats_out     float [rows][2], 8-byte aligned: (sum of h^2, max |h * g'|)
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS, RRF_ERR_SHAPE, RRF_ERR_ALIGN,
 *         RRF_ERR_ALIAS, RRF_ERR_VALUE, RRF_ERR_CUDA. */
rrf_status rrf_sum_rmsnorm_fp8_pre(const void* const* inputs, int num_inputs, int64_t rows,
                                   int64_t cols, const void* residual_in, void* residual_out,
                                   void* h_out, const void* gamma, float weight_offset,
                                   float* stats_out, rrf_stream_t stream);

/* rrf_rmsnorm_fp8_post -- phase 2 on this device's column shard: codes and
 * scales from the norm input and the gathered statistics of all shards.
 * h             bf16 [rows, cols], this shard's norm input (phase 1's h_out
 *               or residual_out), 16-byte aligned
 * stats         float [shards][rows][2]: every shard's phase-1 statistics,
 *               in shard order, 8-byte aligned
 * shards        1..RRF_MAX_SHARDS
 * total_cols    the whole row's columns (the mean's divisor), >= cols
 * gamma         bf16 [cols], this shard's gamma
 * eps, weight_offset, scale_ub  as for rrf_sum_rmsnorm_fp8
 * q_out         fp8 e4m3fn codes [rows, cols], 16-byte aligned
 * scales_out    float [rows] or NULL (every shard derives the same scales,
 *               so one of them may write them)
 * Errors: RRF_ERR_NULL, RRF_ERR_SHAPE, RRF_ERR_ALIGN, RRF_ERR_ALIAS,
 *         RRF_ERR_VALUE, RRF_ERR_CUDA. */
rrf_status rrf_rmsnorm_fp8_post(const void* h, int64_t rows, int64_t cols, const float* stats,
                                int shards, int64_t total_cols, const void* gamma, float eps,
                                float weight_offset, float scale_ub, void* q_out,
                                float* scales_out, rrf_stream_t stream);

/* The host validation of the two phases alone (no GPU needed). */
rrf_status rrf_check_pre_args(const void* const* inputs, int num_inputs, int64_t rows,
                              int64_t cols, const void* residual_in, const void* residual_out,
                              const void* h_out, const void* gamma, float weight_offset,
                              const void* stats_out);
rrf_status rrf_check_post_args(const void* h, int64_t rows, int64_t cols, const float* stats,
                               int shards, int64_t total_cols, const void* gamma, float eps,
                               float weight_offset, float scale_ub, const void* q_out,
                               const void* scales_out);

/* ------------------------------------------------------------------------
 * The multi-GPU form: the `world` partials live on `world` GPUs.
 *
 * Modular docs, `allreduce_rmsnorm_fp8` (its description and the paragraph
 * on signal buffer sizing): one kernel launch does the all-reduce over peer
 * memory and the norm; below a payload threshold every GPU reduces all rows
 * itself (1-stage), above it every GPU reduces ceil(rows / ngpus) rows and
 * the FP8 rows and scales are then gathered (2-stage).  b12x PR #283: a rank
 * takes its rows from every peer and accumulates them in fp32 in fixed rank
 * order, rounding once.  TensorRT-LLM PR #19836: arrivals are counted per
 * CTA.
 *
 * One call is one kernel per rank that reads and writes the other ranks'
 * buffers directly (peer loads and stores over NVLink / NVSwitch):
 *  - start barrier: block b of every rank tells block b of every rank that
 *    it runs (the rank's input, produced earlier in its stream, is ready)
 *    and waits for the same word from every rank;
 *  - one-shot (RRF_AR_ONE_SHOT): every rank computes every row from all
 *    ranks' partials and writes its own outputs;  two-shot
 *    (RRF_AR_TWO_SHOT): rank k computes rows [k*P, min((k+1)*P, rows)),
 *    P = ceil(rows / world), and stores their codes, scales and residual
 *    into every rank's outputs;
 *  - end barrier: the same words again after the stores; when the call has
 *    completed on a rank (stream order) its outputs are whole and no peer
 *    reads its input any more, so the caller may overwrite it.
 * A row's arithmetic is that of rrf_sum_rmsnorm_fp8 with the partials as
 * inputs in rank order: the bf16 sum and residual are the same bits, scales
 * and codes agree within that call's tolerance (the same bits for the same
 * launch shape).
 *
 * Buffers: every pointer array has `world` entries, entry j being rank j's
 * buffer as this GPU addresses it: a peer mapping in a job with one process
 * per GPU (every rank passes the same buffers, each through its own
 * mappings), or another buffer of this GPU when one launch runs all ranks
 * (local_ranks == world, used to run the whole exchange on one GPU).
 * Signal pads: RRF_AR_SIGNAL_WORDS 32-bit words per rank, zeroed once before
 * the first call.  Besides the barrier words a pad holds one call counter
 * per block, which the kernel itself advances, so the calls need no number
 * from the host and a call captured in a CUDA graph stays correct when the
 * graph is replayed.  Every rank must make the same sequence of calls on its
 * pads.  After RRF_DEVICE_ERROR_PEER_TIMEOUT the pads must be zeroed again.
 * ---------------------------------------------------------------------- */

#define RRF_AR_MAX_WORLD 8
#define RRF_AR_MAX_BLOCKS 1024 /* blocks per rank of one launch */
#define RRF_AR_SIGNAL_WORDS ((2 * RRF_AR_MAX_WORLD + 1) * RRF_AR_MAX_BLOCKS)
#define RRF_AR_AUTO 0     /* two-shot when every rank gets a row, else one-shot */
#define RRF_AR_ONE_SHOT 1
#define RRF_AR_TWO_SHOT 2

/* rrf_allreduce_rmsnorm_fp8 -- one call of the multi-GPU form.
 * inputs        [world] bf16 [rows, cols] partials, 16-byte aligned
 * residual_in   [world] bf16 [rows, cols] residuals (rank j reads entry j;
 *               all ranks hold the same residual), or NULL for none
 * residual_out  [world] bf16 [rows, cols], NULL exactly when residual_in is;
 *               entry j may equal residual_in[j] (in place)
 * q_out         [world] fp8 e4m3fn codes [rows, cols], 16-byte aligned
 * scales_out    [world] float [rows], 4-byte aligned
 * signals       [world] pads of RRF_AR_SIGNAL_WORDS words, 16-byte aligned
 * world         1..RRF_AR_MAX_WORLD;  rank: this process's rank (0 when
 *               local_ranks == world);  local_ranks: 1 or world
 * rows, cols, gamma, eps, weight_offset, scale_ub  as for rrf_sum_rmsnorm_fp8
 *               (gamma: this GPU's copy); cols <= 8 * 8 * 512 * 4
 * mode          RRF_AR_*
 * timeout_ns    bound on each barrier wait (0 = one second)
 * Every rank must make the same call (same shape and mode).
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS (world or rank out of range),
 *         RRF_ERR_SHAPE, RRF_ERR_ALIGN, RRF_ERR_ALIAS, RRF_ERR_VALUE,
 *         RRF_ERR_UNSUPPORTED (mode or local_ranks out of
 *         range, or all ranks' blocks cannot be resident on this GPU at
 *         once), RRF_ERR_CUDA. */
rrf_status rrf_allreduce_rmsnorm_fp8(const void* const* inputs, const void* const* residual_in,
                                     void* const* residual_out, void* const* q_out,
                                     float* const* scales_out, unsigned int* const* signals,
                                     int world, int rank, int local_ranks, int64_t rows,
                                     int64_t cols, const void* gamma, float eps,
                                     float weight_offset, float scale_ub, int mode,
                                     uint64_t timeout_ns, rrf_stream_t stream);

/* The host validation of rrf_allreduce_rmsnorm_fp8 alone (no GPU needed). */
rrf_status rrf_check_allreduce_args(const void* const* inputs, const void* const* residual_in,
                                    void* const* residual_out, void* const* q_out,
                                    float* const* scales_out, unsigned int* const* signals,
                                    int world, int rank, int local_ranks, int64_t rows,
                                    int64_t cols, const void* gamma, float eps,
                                    float weight_offset, float scale_ub, int mode);

/* rrf_plan_allreduce -- the mode and row shape rrf_allreduce_rmsnorm_fp8
 * picks on a GPU with sm_count SMs, without touching the GPU: the mode
 * (RRF_AR_ONE_SHOT / RRF_AR_TWO_SHOT), blocks per row, threads per block and
 * 16-byte vectors per thread.  (The blocks per rank also depend on the
 * occupancy of the compiled kernel, known only on the device.)
 * Errors: RRF_ERR_NULL, RRF_ERR_RANKS, RRF_ERR_SHAPE, RRF_ERR_UNSUPPORTED. */
rrf_status rrf_plan_allreduce(int world, int64_t rows, int64_t cols, int residual, int mode,
                              int sm_count, int* mode_out, int* cluster_size,
                              int* block_threads, int* vecs_per_thread);

/* ------------------------------------------------------------------------
 * The multi-GPU form without any allocation by the caller.
 *
 * No page has a counterpart to this entry point; it is a library service.
 * Some callers cannot allocate device memory: a program whose device memory
 * is all owned by another allocator (a framework's caching pool that has
 * reserved the GPU, where an outside cudaMalloc can fail or fragment the
 * pool), code that must not call cudaMalloc / cudaFree because they may
 * synchronise the whole device (a latency-bound serving loop), or a plug-in
 * whose host forbids allocation after start-up.  Such a caller still owns
 * and passes every input and output; the signal pads, the call's only
 * scratch memory, come from a fixed array inside the library.
 * ---------------------------------------------------------------------- */

/* Ranks whose signal pads the library's fixed array holds:
 * RRF_AR_STATIC_MAX_WORLD * RRF_AR_SIGNAL_WORDS 32-bit words (544 KiB),
 * held on every GPU that loads the library until the process exits. */
#define RRF_AR_STATIC_MAX_WORLD 8

/* rrf_allreduce_rmsnorm_fp8_static -- rrf_allreduce_rmsnorm_fp8 with every
 * rank in one launch on the current GPU (local_ranks == world, rank 0) and
 * the signal pads taken from the library's fixed array: the call allocates
 * no memory (no cudaMalloc, cudaFree or allocating library routine).
 * Arguments, results and errors are those of rrf_allreduce_rmsnorm_fp8
 * without `signals`, `rank` and `local_ranks`; every pointer entry is a
 * buffer of this GPU.
 * world    1..RRF_AR_STATIC_MAX_WORLD; a larger world is rejected with
 *          RRF_ERR_RANKS before any CUDA call.
 * Set-up: the first call on a device (with that device current) looks up
 * the array's device address once and keeps it; make that first call
 * before any stream capture.  Failing look-up: RRF_ERR_CUDA.
 * Sharing: every call uses the same array, which keeps the last call's
 * contents; each call zeroes the pads it uses, in stream order, before its
 * kernel.  Calls that overlap on the GPU (on two streams, or from two host
 * threads without ordering between their streams) race on the pads; order
 * them on one stream or with events. */
rrf_status rrf_allreduce_rmsnorm_fp8_static(const void* const* inputs,
                                            const void* const* residual_in,
                                            void* const* residual_out, void* const* q_out,
                                            float* const* scales_out, int world, int64_t rows,
                                            int64_t cols, const void* gamma, float eps,
                                            float weight_offset, float scale_ub, int mode,
                                            uint64_t timeout_ns, rrf_stream_t stream);

/* ------------------------------------------------------------------------
 * A consumer of the per-row scales: the FP8 GEMM that follows the
 * quantisation in a transformer layer.
 *
 * Ascend CANN docs, aclnnAlltoAllQuantMatmul (the formulas of its K-C and
 * per-token dynamic quantisation scenarios): after the activations x1 are
 * quantised per token (row) with scale x1Scale, the product is
 * out = (x1_q @ x2) * x1Scale * x2Scale (+ bias), x2Scale one per output
 * column.  Here x1_q and x1Scale are exactly the codes and scales that
 * rrf_sum_rmsnorm_fp8 writes, and x2 is a weight stored like a linear
 * layer's, one row of K codes per output column:
 *
 *   out[m][n] = RN_bf16( (sum_k e4m3(a[m][k]) * e4m3(b[n][k])) * a_scale[m]
 *                        * b_scale[n] + bias[n] )
 *
 * The products of two e4m3 values are exact; the tensor cores sum them in
 * fp32 (in an order of their own), then the epilogue multiplies by the two
 * scales, adds bias and rounds once to bf16.
 * ---------------------------------------------------------------------- */

/* rrf_scaled_mm_fp8 -- the GEMM above on the tensor cores (sm_100a).
 * a         e4m3fn codes [M, K] row-major (K contiguous), 16-byte aligned
 * a_scale   float [M] (per row: rrf_sum_rmsnorm_fp8's scales_out), 4-byte aligned
 * b         e4m3fn codes [N, K] row-major (K contiguous), 16-byte aligned
 * b_scale   float [N] (per output column), 4-byte aligned
 * bias      bf16 [N] or NULL, 2-byte aligned
 * out       bf16 [M, N] row-major, 16-byte aligned
 * M, N, K   M >= 0 (M == 0 is a no-op); N, K >= 16 and multiples of 16
 * Errors: RRF_ERR_NULL, RRF_ERR_SHAPE, RRF_ERR_ALIGN, RRF_ERR_ALIAS (out
 *         overlapping an operand), RRF_ERR_CUDA. */
rrf_status rrf_scaled_mm_fp8(const void* a, const float* a_scale, const void* b,
                             const float* b_scale, const void* bias, void* out, int64_t M,
                             int64_t N, int64_t K, rrf_stream_t stream);

/* rrf_scaled_mm_mxfp8 -- the GEMM of the mx scenario of the same page:
 * out = (x1 * x1Scale) @ (x2 * x2Scale) + bias with one E8M0 scale per 32
 * values of K on both operands,
 *   out[m][n] = RN_bf16( sum_k e4m3(a[m][k]) 2^(sa[m][k/32] - 127)
 *                              e4m3(b[n][k]) 2^(sb[n][k/32] - 127) + bias[n] )
 * on the tensor cores' block-scaled MMA (fp32 accumulation, one rounding).
 * a, b      e4m3fn codes [M, K] and [N, K], row-major, 16-byte aligned
 * sa, sb    E8M0 codes in the blocked order (RRF_MX_BLOCKED_BYTES(M, K) and
 *           (N, K) bytes; rrf_sum_rmsnorm_mxfp8_blocked writes sa), 16-byte
 *           aligned.  The codes of rounded-up rows may hold anything: they
 *           only scale output rows and columns that are not stored.
 * bias      bf16 [N] or NULL;  out  bf16 [M, N], 16-byte aligned
 * M >= 0 (0 is a no-op); N >= 16 and a multiple of 16; K a multiple of 128
 * Errors: RRF_ERR_NULL, RRF_ERR_SHAPE, RRF_ERR_ALIGN, RRF_ERR_ALIAS,
 *         RRF_ERR_CUDA. */
rrf_status rrf_scaled_mm_mxfp8(const void* a, const void* sa, const void* b, const void* sb,
                               const void* bias, void* out, int64_t M, int64_t N, int64_t K,
                               rrf_stream_t stream);

/* The host validation of rrf_scaled_mm_mxfp8 alone (no GPU needed). */
rrf_status rrf_check_scaled_mm_mx_args(const void* a, const void* sa, const void* b,
                                       const void* sb, const void* bias, const void* out,
                                       int64_t M, int64_t N, int64_t K);

/* The host validation of rrf_scaled_mm_fp8 alone (no GPU needed). */
rrf_status rrf_check_scaled_mm_args(const void* a, const float* a_scale, const void* b,
                                    const float* b_scale, const void* bias, const void* out,
                                    int64_t M, int64_t N, int64_t K);

/* GEMM kernels (rrf_plan_scaled_mm). */
#define RRF_GEMM_KERNEL_PAIR 1 /* 256 x 256 tiles on SM pairs (two-CTA MMA)           */
#define RRF_GEMM_KERNEL_TILE 2 /* one persistent CTA per SM walking 128 x tile_n output
                                  tiles, its A stages a_rows rows                     */
#define RRF_GEMM_KERNEL_SWAP 3 /* operands swapped, 64 weight rows of each of two
                                  k-tiles on the MMA's M side, the call's rows padded
                                  to a_rows (per-token and MX, at most 32 rows)       */

/* rrf_plan_scaled_mm -- the kernel rrf_scaled_mm_fp8 (mx == 0) or
 * rrf_scaled_mm_mxfp8 (mx != 0) runs for an M x N x K product on a GPU with
 * sm_count SMs, without touching the GPU: its RRF_GEMM_KERNEL_*, the rows of
 * an A stage, the output columns of a tile (for RRF_GEMM_KERNEL_SWAP the 64
 * weight rows of a tile), the k-tiles of 128 bytes per TMA box, the output
 * tiles and the CTAs launched (ctas < tiles: CTAs walk several tiles).
 * M == 0 launches nothing: kernel 0, tiles and ctas 0.
 * Errors: RRF_ERR_NULL (an output pointer), RRF_ERR_SHAPE (a shape the call
 * rejects), RRF_ERR_UNSUPPORTED (sm_count < 2). */
rrf_status rrf_plan_scaled_mm(int64_t M, int64_t N, int64_t K, int mx, int sm_count,
                              int* kernel, int* a_rows, int* tile_n, int* k_tiles_per_stage,
                              int64_t* tiles, int64_t* ctas);

/* rrf_plan_fused -- the launch rrf_sum_rmsnorm_fp8 would use on a GPU with
 * sm_count SMs for a call with (residual != 0) or without a residual,
 * without touching the GPU.  Writes the cluster size (1 = one
 * block per row), the threads per block and the 16-byte vectors each thread
 * holds.
 * Returns RRF_ERR_SHAPE / RRF_ERR_RANKS for shapes the library rejects and
 * RRF_ERR_NULL for a null output pointer. */
rrf_status rrf_plan_fused(int num_inputs, int64_t rows, int64_t cols, int residual,
                          int sm_count, int* cluster_size, int* block_threads,
                          int* vecs_per_thread);

/* rrf_plan_fused_ex -- rrf_plan_fused with the launch's L2-prefetch choice
 * (1: each block prefetches its slice before waiting for the previous
 * kernel; see rrf_sum_rmsnorm_fp8_ex).  The launch comes from the library's
 * table of measured launches (the entry nearest to the shape), adjusted so
 * that every block keeps at least 32 vectors and fits its slice.
 * Errors: those of rrf_plan_fused. */
rrf_status rrf_plan_fused_ex(int num_inputs, int64_t rows, int64_t cols, int residual,
                             int sm_count, int* cluster_size, int* block_threads,
                             int* vecs_per_thread, int* prefetch);

/* rrf_check_sum_args / rrf_check_fused_args -- the host-side validation of
 * rrf_sum / rrf_sum_rmsnorm_fp8 alone: the status those calls would return
 * before any CUDA call (RRF_OK if the arguments are valid).  No GPU needed. */
rrf_status rrf_check_sum_args(const void* const* inputs, int num_inputs, int64_t rows,
                              int64_t cols, const void* out);
rrf_status rrf_check_fused_args(const void* const* inputs, int num_inputs, int64_t rows,
                                int64_t cols, const void* residual_in,
                                const void* residual_out, const void* gamma, float eps,
                                float weight_offset, float scale_ub, const void* q_out,
                                const void* scales_out);

/* Device error bits. */
#define RRF_DEVICE_ERROR_EXCHANGE_TIMEOUT 1u /* a cluster block's bounded wait for its
                                               peers' statistics ran out          */
#define RRF_DEVICE_ERROR_PEER_TIMEOUT 2u /* a multi-GPU barrier wait for a peer
                                            rank ran out                      */
#define RRF_DEVICE_ERROR_GEMM_TIMEOUT 4u /* a wait of the FP8 GEMM's operand
                                            pipeline ran out                  */
#define RRF_DEVICE_ERROR_BOUNDS 8u /* the bounds-checking build (librrf_debug.so,
                                      compiled with RRF_DEBUG) found an index
                                      outside its buffer and skipped that
                                      access; never set by the normal build    */

/* rrf_device_error -- the device error word of the current device: the OR
 * of RRF_DEVICE_ERROR_* bits that kernels of this library have set since it
 * was last cleared.  Synchronises the device first (all streams), so call it
 * between steps, not inside stream capture.  clear != 0 resets the word.
 * Errors: RRF_ERR_NULL, RRF_ERR_CUDA. */
rrf_status rrf_device_error(unsigned int* flags, int clear);

/* Text for a status code (static storage, never NULL). */
const char* rrf_status_string(rrf_status status);

/* The cudaError_t of the last RRF_ERR_CUDA returned on this host thread
 * (0 if none). */
int rrf_last_cuda_error(void);

/* Test hook for the error path: the next launch on this host thread reports
 * the given cudaError_t value without launching anything (0 clears it), so
 * the RRF_ERR_CUDA path can be tested without making a GPU fail. */
void rrf_debug_fail_next_launch(int cuda_error);

/* Test hook for the GEMMs' bounded waits: the next rrf_scaled_mm_fp8 or
 * rrf_scaled_mm_mxfp8 call on this host thread that launches (a call
 * rejected on the host, or with M == 0, leaves the hook set) runs, but its
 * epilogue, after each accumulator it drains, also waits for that
 * accumulator's next completion, which cannot come before the epilogue
 * releases it.  The wait runs out (100 ms), the kernel sets
 * RRF_DEVICE_ERROR_GEMM_TIMEOUT in the device error word and finishes; the
 * output of that call is incomplete.  So the failure path is tested without
 * making a GPU fault or hang. */
void rrf_debug_starve_next_gemm(void);

/* Library version, "major.minor.patch". */
const char* rrf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RRF_H */

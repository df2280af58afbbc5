/*
 * cce.h: C ABI of libcce.so, the Cut Cross-Entropy (CCE) hot path for NVIDIA B200 (sm_100a).
 *
 * The problem (Cut Your Losses in Large-Vocabulary Language Models, abstract; mlx-cross-entropy
 * README, "How it works" and "API"): hidden states E [N, D], classifier C [V, D] and targets
 * t [N]. Logits z = E C^T never reach global memory. The forward returns the cross-entropy loss
 * and the per-row log-sum-exp (LSE). The backward recomputes logit tiles, skips tiles whose
 * softmax is below filter_eps (2^-12 by default), and returns dE and dC. An optional classifier
 * bias [V] is added to every row of logits (z = E C^T + bias); its gradient is returned too.
 *
 * Conventions for every call:
 *  - Pointers marked "device" are CUDA device pointers of the current device. The caller owns
 *    every buffer, workspaces included. The library allocates nothing and keeps no state between
 *    calls, with two exceptions: the fixed scratch array of cce_forward_noalloc() and the
 *    optional per-thread instrumentation set by cce_set_kernel_events().
 *  - E and C are bf16, row-major with contiguous rows (row stride = D elements). D must be a
 *    multiple of 8 and every pointer 16-byte aligned. targets is int64 [N].
 *  - All work is enqueued on `stream` and is asynchronous. Argument errors are returned
 *    synchronously, before anything is enqueued. Errors found on the device (a target outside
 *    [0, V) that is not ignore_index; a bounded wait inside a kernel that ran out) are written
 *    into the workspace and reported by cce_check_device_error(); the outputs of that call are
 *    then undefined.
 *  - cce_last_error_message() gives a human-readable detail of the last failing call on the
 *    calling thread.
 */
#ifndef CCE_H_
#define CCE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CCE_API __attribute__((visibility("default")))
#else
#define CCE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL means the legacy default stream. */
typedef struct CUstream_st* cce_stream_t;

typedef enum {
  CCE_OK = 0,
  CCE_ERR_INVALID_ARG = 1,     /* null pointer, bad size, misalignment, bad reduction */
  CCE_ERR_UNSUPPORTED = 2,     /* device is not sm_100 or a size is beyond what the kernels take */
  CCE_ERR_WORKSPACE = 3,       /* workspace smaller than the *_workspace_size() result */
  CCE_ERR_TARGET_RANGE = 4,    /* device: a target outside [0, V) that is not ignore_index */
  CCE_ERR_DEVICE_TIMEOUT = 5,  /* device: a bounded wait in a kernel ran out */
  CCE_ERR_CUDA = 6             /* a CUDA runtime/driver call failed */
} cce_status;

typedef enum {
  CCE_REDUCTION_NONE = 0, /* per-token loss [N] */
  CCE_REDUCTION_MEAN = 1, /* sum over non-ignored tokens / max(count, 1) */
  CCE_REDUCTION_SUM = 2   /* sum over non-ignored tokens */
} cce_reduction;

/* mlx-cross-entropy README, "API" table: flat [N, D] inputs, reduction, ignore_index (-100). */
typedef struct {
  int64_t N;            /* tokens: rows of E and entries of targets; >= 0 */
  int64_t D;            /* hidden size; multiple of 8, >= 8 */
  int64_t V;            /* vocabulary size: rows of C; >= 1 */
  int64_t ignore_index; /* a target equal to this masks the token (no loss, zero gradient) */
  int32_t reduction;    /* cce_reduction */
  int32_t reserved;     /* must be 0 */
  /* Loss variants (Loss functions explainer, "How it works" item 3 and "Implementation notes");
   * 0 and 0 give the plain cross-entropy. Per non-ignored token the loss is
   *   LSE - (1 - label_smoothing) z_t - (label_smoothing / V) sum_v z_v + z_loss LSE^2
   * and its logit gradient (1 + 2 z_loss LSE) p - (1 - label_smoothing) onehot - label_smoothing / V.
   * Tile skipping drops only the softmax part; the rest is exact. */
  float label_smoothing; /* in [0, 1] */
  float z_loss;          /* >= 0 (PaLM uses 1e-4) */
  /* Vocabulary sharding (the classifier split by rows over several GPUs, each holding a contiguous
   * range of the vocabulary). vocab_total = 0: not sharded, C is the whole classifier (vocab_start
   * must then be 0). vocab_total > 0: C holds rows [vocab_start, vocab_start + V) of a classifier of
   * vocab_total rows, targets are ids in [0, vocab_total), and a target outside this shard's range
   * marks a token that is scored here (its logits enter the softmax) but whose onehot term and
   * correct-token logit belong to another shard. Forward: cce_forward_partial on every shard, an
   * exchange of the partial results, then cce_forward_merge. Backward: cce_backward on every shard
   * with the merged LSE and count; dC (and dbias) are this shard's rows, dE is this shard's part of
   * dE, summed over the shards by the caller. */
  int64_t vocab_start;
  int64_t vocab_total;
} cce_problem;

/* Output dtypes of cce_backward (its out_fp32 argument). */
#define CCE_OUT_BF16 0     /* dE, dC, dbias bf16 */
#define CCE_OUT_FP32 1     /* dE, dC, dbias fp32 */
#define CCE_OUT_DE_FP32 2  /* dE fp32 (a shard's part, to be summed over shards), dC and dbias bf16 */

/* Width of the vocabulary sub-tile whose per-row maximum logit the forward saves. */
#define CCE_VOCAB_SUBTILE 64

/* Number of floats in the saved tile-max buffer: ceil(V / 64) * N. Layout [ceil(V/64), N]:
 * entry (j, r) is max_{v in [64 j, 64 j + 64) and v < V} z[r, v]. -1 for a bad problem. */
CCE_API int64_t cce_tile_max_len(const cce_problem* p);

/* Rows and vocabulary columns of one unit of the backward's skip rule (128 x 64): the rule decides
 * per unit of this size (mlx-cross-entropy README, "How it works" item 2); the kernels work on
 * 128 x 128 tiles made of two such units and skip the work of a skipped one. */
CCE_API void cce_backward_tile_shape(int32_t* tile_rows, int32_t* tile_cols);

/* Bytes of device workspace cce_forward() needs (0 for a bad problem). */
CCE_API size_t cce_forward_workspace_size(const cce_problem* p);

/* Bytes of device workspace cce_backward() needs: the tile plan (about 41 bytes per 128 x 128
 * tile), the gradient tiles of two vocabulary chunks (4 MiB per 128 rows, at least 128 MiB) and,
 * with out_fp32 = 0, the fp32 accumulators of dE and dbias, (N * D + V) * 4 bytes. Never anything
 * of size N * V. */
CCE_API size_t cce_backward_workspace_size(const cce_problem* p, int32_t out_fp32);

/*
 * Forward: loss and per-row LSE without materialising the logits z = E C^T + bias.
 * Cut Your Losses abstract (only the correct token's logit is computed; the log-sum-exp over
 * the vocabulary is evaluated on the fly); Cut Cross Entropy from first principles
 * (loss = LSE - z_correct); mlx-cross-entropy README, "How it works" item 1 (tile-wise max and
 * sum-exp) and "API" (bias, reduction, ignore_index).
 *
 *  E        device bf16 [N, D]          C       device bf16 [V, D]
 *  bias     device bf16 [V], added to every row of logits; NULL for none
 *  targets  device int64 [N]
 *  loss     device fp32: [1] for mean/sum, [N] for none (0 at ignored tokens)
 *  lse      device fp32 [N]: log-sum-exp of each row's logits (computed for ignored rows too)
 *  tile_max device fp32 [cce_tile_max_len(p)]: saved for cce_backward()
 *  count    device int64 [1]: number of non-ignored tokens
 *  workspace/workspace_bytes: device scratch of at least cce_forward_workspace_size(p) bytes;
 *           it also holds the device error word read by cce_check_device_error().
 * N = 0 is allowed (loss 0, count 0). After a device error the loss is NaN (every entry for none).
 */
CCE_API cce_status cce_forward(const cce_problem* p, const void* E, const void* C, const void* bias,
                               const int64_t* targets, float* loss, float* lse, float* tile_max, int64_t* count,
                               void* workspace, size_t workspace_bytes, cce_stream_t stream);

/*
 * Backward: dE = G C, dC = G^T E and dbias = sum_r G[r, :] with G = scale_r * (p~ - onehot),
 * p = softmax(z),
 * recomputed tile by tile from E, C and the saved LSE. p~ is p with every skipped unit set to 0:
 * a unit (tile_rows x tile_cols, see cce_backward_tile_shape) is skipped when, for every
 * non-ignored row r in it, max over its columns of z[r, v] - LSE[r] < ln(filter_eps); a unit
 * without a non-ignored row is skipped too. filter_eps <= 0 keeps every unit. The onehot term
 * is never skipped. Loss functions explainer, "How it works" item 2 (gradient p - y);
 * mlx-cross-entropy README, "How it works" items 2 and 3 (skipping, accumulation).
 * scale_r = g / max(count, 1) (mean), g (sum) or g[r] (none); 0 for ignored rows. With the loss
 * variants of cce_problem, G is scale_r times the logit gradient given there; only its softmax
 * part (1 + 2 z_loss LSE) p~ is skipped.
 *
 *  E, C, bias, targets, lse, tile_max, count: as given to / produced by cce_forward() on the
 *           same problem (bias NULL for none)
 *  grad_out device fp32: [1] for mean/sum, [N] for none
 *  dE       device [N, D], dC device [V, D], dbias device [V] or NULL (not computed): all bf16 when
 *           out_fp32 = CCE_OUT_BF16, all fp32 when CCE_OUT_FP32, dE fp32 and the others bf16 when
 *           CCE_OUT_DE_FP32. Fully overwritten. Rows of ignored tokens in dE are exactly +0. dbias is
 *           the gradient of the bias (also when bias is NULL, i.e. zero).
 *  For a vocabulary shard (p->vocab_total > 0): lse and count are the merged values of
 *  cce_forward_merge, tile_max is this shard's from cce_forward_partial; dE is this shard's part.
 *  filtered_tiles device int64 [1]: number of skipped units (tile_rows x tile_cols)
 *  workspace: device scratch of at least cce_backward_workspace_size(p, out_fp32) bytes.
 */
CCE_API cce_status cce_backward(const cce_problem* p, const void* E, const void* C, const void* bias,
                                const int64_t* targets, const float* lse, const float* tile_max,
                                const int64_t* count, const float* grad_out, float filter_eps, void* dE, void* dC,
                                void* dbias, int32_t out_fp32, int64_t* filtered_tiles, void* workspace,
                                size_t workspace_bytes, cce_stream_t stream);

/* The skip decision of every unit of the skip rule taken by the last cce_backward() that ran on
 * `workspace` for the same problem: skipped[b * nt + t] = 1 when unit (row block b, vocabulary
 * block t) was skipped and 0 when it was kept, with nb = ceil(N / tile_rows) row blocks,
 * nt = ceil(V / tile_cols) vocabulary blocks (cce_backward_tile_shape) and b < nb, t < nt. A
 * diagnostic of the skip rule of mlx-cross-entropy README, "How it works" item 2: the count of ones
 * equals filtered_tiles.
 *  workspace: the backward workspace of that call (workspace_bytes as given to it); it is read,
 *             not changed, so call this after the backward on the same stream.
 *  skipped:   device uint8 [nb * nt].
 * Enqueued on `stream`; argument errors return synchronously. N = 0 writes nothing. */
CCE_API cce_status cce_backward_skip_map(const cce_problem* p, const void* workspace, size_t workspace_bytes,
                                         uint8_t* skipped, cce_stream_t stream);

/*
 * Forward of one vocabulary shard (p->vocab_total > 0; also valid for an unsharded problem). Per row
 * it returns the partial results that cce_forward_merge combines over all shards:
 *  partial  device fp32 [3, N]: row 0 the log-sum-exp of the row's logits over this shard's
 *           columns, row 1 the correct-token logit when the target lies in this shard (else 0),
 *           row 2 the sum of the row's logits over this shard (label smoothing only; else 0).
 *  tile_max device fp32 [cce_tile_max_len(p)]: this shard's saved maxima, for cce_backward.
 *  E, C (this shard's rows), bias (this shard's entries, or NULL), targets (global ids) and the
 *  workspace (cce_forward_workspace_size(p) bytes; it holds the device error word: a target outside
 *  [0, vocab_total) that is not ignore_index) as for cce_forward.
 * The log-sum-exp over the whole vocabulary is the log-sum-exp of the shards' row-0 values (Loss
 * functions explainer, "How it works" item 1: stable log-sum-exp; mlx-cross-entropy README, "How it
 * works" item 1: partial maxima and sums combine).
 */
CCE_API cce_status cce_forward_partial(const cce_problem* p, const void* E, const void* C, const void* bias,
                                       const int64_t* targets, float* partial, float* tile_max, void* workspace,
                                       size_t workspace_bytes, cce_stream_t stream);

/*
 * Combines the partial results of `shards` vocabulary shards (each [3, N] from cce_forward_partial,
 * stacked as device fp32 [shards, 3, N] in any shard order) into the loss, the LSE over the whole
 * vocabulary and the count, as cce_forward returns them. p describes the whole problem: V is the
 * full vocabulary size (vocab_total of the shards), vocab_start = 0 and vocab_total = 0 or V.
 * Needs no workspace; the reduction over rows runs in a fixed order (deterministic).
 */
CCE_API cce_status cce_forward_merge(const cce_problem* p, const float* partials, int32_t shards,
                                     const int64_t* targets, float* loss, float* lse, int64_t* count,
                                     cce_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word kept at the start of
 * `workspace` (a forward or backward workspace passed to an earlier call on that stream).
 * Returns CCE_OK, CCE_ERR_TARGET_RANGE, CCE_ERR_DEVICE_TIMEOUT or CCE_ERR_CUDA. */
CCE_API cce_status cce_check_device_error(void* workspace, cce_stream_t stream);

/* Static description of a status code. */
CCE_API const char* cce_status_string(cce_status s);

/* Detail of the last failing call on the calling thread ("" if none). */
CCE_API const char* cce_last_error_message(void);

/* Bytes of device scratch the library holds, per GPU that loads it, for cce_forward_noalloc(). */
#define CCE_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * Forward that allocates nothing and takes no workspace, for callers that cannot allocate device
 * memory where they compute the loss: an embedding host that hands the library only fixed,
 * pre-registered buffers for inputs and outputs and owns all other device memory, or a runtime
 * whose allocator must not be re-entered from inside a loss callback. The pages have no
 * counterpart; it is an addition for such callers. Arguments and results are those of
 * cce_forward() without the workspace.
 *  - Scratch lives in one device array of CCE_NOALLOC_SCRATCH_BYTES that every GPU loading the
 *    library holds until exit. Problems needing more (about ceil(V/64) * N * 4 + 5 N + 4 D bytes; at
 *    V = 128256 up to N of about 4100) are rejected with CCE_ERR_UNSUPPORTED before anything runs.
 *  - The first call on each device looks up the array's device address (with that device
 *    current); make that first call before any stream capture.
 *  - Every call shares the array and the array keeps the last call's contents (the call clears
 *    what must start at zero), so calls whose work overlaps on the GPU (other streams, other
 *    threads) race and give undefined results; serialise them.
 *  - Device-side errors (a target outside [0, V) that is not ignore_index; a bounded wait inside a
 *    kernel that ran out, after CCE_WAIT_TIMEOUT_MS milliseconds as for cce_forward) cannot be
 *    returned, since the call does not wait for the GPU: the loss (every entry for reduction none)
 *    is then written as NaN, and lse / tile_max are undefined. cce_forward() with
 *    cce_check_device_error() names the error.
 */
CCE_API cce_status cce_forward_noalloc(const cce_problem* p, const void* E, const void* C, const void* bias,
                                       const int64_t* targets, float* loss, float* lse, float* tile_max,
                                       int64_t* count, cce_stream_t stream);

/* Optional instrumentation, off by default and per calling thread. When an event pair is set
 * (cudaEvent_t handles created by the caller; NULL clears), cce_forward() records fwd_start and
 * fwd_stop on its stream immediately before and after launching its tensor-core kernel, and
 * cce_backward() does the same with bwd_start and bwd_stop, so the caller can time that kernel
 * alone. */
CCE_API void cce_set_kernel_events(void* fwd_start, void* fwd_stop, void* bwd_start, void* bwd_stop);

/* Number of kernels this library has launched from the calling thread since it was loaded. */
CCE_API int64_t cce_kernel_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
CCE_API int32_t cce_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CCE_H_ */

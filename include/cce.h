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
} cce_problem;

/* Width of the vocabulary sub-tile whose per-row maximum logit the forward saves. */
#define CCE_VOCAB_SUBTILE 128

/* Number of floats in the saved tile-max buffer: ceil(V / 128) * N. Layout [ceil(V/128), N]:
 * entry (j, r) is max_{v in [128 j, 128 j + 128) and v < V} z[r, v]. -1 for a bad problem. */
CCE_API int64_t cce_tile_max_len(const cce_problem* p);

/* Rows and vocabulary columns of one backward tile. The skip rule of the backward decides per
 * tile of this size (mlx-cross-entropy README, "How it works" item 2). */
CCE_API void cce_backward_tile_shape(int32_t* tile_rows, int32_t* tile_cols);

/* Bytes of device workspace cce_forward() needs (0 for a bad problem). */
CCE_API size_t cce_forward_workspace_size(const cce_problem* p);

/* Bytes of device workspace cce_backward() needs: the tile plan (about 37 bytes per 128 x 128
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
 * N = 0 is allowed (loss 0, count 0).
 */
CCE_API cce_status cce_forward(const cce_problem* p, const void* E, const void* C, const void* bias,
                               const int64_t* targets, float* loss, float* lse, float* tile_max, int64_t* count,
                               void* workspace, size_t workspace_bytes, cce_stream_t stream);

/*
 * Backward: dE = G C, dC = G^T E and dbias = sum_r G[r, :] with G = scale_r * (p~ - onehot),
 * p = softmax(z),
 * recomputed tile by tile from E, C and the saved LSE. p~ is p with every skipped tile set to 0:
 * a tile (tile_rows x tile_cols, see cce_backward_tile_shape) is skipped when, for every
 * non-ignored row r in it, max over its columns of z[r, v] - LSE[r] < ln(filter_eps); a tile
 * without a non-ignored row is skipped too. filter_eps <= 0 keeps every tile. The onehot term
 * is never skipped. Loss functions explainer, "How it works" item 2 (gradient p - y);
 * mlx-cross-entropy README, "How it works" items 2 and 3 (skipping, accumulation).
 * scale_r = g / max(count, 1) (mean), g (sum) or g[r] (none); 0 for ignored rows. With the loss
 * variants of cce_problem, G is scale_r times the logit gradient given there; only its softmax
 * part (1 + 2 z_loss LSE) p~ is skipped.
 *
 *  E, C, bias, targets, lse, tile_max, count: as given to / produced by cce_forward() on the
 *           same problem (bias NULL for none)
 *  grad_out device fp32: [1] for mean/sum, [N] for none
 *  dE       device [N, D], dC device [V, D], dbias device [V] or NULL (not computed): bf16 when
 *           out_fp32 = 0, fp32 when out_fp32 = 1. Fully overwritten. Rows of ignored tokens in dE
 *           are exactly +0. dbias is the gradient of the bias (also when bias is NULL, i.e. zero).
 *  filtered_tiles device int64 [1]: number of skipped tiles
 *  workspace: device scratch of at least cce_backward_workspace_size(p, out_fp32) bytes.
 */
CCE_API cce_status cce_backward(const cce_problem* p, const void* E, const void* C, const void* bias,
                                const int64_t* targets, const float* lse, const float* tile_max,
                                const int64_t* count, const float* grad_out, float filter_eps, void* dE, void* dC,
                                void* dbias, int32_t out_fp32, int64_t* filtered_tiles, void* workspace,
                                size_t workspace_bytes, cce_stream_t stream);

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
 * memory where they compute the loss (for example code running during CUDA graph capture, or an
 * embedding that only hands the library fixed buffers for inputs and outputs). The pages have no
 * counterpart; it is an addition for such callers. Arguments and results are those of
 * cce_forward() without the workspace.
 *  - Scratch lives in one device array of CCE_NOALLOC_SCRATCH_BYTES that every GPU loading the
 *    library holds until exit. Problems needing more (about ceil(V/128) * N * 4 + 12 N + 4 D bytes; at
 *    V = 128256 up to N of about 8000) are rejected with CCE_ERR_UNSUPPORTED before anything runs.
 *  - The first call on each device looks up the array's device address; make that first call
 *    before any stream capture.
 *  - Every call shares the array, so calls whose work overlaps on the GPU (other streams, other
 *    threads) race and give undefined results; serialise them.
 *  - Device-side errors (a target outside [0, V)) are not reported by this variant; use
 *    cce_forward() and cce_check_device_error() to diagnose them.
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

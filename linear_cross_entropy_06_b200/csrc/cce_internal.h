// Internal interface between the C ABI (cce_api.cu) and the kernel files. Not installed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <stdint.h>

#include <utility>

namespace cce {

// Forward tile: 128 rows x 256 vocabulary columns, K in blocks of 64 (one 128-byte swizzle row).
constexpr int kFwdBM = 128;
constexpr int kFwdBN = 256;
constexpr int kSubTile = 64;  // vocabulary width of one saved tile max (and of a skip-rule unit)

// Backward tile: 128 rows x 128 vocabulary columns (a gradient tile and the unit of the work lists),
// made of two 64-column halves. The skip rule decides each half (128 rows x kSubTile columns) on its
// own; a tile is listed when either half is kept, and only its kept halves are recomputed, stored and
// multiplied into dE.
constexpr int kBwdBM = 128;
constexpr int kBwdBN = 128;
static_assert(kBwdBN == 2 * kSubTile, "a backward tile is two skip-rule halves");

// Tile flags of the plan, one byte per (row block, vocabulary tile): bits 0-1 the state (0 nothing,
// 1 listed, 2 onehot only: no half kept but a row of the block has its target in the tile), bits 2-3
// the kept halves of a listed tile.
constexpr int kFlagListed = 1;
constexpr int kFlagOnehotOnly = 2;
__host__ __device__ constexpr int flag_state(int f) { return f & 3; }
__host__ __device__ constexpr int flag_halves(int f) { return (f >> 2) & 3; }
// Slots in entries_b carry the tile's kept halves in bits 29-30.
constexpr int kSlotBits = 29;
constexpr int kSlotMask = (1 << kSlotBits) - 1;
// Zeros standing for one 64-row K-block of a skipped half in the dC MMAs (64 x 64 bf16).
constexpr int kZeroHalfBytes = 64 * kSubTile * 2;

struct FwdLaunch {
  CUtensorMap tmE;  // bf16 [N, D], box 64 x 128, 128B swizzle
  CUtensorMap tmC;  // bf16 [V, D], box 64 x 256, 128B swizzle
  int N, D, V, T;   // T = ceil(V / kSubTile)
  const __nv_bfloat16* bias;  // [V] added to every row of logits, or null
  float* tile_max;  // [T, N]
  float* tile_sum;  // [T, N]: sum over the sub-tile of exp(z - tile_max)
  const int64_t* targets;  // [N]: rows whose target v lies in C (vs <= v < vs + V, v != ignore_index) ...
  int64_t vs, ignore_index;
  float* zt;              // ... get zt[r] = z[r, v] (bias included), taken from the logit tile; others untouched
  int* err;
  uint64_t timeout_ns;
  int num_sms;
  int inject_stall;  // test hook: the producer issues nothing, so a bounded wait runs out
};

// Counts every kernel launch of the calling thread (instrumentation for benchmarks).
void note_launches(int n);

// Launches `kernel` on `s` with programmatic stream serialisation: it may be scheduled while the
// previous kernel of the stream finishes, and must call wait_for_previous_grid() before it reads
// that kernel's results. Used only where the previous operation on the stream is a kernel.
template <typename... Params, typename... Args>
cudaError_t launch_after_previous(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Limit of one bounded wait inside a kernel: CCE_WAIT_TIMEOUT_MS milliseconds (default 4000).
uint64_t wait_timeout_ns();

// Sets the message cce_last_error_message() returns on the calling thread.
void set_last_error(const char* msg);

// Backward (cce_bwd_plan.cu: tile plan and work lists; cce_bwd.cu: the persistent kernel).
constexpr int kGradTileBytes = kBwdBM * kBwdBN * 2;      // one bf16 gradient tile, 128B-swizzled
constexpr int kGemmSlice = 256;                           // columns of D per dC/dE work item
// A vocabulary chunk spans at most kChunkCBytes of C. Each chunk adds a full N x D fp32 partial
// into dE, so fewer chunks move fewer bytes there; smaller chunks keep more of a chunk's C rows in
// L2 between their recompute and their dE items. 128 MiB measured best on B200 (N = 4096,
// D = 4096, V = 128256: 7.3 GB of DRAM traffic per backward against 8.3 GB at 64 MiB and 8.5 GB at
// 256 MiB) ...
constexpr int64_t kChunkCBytes = int64_t(128) << 20;
// ... and the gradient tiles of kGradBuffers chunks (at most one per listed row block and
// vocabulary tile; a chunk is written while the one before it is read) fit in the scratch: 4 MiB
// per 128-row block, at least 128 MiB. The scratch grows with N, not with V, so that a chunk keeps
// the same number of vocabulary tiles as N grows: each chunk adds a full N x D fp32 partial into
// dE. The backward's queue places the dE/dC items of chunk c - 2 before the quads of chunk c, so
// two buffers are the fewest that keep every wait pointing to an earlier item.
constexpr int64_t kGradScratchPerRowBlock = int64_t(4) << 20;
constexpr int64_t kGradScratchMin = int64_t(128) << 20;
constexpr int kGradBuffers = 2;
static_assert(kGradBuffers >= 2, "the quads of chunk c reuse the buffer of chunk c - kGradBuffers");

struct BwdPlan {
  int nb, nt;
  uint8_t* flags;   // [nb * nt]: state and kept halves (kFlagListed, kFlagOnehotOnly, flag_halves)
  int* rank;        // [nb * nt]: position of (b, t) among the listed row blocks of t
  int* cnt_t;       // [nt]
  int* offsets_t;   // [nt + 1]
  int2* entries_t;  // [nb * nt]: (b * 16 + flag, t), by vocabulary tile then row block
  int* cnt_b;       // [nb]
  int* offsets_b;   // [nb + 1]
  int* cnt_hb;      // [nb]: kept halves per row block
  int* off_hb;      // [nb + 1]: their prefix sums
  int2* entries_b;  // [nb * nt]: (t, slot in entries_t | kept halves << kSlotBits), by row block then
                    // vocabulary tile
  int* hp_b;        // [nb * nt + 1]: kept halves before each entries_b position (over all row blocks)
  int* pos_b;       // [nb * nt]: for each entries_t position, the tile's position in entries_b
  int* kept_total;  // kept halves
  int chunk_vt;     // vocabulary tiles per chunk at most once every tile is listed (sizes the arrays)
  int nchunks;      // chunks at most (arrays are sized for it); the plan's own count is *nchunks_dev
  int* nchunks_dev; // [1]: chunks of this plan
  int* chunk_of;    // [nt]: chunk of each vocabulary tile
  int S;            // 256-column slices of D
  int* chunk_t;     // [nchunks + 1]: first vocabulary tile of each chunk
  int64_t chunk_c_tiles;  // vocabulary tiles with a listed tile a chunk may hold (kChunkCBytes of C)
  int64_t chunk_g_tiles;  // listed tiles a chunk may hold (one gradient-tile buffer)
  int2* rb_range;   // [nchunks * nb]: entries [lo, hi) of each row block inside each chunk
  int* pstart_t;    // [nt + 1]: first quad whose first half is in vocabulary tile t
  int* quad_b;      // [quad capacity]: row block of each quad (up to four kept halves of one row block
                    // in a chunk), by the tile of its first half then row block
  int4* quad_h;     // [quad capacity]: its halves, each 2 t + h (-1 when absent)
  int4* quad_s;     // [quad capacity]: their tiles' gradient slots, relative to the chunk
  int* cnt_ht;      // [nt]: kept halves of each vocabulary tile (over its listed row blocks)
  int* grp_size;    // [2 * nchunks]: work items of each queue group (quads of chunk c, then its dE/dC)
  int* grp_start;   // [2 * nchunks + 1]: their prefix sums
  int* vt_order;    // [nt]: chunk c's vocabulary tiles at [chunk_t[c], chunk_t[c + 1]): first the ndc[c]
                    // with a listed tile (dC items), ascending, then the empty ones, ascending
  int* ndc;         // [nchunks]
  int* de_list;     // [nchunks * nb]: row blocks with a listed tile in chunk c, ascending, at c * nb
  int* nde;         // [nchunks]
  int* empty_list;  // [nt]: the vocabulary tiles no row block lists (their dC rows are filled directly)
  int* n_empty;     // [1], zero before planning
  int* oh_cnt;      // [nt]: rows whose target tile is onehot only, per vocabulary tile (scratch)
  int* oh_cur;      // [nt]: cursors while those rows are written (scratch)
  int* oh_off;      // [nt + 1]: their prefix sums
  int* oh_rows;     // [N]: those rows, grouped by the vocabulary tile of their target
};

// Everything the persistent backward kernel reads besides its tensor maps.
struct BwdArgs {
  int N, D, V, nb, nt, S;
  const int* nchunks;  // [1] the plan's chunk count
  int out_bf16;
  int slab3d;  // operand slices by one 3-D TMA load (D a multiple of 256)
  int64_t ignore_index;
  int64_t vocab_start;  // C holds vocabulary rows [vocab_start, vocab_start + V); targets are global ids
  size_t buf_bytes;  // one of the kGradBuffers gradient-tile buffers
  const float* lse;
  const float* scale;
  const int64_t* targets;
  const __nv_bfloat16* bias;  // [V] or null
  float* dbias;               // [V] fp32 accumulator of the column sums of G, or null
  float z_loss;               // softmax part of G scaled by 1 + 2 z_loss LSE_r
  float onehot_coef;          // 1 - label_smoothing: weight of the onehot part of G
  const float* dc_add;        // [D] or null: added, times dc_coef, to every row of dC
  float dc_coef;
  const __nv_bfloat16* E;     // rows of the onehot-only targets, added into their dC rows
  const int* oh_off;          // [nt + 1]
  const int* oh_rows;         // rows whose target tile is onehot only, by vocabulary tile
  const int* grp_start;
  const int* vt_order;
  const int* ndc;
  const int* de_list;
  const int* nde;
  const int* chunk_t;
  const int* pstart_t;
  const int* quad_b;
  const int4* quad_h;
  const int4* quad_s;
  const int* cnt_ht;
  const int2* rb_range;
  const int* offsets_t;
  const int2* entries_t;
  const int2* entries_b;
  const int* hp_b;
  const void* zero_half;  // 8 KB of zeros: the gradient of a skipped half, as the dC MMAs read it
  uint8_t* gscratch;
  int* qctr;      // queue position, zero at launch
  int* counters;  // zero at launch: [ctr_g_b] gradient halves stored per (chunk, row block),
                  // [ctr_g_t] per vocabulary tile, [ctr_b_done] dE / dC items finished per chunk
  int ctr_g_b, ctr_g_t, ctr_b_done;
  int* err;
  uint64_t timeout_ns;
  int inject_stall;  // test hook: the first dE item waits for a count no item produces
};

struct BwdLaunch {
  CUtensorMap tmE128;          // bf16, box 64 x 128: E K-blocks of the recompute
  CUtensorMap tmC128;          // bf16, box 64 x 64: C K-blocks of one kept half of the recompute
  CUtensorMap tmE64, tmC64;    // bf16 operand slices of the dC / dE MMAs: 3-D box 64 x 64 x 4 (D % 256 == 0)
                               // or 2-D box 64 x 64
  CUtensorMap tmdC;            // dC output: bf16 box 64 x 32, or fp32 box 32 x 32
  CUtensorMap tmdE;            // fp32 dE accumulator, box 32 x 32 (reduce-add)
  BwdArgs args;
  int num_sms;
};

// Everything the backward's planning launch reads and writes besides the plan itself (cce_bwd_plan.cu).
struct PlanArgs {
  BwdPlan P;
  const float* tile_max;   // [T, N] from the forward
  const float* lse;        // [N]
  const int64_t* targets;  // [N] ids in [0, vtot); this problem's C holds rows [vs, vs + V)
  const int64_t* count;    // [1] non-ignored rows (from the forward)
  const float* grad_out;   // [1] or [N]
  int64_t N, D, V, T, vs, vtot, ignore_index;
  int reduction;
  int filter_on;
  float ln_eps;
  float* scale;            // [N] out: the row scales of the gradient
  float onehot_coef;       // 1 - label_smoothing
  float* dE_acc;           // [N, D] fp32, zeroed here
  float* dbias_acc;        // [V] fp32 or null, zeroed here; receives the onehot-only rows' terms
  void* zero_half;         // [kZeroHalfBytes] zeroed here, read by the backward kernel
  int64_t* filtered_tiles;
  int* sync;               // [sync_ints] the backward kernel's queue position and counters, zeroed here
  int64_t sync_ints;
  int* bar;                // grid barrier counter, zero at launch
  int* err;
  uint64_t timeout_ns;
  int inject_stall;        // test hook: block 0 leaves before the first grid barrier, whose wait then runs out
};
// One cooperative launch: the row scales, the tile flags, both tile lists, the quad list, the
// chunks' work lists and queue groups, the onehot-only rows, and the skipped count.
cudaError_t launch_bwd_plan(const PlanArgs& A, int num_sms, cudaStream_t s);
// after_kernel: the previous operation on s is a kernel (the planning launch or a column sum).
cudaError_t launch_bwd(const BwdLaunch& L, bool after_kernel, cudaStream_t s);
// Everything the backward computes after its tensor-core kernel (cce_bwd_plan.cu, two launches): the
// dC rows of the vocabulary tiles no row block lists (empty_tiles_kernel), the last terms of dE and
// its conversion, and dbias (bwd_finalize_kernel).
struct BwdFinalize {
  int64_t N, D, V, vs, ignore_index;
  int nt;
  const uint8_t* flags;       // the plan's tile flags [nb * nt] (state and kept halves)
  const int* empty_list;
  const int* n_empty;
  const int* oh_off;
  const int* oh_rows;
  const int64_t* targets;
  const float* scale;
  float onehot_coef;          // 1 - label_smoothing
  float ls_v;                 // label_smoothing / vocab_total
  const __nv_bfloat16* E;
  const __nv_bfloat16* C;
  const float* csum;          // [D] column sums of C (label smoothing) or null
  const float* wsum;          // [D + 1] sum_r scale_r E_r and sum_r scale_r (label smoothing) or null
  float* dE_acc;              // [N, D] fp32
  void* dE_out;               // bf16 [N, D], or null: dE_acc is the output (fp32)
  void* dC;                   // [V, D]
  int dc_bf16;
  float* dbias_acc;           // [V] fp32, or null (no dbias)
  void* dbias_out;            // bf16 [V], or null: dbias_acc is the output (fp32)
};
// dC rows of the vocabulary tiles no row block lists.
cudaError_t launch_empty_tiles(const BwdFinalize& F, int num_sms, bool after_kernel, cudaStream_t s);
// dE's last terms and conversion, dbias (after the tensor-core kernel and launch_empty_tiles).
cudaError_t launch_bwd_finalize(const BwdFinalize& F, int num_sms, cudaStream_t s);
// out[b * T + j] = 1 if half j of row block b was skipped, 0 if it was kept (b < nb, j < T).
cudaError_t launch_skip_map(const uint8_t* flags, int nb, int nt, int64_t T, uint8_t* out, cudaStream_t s);

cudaError_t launch_fwd_lse(const FwdLaunch& L, cudaStream_t s);

// Small kernels (cce_aux.cu).
// Everything the forward computes after its tensor-core kernel (one launch).
struct FwdFinish {
  const float* tile_max;  // [T, N]
  const float* tile_sum;  // [T, N]
  int64_t N, T, D, V;
  int64_t vs, vtot;       // C holds vocabulary rows [vs, vs + V) of vtot (0 and V: the whole vocabulary)
  int64_t ignore_index;
  const __nv_bfloat16* E;
  const int64_t* targets;
  const float* zt;            // [N] correct-token logits written by the forward kernel (rows with a local target)
  const float* csum;          // [D + 1] column sums of C and the bias sum (label smoothing), or null
  float label_smoothing, z_loss;
  float* lse;                 // [N]
  float* zt_out;              // vocabulary shard: [N] correct-token logits and [N] logit sums; else null
  float* zs_out;
  float* loss;                // [1] or [N] (reduction none); null for a vocabulary shard
  int reduction;
  int64_t* count;
  double* block_sums;         // [ceil(N / kFinishRows)] scratch
  long long* block_counts;    // [ceil(N / kFinishRows)] scratch
  int* done;                  // zero at launch
  int* err;
};
constexpr int kFinishRows = 32;  // rows per block of the finish kernel
// after_kernel: the previous operation on s is the forward's tensor-core kernel (launched to overlap
// its tail).
cudaError_t launch_fwd_finish(const FwdFinish& F, bool after_kernel, cudaStream_t s);
// out[0:D] = sum_r w_r X[r, :] (w_r = 1 when w is null); out[D] = sum_r w_r, or the sum of extra[0:rows].
cudaError_t launch_weighted_colsum(const __nv_bfloat16* X, int64_t rows, int64_t D, const float* w,
                                   const __nv_bfloat16* extra, float* out, cudaStream_t s);
// LSE over the whole vocabulary, loss, count and reduction from the shards' partial results [shards, 3, N].
cudaError_t launch_shard_merge(const float* partials, int shards, const int64_t* targets, int64_t N, int64_t V,
                               int64_t ignore_index, float label_smoothing, float z_loss, int reduction, float* loss,
                               float* lse, int64_t* count, cudaStream_t s);
cudaError_t launch_fill_zero(void* dst, int64_t bytes, cudaStream_t s);

}  // namespace cce

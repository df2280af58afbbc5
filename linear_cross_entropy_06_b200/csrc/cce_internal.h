// Internal interface between the C ABI (cce_api.cu) and the kernel files. Not installed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cce {

// Forward tile: 128 rows x 256 vocabulary columns, K in blocks of 64 (one 128-byte swizzle row).
constexpr int kFwdBM = 128;
constexpr int kFwdBN = 256;
constexpr int kSubTile = 128;  // vocabulary width of one saved tile max

// Backward tile: 128 rows x 128 vocabulary columns; gradients in D-chunks of 64 columns.
constexpr int kBwdBM = 128;
constexpr int kBwdBN = 128;

struct FwdLaunch {
  CUtensorMap tmE;  // bf16 [N, D], box 64 x 128, 128B swizzle
  CUtensorMap tmC;  // bf16 [V, D], box 64 x 256, 128B swizzle
  int N, D, V, T;   // T = ceil(V / 128)
  float* tile_max;  // [T, N]
  float* tile_sum;  // [T, N]: sum over the sub-tile of exp(z - tile_max)
  int* err;
  uint64_t timeout_ns;
  int num_sms;
};

struct BwdLaunch {
  CUtensorMap tmE;      // bf16 [N, D], box 64 x 128, 128B swizzle
  CUtensorMap tmC;      // bf16 [V, D], box 64 x 128, 128B swizzle
  CUtensorMap tmdE;     // fp32 [N, D] accumulator, box 32 x 32, 128B swizzle (reduce-add)
  CUtensorMap tmdC;     // fp32 [V, D] accumulator, box 32 x 32, 128B swizzle (reduce-add)
  int N, D, V;
  const float* lse;     // [N]
  const float* scale;   // [N]: per-row gradient factor, 0 for ignored rows
  const int64_t* targets;  // [N]: the onehot term of a kept tile is applied inside the kernel
  int64_t ignore_index;
  const int2* tiles;    // kept tiles (row block, vocab tile)
  const int* num_tiles; // device count of kept tiles
  int* err;
  uint64_t timeout_ns;
  int num_sms;
};

// Counts every kernel launch of the calling thread (instrumentation for benchmarks).
void note_launches(int n);

// Sets the message cce_last_error_message() returns on the calling thread.
void set_last_error(const char* msg);

cudaError_t launch_fwd_lse(const FwdLaunch& L, cudaStream_t s);
cudaError_t launch_bwd_grad(const BwdLaunch& L, cudaStream_t s);

// Small kernels (cce_aux.cu).
cudaError_t launch_target_logit(const __nv_bfloat16* E, const __nv_bfloat16* C, const int64_t* targets, int64_t N,
                                int64_t D, int64_t V, int64_t ignore_index, float* z_target, int* err,
                                cudaStream_t s);
cudaError_t launch_lse_loss(const float* tile_max, const float* tile_sum, const float* z_target,
                            const int64_t* targets, int64_t N, int64_t T, int64_t ignore_index, int64_t V,
                            float* lse, float* loss_rows, cudaStream_t s);
cudaError_t launch_loss_reduce(const float* loss_rows, const int64_t* targets, int64_t N, int64_t ignore_index,
                               int reduction, float* loss, int64_t* count, cudaStream_t s);
cudaError_t launch_row_scale(const int64_t* targets, const int64_t* count, const float* grad_out, int64_t N,
                             int64_t ignore_index, int reduction, float* scale, int* num_tiles, cudaStream_t s);
cudaError_t launch_tile_mask(const float* tile_max, const float* lse, const int64_t* targets, int64_t N, int64_t V,
                             int64_t T, int64_t ignore_index, float filter_eps, int2* tiles, uint8_t* keep,
                             int* num_tiles, int64_t* filtered_tiles, cudaStream_t s);
cudaError_t launch_grad_init(const __nv_bfloat16* E, const __nv_bfloat16* C, const int64_t* targets,
                             const float* scale, const uint8_t* keep, int64_t N, int64_t D, int64_t V,
                             int64_t ignore_index, float* dE_acc, float* dC_acc, int* err, cudaStream_t s);
cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, int64_t n, cudaStream_t s);
cudaError_t launch_fill_zero(void* dst, int64_t bytes, cudaStream_t s);

}  // namespace cce

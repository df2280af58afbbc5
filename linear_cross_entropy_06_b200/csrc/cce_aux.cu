// The bandwidth-bound and bookkeeping kernels around the tensor-core kernels:
//  target_logit   z_t[r] = E[r] . C[t_r] (fp32 accumulation of bf16 products), target validation.
//                 Cut Your Losses abstract: only the correct token's logit is computed.
//  lse_loss       LSE_r = M + ln sum_j s_j exp(m_j - M) over the saved sub-tile (max, sum-exp)
//                 pairs, and loss_r = LSE_r - z_t[r] (0 for ignored rows). Loss functions
//                 explainer, "How it works" item 1; Cut Cross Entropy from first principles.
//  loss_reduce    count of non-ignored rows and sum/mean of the loss, in a fixed order (fp64 sum).
//                 mlx-cross-entropy README, "API" (reduction); explainer item 4 (mean over
//                 non-ignored tokens).
//  row_scale      per-row factor of the gradient: g/max(count,1), g or g[r]; 0 for ignored rows.
//  to_bf16        fp32 dE accumulator -> bf16 output (round to nearest even).
#include <cuda_bf16.h>

#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

__device__ __forceinline__ bool valid_target(int64_t t, int64_t V, int64_t ignore_index) {
  return t != ignore_index && t >= 0 && t < V;
}

__device__ __forceinline__ float dot8_bf16(uint4 a, uint4 b, float acc) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 fx = __bfloat1622float2(x[i]);
    const float2 fy = __bfloat1622float2(y[i]);
    acc = fmaf(fx.x, fy.x, acc);
    acc = fmaf(fx.y, fy.y, acc);
  }
  return acc;
}

// One warp per row; lanes read 16-byte pieces, so a warp reads 512 contiguous bytes per step.
__global__ void target_logit_kernel(const __nv_bfloat16* __restrict__ E, const __nv_bfloat16* __restrict__ C,
                                    const __nv_bfloat16* __restrict__ bias, const int64_t* __restrict__ targets,
                                    int64_t N, int64_t D, int64_t V, int64_t ignore_index,
                                    float* __restrict__ z_target, int* err) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t t = targets[row];
  if (!valid_target(t, V, ignore_index)) {
    if (lane == 0) {
      z_target[row] = 0.f;
      if (t != ignore_index) record_error(err, kErrTargetRange);
    }
    return;
  }
  const __nv_bfloat16* e = E + row * D;
  const __nv_bfloat16* c = C + t * D;
  float acc0 = 0.f, acc1 = 0.f;
  int64_t d = static_cast<int64_t>(lane) * 8;
  for (; d + 256 < D; d += 512) {
    acc0 = dot8_bf16(ld_global_nc_v4(e + d), ld_global_nc_v4(c + d), acc0);
    acc1 = dot8_bf16(ld_global_nc_v4(e + d + 256), ld_global_nc_v4(c + d + 256), acc1);
  }
  if (d < D) acc0 = dot8_bf16(ld_global_nc_v4(e + d), ld_global_nc_v4(c + d), acc0);
  const float s = warp_sum(acc0 + acc1);
  if (lane == 0) z_target[row] = bias != nullptr ? s + __bfloat162float(bias[t]) : s;
}

__device__ __forceinline__ void lse_merge(float& M, float& S, float m, float s) {
  if (m == -INFINITY) return;
  if (m > M) {
    S = S * exp2f((M - m) * kLog2e) + s;
    M = m;
  } else {
    S += s * exp2f((m - M) * kLog2e);
  }
}

constexpr int kLseWarps = 32;

// Block = 32 warps x 32 rows. Warp w merges sub-tiles j = w, w + 32, ... of its 32 rows (lane = row,
// so each load is 128 contiguous bytes), four sub-tiles per step so that eight loads are in flight;
// the 32 partial results merge in shared memory.
__global__ void __launch_bounds__(kLseWarps * 32)
    lse_loss_kernel(const float* __restrict__ tile_max, const float* __restrict__ tile_sum,
                    const float* __restrict__ z_target, const int64_t* __restrict__ targets, int64_t N, int64_t T,
                    int64_t ignore_index, int64_t V, float* __restrict__ lse, float* __restrict__ loss_rows) {
  __shared__ float sm_m[kLseWarps][32], sm_s[kLseWarps][32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  float M = -INFINITY, S = 0.f;
  if (r < N) {
    for (int64_t j = w; j < T; j += 4 * kLseWarps) {
      float m[4], s[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t jj = j + u * kLseWarps;
        m[u] = jj < T ? tile_max[jj * N + r] : -INFINITY;
        s[u] = jj < T ? tile_sum[jj * N + r] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) lse_merge(M, S, m[u], s[u]);
    }
  }
  sm_m[w][lane] = M;
  sm_s[w][lane] = S;
  __syncthreads();
  if (w == 0 && r < N) {
    float Mt = -INFINITY, St = 0.f;
    for (int k = 0; k < kLseWarps; ++k) lse_merge(Mt, St, sm_m[k][lane], sm_s[k][lane]);
    const float L = Mt + logf(St);
    lse[r] = L;
    const int64_t t = targets[r];
    loss_rows[r] = valid_target(t, V, ignore_index) ? L - z_target[r] : 0.f;
  }
}

constexpr int kReduceThreads = 1024;

// Single block: deterministic order (strided fp64 partial sums, then a fixed tree).
__global__ void loss_reduce_kernel(const float* __restrict__ loss_rows, const int64_t* __restrict__ targets,
                                   int64_t N, int64_t ignore_index, int reduction, float* __restrict__ loss,
                                   int64_t* __restrict__ count) {
  __shared__ double ssum[kReduceThreads];
  __shared__ long long scnt[kReduceThreads];
  double acc = 0.0;
  long long cnt = 0;
  for (int64_t r = threadIdx.x; r < N; r += kReduceThreads) {
    if (targets[r] != ignore_index) ++cnt;
    if (reduction != 0) acc += static_cast<double>(loss_rows[r]);
  }
  ssum[threadIdx.x] = acc;
  scnt[threadIdx.x] = cnt;
  __syncthreads();
  for (int o = kReduceThreads / 2; o > 0; o >>= 1) {
    if (static_cast<int>(threadIdx.x) < o) {
      ssum[threadIdx.x] += ssum[threadIdx.x + o];
      scnt[threadIdx.x] += scnt[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const long long c = scnt[0];
    *count = c;
    if (reduction == 1) *loss = static_cast<float>(ssum[0] / static_cast<double>(c > 0 ? c : 1));
    if (reduction == 2) *loss = static_cast<float>(ssum[0]);
  }
}

__global__ void row_scale_kernel(const int64_t* __restrict__ targets, const int64_t* __restrict__ count,
                                 const float* __restrict__ grad_out, int64_t N, int64_t ignore_index, int reduction,
                                 float* __restrict__ scale) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= N) return;
  float s;
  if (reduction == 1) {
    const long long c = *count;
    s = grad_out[0] / static_cast<float>(c > 0 ? c : 1);
  } else if (reduction == 2) {
    s = grad_out[0];
  } else {
    s = grad_out[r];
  }
  scale[r] = (targets[r] != ignore_index) ? s : 0.f;
}

// Eight elements per thread and step (16-byte stores), then the last n % 8 one by one.
__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n) {
  const int64_t n8 = n / 8;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid < n - 8 * n8) dst[8 * n8 + tid] = __float2bfloat16_rn(src[8 * n8 + tid]);
  for (int64_t i = tid; i < n8; i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(src)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(src)[2 * i + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x, a.y);
    o.y = pack_bf16x2(a.z, a.w);
    o.z = pack_bf16x2(b.x, b.y);
    o.w = pack_bf16x2(b.z, b.w);
    reinterpret_cast<uint4*>(dst)[i] = o;
  }
}

// 16 bytes per thread and step, then the last bytes % 16 one by one.
__global__ void fill_zero_kernel(uint4* __restrict__ dst, int64_t bytes) {
  const int64_t n16 = bytes / 16;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid < bytes - 16 * n16) reinterpret_cast<uint8_t*>(dst)[16 * n16 + tid] = 0;
  for (int64_t i = tid; i < n16; i += static_cast<int64_t>(gridDim.x) * blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
}

int grid_for(int64_t items, int per_block, int cap) {
  const int64_t g = (items + per_block - 1) / per_block;
  return static_cast<int>(g < cap ? (g > 0 ? g : 1) : cap);
}

}  // namespace

cudaError_t launch_target_logit(const __nv_bfloat16* E, const __nv_bfloat16* C, const __nv_bfloat16* bias,
                                const int64_t* targets, int64_t N, int64_t D, int64_t V, int64_t ignore_index,
                                float* z_target, int* err, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 7) / 8);
  target_logit_kernel<<<grid, 256, 0, s>>>(E, C, bias, targets, N, D, V, ignore_index, z_target, err);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_lse_loss(const float* tile_max, const float* tile_sum, const float* z_target,
                            const int64_t* targets, int64_t N, int64_t T, int64_t ignore_index, int64_t V,
                            float* lse, float* loss_rows, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 31) / 32);
  lse_loss_kernel<<<grid, kLseWarps * 32, 0, s>>>(tile_max, tile_sum, z_target, targets, N, T, ignore_index, V, lse,
                                                  loss_rows);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_loss_reduce(const float* loss_rows, const int64_t* targets, int64_t N, int64_t ignore_index,
                               int reduction, float* loss, int64_t* count, cudaStream_t s) {
  loss_reduce_kernel<<<1, kReduceThreads, 0, s>>>(loss_rows, targets, N, ignore_index, reduction, loss, count);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_row_scale(const int64_t* targets, const int64_t* count, const float* grad_out, int64_t N,
                             int64_t ignore_index, int reduction, float* scale, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 255) / 256);
  row_scale_kernel<<<grid, 256, 0, s>>>(targets, count, grad_out, N, ignore_index, reduction, scale);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, int64_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  // src and dst 16-byte aligned; the tail of fewer than 8 elements is taken by the first threads
  to_bf16_kernel<<<grid_for(n / 8, 256, 148 * 16), 256, 0, s>>>(src, dst, n);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fill_zero(void* dst, int64_t bytes, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  // dst 16-byte aligned; the tail of fewer than 16 bytes is taken by the first threads
  fill_zero_kernel<<<grid_for(bytes / 16, 256, 148 * 16), 256, 0, s>>>(static_cast<uint4*>(dst), bytes);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

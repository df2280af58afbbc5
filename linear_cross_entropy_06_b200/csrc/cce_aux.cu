// The bandwidth-bound and bookkeeping kernels around the two tensor-core kernels:
//  target_logit   z_t[r] = E[r] . C[t_r] (fp32 accumulation of bf16 products), target validation.
//                 Cut Your Losses abstract: only the correct token's logit is computed.
//  lse_loss       LSE_r = M + ln sum_j s_j exp(m_j - M) over the saved sub-tile (max, sum-exp)
//                 pairs, and loss_r = LSE_r - z_t[r] (0 for ignored rows). Loss functions
//                 explainer, "How it works" item 1; Cut Cross Entropy from first principles.
//  loss_reduce    count of non-ignored rows and sum/mean of the loss, in a fixed order (fp64 sum).
//                 mlx-cross-entropy README, "API" (reduction); explainer item 4 (mean over
//                 non-ignored tokens).
//  row_scale      per-row factor of the gradient: g/max(count,1), g or g[r]; 0 for ignored rows.
//  tile_mask      keep/skip decision per backward tile from the saved maxima and LSE, compacted
//                 into a list. mlx-cross-entropy README, "How it works" item 2.
//  grad_init      dC_acc = 0 and dE_acc[r] = -scale_r C[t_r] when the tile holding (r, t_r) is
//                 skipped, else +0; onehot_dC adds -scale_r E[r] into dC_acc[t_r] for the same
//                 rows. The onehot part of p - y of a kept tile is folded into the gradient tile
//                 by the backward kernel (before rounding to bf16), so it is never skipped and
//                 never cancels against a rounded p.
//  to_bf16        fp32 accumulators -> bf16 outputs (round to nearest even).
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
                                    const int64_t* __restrict__ targets, int64_t N, int64_t D, int64_t V,
                                    int64_t ignore_index, float* __restrict__ z_target, int* err) {
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
  if (lane == 0) z_target[row] = s;
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
                                 float* __restrict__ scale, int* num_tiles) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r == 0) *num_tiles = 0;
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

// One block (128 threads, one per tile row) per vocabulary tile. Tile (b, t) is kept iff some
// non-ignored row r of block b has tile_max[t, r] - LSE_r >= ln(eps), or eps <= 0. The block
// counts its kept tiles, reserves a contiguous range with one atomic, then writes (b, t) in b order,
// so each vocabulary tile's row blocks are adjacent in the list.
__global__ void tile_mask_kernel(const float* __restrict__ tile_max, const float* __restrict__ lse,
                                 const int64_t* __restrict__ targets, int64_t N, int64_t V, int64_t T,
                                 int64_t ignore_index, float ln_eps, int filter_on, int2* __restrict__ tiles,
                                 uint8_t* __restrict__ keep, int* num_tiles) {
  __shared__ float wmax[4];
  __shared__ int base;
  const int t = blockIdx.x;
  const int nb = static_cast<int>((N + kBwdBM - 1) / kBwdBM);
  int kept_count = 0;
  for (int pass = 0; pass < 2; ++pass) {
    int k = 0;
    for (int b = 0; b < nb; ++b) {
      bool keep_tile = true;
      if (filter_on) {
        const int64_t r = static_cast<int64_t>(b) * kBwdBM + threadIdx.x;
        float m = -INFINITY;
        if (r < N && valid_target(targets[r], V, ignore_index)) {
          const int64_t j0 = static_cast<int64_t>(t) * (kBwdBN / kSubTile);
          const int64_t j1 = j0 + kBwdBN / kSubTile < T ? j0 + kBwdBN / kSubTile : T;
          for (int64_t j = j0; j < j1; ++j) m = fmaxf(m, tile_max[j * N + r]);
          m -= lse[r];
        }
        m = warp_max(m);
        if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
        __syncthreads();
        const float bm = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
        __syncthreads();
        keep_tile = bm >= ln_eps;
      }
      if (pass == 0 && threadIdx.x == 0) keep[static_cast<int64_t>(b) * gridDim.x + t] = keep_tile ? 1 : 0;
      if (keep_tile) {
        if (pass == 1 && threadIdx.x == 0) tiles[base + k] = make_int2(b, t);
        ++k;
      }
    }
    if (pass == 0) {
      kept_count = k;
      if (threadIdx.x == 0) base = atomicAdd(num_tiles, kept_count);
      __syncthreads();
    }
  }
}

__global__ void mask_finish_kernel(const int* __restrict__ num_tiles, int64_t total, int64_t* __restrict__ filtered) {
  *filtered = total - static_cast<int64_t>(*num_tiles);
}

// True when row r has a valid target whose tile (r's row block, t_r's vocabulary tile) was skipped:
// then the onehot term of that row is added here instead of inside the backward kernel.
__device__ __forceinline__ bool onehot_outside(int64_t r, int64_t t, int64_t V, int64_t ignore_index,
                                               const uint8_t* keep, int64_t nt) {
  return valid_target(t, V, ignore_index) && keep[(r / kBwdBM) * nt + t / kBwdBN] == 0;
}

// dE_acc[r, :] = -scale_r * C[t_r, :] for rows whose target tile is skipped, +0 otherwise. One warp
// per row, 8 elements per lane per step.
__global__ void grad_init_dE_kernel(const __nv_bfloat16* __restrict__ C, const int64_t* __restrict__ targets,
                                    const float* __restrict__ scale, const uint8_t* __restrict__ keep, int64_t N,
                                    int64_t D, int64_t V, int64_t ignore_index, float* __restrict__ dE_acc,
                                    int* err) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t t = targets[row];
  float* out = dE_acc + row * D;
  if (lane == 0 && t != ignore_index && !valid_target(t, V, ignore_index)) record_error(err, kErrTargetRange);
  const int64_t nt = (V + kBwdBN - 1) / kBwdBN;
  if (!onehot_outside(row, t, V, ignore_index, keep, nt)) {
    for (int64_t d = static_cast<int64_t>(lane) * 4; d < D; d += 128)
      *reinterpret_cast<float4*>(out + d) = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const float s = -scale[row];
  const __nv_bfloat16* c = C + t * D;
  for (int64_t d = static_cast<int64_t>(lane) * 8; d < D; d += 256) {
    const uint4 raw = ld_global_nc_v4(c + d);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    const float2 cc = __bfloat1622float2(h[2]), dd = __bfloat1622float2(h[3]);
    *reinterpret_cast<float4*>(out + d) = make_float4(s * a.x, s * a.y, s * b.x, s * b.y);
    *reinterpret_cast<float4*>(out + d + 4) = make_float4(s * cc.x, s * cc.y, s * dd.x, s * dd.y);
  }
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// dC_acc[t_r, :] += -scale_r * E[r, :] for non-ignored rows (targets repeat, hence atomics).
__global__ void onehot_dC_kernel(const __nv_bfloat16* __restrict__ E, const int64_t* __restrict__ targets,
                                 const float* __restrict__ scale, const uint8_t* __restrict__ keep, int64_t N,
                                 int64_t D, int64_t V, int64_t ignore_index, float* __restrict__ dC_acc) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t t = targets[row];
  if (!onehot_outside(row, t, V, ignore_index, keep, (V + kBwdBN - 1) / kBwdBN)) return;
  const float s = -scale[row];
  const __nv_bfloat16* e = E + row * D;
  float* out = dC_acc + t * D;
  for (int64_t d = static_cast<int64_t>(lane) * 8; d < D; d += 256) {
    const uint4 raw = ld_global_nc_v4(e + d);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    const float2 cc = __bfloat1622float2(h[2]), dd = __bfloat1622float2(h[3]);
    red_add_v4(out + d, s * a.x, s * a.y, s * b.x, s * b.y);
    red_add_v4(out + d + 4, s * cc.x, s * cc.y, s * dd.x, s * dd.y);
  }
}

__global__ void to_bf16_kernel(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
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

__global__ void fill_zero_kernel(uint4* __restrict__ dst, int64_t n16) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = make_uint4(0, 0, 0, 0);
}

int grid_for(int64_t items, int per_block, int cap) {
  const int64_t g = (items + per_block - 1) / per_block;
  return static_cast<int>(g < cap ? (g > 0 ? g : 1) : cap);
}

}  // namespace

cudaError_t launch_target_logit(const __nv_bfloat16* E, const __nv_bfloat16* C, const int64_t* targets, int64_t N,
                                int64_t D, int64_t V, int64_t ignore_index, float* z_target, int* err,
                                cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 7) / 8);
  target_logit_kernel<<<grid, 256, 0, s>>>(E, C, targets, N, D, V, ignore_index, z_target, err);
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
                             int64_t ignore_index, int reduction, float* scale, int* num_tiles, cudaStream_t s) {
  const int grid = static_cast<int>(N > 0 ? (N + 255) / 256 : 1);
  row_scale_kernel<<<grid, 256, 0, s>>>(targets, count, grad_out, N, ignore_index, reduction, scale, num_tiles);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tile_mask(const float* tile_max, const float* lse, const int64_t* targets, int64_t N, int64_t V,
                             int64_t T, int64_t ignore_index, float filter_eps, int2* tiles, uint8_t* keep,
                             int* num_tiles, int64_t* filtered_tiles, cudaStream_t s) {
  const int64_t nb = (N + kBwdBM - 1) / kBwdBM;
  const int64_t nt = (V + kBwdBN - 1) / kBwdBN;
  const int filter_on = filter_eps > 0.f ? 1 : 0;
  const float ln_eps = filter_on ? logf(filter_eps) : -INFINITY;
  if (nb > 0) {
    tile_mask_kernel<<<static_cast<int>(nt), kBwdBM, 0, s>>>(tile_max, lse, targets, N, V, T, ignore_index, ln_eps,
                                                             filter_on, tiles, keep, num_tiles);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  mask_finish_kernel<<<1, 1, 0, s>>>(num_tiles, nb * nt, filtered_tiles);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_grad_init(const __nv_bfloat16* E, const __nv_bfloat16* C, const int64_t* targets,
                             const float* scale, const uint8_t* keep, int64_t N, int64_t D, int64_t V,
                             int64_t ignore_index, float* dE_acc, float* dC_acc, int* err, cudaStream_t s) {
  cudaError_t e = launch_fill_zero(dC_acc, V * D * 4, s);
  if (e != cudaSuccess) return e;
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 7) / 8);
  grad_init_dE_kernel<<<grid, 256, 0, s>>>(C, targets, scale, keep, N, D, V, ignore_index, dE_acc, err);
  note_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  onehot_dC_kernel<<<grid, 256, 0, s>>>(E, targets, scale, keep, N, D, V, ignore_index, dC_acc);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float* src, __nv_bfloat16* dst, int64_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const int64_t n8 = n / 8;  // n is a multiple of 8 (D is)
  to_bf16_kernel<<<grid_for(n8, 256, 148 * 16), 256, 0, s>>>(src, dst, n8);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_fill_zero(void* dst, int64_t bytes, cudaStream_t s) {
  if (bytes == 0) return cudaSuccess;
  const int64_t n16 = bytes / 16;  // callers pass multiples of 16 bytes
  fill_zero_kernel<<<grid_for(n16, 256, 148 * 16), 256, 0, s>>>(static_cast<uint4*>(dst), n16);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

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
__device__ __forceinline__ float dot8_f32(uint4 a, const float* __restrict__ b, float acc) {
  const float4 b0 = *reinterpret_cast<const float4*>(b), b1 = *reinterpret_cast<const float4*>(b + 4);
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 h;
    *reinterpret_cast<uint32_t*>(&h) = w[k];
    acc = fmaf(__low2float(h), bb[2 * k], acc);
    acc = fmaf(__high2float(h), bb[2 * k + 1], acc);
  }
  return acc;
}

// One warp per row: z_target[r] = E_r . C_{t_r} (+ bias[t_r]); with csum (the column sums of C
// and, at index D, the sum of the bias) also z_sum[r] = sum_v z[r, v] = E_r . csum + csum[D].
// C holds vocabulary rows [vs, vs + V) of vtot (a shard, or the whole vocabulary with vs = 0 and
// vtot = V): a target outside the shard but inside [0, vtot) gets z_target 0 here (another shard
// holds its logit); a target outside [0, vtot) that is not ignore_index is a device error.
__global__ void target_logit_kernel(const __nv_bfloat16* __restrict__ E, const __nv_bfloat16* __restrict__ C,
                                    const __nv_bfloat16* __restrict__ bias, const int64_t* __restrict__ targets,
                                    int64_t N, int64_t D, int64_t V, int64_t vs, int64_t vtot, int64_t ignore_index,
                                    float* __restrict__ z_target, const float* __restrict__ csum,
                                    float* __restrict__ z_sum, int* err) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const int64_t t = targets[row];
  const __nv_bfloat16* e = E + row * D;
  if (csum != nullptr) {  // every row, ignored ones included (their loss is 0 anyway)
    float zs = 0.f;
    for (int64_t d = static_cast<int64_t>(lane) * 8; d < D; d += 256) zs = dot8_f32(ld_global_nc_v4(e + d), csum + d, zs);
    zs = warp_sum(zs);
    if (lane == 0) z_sum[row] = zs + csum[D];
  }
  if (!valid_target(t - vs, V, ignore_index - vs)) {  // not ignored and inside this shard
    if (lane == 0) {
      z_target[row] = 0.f;
      if (!valid_target(t, vtot, ignore_index) && t != ignore_index) record_error(err, kErrTargetRange);
    }
    return;
  }
  const int64_t tl = t - vs;
  const __nv_bfloat16* c = C + tl * D;
  float acc0 = 0.f, acc1 = 0.f;
  int64_t d = static_cast<int64_t>(lane) * 8;
  for (; d + 256 < D; d += 512) {
    acc0 = dot8_bf16(ld_global_nc_v4(e + d), ld_global_nc_v4(c + d), acc0);
    acc1 = dot8_bf16(ld_global_nc_v4(e + d + 256), ld_global_nc_v4(c + d + 256), acc1);
  }
  if (d < D) acc0 = dot8_bf16(ld_global_nc_v4(e + d), ld_global_nc_v4(c + d), acc0);
  const float s = warp_sum(acc0 + acc1);
  if (lane == 0) z_target[row] = bias != nullptr ? s + __bfloat162float(bias[tl]) : s;
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
                    const float* __restrict__ z_target, const float* __restrict__ z_sum,
                    const int64_t* __restrict__ targets, int64_t N, int64_t T, int64_t ignore_index, int64_t V,
                    float label_smoothing, float z_loss, float* __restrict__ lse, float* __restrict__ loss_rows) {
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
    if (loss_rows == nullptr) return;  // a vocabulary shard: the loss needs every shard's LSE
    const int64_t t = targets[r];
    // LSE - (1 - ls) z_t - (ls / V) sum_v z_v + zl LSE^2 (ls and zl are 0 unless requested)
    float l = L - (1.f - label_smoothing) * z_target[r] + z_loss * L * L;
    if (z_sum != nullptr) l -= label_smoothing / static_cast<float>(V) * z_sum[r];
    loss_rows[r] = valid_target(t, V, ignore_index) ? l : 0.f;
  }
}

constexpr int kReduceThreads = 1024;

// Single block: deterministic order (strided fp64 partial sums, then a fixed tree). When an earlier
// kernel of the call recorded a device error (err != 0), the loss is written as NaN instead (every
// entry for reduction none, whose per-row losses live in `loss`), so that a caller who never reads
// the error word still sees that the result is not valid.
__global__ void loss_reduce_kernel(const float* __restrict__ loss_rows, const int64_t* __restrict__ targets,
                                   int64_t N, int64_t ignore_index, int reduction, float* __restrict__ loss,
                                   int64_t* __restrict__ count, const int* err) {
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
  const bool failed = *reinterpret_cast<const volatile int*>(err) != 0;
  if (threadIdx.x == 0) {
    const long long c = scnt[0];
    *count = c;
    if (reduction == 1) *loss = failed ? NAN : static_cast<float>(ssum[0] / static_cast<double>(c > 0 ? c : 1));
    if (reduction == 2) *loss = failed ? NAN : static_cast<float>(ssum[0]);
  }
  if (failed && reduction == 0)
    for (int64_t r = threadIdx.x; r < N; r += kReduceThreads) loss[r] = NAN;
}

// The vocabulary shards' partial results [shards, 3, N] (per row: the shard's log-sum-exp, the
// correct-token logit if the target lies in the shard, the sum of the shard's logits) combined into
// the row's LSE over the whole vocabulary, LSE = M + ln sum_s exp(lse_s - M) with M = max_s lse_s
// (Loss functions explainer, "How it works" item 1), its loss
// LSE - (1 - ls) z_t - (ls / V) sum_v z_v + zl LSE^2 (0 for ignored rows), and the count and
// reduction of loss_reduce_kernel, in one block with the same fixed summation order.
__global__ void shard_merge_kernel(const float* __restrict__ partials, int shards, const int64_t* __restrict__ targets,
                                   int64_t N, int64_t V, int64_t ignore_index, float label_smoothing, float z_loss,
                                   int reduction, float* __restrict__ loss, float* __restrict__ lse,
                                   int64_t* __restrict__ count) {
  __shared__ double ssum[kReduceThreads];
  __shared__ long long scnt[kReduceThreads];
  double acc = 0.0;
  long long cnt = 0;
  for (int64_t r = threadIdx.x; r < N; r += kReduceThreads) {
    float M = -INFINITY;
    for (int k = 0; k < shards; ++k) M = fmaxf(M, partials[(static_cast<int64_t>(k) * 3) * N + r]);
    float S = 0.f, zt = 0.f, zs = 0.f;
    for (int k = 0; k < shards; ++k) {
      const float* q = partials + static_cast<int64_t>(k) * 3 * N;
      if (q[r] != -INFINITY) S += exp2f((q[r] - M) * kLog2e);
      zt += q[N + r];
      zs += q[2 * N + r];
    }
    const float L = M + logf(S);
    lse[r] = L;
    const bool valid = valid_target(targets[r], V, ignore_index);
    const float l = valid ? L - (1.f - label_smoothing) * zt - label_smoothing / static_cast<float>(V) * zs +
                                z_loss * L * L
                          : 0.f;
    if (reduction == 0) loss[r] = l;
    if (targets[r] != ignore_index) ++cnt;
    acc += static_cast<double>(l);
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

// out[d] += sum_r w_r X[r, d] for d < D (w_r = 1 without weights), and out[D] += sum_r w_r (with
// weights) or sum_r extra[r] (with an extra bf16 vector). One block per kRowsPerBlock rows; each
// thread owns 8 columns at a time and adds its partial sums atomically (fp32).
constexpr int kColsumRows = 512;

__global__ void weighted_colsum_kernel(const __nv_bfloat16* __restrict__ X, int64_t rows, int64_t D,
                                       const float* __restrict__ w, const __nv_bfloat16* __restrict__ extra,
                                       float* __restrict__ out) {
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kColsumRows;
  const int64_t r1 = r0 + kColsumRows < rows ? r0 + kColsumRows : rows;
  for (int64_t c = static_cast<int64_t>(threadIdx.x) * 8; c < D; c += static_cast<int64_t>(blockDim.x) * 8) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t r = r0; r < r1; ++r) {
      const float wr = w != nullptr ? w[r] : 1.f;
      const uint4 u = ld_global_nc_v4(X + r * D + c);
      const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 h;
        *reinterpret_cast<uint32_t*>(&h) = q[k];
        acc[2 * k] = fmaf(wr, __low2float(h), acc[2 * k]);
        acc[2 * k + 1] = fmaf(wr, __high2float(h), acc[2 * k + 1]);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) atomicAdd(out + c + k, acc[k]);
  }
  if (threadIdx.x < 32 && (w != nullptr || extra != nullptr)) {
    float a = 0.f;
    for (int64_t r = r0 + threadIdx.x; r < r1; r += 32) a += w != nullptr ? w[r] : __bfloat162float(extra[r]);
    a = warp_sum(a);
    if (threadIdx.x == 0) atomicAdd(out + D, a);
  }
}

// X[r, d] += coef * scale[r] * u[d] (fp32, in place).
__global__ void add_rank1_kernel(float* __restrict__ X, int64_t rows, int64_t D, const float* __restrict__ scale,
                                 float coef, const float* __restrict__ u) {
  const int64_t n = rows * D;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    X[i] = fmaf(coef * scale[i / D], u[i % D], X[i]);
}

// X[i] += coef * (*c) (fp32, in place).
__global__ void add_scalar_kernel(float* __restrict__ X, int64_t n, float coef, const float* __restrict__ c) {
  const float v = coef * *c;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    X[i] += v;
}

// One warp per listed row r (rows[i], i < off[nt]): dE_acc[r, :] -= coef * scale[r] * C[t_r, :]
// and dbias_acc[t_r] -= coef * scale[r]. Each row is listed once, so the dE rows need no atomics.
__global__ void onehot_rows_apply_kernel(const int* __restrict__ off, int nt, const int* __restrict__ rows,
                                         const int64_t* __restrict__ targets, int64_t vs,
                                         const float* __restrict__ scale, float coef,
                                         const __nv_bfloat16* __restrict__ C, int64_t D, float* __restrict__ dE_acc,
                                         float* __restrict__ dbias_acc) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= off[nt]) return;
  const int64_t r = rows[i];
  const int64_t t = targets[r] - vs;  // listed rows have their target in this shard
  const float a = -coef * scale[r];
  if (dbias_acc != nullptr && lane == 0) atomicAdd(dbias_acc + t, a);
  const __nv_bfloat16* c = C + t * D;
  float* out = dE_acc + r * D;
  for (int64_t d = static_cast<int64_t>(lane) * 8; d < D; d += 256) {
    const uint4 u = ld_global_nc_v4(c + d);
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
    float4 o0 = *reinterpret_cast<float4*>(out + d), o1 = *reinterpret_cast<float4*>(out + d + 4);
    float cv[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 h;
      *reinterpret_cast<uint32_t*>(&h) = q[k];
      cv[2 * k] = __low2float(h);
      cv[2 * k + 1] = __high2float(h);
    }
    o0.x = fmaf(a, cv[0], o0.x);
    o0.y = fmaf(a, cv[1], o0.y);
    o0.z = fmaf(a, cv[2], o0.z);
    o0.w = fmaf(a, cv[3], o0.w);
    o1.x = fmaf(a, cv[4], o1.x);
    o1.y = fmaf(a, cv[5], o1.y);
    o1.z = fmaf(a, cv[6], o1.z);
    o1.w = fmaf(a, cv[7], o1.w);
    *reinterpret_cast<float4*>(out + d) = o0;
    *reinterpret_cast<float4*>(out + d + 4) = o1;
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
                                const int64_t* targets, int64_t N, int64_t D, int64_t V, int64_t vs, int64_t vtot,
                                int64_t ignore_index, float* z_target, const float* csum, float* z_sum, int* err,
                                cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 7) / 8);  // 8 warps (rows) per block
  target_logit_kernel<<<grid, 256, 0, s>>>(E, C, bias, targets, N, D, V, vs, vtot, ignore_index, z_target, csum,
                                           z_sum, err);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_lse_loss(const float* tile_max, const float* tile_sum, const float* z_target, const float* z_sum,
                            const int64_t* targets, int64_t N, int64_t T, int64_t ignore_index, int64_t V,
                            float label_smoothing, float z_loss, float* lse, float* loss_rows, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int grid = static_cast<int>((N + 31) / 32);
  lse_loss_kernel<<<grid, kLseWarps * 32, 0, s>>>(tile_max, tile_sum, z_target, z_sum, targets, N, T, ignore_index,
                                                  V, label_smoothing, z_loss, lse, loss_rows);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_loss_reduce(const float* loss_rows, const int64_t* targets, int64_t N, int64_t ignore_index,
                               int reduction, float* loss, int64_t* count, const int* err, cudaStream_t s) {
  loss_reduce_kernel<<<1, kReduceThreads, 0, s>>>(loss_rows, targets, N, ignore_index, reduction, loss, count, err);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_shard_merge(const float* partials, int shards, const int64_t* targets, int64_t N, int64_t V,
                               int64_t ignore_index, float label_smoothing, float z_loss, int reduction, float* loss,
                               float* lse, int64_t* count, cudaStream_t s) {
  shard_merge_kernel<<<1, kReduceThreads, 0, s>>>(partials, shards, targets, N, V, ignore_index, label_smoothing,
                                                  z_loss, reduction, loss, lse, count);
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

cudaError_t launch_weighted_colsum(const __nv_bfloat16* X, int64_t rows, int64_t D, const float* w,
                                   const __nv_bfloat16* extra, float* out, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * static_cast<size_t>(D + 1), s);
  if (e != cudaSuccess || rows == 0) return e;
  weighted_colsum_kernel<<<static_cast<int>((rows + kColsumRows - 1) / kColsumRows), 256, 0, s>>>(X, rows, D, w,
                                                                                                 extra, out);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_add_rank1(float* X, int64_t rows, int64_t D, const float* scale, float coef, const float* u,
                             cudaStream_t s) {
  if (rows * D == 0) return cudaSuccess;
  add_rank1_kernel<<<grid_for(rows * D, 256, 148 * 16), 256, 0, s>>>(X, rows, D, scale, coef, u);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_add_scalar(float* X, int64_t n, float coef, const float* c, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  add_scalar_kernel<<<grid_for(n, 256, 148 * 16), 256, 0, s>>>(X, n, coef, c);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_onehot_rows(const int* off, int nt, const int* rows, const int64_t* targets, int64_t vs,
                               const float* scale, float coef, const __nv_bfloat16* C, int64_t D, float* dE_acc,
                               float* dbias_acc, int64_t max_rows, cudaStream_t s) {
  if (max_rows == 0) return cudaSuccess;
  const int grid = static_cast<int>((max_rows + 7) / 8);  // 8 warps per block, one listed row each
  onehot_rows_apply_kernel<<<grid, 256, 0, s>>>(off, nt, rows, targets, vs, scale, coef, C, D, dE_acc, dbias_acc);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

// The bandwidth-bound and bookkeeping kernels around the tensor-core kernels:
//  fwd_finish     per row LSE = M + ln sum_j s_j exp(m_j - M) over the saved sub-tile (max, sum-exp)
//                 pairs, target validation, loss_r = LSE_r - z_t with the correct-token logit z_t
//                 the forward kernel picked from its logit tile (0 for ignored rows), and the count
//                 and mean/sum in a fixed order (fp64). Loss functions explainer, "How it works"
//                 items 1 and 4; Cut Cross Entropy from first principles; mlx-cross-entropy README,
//                 "API".
//  shard_merge    the same loss from the partial results of several vocabulary shards.
//  weighted_colsum  column sums of C or of scale_r E_r (label smoothing's rank-one terms).
//  fill_zero      zeroes a buffer (the fp32 accumulators of dE and dbias).
#include <cuda_bf16.h>

#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

__device__ __forceinline__ bool valid_target(int64_t t, int64_t V, int64_t ignore_index) {
  return t != ignore_index && t >= 0 && t < V;
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

__device__ __forceinline__ void lse_merge(float& M, float& S, float m, float s) {
  if (m == -INFINITY) return;
  if (m > M) {
    S = S * exp2f((M - m) * kLog2e) + s;
    M = m;
  } else {
    S += s * exp2f((m - M) * kLog2e);
  }
}

constexpr int kFinishWarps = kFinishRows;  // rows per block; one warp per row for the dot product
constexpr int kFinishBatch = 8;            // sub-tiles a warp loads before merging them
constexpr int kReduceThreads = 1024;

// The rest of the forward after the tensor-core kernel, one block of 32 warps per 32 rows:
//  1. LSE_r = M + ln sum_j s_j exp(m_j - M) over the saved per-sub-tile (max, sum-exp) pairs
//     (Loss functions explainer, "How it works" item 1). Warp w merges sub-tiles j = w, w + 32, ...
//     of the block's rows (lane = row: 128-byte loads), kFinishBatch sub-tiles per step.
//  2. warp w, row r0 + w: the correct-token logit z_t, which the forward kernel took from its fp32
//     logit tile (Cut Your Losses abstract: only the correct token's logit is computed); with label
//     smoothing also z_sum = sum_v z[r, v] = E_r . colsum(C) (+ sum of the bias), fp32 accumulation
//     of bf16 products, 16-byte loads. C holds vocabulary rows [vs, vs + V) of vtot: a target
//     elsewhere gets z_t = 0 (another shard's), and a target outside [0, vtot) that is not
//     ignore_index is a device error.
//  3. the loss of each row, LSE - (1 - ls) z_t - (ls / V) z_sum + zl LSE^2 (0 for ignored rows; Cut
//     Cross Entropy from first principles; explainer items 3 and 4, z-loss), and the block's fp64
//     sum and count; the last block to finish adds the blocks' sums in block order (a fixed order:
//     deterministic) into the mean / sum and the count. When a device error was recorded the loss is
//     written as NaN (every entry for reduction none).
// A vocabulary shard (loss == null) writes its partial results instead: lse, z_t and z_sum per row.
__global__ void __launch_bounds__(kFinishWarps * 32) fwd_finish_kernel(const __grid_constant__ FwdFinish F) {
  __shared__ float sm_m[kFinishWarps][32], sm_s[kFinishWarps][32];
  __shared__ float s_zt[kFinishWarps], s_zs[kFinishWarps];
  __shared__ double s_sum[kReduceThreads];
  __shared__ long long s_cnt[kReduceThreads];
  __shared__ int s_last;
  wait_for_previous_grid();  // the tensor-core kernel's sub-tile statistics and picked logits
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kFinishWarps;
  const int64_t N = F.N, T = F.T, D = F.D;
  {  // 1. per-sub-tile partials of rows r0 + lane
    const int64_t r = r0 + lane;
    float M = -INFINITY, S = 0.f;
    if (r < N) {
      for (int64_t j = w; j < T; j += kFinishBatch * kFinishWarps) {
        float m[kFinishBatch], sv[kFinishBatch];
#pragma unroll
        for (int u = 0; u < kFinishBatch; ++u) {
          const int64_t jj = j + u * kFinishWarps;
          m[u] = jj < T ? F.tile_max[jj * N + r] : -INFINITY;
          sv[u] = jj < T ? F.tile_sum[jj * N + r] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kFinishBatch; ++u) lse_merge(M, S, m[u], sv[u]);
      }
    }
    sm_m[w][lane] = M;
    sm_s[w][lane] = S;
  }
  {  // 2. dot products of row r0 + w
    const int64_t r = r0 + w;
    float zt = 0.f, zs = 0.f;
    if (r < N) {
      const int64_t t = F.targets[r];
      const __nv_bfloat16* e = F.E + r * D;
      if (F.csum != nullptr) {
        for (int64_t d = static_cast<int64_t>(lane) * 8; d < D; d += 256)
          zs = dot8_f32(ld_global_nc_v4(e + d), F.csum + d, zs);
        zs = warp_sum(zs) + F.csum[D];
      }
      if (valid_target(t - F.vs, F.V, F.ignore_index - F.vs)) {  // not ignored, inside this shard
        zt = F.zt[r];
      } else if (lane == 0 && t != F.ignore_index && !valid_target(t, F.vtot, F.ignore_index)) {
        record_error(F.err, kErrTargetRange);
      }
    }
    if (lane == 0) {
      s_zt[w] = zt;
      s_zs[w] = zs;
    }
  }
  __syncthreads();
  // 3. rows r0 + lane in warp 0
  if (w == 0) {
    const int64_t r = r0 + lane;
    double l = 0.0;
    long long c = 0;
    if (r < N) {
      float Mt = -INFINITY, St = 0.f;
      for (int k = 0; k < kFinishWarps; ++k) lse_merge(Mt, St, sm_m[k][lane], sm_s[k][lane]);
      const float L = Mt + logf(St);
      F.lse[r] = L;
      if (F.zt_out != nullptr) {
        F.zt_out[r] = s_zt[lane];
        F.zs_out[r] = s_zs[lane];
      }
      if (F.loss != nullptr) {
        const int64_t t = F.targets[r];
        float lr = L - (1.f - F.label_smoothing) * s_zt[lane] + F.z_loss * L * L;
        if (F.csum != nullptr) lr -= F.label_smoothing / static_cast<float>(F.V) * s_zs[lane];
        lr = valid_target(t, F.V, F.ignore_index) ? lr : 0.f;
        if (F.reduction == 0) F.loss[r] = lr;
        l = lr;
        c = t != F.ignore_index ? 1 : 0;
      }
    }
    if (F.loss != nullptr) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
      }
      if (lane == 0) {
        F.block_sums[blockIdx.x] = l;
        F.block_counts[blockIdx.x] = c;
        __threadfence();
        s_last = atomicAdd(F.done, 1) == static_cast<int>(gridDim.x) - 1;
      }
    }
  }
  __syncthreads();
  if (F.loss == nullptr || !s_last) return;
  __threadfence();  // the other blocks' sums, counts and per-row losses are visible
  double acc = 0.0;
  long long cnt = 0;
  for (int b = threadIdx.x; b < static_cast<int>(gridDim.x); b += kReduceThreads) {
    acc += reinterpret_cast<volatile double*>(F.block_sums)[b];
    cnt += reinterpret_cast<volatile long long*>(F.block_counts)[b];
  }
  s_sum[threadIdx.x] = acc;
  s_cnt[threadIdx.x] = cnt;
  __syncthreads();
  for (int o = kReduceThreads / 2; o > 0; o >>= 1) {
    if (static_cast<int>(threadIdx.x) < o) {
      s_sum[threadIdx.x] += s_sum[threadIdx.x + o];
      s_cnt[threadIdx.x] += s_cnt[threadIdx.x + o];
    }
    __syncthreads();
  }
  const bool failed = *reinterpret_cast<const volatile int*>(F.err) != 0;
  if (threadIdx.x == 0) {
    const long long c = s_cnt[0];
    *F.count = c;
    if (F.reduction == 1) *F.loss = failed ? NAN : static_cast<float>(s_sum[0] / static_cast<double>(c > 0 ? c : 1));
    if (F.reduction == 2) *F.loss = failed ? NAN : static_cast<float>(s_sum[0]);
  }
  if (failed && F.reduction == 0)
    for (int64_t r = threadIdx.x; r < N; r += kReduceThreads) F.loss[r] = NAN;
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

cudaError_t launch_fwd_finish(const FwdFinish& F, bool after_kernel, cudaStream_t s) {
  const int64_t blocks = (F.N + kFinishWarps - 1) / kFinishWarps;
  const dim3 grid(static_cast<unsigned>(blocks > 0 ? blocks : 1)), block(kFinishWarps * 32);
  if (after_kernel) {
    const cudaError_t e = launch_after_previous(fwd_finish_kernel, grid, block, 0, s, F);
    if (e != cudaSuccess) return e;
  } else {
    fwd_finish_kernel<<<grid, block, 0, s>>>(F);
  }
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

}  // namespace cce

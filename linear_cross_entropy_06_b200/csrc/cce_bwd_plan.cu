// Planning of the backward: which (row block b, vocabulary tile t) tiles carry gradient, and two
// compact lists of them.
//
// A tile of 128 rows x 128 vocabulary columns is kept when some non-ignored row r of block b has
// max over the tile of z[r, v] - LSE_r >= ln(eps) (mlx-cross-entropy README, "How it works" item 2:
// skip tiles whose softmax is below 2^-12), judged from the forward's saved per-sub-tile maxima.
// A skipped tile that holds the target of one of its rows still carries the onehot term of
// p - y (Loss functions explainer, "How it works" item 2), which is never skipped. Such a tile
// ("onehot only") is not listed: its rows' onehot terms are applied one row at a time, listed by
// vocabulary tile in oh_off / oh_rows (dC adds -scale_r (1 - ls) E_r to row t_r, dE adds
// -scale_r (1 - ls) C_{t_r} to row r).
//
// flags[b * nt + t]: 0 = no gradient, 1 = kept (listed), 2 = onehot only.
// By vocabulary tile (recompute and dC kernels): offsets_t[t] .. offsets_t[t+1] index entries_t,
//   each (b * 4 + flag, t), row blocks ascending. An entry's position is also its gradient-tile slot.
// By row block (dE kernel): offsets_b[b] .. offsets_b[b+1] index entries_b, each (t, slot),
//   vocabulary tiles ascending.
// Flat work lists the backward kernel reads with one load per item:
//   rb_range[c * nb + b]   the entries [lo, hi) of row block b inside vocabulary chunk c;
//   pair_desc/pair_slot    the pairs of consecutive listed tiles of a row block inside a chunk,
//                          by the vocabulary tile of their first tile (pstart_t[t] is the first
//                          pair starting in tile t, so a chunk's pairs are contiguous).
#include <algorithm>

#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

__device__ __forceinline__ bool valid_target(int64_t t, int64_t V, int64_t ignore_index) {
  return t != ignore_index && t >= 0 && t < V;
}

// One block of 128 threads (one per tile row) per row block b and run of kFlagTiles vocabulary
// tiles: the flags of those tiles. The rows' targets and LSE are read once for the whole run.
constexpr int kFlagTiles = 8;

__global__ void tile_flags_kernel(const float* __restrict__ tile_max, const float* __restrict__ lse,
                                  const int64_t* __restrict__ targets, int64_t N, int64_t V, int64_t T,
                                  int64_t ignore_index, float ln_eps, int filter_on, int nt, int runs,
                                  uint8_t* __restrict__ flags) {
  __shared__ float wmax[kFlagTiles][4];
  __shared__ int any_target[kFlagTiles];
  const int b = static_cast<int>(blockIdx.x / runs), t0 = static_cast<int>(blockIdx.x % runs) * kFlagTiles;
  const int64_t r = static_cast<int64_t>(b) * kBwdBM + threadIdx.x;
  if (threadIdx.x < kFlagTiles) any_target[threadIdx.x] = 0;
  __syncthreads();
  bool valid = false;
  float l = 0.f;
  int64_t tr = -1;
  if (r < N) {
    tr = targets[r];
    valid = valid_target(tr, V, ignore_index);
    if (valid && filter_on) l = lse[r];
  }
  if (valid && tr / kBwdBN >= t0 && tr / kBwdBN < t0 + kFlagTiles) any_target[tr / kBwdBN - t0] = 1;
#pragma unroll
  for (int k = 0; k < kFlagTiles; ++k) {
    const int t = t0 + k;
    float m = -INFINITY;
    if (valid && filter_on && t < nt) {
      const int64_t j0 = static_cast<int64_t>(t) * (kBwdBN / kSubTile);
      const int64_t j1 = j0 + kBwdBN / kSubTile < T ? j0 + kBwdBN / kSubTile : T;
      for (int64_t j = j0; j < j1; ++j) m = fmaxf(m, tile_max[j * N + r]);
      m -= l;
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) wmax[k][threadIdx.x >> 5] = m;
  }
  __syncthreads();
  if (threadIdx.x < kFlagTiles && t0 + threadIdx.x < nt) {
    const int k = threadIdx.x;
    const bool keep = !filter_on || fmaxf(fmaxf(wmax[k][0], wmax[k][1]), fmaxf(wmax[k][2], wmax[k][3])) >= ln_eps;
    flags[static_cast<int64_t>(b) * nt + t0 + k] = keep ? 1 : (any_target[k] ? 2 : 0);
  }
}

// One warp per vocabulary tile t: the rank of each listed (b, t) among the listed row blocks of t,
// the number of listed tiles of t, and the kept total.
__global__ void tile_rank_kernel(const uint8_t* __restrict__ flags, int nb, int nt, int* __restrict__ rank,
                                 int* __restrict__ cnt_t, int* __restrict__ cnt_b, int* __restrict__ kept_total) {
  const int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= nt) return;
  int listed = 0, kept = 0;
  for (int b0 = 0; b0 < nb; b0 += 32) {
    const int b = b0 + lane;
    const uint8_t f = b < nb ? flags[static_cast<int64_t>(b) * nt + t] : 0;
    const unsigned on = __ballot_sync(0xffffffffu, f == 1);
    if (f == 1) {
      rank[static_cast<int64_t>(b) * nt + t] = listed + __popc(on & ((1u << lane) - 1u));
      atomicAdd(cnt_b + b, 1);
    }
    listed += __popc(on);
    kept += __popc(__ballot_sync(0xffffffffu, f == 1));
  }
  if (lane == 0) {
    cnt_t[t] = listed;
    atomicAdd(kept_total, kept);
  }
}

// Exclusive scan of cnt[0..n) into off[0..n]; one block of 1024 threads, in chunks.
__global__ void scan_kernel(const int* __restrict__ cnt, int n, int* __restrict__ off) {
  __shared__ int buf[1024];
  __shared__ int carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    const int v = i < n ? cnt[i] : 0;
    buf[threadIdx.x] = v;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int add = threadIdx.x >= o ? buf[threadIdx.x - o] : 0;
      __syncthreads();
      buf[threadIdx.x] += add;
      __syncthreads();
    }
    if (i < n) off[i] = carry + buf[threadIdx.x] - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += buf[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) off[n] = carry;
}

__global__ void fill_col_kernel(const uint8_t* __restrict__ flags, const int* __restrict__ rank,
                                const int* __restrict__ offsets_t, int nb, int nt, int2* __restrict__ entries_t) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<int64_t>(nb) * nt) return;
  const uint8_t f = flags[i];
  if (f != 1) return;
  const int b = static_cast<int>(i / nt), t = static_cast<int>(i % nt);
  entries_t[offsets_t[t] + rank[i]] = make_int2(b * 4 + f, t);
}

// One block of 1024 threads per row block: writes its listed tiles in vocabulary order (a block-wide
// scan of the listed flags, 1024 vocabulary tiles per step), and the inverse map pos_b.
__global__ void row_list_kernel(const uint8_t* __restrict__ flags, const int* __restrict__ rank,
                                const int* __restrict__ offsets_t, int nt, const int* __restrict__ offsets_b,
                                int2* __restrict__ entries_b, int* __restrict__ pos_b) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint8_t* row = flags + static_cast<int64_t>(b) * nt;
  if (threadIdx.x == 0) carry = offsets_b[b];
  __syncthreads();
  for (int t0 = 0; t0 < nt; t0 += 1024) {
    const int t = t0 + threadIdx.x;
    const bool on = t < nt && row[t] == 1;
    const unsigned m = __ballot_sync(0xffffffffu, on);
    if (lane == 0) wsum[w] = __popc(m);
    __syncthreads();
    int before = 0, total = 0;
    for (int k = 0; k < 32; ++k) {
      before += k < w ? wsum[k] : 0;
      total += wsum[k];
    }
    if (on) {
      const int pos = carry + before + __popc(m & ((1u << lane) - 1u));
      const int slot = offsets_t[t] + rank[static_cast<int64_t>(b) * nt + t];
      entries_b[pos] = make_int2(t, slot);
      pos_b[slot] = pos;
    }
    __syncthreads();  // everyone has read carry and wsum
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
}

__device__ __forceinline__ int lower_bound_t(const int2* e, int lo, int hi, int t) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (e[mid].x < t) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Chunk boundaries: chunk c covers vocabulary tiles [c * chunk_vt, min(nt, (c + 1) * chunk_vt)).
__global__ void chunk_plan_kernel(int nt, int chunk_vt, int nchunks, int* __restrict__ chunk_t) {
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c <= nchunks; c += gridDim.x * blockDim.x)
    chunk_t[c] = min(nt, c * chunk_vt);
}

// For every chunk c and row block b, the range [lo, hi) of b's entries_b inside the chunk.
__global__ void row_range_kernel(const int2* __restrict__ entries_b, const int* __restrict__ offsets_b, int nb,
                                 int nchunks, const int* __restrict__ chunk_t, int2* __restrict__ rb_range) {
  const int64_t total = static_cast<int64_t>(nb) * nchunks;
  for (int64_t cb = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; cb < total;
       cb += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(cb / nb), b = static_cast<int>(cb % nb);
    const int lo = lower_bound_t(entries_b, offsets_b[b], offsets_b[b + 1], chunk_t[c]);
    const int hi = lower_bound_t(entries_b, lo, offsets_b[b + 1], chunk_t[c + 1]);
    rb_range[cb] = make_int2(lo, hi);
  }
}

// A listed tile (b, t) starts a pair when its position in row block b's list inside t's chunk is
// even; the pair is (b, t) and b's next listed tile in the chunk, if any. Pairs are listed by the
// vocabulary tile of their first tile (then row block), so that the recompute of concurrent pairs
// shares C tiles in L2. One warp per vocabulary tile; pass 0 counts the pairs starting in tile t,
// pass 1 (after the scan of those counts into pstart_t) writes them.
__global__ void pair_list_kernel(const int2* __restrict__ entries_t, const int* __restrict__ offsets_t,
                                 const int2* __restrict__ entries_b, const int* __restrict__ pos_b,
                                 const int2* __restrict__ rb_range, const uint8_t* __restrict__ flags, int nb, int nt,
                                 int chunk_vt, const int* __restrict__ chunk_t, int* __restrict__ cnt,
                                 const int* __restrict__ pstart_t, int4* __restrict__ pair_desc,
                                 int2* __restrict__ pair_slot, int pass) {
  const int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= nt) return;
  const int c = t / chunk_vt;
  const int slot_base = offsets_t[chunk_t[c]];
  const int i0 = offsets_t[t], i1 = offsets_t[t + 1];
  int k = 0;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    bool start = false;
    int b = 0, p = 0;
    int2 rr = make_int2(0, 0);
    if (i < i1) {
      b = entries_t[i].x >> 2;
      p = pos_b[i];
      rr = rb_range[static_cast<int64_t>(c) * nb + b];
      start = ((p - rr.x) & 1) == 0;
    }
    const unsigned mask = __ballot_sync(0xffffffffu, start);
    if (pass == 1 && start) {
      const int out = pstart_t[t] + k + __popc(mask & ((1u << lane) - 1u));
      const bool two = p + 1 < rr.y;
      const int t1 = two ? entries_b[p + 1].x : -1;
      const int slot1 = two ? entries_b[p + 1].y : i;
      const uint8_t* row = flags + static_cast<int64_t>(b) * nt;
      const int kept = (row[t] == 1 ? 1 : 0) | (two && row[t1] == 1 ? 2 : 0);
      pair_desc[out] = make_int4(b, t, t1, kept);
      pair_slot[out] = make_int2(i - slot_base, slot1 - slot_base);
    }
    k += __popc(mask);
  }
  if (pass == 0 && lane == 0) cnt[t] = k;
}

// Sizes of the backward's queue groups, in queue order: pairs(0), then pairs(c) and dE/dC(c - 1)
// for c = 1 .. n-1, then dE/dC(n - 1). A chunk's pairs are those starting in its vocabulary tiles;
// its dE/dC group holds nb * S dE items and one dC item per vocabulary tile and slice.
__global__ void group_size_kernel(const int* __restrict__ pstart_t, const int* __restrict__ chunk_t, int nb, int S,
                                  int nchunks, int* __restrict__ grp_size) {
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < 2 * nchunks; g += gridDim.x * blockDim.x) {
    int c, pairs;
    if (g == 0) {
      c = 0;
      pairs = 1;
    } else if (g == 2 * nchunks - 1) {
      c = nchunks - 1;
      pairs = 0;
    } else {
      const int pos = g - 1;
      c = pos / 2 + 1 - (pos & 1);
      pairs = (pos & 1) == 0;
    }
    grp_size[g] = pairs ? pstart_t[chunk_t[c + 1]] - pstart_t[chunk_t[c]] : (nb + chunk_t[c + 1] - chunk_t[c]) * S;
  }
}

// Rows whose target tile is onehot only: counted (pass 0) or written (pass 1, positions from the
// scanned counts and a per-tile cursor) per vocabulary tile of the target.
__global__ void onehot_rows_kernel(const uint8_t* __restrict__ flags, const int64_t* __restrict__ targets,
                                   int64_t N, int64_t V, int64_t ignore_index, int nt, int* __restrict__ cnt,
                                   const int* __restrict__ off, int* __restrict__ rows, int pass) {
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < N;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tr = targets[r];
    if (!valid_target(tr, V, ignore_index)) continue;
    const int t = static_cast<int>(tr / kBwdBN);
    if (flags[(r / kBwdBM) * nt + t] != 2) continue;
    const int k = atomicAdd(cnt + t, 1);
    if (pass == 1) rows[off[t] + k] = static_cast<int>(r);
  }
}

__global__ void plan_finish_kernel(const int* __restrict__ kept_total, int64_t total, int64_t* __restrict__ filtered) {
  *filtered = total - static_cast<int64_t>(*kept_total);
}

}  // namespace

cudaError_t launch_bwd_plan(const BwdPlan& P, const float* tile_max, const float* lse, const int64_t* targets,
                            int64_t N, int64_t V, int64_t T, int64_t ignore_index, float filter_eps,
                            int64_t* filtered_tiles, cudaStream_t s) {
  const int nb = P.nb, nt = P.nt;
  const int filter_on = filter_eps > 0.f ? 1 : 0;
  const float ln_eps = filter_on ? logf(filter_eps) : -INFINITY;
  cudaError_t e = cudaMemsetAsync(P.kept_total, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  if (nb > 0) {
    const int64_t tiles = static_cast<int64_t>(nb) * nt;
    const int runs = (nt + kFlagTiles - 1) / kFlagTiles;
    tile_flags_kernel<<<static_cast<unsigned>(static_cast<int64_t>(nb) * runs), kBwdBM, 0, s>>>(
        tile_max, lse, targets, N, V, T, ignore_index, ln_eps, filter_on, nt, runs, P.flags);
    note_launches(1);
    e = cudaMemsetAsync(P.cnt_b, 0, sizeof(int) * static_cast<size_t>(nb), s);
    if (e != cudaSuccess) return e;
    tile_rank_kernel<<<static_cast<int>((static_cast<int64_t>(nt) * 32 + 255) / 256), 256, 0, s>>>(
        P.flags, nb, nt, P.rank, P.cnt_t, P.cnt_b, P.kept_total);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.cnt_t, nt, P.offsets_t);
    note_launches(1);
    fill_col_kernel<<<static_cast<int>((tiles + 255) / 256), 256, 0, s>>>(P.flags, P.rank, P.offsets_t, nb, nt,
                                                                          P.entries_t);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.cnt_b, nb, P.offsets_b);
    note_launches(1);
    row_list_kernel<<<nb, 1024, 0, s>>>(P.flags, P.rank, P.offsets_t, nt, P.offsets_b, P.entries_b, P.pos_b);
    note_launches(1);
    chunk_plan_kernel<<<(P.nchunks + 256) / 256, 256, 0, s>>>(nt, P.chunk_vt, P.nchunks, P.chunk_t);
    note_launches(1);
    const int64_t cbs = static_cast<int64_t>(nb) * P.nchunks;
    row_range_kernel<<<static_cast<int>(std::min<int64_t>((cbs + 255) / 256, 4096)), 256, 0, s>>>(
        P.entries_b, P.offsets_b, nb, P.nchunks, P.chunk_t, P.rb_range);
    note_launches(1);
    // the pair counts per vocabulary tile reuse cnt_t (its counts are already scanned into offsets_t)
    const int grid_t = static_cast<int>((static_cast<int64_t>(nt) * 32 + 255) / 256);
    pair_list_kernel<<<grid_t, 256, 0, s>>>(P.entries_t, P.offsets_t, P.entries_b, P.pos_b, P.rb_range, P.flags, nb,
                                            nt, P.chunk_vt, P.chunk_t, P.cnt_t, P.pstart_t, P.pair_desc, P.pair_slot,
                                            0);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.cnt_t, nt, P.pstart_t);
    note_launches(1);
    pair_list_kernel<<<grid_t, 256, 0, s>>>(P.entries_t, P.offsets_t, P.entries_b, P.pos_b, P.rb_range, P.flags, nb,
                                            nt, P.chunk_vt, P.chunk_t, P.cnt_t, P.pstart_t, P.pair_desc, P.pair_slot,
                                            1);
    note_launches(1);
    group_size_kernel<<<(P.nchunks + 255) / 256, 256, 0, s>>>(P.pstart_t, P.chunk_t, nb, P.S, P.nchunks, P.grp_size);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.grp_size, 2 * P.nchunks, P.grp_start);
    note_launches(1);
  }
  if (nb > 0) {
    e = cudaMemsetAsync(P.oh_cnt, 0, sizeof(int) * static_cast<size_t>(nt), s);
    if (e != cudaSuccess) return e;
    const int grid_r = static_cast<int>(std::min<int64_t>((N + 255) / 256, 4096));
    onehot_rows_kernel<<<grid_r, 256, 0, s>>>(P.flags, targets, N, V, ignore_index, nt, P.oh_cnt, P.oh_off,
                                              P.oh_rows, 0);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.oh_cnt, nt, P.oh_off);
    note_launches(1);
    e = cudaMemsetAsync(P.oh_cnt, 0, sizeof(int) * static_cast<size_t>(nt), s);
    if (e != cudaSuccess) return e;
    onehot_rows_kernel<<<grid_r, 256, 0, s>>>(P.flags, targets, N, V, ignore_index, nt, P.oh_cnt, P.oh_off,
                                              P.oh_rows, 1);
    note_launches(1);
  }
  plan_finish_kernel<<<1, 1, 0, s>>>(P.kept_total, static_cast<int64_t>(nb) * nt, filtered_tiles);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

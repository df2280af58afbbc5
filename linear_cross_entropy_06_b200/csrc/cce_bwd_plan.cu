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
                                  const int64_t* __restrict__ targets, int64_t N, int64_t V, int64_t vs,
                                  int64_t vtot, int64_t T, int64_t ignore_index, float ln_eps, int filter_on, int nt,
                                  int runs, uint8_t* __restrict__ flags) {
  __shared__ float wmax[kFlagTiles][4];
  __shared__ int any_target[kFlagTiles];
  const int b = static_cast<int>(blockIdx.x / runs), t0 = static_cast<int>(blockIdx.x % runs) * kFlagTiles;
  const int64_t r = static_cast<int64_t>(b) * kBwdBM + threadIdx.x;
  if (threadIdx.x < kFlagTiles) any_target[threadIdx.x] = 0;
  __syncthreads();
  bool valid = false, local = false;
  float l = 0.f;
  int64_t tr = -1;
  if (r < N) {
    tr = targets[r];
    valid = valid_target(tr, vtot, ignore_index);      // the row is scored (by every shard)
    local = valid && valid_target(tr - vs, V, ignore_index - vs);  // its target lies in this shard
    if (valid && filter_on) l = lse[r];
    tr -= vs;
  }
  if (local && tr / kBwdBN >= t0 && tr / kBwdBN < t0 + kFlagTiles) any_target[tr / kBwdBN - t0] = 1;
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

// For every chunk c and row block b, the range [lo, hi) of b's entries_b inside the chunk.
// Chunk c covers vocabulary tiles [c * chunk_vt, min(nt, (c + 1) * chunk_vt)).
__global__ void row_range_kernel(const int2* __restrict__ entries_b, const int* __restrict__ offsets_b, int nb,
                                 int nchunks, int nt, int chunk_vt, int2* __restrict__ rb_range) {
  const int64_t total = static_cast<int64_t>(nb) * nchunks;
  for (int64_t cb = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; cb < total;
       cb += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(cb / nb), b = static_cast<int>(cb % nb);
    const int lo = lower_bound_t(entries_b, offsets_b[b], offsets_b[b + 1], min(nt, c * chunk_vt));
    const int hi = lower_bound_t(entries_b, lo, offsets_b[b + 1], min(nt, (c + 1) * chunk_vt));
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
                                 int chunk_vt, int* __restrict__ cnt,
                                 const int* __restrict__ pstart_t, int4* __restrict__ pair_desc,
                                 int2* __restrict__ pair_slot, int pass) {
  const int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= nt) return;
  const int c = t / chunk_vt;
  const int slot_base = offsets_t[c * chunk_vt];
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

// Block-wide ordered compaction helper: every thread holds one flag; returns the number of set flags
// before this thread in the block (ascending thread order) and sets *total to the block's count.
// blockDim.x is a multiple of 32, at most 1024; `warps` is shared scratch of 32 ints.
__device__ __forceinline__ int block_rank(bool flag, int* warps, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warps[w] = __popc(m);
  __syncthreads();
  int before = 0, all = 0;
  for (int k = 0; k < nw; ++k) {
    before += k < w ? warps[k] : 0;
    all += warps[k];
  }
  __syncthreads();  // warps[] may be rewritten by the next call
  *total = all;
  return before + __popc(m & ((1u << lane) - 1u));
}

// One block per vocabulary chunk c: its work lists and the sizes of its two queue groups.
//  - vt_order: the chunk's vocabulary tiles with a listed tile first (they get dC items), then the
//    empty ones (no row block lists them: their dC rows hold only onehot and smoothing terms and are
//    written by dc_fill_empty_kernel); both ascending.
//  - de_list: the row blocks with a listed tile in the chunk (they get dE items), ascending.
//  - empty_list: the chunk's empty tiles, appended to one list for the whole vocabulary.
//  - grp_size: pairs(c) and dE/dC(c), at their places in the queue order pairs(0), then pairs(c) and
//    dE/dC(c - 1) for c = 1 .. n-1, then dE/dC(n - 1): pairs(c) is group 2c - 1 (0 for c = 0) and
//    dE/dC(c) group min(2c + 2, 2n - 1).
__global__ void chunk_items_kernel(const int* __restrict__ offsets_t, const int2* __restrict__ rb_range,
                                   const int* __restrict__ pstart_t, int nt, int chunk_vt, int nb, int S,
                                   int nchunks, int* __restrict__ chunk_t, int* __restrict__ vt_order,
                                   int* __restrict__ ndc, int* __restrict__ de_list, int* __restrict__ nde,
                                   int* __restrict__ empty_list, int* __restrict__ n_empty,
                                   int* __restrict__ grp_size) {
  __shared__ int warps[32];
  __shared__ int em_base;
  const int c = blockIdx.x;
  const int t0 = min(nt, c * chunk_vt), t1 = min(nt, (c + 1) * chunk_vt);
  if (threadIdx.x == 0) {
    chunk_t[c] = t0;
    if (c == nchunks - 1) chunk_t[nchunks] = t1;
  }
  // vocabulary tiles: count the listed ones first, so that the empty ones can follow them
  int n_listed = 0;
  for (int base = t0; base < t1; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const bool on = t < t1 && offsets_t[t + 1] > offsets_t[t];
    int total;
    const int pos = block_rank(on, warps, &total);
    if (on) vt_order[t0 + n_listed + pos] = t;
    n_listed += total;
  }
  const int n_em = (t1 - t0) - n_listed;
  if (threadIdx.x == 0) em_base = n_em > 0 ? atomicAdd(n_empty, n_em) : 0;
  __syncthreads();
  int n_seen = 0;
  for (int base = t0; base < t1; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const bool em = t < t1 && offsets_t[t + 1] == offsets_t[t];
    int total;
    const int pos = block_rank(em, warps, &total);
    if (em) {
      vt_order[t0 + n_listed + n_seen + pos] = t;
      empty_list[em_base + n_seen + pos] = t;
    }
    n_seen += total;
  }
  // row blocks with a listed tile in the chunk
  int n_rb = 0;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int b = base + threadIdx.x;
    bool on = false;
    if (b < nb) {
      const int2 r = rb_range[static_cast<int64_t>(c) * nb + b];
      on = r.x < r.y;
    }
    int total;
    const int pos = block_rank(on, warps, &total);
    if (on) de_list[static_cast<int64_t>(c) * nb + n_rb + pos] = b;
    n_rb += total;
  }
  if (threadIdx.x == 0) {
    ndc[c] = n_listed;
    nde[c] = n_rb;
    grp_size[c == 0 ? 0 : 2 * c - 1] = pstart_t[t1] - pstart_t[t0];
    grp_size[min(2 * c + 2, 2 * nchunks - 1)] = (n_rb + n_listed) * S;
  }
}

// dC rows of the vocabulary tiles that no row block lists. Every logit of such a tile is skipped,
// so only the target part of the logit gradient reaches them (Loss functions explainer, "How it
// works" items 2 and 3): -scale_r (1 - ls) E_r for each row r whose target v lies there, and the
// smoothing term dc_coef * dc_add shared by every row of dC. No tensor core is involved: a work unit
// is 4 vocabulary rows x 512 columns, one thread per 8 columns, 16-byte loads and stores along a
// row. The target rows of tile t are oh_rows[oh_off[t] .. oh_off[t + 1]) (for an empty tile every
// non-ignored row targeting it is listed there), scanned in order, so the result is deterministic.
constexpr int kFillCols = 512;

__global__ void __launch_bounds__(256, 4) dc_fill_empty_kernel(
    const int* __restrict__ empty_list, const int* __restrict__ n_empty, const int* __restrict__ oh_off,
    const int* __restrict__ oh_rows, const int64_t* __restrict__ targets, int64_t vs, const float* __restrict__ scale,
    float onehot_coef, const __nv_bfloat16* __restrict__ E, int64_t D, int64_t V, const float* __restrict__ dc_add,
    float dc_coef, void* __restrict__ dC, int out_bf16) {
  const int col_chunks = static_cast<int>((D + kFillCols - 1) / kFillCols);
  const int units_per_tile = (kBwdBN / 4) * col_chunks;
  const int64_t units = static_cast<int64_t>(*n_empty) * units_per_tile;
  const int row_in_unit = threadIdx.x >> 6;  // 4 rows of 64 threads
  const int col_thread = (threadIdx.x & 63) * 8;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int e = static_cast<int>(u / units_per_tile);
    const int rem = static_cast<int>(u % units_per_tile);
    const int t = empty_list[e];
    const int row = (rem / col_chunks) * 4 + row_in_unit;
    const int64_t v = static_cast<int64_t>(t) * kBwdBN + row;
    const int64_t d = static_cast<int64_t>(rem % col_chunks) * kFillCols + col_thread;
    if (v >= V || d >= D) continue;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = dc_add != nullptr ? dc_coef * dc_add[d + k] : 0.f;
    const int i1 = oh_off[t + 1];
    for (int i = oh_off[t]; i < i1; ++i) {
      const int r = oh_rows[i];
      if (targets[r] - vs != v) continue;
      const float a = -scale[r] * onehot_coef;
      const uint4 q = ld_global_nc_v4(E + static_cast<int64_t>(r) * D + d);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 h;
        *reinterpret_cast<uint32_t*>(&h) = w[k];
        acc[2 * k] = fmaf(a, __low2float(h), acc[2 * k]);
        acc[2 * k + 1] = fmaf(a, __high2float(h), acc[2 * k + 1]);
      }
    }
    if (out_bf16) {
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dC) + v * D + d) = o;
    } else {
      float4* out = reinterpret_cast<float4*>(static_cast<float*>(dC) + v * D + d);
      out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// Rows whose target tile is onehot only: counted (pass 0) or written (pass 1, positions from the
// scanned counts and a per-tile cursor) per vocabulary tile of the target.
__global__ void onehot_rows_kernel(const uint8_t* __restrict__ flags, const int64_t* __restrict__ targets,
                                   int64_t N, int64_t V, int64_t vs, int64_t ignore_index, int nt,
                                   int* __restrict__ cnt, const int* __restrict__ off, int* __restrict__ rows,
                                   int pass) {
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < N;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tr = targets[r] - vs;  // only targets inside this shard have an onehot term here
    if (!valid_target(tr, V, ignore_index - vs)) continue;
    const int t = static_cast<int>(tr / kBwdBN);
    if (flags[(r / kBwdBM) * nt + t] != 2) continue;
    const int k = atomicAdd(cnt + t, 1);
    if (pass == 1) rows[off[t] + k] = static_cast<int>(r);
  }
}

// out[i] = 1 when backward tile i (row block i / nt, vocabulary tile i % nt) was skipped, 0 when kept.
__global__ void skip_map_kernel(const uint8_t* __restrict__ flags, int64_t n, uint8_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = flags[i] == 1 ? 0 : 1;
}

__global__ void plan_finish_kernel(const int* __restrict__ kept_total, int64_t total, int64_t* __restrict__ filtered) {
  *filtered = total - static_cast<int64_t>(*kept_total);
}

}  // namespace

cudaError_t launch_dc_fill_empty(const BwdPlan& P, const int64_t* targets, int64_t vs, const float* scale,
                                 float onehot_coef, const __nv_bfloat16* E, int64_t D, int64_t V, const float* dc_add,
                                 float dc_coef, void* dC, int out_bf16, int num_sms, cudaStream_t s) {
  if (P.nb == 0) return cudaSuccess;
  // persistent: the number of empty tiles is known on the device only
  dc_fill_empty_kernel<<<num_sms * 8, 256, 0, s>>>(P.empty_list, P.n_empty, P.oh_off, P.oh_rows, targets, vs,
                                                   scale, onehot_coef, E, D, V, dc_add, dc_coef, dC, out_bf16);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_skip_map(const uint8_t* flags, int64_t tiles, uint8_t* out, cudaStream_t s) {
  if (tiles == 0) return cudaSuccess;
  skip_map_kernel<<<static_cast<int>(std::min<int64_t>((tiles + 255) / 256, 4096)), 256, 0, s>>>(flags, tiles, out);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_plan(const BwdPlan& P, const float* tile_max, const float* lse, const int64_t* targets,
                            int64_t N, int64_t V, int64_t vs, int64_t vtot, int64_t T, int64_t ignore_index,
                            float filter_eps, int64_t* filtered_tiles, cudaStream_t s) {
  const int nb = P.nb, nt = P.nt;
  const int filter_on = filter_eps > 0.f ? 1 : 0;
  const float ln_eps = filter_on ? logf(filter_eps) : -INFINITY;
  cudaError_t e = cudaMemsetAsync(P.kept_total, 0, 2 * sizeof(int), s);  // kept_total and n_empty
  if (e != cudaSuccess) return e;
  if (nb > 0) {
    const int64_t tiles = static_cast<int64_t>(nb) * nt;
    const int runs = (nt + kFlagTiles - 1) / kFlagTiles;
    tile_flags_kernel<<<static_cast<unsigned>(static_cast<int64_t>(nb) * runs), kBwdBM, 0, s>>>(
        tile_max, lse, targets, N, V, vs, vtot, T, ignore_index, ln_eps, filter_on, nt, runs, P.flags);
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
    const int64_t cbs = static_cast<int64_t>(nb) * P.nchunks;
    row_range_kernel<<<static_cast<int>(std::min<int64_t>((cbs + 255) / 256, 4096)), 256, 0, s>>>(
        P.entries_b, P.offsets_b, nb, P.nchunks, nt, P.chunk_vt, P.rb_range);
    note_launches(1);
    // the pair counts per vocabulary tile reuse cnt_t (its counts are already scanned into offsets_t)
    const int grid_t = static_cast<int>((static_cast<int64_t>(nt) * 32 + 255) / 256);
    pair_list_kernel<<<grid_t, 256, 0, s>>>(P.entries_t, P.offsets_t, P.entries_b, P.pos_b, P.rb_range, P.flags, nb,
                                            nt, P.chunk_vt, P.cnt_t, P.pstart_t, P.pair_desc, P.pair_slot,
                                            0);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.cnt_t, nt, P.pstart_t);
    note_launches(1);
    pair_list_kernel<<<grid_t, 256, 0, s>>>(P.entries_t, P.offsets_t, P.entries_b, P.pos_b, P.rb_range, P.flags, nb,
                                            nt, P.chunk_vt, P.cnt_t, P.pstart_t, P.pair_desc, P.pair_slot,
                                            1);
    note_launches(1);
    // (pair_list pass 0 left each vocabulary tile's pair count in cnt_t; chunk_items reads the
    // listed-tile counts as differences of offsets_t)
    chunk_items_kernel<<<P.nchunks, 256, 0, s>>>(P.offsets_t, P.rb_range, P.pstart_t, nt, P.chunk_vt, nb, P.S,
                                                 P.nchunks, P.chunk_t, P.vt_order, P.ndc, P.de_list, P.nde,
                                                 P.empty_list, P.n_empty, P.grp_size);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.grp_size, 2 * P.nchunks, P.grp_start);
    note_launches(1);
  }
  if (nb > 0) {
    e = cudaMemsetAsync(P.oh_cnt, 0, sizeof(int) * static_cast<size_t>(nt), s);
    if (e != cudaSuccess) return e;
    const int grid_r = static_cast<int>(std::min<int64_t>((N + 255) / 256, 4096));
    onehot_rows_kernel<<<grid_r, 256, 0, s>>>(P.flags, targets, N, V, vs, ignore_index, nt, P.oh_cnt, P.oh_off,
                                              P.oh_rows, 0);
    note_launches(1);
    scan_kernel<<<1, 1024, 0, s>>>(P.oh_cnt, nt, P.oh_off);
    note_launches(1);
    e = cudaMemsetAsync(P.oh_cnt, 0, sizeof(int) * static_cast<size_t>(nt), s);
    if (e != cudaSuccess) return e;
    onehot_rows_kernel<<<grid_r, 256, 0, s>>>(P.flags, targets, N, V, vs, ignore_index, nt, P.oh_cnt, P.oh_off,
                                              P.oh_rows, 1);
    note_launches(1);
  }
  plan_finish_kernel<<<1, 1, 0, s>>>(P.kept_total, static_cast<int64_t>(nb) * nt, filtered_tiles);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

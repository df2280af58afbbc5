// Planning of the backward: which (row block b, vocabulary tile t) tiles carry gradient, and two
// compact lists of them.
//
// The skip rule works on halves of a tile: 128 rows x 64 vocabulary columns. A half is kept when some
// non-ignored row r of block b has max over the half of z[r, v] - LSE_r >= ln(eps) (mlx-cross-entropy
// README, "How it works" item 2: skip tiles whose softmax is below 2^-12), judged from the forward's
// saved per-64-column maxima. A tile (128 x 128) with a kept half is listed; only its kept halves are
// recomputed and multiplied into dE, and its skipped half reads as zeros in the dC MMAs.
// The onehot term of p - y (Loss functions explainer, "How it works" item 2) is never skipped. A row
// whose target lies in a skipped half (of a listed tile, or of a tile with no kept half, "onehot
// only") gets its onehot term one row at a time, listed by vocabulary tile in oh_off / oh_rows (dC
// adds -scale_r (1 - ls) E_r to row t_r, dE adds -scale_r (1 - ls) C_{t_r} to row r).
//
// flags[b * nt + t]: the state (nothing, listed, onehot only) and the kept halves (cce_internal.h).
// By vocabulary tile (recompute and dC kernels): offsets_t[t] .. offsets_t[t+1] index entries_t,
//   each (b * 16 + flag, t), row blocks ascending. An entry's position is also its gradient-tile slot.
// By row block (dE kernel): offsets_b[b] .. offsets_b[b+1] index entries_b, each (t, slot | kept
//   halves << kSlotBits), vocabulary tiles ascending; hp_b counts the kept halves before each entry.
// Flat work lists the backward kernel reads with one load per item:
//   rb_range[c * nb + b]   the entries [lo, hi) of row block b inside vocabulary chunk c;
//   quad_b/quad_h/quad_s   the quads (up to four consecutive kept halves of a row block inside a chunk),
//                          by the vocabulary tile of their first half (pstart_t[t] is the first quad
//                          starting in tile t, so a chunk's quads are contiguous).
#include <algorithm>

#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

__device__ __forceinline__ bool valid_target(int64_t t, int64_t V, int64_t ignore_index) {
  return t != ignore_index && t >= 0 && t < V;
}

// Whether the onehot term of a row whose target is column tr (of this problem's vocabulary) is
// applied on its own: the half of the target's tile that holds tr is not kept. f is the flag of the
// row's block and the target's tile.
__device__ __forceinline__ bool target_half_skipped(int f, int64_t tr) {
  const int h = static_cast<int>((tr % kBwdBN) / kSubTile);
  return flag_state(f) == kFlagOnehotOnly || (flag_state(f) == kFlagListed && !((flag_halves(f) >> h) & 1));
}

// The planning runs as one cooperative launch of one 1024-thread block per SM: a sequence of
// phases separated by grid-wide barriers (bounded waits; a block that gives up records
// CCE_ERR_DEVICE_TIMEOUT and every block then leaves). Each phase spreads its work over the grid.
constexpr int kPlanThreads = 1024;
static_assert(kPlanThreads == 32 * 32, "block_scan keeps one total per warp in 32 lanes");
constexpr int kFlagTiles = 16;   // vocabulary tiles per flag unit (32 halves: one per lane of a column max)
constexpr int kFlagGroups = kPlanThreads / kBwdBM;  // flag units per block at a time (128 threads each)

struct PlanCtl {
  int* bar;        // barrier counter, zero at launch
  int* err;
  uint64_t timeout_ns;
};

// Grid-wide barrier number `round` (1, 2, ...): every block's writes before it are visible to every
// block after it. Returns false when the wait ran out or another block recorded an error.
__device__ bool grid_barrier(const PlanCtl& ctl, int round) {
  __shared__ int ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    ok = 1;
    __threadfence();
    red_release_add(ctl.bar, 1);
    const int target = round * static_cast<int>(gridDim.x);
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire(ctl.bar) < target) {
      if (ld_relaxed(ctl.err) != 0) {
        ok = 0;
        break;
      }
      if (global_timer_ns() - t0 > ctl.timeout_ns) {
        record_error(ctl.err, kErrDeviceTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  return ok != 0;
}

// Exclusive scan of cnt[0..n) into off[0..n] by the calling block (1024 threads = 32 warps), in
// chunks of 1024: a shuffle scan inside each warp, then one over the 32 warp totals.
__device__ void block_scan(const int* __restrict__ cnt, int n, int* __restrict__ off) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kPlanThreads) {
    const int i = base + threadIdx.x;
    const int v = i < n ? cnt[i] : 0;
    int x = v;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[w] = x;
    __syncthreads();
    if (w == 0) {  // inclusive scan of the warp totals
      int t = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      wsum[lane] = t;
    }
    __syncthreads();
    if (i < n) off[i] = carry + (w > 0 ? wsum[w - 1] : 0) + x - v;
    __syncthreads();  // every thread has read carry and wsum
    if (threadIdx.x == 0) carry += wsum[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) off[n] = carry;
  __syncthreads();
}

// Block-wide ordered compaction: every thread holds one flag; returns the number of set flags
// before this thread (ascending thread order) and sets *total to the block's count.
__device__ __forceinline__ int block_rank(bool flag, int* total) {
  __shared__ int warps[32];
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

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Column maxima of a warp's 32 x 32 block (lane = row, v[i] = column i): afterwards lane l returns the
// maximum over the 32 lanes of v[l]. Recursive halving, 31 shuffles. Clobbers v.
__device__ __forceinline__ float warp_column_max32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
    }
  }
  return v[0];
}

// Flags of one row block b and run of kFlagTiles vocabulary tiles from t0, by 128 threads (one per
// tile row; named barrier `group + 1`). Every load of the unit (the rows' targets and LSE, the run's
// saved maxima) is issued before any of them is used, so they are in flight together.
__device__ void tile_flags_unit(const PlanArgs& A, int group, int b, int t0) {
  __shared__ float wmax[kFlagGroups][4][2 * kFlagTiles];
  __shared__ int any_target[kFlagGroups][kFlagTiles];
  const int tid = threadIdx.x & (kBwdBM - 1), lane = tid & 31;
  const int nt = A.P.nt;
  const int64_t r = static_cast<int64_t>(b) * kBwdBM + tid;
  const bool row_in = r < A.N;
  if (tid < kFlagTiles) any_target[group][tid] = 0;
  const int64_t j0 = 2 * static_cast<int64_t>(t0);  // the run's first half (saved sub-tile)
  float mt[2 * kFlagTiles];
#pragma unroll
  for (int k = 0; k < 2 * kFlagTiles; ++k)
    mt[k] = (row_in && A.filter_on && j0 + k < A.T) ? A.tile_max[(j0 + k) * A.N + r] : -INFINITY;
  int64_t tr = row_in ? A.targets[r] : A.ignore_index;
  const float l = (row_in && A.filter_on) ? A.lse[r] : 0.f;
  named_barrier(group + 1, kBwdBM);
  const bool valid = row_in && valid_target(tr, A.vtot, A.ignore_index);  // the row is scored (by every shard)
  const bool local = valid && valid_target(tr - A.vs, A.V, A.ignore_index - A.vs);  // its target is in this shard
  tr -= A.vs;
  if (local && tr / kBwdBN >= t0 && tr / kBwdBN < t0 + kFlagTiles) any_target[group][tr / kBwdBN - t0] = 1;
#pragma unroll
  for (int k = 0; k < 2 * kFlagTiles; ++k) mt[k] = valid ? mt[k] - l : -INFINITY;
  wmax[group][tid >> 5][lane] = warp_column_max32(mt, lane);  // lane k: the warp's max of half j0 + k
  named_barrier(group + 1, kBwdBM);
  if (tid < kFlagTiles && t0 + tid < nt) {
    int halves = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = 2 * tid + h;
      const float m = fmaxf(fmaxf(wmax[group][0][k], wmax[group][1][k]), fmaxf(wmax[group][2][k], wmax[group][3][k]));
      if (j0 + k < A.T && (!A.filter_on || m >= A.ln_eps)) halves |= 1 << h;
    }
    A.P.flags[static_cast<int64_t>(b) * nt + t0 + tid] = static_cast<uint8_t>(
        halves != 0 ? (kFlagListed | (halves << 2)) : (any_target[group][tid] ? kFlagOnehotOnly : 0));
  }
  named_barrier(group + 1, kBwdBM);  // the shared arrays are reused by the group's next unit
}

// The listed tiles of row block b in vocabulary order (a block-wide scan of its flags, 1024 vocabulary
// tiles per step), the kept halves before each of them (hp_b, counted from the row block's offset
// off_hb[b]) and the inverse map pos_b; the whole block.
__device__ void row_list_block(const PlanArgs& A, int b) {
  __shared__ int wsum[32], hsum[32];
  __shared__ int carry, hcarry;
  const BwdPlan& P = A.P;
  const int nt = P.nt;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const uint8_t* row = P.flags + static_cast<int64_t>(b) * nt;
  if (threadIdx.x == 0) {
    carry = P.offsets_b[b];
    hcarry = P.off_hb[b];
  }
  __syncthreads();
  for (int t0 = 0; t0 < nt; t0 += kPlanThreads) {
    const int t = t0 + threadIdx.x;
    const int f = t < nt ? row[t] : 0;
    const bool on = flag_state(f) == kFlagListed;
    const int nh = on ? __popc(flag_halves(f)) : 0;
    const unsigned m = __ballot_sync(0xffffffffu, on);
    int hx = nh;  // inclusive scan of the kept halves within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, hx, o);
      if (lane >= o) hx += y;
    }
    if (lane == 31) {
      wsum[w] = __popc(m);
      hsum[w] = hx;
    }
    __syncthreads();
    int before = 0, total = 0, hbefore = 0, htotal = 0;
    for (int k = 0; k < 32; ++k) {
      before += k < w ? wsum[k] : 0;
      total += wsum[k];
      hbefore += k < w ? hsum[k] : 0;
      htotal += hsum[k];
    }
    if (on) {
      const int pos = carry + before + __popc(m & ((1u << lane) - 1u));
      const int slot = P.offsets_t[t] + P.rank[static_cast<int64_t>(b) * nt + t];
      P.entries_b[pos] = make_int2(t, slot | (flag_halves(f) << kSlotBits));
      P.hp_b[pos] = hcarry + hbefore + hx - nh;
      P.pos_b[slot] = pos;
    }
    __syncthreads();  // everyone has read carry and the warp sums
    if (threadIdx.x == 0) {
      carry += total;
      hcarry += htotal;
    }
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

// The recompute's items are quads: up to four consecutive kept halves of one row block inside a chunk,
// from one or several of its listed tiles. A kept half starts a quad when its position among the kept
// halves of its row block in the chunk (hp_b, counted from the row block's first entry there) is a
// multiple of four. Quads are listed by the vocabulary tile of their first half (then row block), so
// that the recompute of concurrent quads shares C rows in L2. One warp per vocabulary tile; pass 0
// counts the quads starting in tile t (into cnt_t, whose tile counts are already scanned into
// offsets_t), pass 1 (after the scan of those counts into pstart_t) writes them.
__device__ void quad_list_warp(const PlanArgs& A, int t, int lane, int pass) {
  const BwdPlan& P = A.P;
  const int nb = P.nb;
  const int c = P.chunk_of[t];
  const int slot_base = P.offsets_t[P.chunk_t[c]];
  const int i0 = P.offsets_t[t], i1 = P.offsets_t[t + 1];
  int k = 0;
  for (int base = i0; base < i1; base += 32) {
    const int i = base + lane;
    int b = 0, p = 0, hm = 0, hrel = 0, nstart = 0;
    int2 rr = make_int2(0, 0);
    if (i < i1) {
      const int x = P.entries_t[i].x;
      b = x >> 4;
      hm = flag_halves(x & 15);
      p = P.pos_b[i];
      rr = P.rb_range[static_cast<int64_t>(c) * nb + b];
      hrel = P.hp_b[p] - P.hp_b[rr.x];  // kept halves of b in the chunk before this tile
      for (int q = 0; q < __popc(hm); ++q) nstart += ((hrel + q) & 3) == 0 ? 1 : 0;
    }
    int incl = nstart;  // inclusive scan of the quad starts over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (pass == 1 && nstart > 0) {
      int out = P.pstart_t[t] + k + incl - nstart;
      for (int q = 0; q < __popc(hm); ++q) {
        if (((hrel + q) & 3) != 0) continue;
        // this tile's q-th kept half and the row block's next kept halves in the chunk, up to four
        int th[4] = {-1, -1, -1, -1}, sl[4] = {0, 0, 0, 0};
        int n = 0, skip = q;
        for (int pp = p; pp < rr.y && n < 4; ++pp) {
          const int2 e = P.entries_b[pp];
          const int m = e.y >> kSlotBits;
          for (int h = 0; h < 2 && n < 4; ++h) {
            if (!((m >> h) & 1)) continue;
            if (skip > 0) {
              --skip;
              continue;
            }
            th[n] = 2 * e.x + h;
            sl[n] = (e.y & kSlotMask) - slot_base;
            ++n;
          }
        }
        P.quad_b[out] = b;
        P.quad_h[out] = make_int4(th[0], th[1], th[2], th[3]);
        P.quad_s[out] = make_int4(sl[0], sl[1], sl[2], sl[3]);
        ++out;
      }
    }
    k += total;
  }
  if (pass == 0 && lane == 0) P.cnt_t[t] = k;
}

// Work lists of vocabulary chunk c and the sizes of its two queue groups; the whole block.
//  - vt_order: the chunk's vocabulary tiles with a listed tile first (they get dC items), then the
//    empty ones (no row block lists them: their dC rows hold only onehot and smoothing terms and are
//    written by bwd_finalize_kernel); both ascending.
//  - de_list: the row blocks with a listed tile in the chunk (they get dE items), ascending.
//  - empty_list: the chunk's empty tiles, appended to one list for the whole vocabulary.
//  - grp_size: quads(c) and dE/dC(c), at their places in the queue order quads(0), then quads(c) and
//    dE/dC(c - 1) for c = 1 .. n-1, then dE/dC(n - 1): quads(c) is group 2c - 1 (0 for c = 0) and
//    dE/dC(c) group min(2c + 2, 2n - 1).
__device__ void chunk_items_block(const PlanArgs& A, int c, int nchunks) {
  __shared__ int em_base;
  const BwdPlan& P = A.P;
  const int nb = P.nb;
  const int t0 = P.chunk_t[c], t1 = P.chunk_t[c + 1];
  int n_listed = 0;
  for (int base = t0; base < t1; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const bool on = t < t1 && P.offsets_t[t + 1] > P.offsets_t[t];
    int total;
    const int pos = block_rank(on, &total);
    if (on) P.vt_order[t0 + n_listed + pos] = t;
    n_listed += total;
  }
  const int n_em = (t1 - t0) - n_listed;
  if (threadIdx.x == 0) em_base = n_em > 0 ? atomicAdd(P.n_empty, n_em) : 0;
  __syncthreads();
  int n_seen = 0;
  for (int base = t0; base < t1; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const bool em = t < t1 && P.offsets_t[t + 1] == P.offsets_t[t];
    int total;
    const int pos = block_rank(em, &total);
    if (em) {
      P.vt_order[t0 + n_listed + n_seen + pos] = t;
      P.empty_list[em_base + n_seen + pos] = t;
    }
    n_seen += total;
  }
  int n_rb = 0;
  for (int base = 0; base < nb; base += blockDim.x) {
    const int b = base + threadIdx.x;
    bool on = false;
    if (b < nb) {
      const int2 r = P.rb_range[static_cast<int64_t>(c) * nb + b];
      on = r.x < r.y;
    }
    int total;
    const int pos = block_rank(on, &total);
    if (on) P.de_list[static_cast<int64_t>(c) * nb + n_rb + pos] = b;
    n_rb += total;
  }
  if (threadIdx.x == 0) {
    P.ndc[c] = n_listed;
    P.nde[c] = n_rb;
    P.grp_size[c == 0 ? 0 : 2 * c - 1] = P.pstart_t[t1] - P.pstart_t[t0];
    P.grp_size[min(2 * c + 2, 2 * nchunks - 1)] = (n_rb + n_listed) * P.S;
  }
  __syncthreads();  // em_base is reused by the block's next chunk
}

// Vocabulary chunks, by the calling block: consecutive vocabulary tiles, each chunk as long as its
// gradient tiles fit one buffer (at most chunk_g_tiles listed tiles) and the C rows its tiles read
// stay within kChunkCBytes (at most chunk_c_tiles vocabulary tiles with a listed tile), so that a
// sparse stretch of the vocabulary forms one long chunk: fewer chunks mean fewer partial sums of dE
// and longer groups of quads ahead of each chunk's dE / dC items. A chunk of the fixed length
// chunk_vt always satisfies both limits, so there are never more than P.nchunks chunks.
// Greedy, decided by warp 0 over 32 vocabulary tiles at a time (the prefix sums offsets_t staged in
// shared memory by the block): each lane tests whether its tile still fits the open chunk, and the
// first lane that does not starts the next one.
__device__ void chunk_partition(const PlanArgs& A) {
  __shared__ int off[kPlanThreads + 1];
  const BwdPlan& P = A.P;
  const int nt = P.nt;
  const int lane = threadIdx.x & 31;
  const bool decider = threadIdx.x < 32;
  int n = 0, start = 0, start_listed = 0, ne = 0;  // closed chunks; the open chunk's first tile,
                                                   // listed tiles before it, its non-empty tiles
  if (threadIdx.x == 0) P.chunk_t[0] = 0;
  for (int base = 0; base < nt; base += kPlanThreads) {
    __syncthreads();
    for (int i = threadIdx.x; i <= kPlanThreads; i += blockDim.x) off[i] = P.offsets_t[min(base + i, nt)];
    __syncthreads();
    if (!decider) continue;
    for (int sub = 0; sub < kPlanThreads && base + sub < nt; sub += 32) {
      const int i = sub + lane;
      const bool in = base + i < nt;
      const int end_listed = in ? off[i + 1] : 0;  // listed tiles before the end of tile base + i
      const bool nonempty = in && off[i + 1] > off[i];
      const unsigned ne_mask = __ballot_sync(0xffffffffu, nonempty);
      const unsigned le = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);  // lanes <= this one
      int from = 0;
      for (int guard = 0; guard <= 32; ++guard) {
        const unsigned live = from >= 32 ? 0u : (0xffffffffu << from);
        const int cum_ne = __popc(ne_mask & live & le);
        const bool bad = in && lane >= from &&
                         (end_listed - start_listed > P.chunk_g_tiles || ne + cum_ne > P.chunk_c_tiles);
        const unsigned bad_mask = __ballot_sync(0xffffffffu, bad);
        const int j = bad_mask ? __ffs(bad_mask) - 1 : 32;
        if (j == 32 || base + sub + j <= start) {  // the rest of this group fits the open chunk
          ne += __popc(ne_mask & live);
          break;
        }
        // close the open chunk before tile base + sub + j, which starts the next one
        ++n;
        if (lane == 0 && n < P.nchunks) P.chunk_t[n] = base + sub + j;
        start = base + sub + j;
        start_listed = off[sub + j];
        ne = 0;
        from = j;
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (n + 1 <= P.nchunks) {
      P.chunk_t[n + 1] = nt;
      *P.nchunks_dev = n + 1;
    } else {  // defensive: the fixed partition, which always fits the arrays and the buffers
      for (int c = 0; c <= P.nchunks; ++c) P.chunk_t[c] = min(nt, c * P.chunk_vt);
      *P.nchunks_dev = P.nchunks;
    }
  }
}

__device__ __forceinline__ int chunk_containing(const int* chunk_t, int n, int t) {
  int lo = 0, hi = n;  // chunk_t[lo] <= t < chunk_t[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (chunk_t[mid] <= t) lo = mid;
    else hi = mid;
  }
  return lo;
}

// The whole plan. Phases (each spread over the grid; a grid barrier after each from phase 1 on):
//  0  zero the counters (the backward kernel's too) and the fp32 accumulator of dbias; the row
//     scales (the fp32 accumulator of dE is zeroed a tenth per phase)
//  1  tile flags (run with phase 0, whose results they do not read)
//  2  per vocabulary tile: ranks of its listed tiles and their count; per row block: its listed tiles
//     and kept halves; the kept halves in all; per vocabulary tile: rows whose target half is skipped,
//     and their dbias terms
//  3  scans: offsets_t, offsets_b, off_hb, oh_off (four blocks)
//  4  entries_t; row lists (entries_b, hp_b, pos_b); the rows whose target half is skipped, grouped
//     by vocabulary tile; the vocabulary chunks (one block)
//  5  row ranges per chunk; the chunk of every vocabulary tile
//  6  quad counts per vocabulary tile
//  7  scan of the quad counts (pstart_t)
//  8  quads; chunk work lists and queue group sizes
//  9  scan of the group sizes (grp_start); the skipped count: by the last block to finish phase 8
__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(const __grid_constant__ PlanArgs A) {
  const BwdPlan& P = A.P;
  const int nb = P.nb, nt = P.nt;
  const int64_t tiles = static_cast<int64_t>(nb) * nt;
  const int64_t gthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int gwarps = static_cast<int>(gthreads >> 5), gwarp = static_cast<int>(gtid >> 5), lane = threadIdx.x & 31;
  const PlanCtl ctl{A.bar, A.err, A.timeout_ns};
  int round = 0;

  // 0
  if (gtid < 2) P.kept_total[gtid] = 0;  // kept_total and n_empty
  for (int64_t i = gtid; i < A.sync_ints; i += gthreads) A.sync[i] = 0;
  for (int64_t i = gtid; i < nb; i += gthreads) {
    P.cnt_b[i] = 0;
    P.cnt_hb[i] = 0;
  }
  for (int64_t i = gtid; i < kZeroHalfBytes / 16; i += gthreads)
    reinterpret_cast<float4*>(A.zero_half)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t i = gtid; i < nt; i += gthreads) {
    P.oh_cnt[i] = 0;
    P.oh_cur[i] = 0;
  }
  // dE_acc is first read by the tensor-core kernel, so its zeroing (bandwidth-bound) is spread over
  // the phases, beside their latency-bound work: one tenth at the start of each phase.
  const int64_t n4 = A.N * A.D / 4;  // D is a multiple of 8
  auto zero_part = [&](int k) {  // k = 0 .. 9
    float4* z = reinterpret_cast<float4*>(A.dE_acc);
    const int64_t lo = n4 * k / 10, hi = n4 * (k + 1) / 10;
    for (int64_t i = lo + gtid; i < hi; i += gthreads) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  };
  zero_part(0);
  if (A.dbias_acc != nullptr)  // receives atomics in phase 2
    for (int64_t i = gtid; i < A.V; i += gthreads) A.dbias_acc[i] = 0.f;
  for (int64_t r = gtid; r < A.N; r += gthreads) {
    float s;
    if (A.reduction == 1) {
      const long long c = *A.count;
      s = A.grad_out[0] / static_cast<float>(c > 0 ? c : 1);
    } else if (A.reduction == 2) {
      s = A.grad_out[0];
    } else {
      s = A.grad_out[r];
    }
    A.scale[r] = A.targets[r] != A.ignore_index ? s : 0.f;
  }
  // 1 (no barrier before it: the flags read none of the above)
  zero_part(1);
  {
    const int runs = (nt + kFlagTiles - 1) / kFlagTiles;
    const int64_t units = static_cast<int64_t>(nb) * runs;
    const int group = threadIdx.x / kBwdBM;
    for (int64_t u0 = static_cast<int64_t>(blockIdx.x) * kFlagGroups; u0 < units;
         u0 += static_cast<int64_t>(gridDim.x) * kFlagGroups) {
      const int64_t u = u0 + group;
      if (u < units) tile_flags_unit(A, group, static_cast<int>(u / runs), static_cast<int>(u % runs) * kFlagTiles);
    }
  }
  if (A.inject_stall && blockIdx.x == 0) return;  // test hook: the other blocks' barrier wait runs out
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 2
  for (int t = gwarp; t < nt; t += gwarps) {
    int listed = 0, halves = 0;
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int b = b0 + lane;
      const int f = b < nb ? P.flags[static_cast<int64_t>(b) * nt + t] : 0;
      const bool on = flag_state(f) == kFlagListed;
      const unsigned m = __ballot_sync(0xffffffffu, on);
      if (on) {
        const int nh = __popc(flag_halves(f));
        P.rank[static_cast<int64_t>(b) * nt + t] = listed + __popc(m & ((1u << lane) - 1u));
        atomicAdd(P.cnt_b + b, 1);
        atomicAdd(P.cnt_hb + b, nh);
        halves += nh;
      }
      listed += __popc(m);
    }
    halves = __reduce_add_sync(0xffffffffu, halves);
    if (lane == 0) {
      P.cnt_t[t] = listed;
      P.cnt_ht[t] = halves;
      atomicAdd(P.kept_total, halves);
    }
  }
  for (int64_t r = gtid; r < A.N; r += gthreads) {
    const int64_t tr = A.targets[r] - A.vs;  // only targets inside this shard have an onehot term here
    if (!valid_target(tr, A.V, A.ignore_index - A.vs)) continue;
    const int t = static_cast<int>(tr / kBwdBN);
    if (!target_half_skipped(P.flags[(r / kBwdBM) * nt + t], tr)) continue;
    atomicAdd(P.oh_cnt + t, 1);
    if (A.dbias_acc != nullptr) atomicAdd(A.dbias_acc + tr, -A.onehot_coef * A.scale[r]);
  }
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 3
  if (blockIdx.x == 0) block_scan(P.cnt_t, nt, P.offsets_t);
  if (blockIdx.x == 1 % gridDim.x) block_scan(P.cnt_b, nb, P.offsets_b);
  if (blockIdx.x == 2 % gridDim.x) block_scan(P.oh_cnt, nt, P.oh_off);
  if (blockIdx.x == 3 % gridDim.x) block_scan(P.cnt_hb, nb, P.off_hb);
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 4
  for (int64_t i = gtid; i < tiles; i += gthreads) {
    const int f = P.flags[i];
    if (flag_state(f) != kFlagListed) continue;
    const int b = static_cast<int>(i / nt), t = static_cast<int>(i % nt);
    P.entries_t[P.offsets_t[t] + P.rank[i]] = make_int2(b * 16 + f, t);
  }
  if (gtid == 0) P.hp_b[P.offsets_b[nb]] = P.off_hb[nb];  // one past the last entry
  for (int b = blockIdx.x; b < nb; b += gridDim.x) row_list_block(A, b);
  for (int64_t r = gtid; r < A.N; r += gthreads) {
    const int64_t tr = A.targets[r] - A.vs;
    if (!valid_target(tr, A.V, A.ignore_index - A.vs)) continue;
    const int t = static_cast<int>(tr / kBwdBN);
    if (!target_half_skipped(P.flags[(r / kBwdBM) * nt + t], tr)) continue;
    P.oh_rows[P.oh_off[t] + atomicAdd(P.oh_cur + t, 1)] = static_cast<int>(r);
  }
  if (blockIdx.x == gridDim.x - 1) chunk_partition(A);
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);
  const int nchunks = *reinterpret_cast<volatile int*>(P.nchunks_dev);

  // 5
  for (int64_t cb = gtid; cb < static_cast<int64_t>(nb) * nchunks; cb += gthreads) {
    const int c = static_cast<int>(cb / nb), b = static_cast<int>(cb % nb);
    const int lo = lower_bound_t(P.entries_b, P.offsets_b[b], P.offsets_b[b + 1], P.chunk_t[c]);
    const int hi = lower_bound_t(P.entries_b, lo, P.offsets_b[b + 1], P.chunk_t[c + 1]);
    P.rb_range[cb] = make_int2(lo, hi);
  }
  for (int64_t t = gtid; t < nt; t += gthreads)
    P.chunk_of[t] = chunk_containing(P.chunk_t, nchunks, static_cast<int>(t));
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 6
  for (int t = gwarp; t < nt; t += gwarps) quad_list_warp(A, t, lane, 0);
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 7
  if (blockIdx.x == 0) block_scan(P.cnt_t, nt, P.pstart_t);
  if (!grid_barrier(ctl, ++round)) return;
  zero_part(round + 1);

  // 8
  for (int t = gwarp; t < nt; t += gwarps) quad_list_warp(A, t, lane, 1);
  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) chunk_items_block(A, c, nchunks);
  zero_part(9);

  // 9, by the last block to finish phase 8 (counted on the barrier counter; no grid barrier)
  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(ctl.bar, 1) == (round + 1) * static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();  // the other blocks' grp_size entries are visible
  block_scan(P.grp_size, 2 * nchunks, P.grp_start);
  if (threadIdx.x == 0) *A.filtered_tiles = static_cast<int64_t>(nb) * A.T - static_cast<int64_t>(*P.kept_total);
}

// The element-wise steps of the backward after the tensor-core kernel, in two launches:
//  empty_tiles_kernel: dC rows of the vocabulary tiles no row block lists. Every logit of such a
//   tile is skipped, so only the target part of the logit gradient reaches them (Loss functions
//   explainer, "How it works" items 2 and 3): -scale_r (1 - ls) E_r for each row r whose target v
//   lies there, and the smoothing term -(ls / V) wsum shared by every row of dC. The target rows
//   (oh_rows[oh_off[t] .. oh_off[t + 1]]: for an empty tile every non-ignored row targeting it is
//   listed there) are added in list order, so the result is deterministic. The constant rows go out
//   as bulk copies from shared memory.
//  bwd_finalize_kernel (256 threads; 64 threads x 8 columns cover 512 columns of a row, 16-byte
//  loads and stores, four rows at a time):
//   A. dE, 32 rows x 512 columns per unit: dE_acc plus, for a row whose target tile was skipped
//      ("onehot only"), its onehot term -scale_r (1 - ls) C_{t_r}, and with label smoothing the
//      rank-one term -scale_r (ls / V) sum_v C_v; written as bf16 (or in place in fp32).
//   C. dbias, 2048 entries per unit: dbias_acc (the G column sums and the onehot terms) plus the
//      smoothing constant, written as bf16 (or in place in fp32).
constexpr int kFinCols = 512;
constexpr int kFillThreads = 128;
constexpr int64_t kFillImageBytes = 64 << 10;  // shared-memory image of the constant rows
constexpr int kFinRowsA = 32;
constexpr int kFinBias = 2048;

__device__ __forceinline__ void store8(void* base, int bf16, int64_t idx, const float (&acc)[8]) {
  if (bf16) {
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx) = o;
  } else {
    float4* out = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
    out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const __nv_bfloat16* src, float a) {
  const uint4 q = ld_global_nc_v4(src);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 h;
    *reinterpret_cast<uint32_t*>(&h) = w[k];
    acc[2 * k] = fmaf(a, __low2float(h), acc[2 * k]);
    acc[2 * k + 1] = fmaf(a, __high2float(h), acc[2 * k + 1]);
  }
}

// One warp per empty vocabulary tile t. Its rows of dC are the constant row c = -(ls / V) wsum
// (zeros without label smoothing) except the rows of tokens some row r targets. The block keeps
// image_rows copies of c (columns [d0, d0 + win) of it when a row is wider than the image) in
// shared memory, and lane 0 writes every run of constant rows of t with bulk copies from that
// image, so the copy engine streams the bytes out while the warp computes the target rows:
// c + sum of a_r E_r over the list entries of that token, in list order, 16-byte loads and stores.
__global__ void __launch_bounds__(kFillThreads) empty_tiles_kernel(const __grid_constant__ BwdFinalize F,
                                                                   int64_t win, int image_rows) {
  extern __shared__ __align__(128) uint8_t img[];
  wait_for_previous_grid();  // the plan's empty tiles; dC rows the tensor-core kernel does not write
  const int64_t D = F.D;
  const int es = F.dc_bf16 ? 2 : 4;
  const int64_t rowbytes = D * es;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kFillThreads / 32;
  const int n_empty = *F.n_empty;
  const uint32_t img_u32 = smem_u32(img);
  char* dC = static_cast<char*>(F.dC);
  for (int64_t d0 = 0; d0 < D; d0 += win) {
    const int64_t w = D - d0 < win ? D - d0 : win;
    __syncthreads();  // every bulk copy of the previous window has read the image
    for (int64_t i = threadIdx.x; i < image_rows * w; i += kFillThreads) {
      const float c = F.wsum != nullptr ? -F.ls_v * F.wsum[d0 + i % w] : 0.f;
      if (F.dc_bf16) reinterpret_cast<__nv_bfloat16*>(img)[i] = __float2bfloat16_rn(c);
      else reinterpret_cast<float*>(img)[i] = c;
    }
    fence_proxy_async_smem();  // the image, written by threads, is read by the copy engine
    __syncthreads();
    for (int u = warp * gridDim.x + blockIdx.x; u < n_empty; u += gridDim.x * kWarps) {  // blocks first
      const int t = F.empty_list[u];
      const int64_t v0 = static_cast<int64_t>(t) * kBwdBN;
      const int rows = F.V - v0 < kBwdBN ? static_cast<int>(F.V - v0) : kBwdBN;
      const int i0 = F.oh_off[t], i1 = F.oh_off[t + 1];
      // rows of t that some row targets: bit k % 32 of mk, k / 32 = 0..3
      uint32_t m0 = 0u, m1 = 0u, m2 = 0u, m3 = 0u;
      for (int c0 = i0; c0 < i1; c0 += 32) {
        const int col = c0 + lane < i1 ? static_cast<int>(F.targets[F.oh_rows[c0 + lane]] - F.vs - v0) : -1;
        const uint32_t bit = col >= 0 ? 1u << (col & 31) : 0u;
        m0 |= __reduce_or_sync(0xffffffffu, (col >> 5) == 0 ? bit : 0u);
        m1 |= __reduce_or_sync(0xffffffffu, (col >> 5) == 1 ? bit : 0u);
        m2 |= __reduce_or_sync(0xffffffffu, (col >> 5) == 2 ? bit : 0u);
        m3 |= __reduce_or_sync(0xffffffffu, (col >> 5) == 3 ? bit : 0u);
      }
      const uint64_t lo = (static_cast<uint64_t>(m1) << 32) | m0, hi = (static_cast<uint64_t>(m3) << 32) | m2;
      auto target_row = [lo, hi](int row) { return (((row < 64 ? lo : hi) >> (row & 63)) & 1u) != 0; };
      if (lane == 0) {
        for (int row = 0; row < rows;) {
          if (target_row(row)) {
            ++row;
            continue;
          }
          int end = row + 1;
          while (end < rows && end - row < image_rows && !target_row(end)) ++end;
          char* dst = dC + ((v0 + row) * D + d0) * es;
          bulk_store(dst, img_u32, static_cast<uint32_t>(w == D ? (end - row) * rowbytes : w * es));
          row = end;
        }
        bulk_commit_group();
      }
      if (d0 != 0) continue;  // target rows are written whole, with the first window
      for (int k = 0; k < 2; ++k) {
        for (uint64_t bits = k == 0 ? lo : hi; bits != 0; bits &= bits - 1) {
          const int row = k * 64 + __ffsll(static_cast<long long>(bits)) - 1;
          for (int64_t db = 0; db < D; db += 256) {
            const int64_t d = db + lane * 8;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = F.wsum != nullptr && d < D ? -F.ls_v * F.wsum[d + j] : 0.f;
            for (int c0 = i0; c0 < i1; c0 += 32) {
              int r = 0, col = -1;
              float a = 0.f;
              if (c0 + lane < i1) {
                r = F.oh_rows[c0 + lane];
                col = static_cast<int>(F.targets[r] - F.vs - v0);
                a = -F.scale[r] * F.onehot_coef;
              }
              for (unsigned m = __ballot_sync(0xffffffffu, col == row); m != 0; m &= m - 1) {  // list order
                const int q = __ffs(m) - 1;
                const int rq = __shfl_sync(0xffffffffu, r, q);
                const float aq = __shfl_sync(0xffffffffu, a, q);
                if (d < D) add_bf16x8(acc, F.E + static_cast<int64_t>(rq) * D + d, aq);
              }
            }
            if (d < D) store8(F.dC, F.dc_bf16, (v0 + row) * D + d, acc);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group_read0();  // before the image is rewritten
  }
  if (lane == 0) bulk_wait_group0();  // the bulk copies are complete before the block exits
}

__global__ void __launch_bounds__(256, 2) bwd_finalize_kernel(const __grid_constant__ BwdFinalize F) {
  wait_for_previous_grid();  // dE_acc and dbias_acc of the tensor-core kernel, complete
  const int64_t D = F.D;
  const int col_chunks = static_cast<int>((D + kFinCols - 1) / kFinCols);
  const int64_t units_a = (F.N + kFinRowsA - 1) / kFinRowsA * col_chunks;
  const int64_t units_c = F.dbias_acc != nullptr ? (F.V + kFinBias - 1) / kFinBias : 0;
  const int row0 = threadIdx.x >> 6;
  const int col_thread = (threadIdx.x & 63) * 8;
  for (int64_t u = blockIdx.x; u < units_a + units_c; u += gridDim.x) {
    if (u < units_a) {  // A: dE rows
      const int64_t d = (u % col_chunks) * kFinCols + col_thread;
      if (d >= D) continue;
      float cs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (F.csum != nullptr) {
        const float4 c0 = *reinterpret_cast<const float4*>(F.csum + d);
        const float4 c1 = *reinterpret_cast<const float4*>(F.csum + d + 4);
        cs[0] = c0.x; cs[1] = c0.y; cs[2] = c0.z; cs[3] = c0.w;
        cs[4] = c1.x; cs[5] = c1.y; cs[6] = c1.z; cs[7] = c1.w;
      }
      const int64_t rbase = (u / col_chunks) * kFinRowsA;
      for (int i = row0; i < kFinRowsA; i += 4) {
        const int64_t r = rbase + i;
        if (r >= F.N) break;
        const float* src = F.dE_acc + r * D + d;
        const float4 a0 = *reinterpret_cast<const float4*>(src);
        const float4 a1 = *reinterpret_cast<const float4*>(src + 4);
        float acc[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float sc = F.scale[r];
        if (F.csum != nullptr) {
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = fmaf(-F.ls_v * sc, cs[k], acc[k]);
        }
        const int64_t tl = F.targets[r] - F.vs;
        if (tl >= 0 && tl < F.V && F.targets[r] != F.ignore_index &&
            target_half_skipped(F.flags[(r / kBwdBM) * F.nt + tl / kBwdBN], tl))
          add_bf16x8(acc, F.C + tl * D + d, -F.onehot_coef * sc);
        store8(F.dE_out != nullptr ? F.dE_out : static_cast<void*>(F.dE_acc), F.dE_out != nullptr, r * D + d, acc);
      }
    } else {  // C: dbias
      const int64_t v0 = (u - units_a) * kFinBias;
      const float add = F.wsum != nullptr ? -F.ls_v * F.wsum[D] : 0.f;
      for (int64_t v = v0 + threadIdx.x; v < v0 + kFinBias && v < F.V; v += blockDim.x) {
        const float x = F.dbias_acc[v] + add;
        if (F.dbias_out != nullptr) static_cast<__nv_bfloat16*>(F.dbias_out)[v] = __float2bfloat16_rn(x);
        else F.dbias_acc[v] = x;
      }
    }
  }
}

// out[i] = 1 when backward tile i (row block i / nt, vocabulary tile i % nt) was skipped, 0 when kept.
__global__ void skip_map_kernel(const uint8_t* __restrict__ flags, int nt, int64_t T, int64_t n,
                                uint8_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / T, j = i % T;
    const int f = flags[b * nt + j / 2];
    out[i] = flag_state(f) == kFlagListed && ((flag_halves(f) >> (j & 1)) & 1) ? 0 : 1;
  }
}

}  // namespace

cudaError_t launch_empty_tiles(const BwdFinalize& F, int num_sms, bool after_kernel, cudaStream_t s) {
  if (F.N == 0) return cudaSuccess;
  const int64_t es = F.dc_bf16 ? 2 : 4, rowbytes = F.D * es;
  // whole rows when one fits the image (up to 128 of them); otherwise windows of whole 16-byte pieces
  const int64_t win = rowbytes <= kFillImageBytes ? F.D : kFillImageBytes / es / 8 * 8;
  const int image_rows =
      static_cast<int>(rowbytes <= kFillImageBytes ? std::min<int64_t>(kBwdBN, kFillImageBytes / rowbytes) : 1);
  const size_t smem = static_cast<size_t>(image_rows * win * es);
  cudaError_t e = cudaFuncSetAttribute(empty_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFillImageBytes));
  if (e != cudaSuccess) return e;
  if (after_kernel) {
    e = launch_after_previous(empty_tiles_kernel, dim3(num_sms * 2), dim3(kFillThreads), smem, s, F, win, image_rows);
    if (e != cudaSuccess) return e;
  } else {
    empty_tiles_kernel<<<num_sms * 2, kFillThreads, smem, s>>>(F, win, image_rows);
  }
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_finalize(const BwdFinalize& F, int num_sms, cudaStream_t s) {
  if (F.N == 0) return cudaSuccess;
  const cudaError_t e = launch_after_previous(bwd_finalize_kernel, dim3(num_sms * 4), dim3(256), 0, s, F);
  if (e != cudaSuccess) return e;
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_skip_map(const uint8_t* flags, int nb, int nt, int64_t T, uint8_t* out, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(nb) * T;
  if (n == 0) return cudaSuccess;
  skip_map_kernel<<<static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096)), 256, 0, s>>>(flags, nt, T, n, out);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_plan(const PlanArgs& A, int num_sms, cudaStream_t s) {
  if (A.P.nb == 0) return cudaSuccess;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, plan_kernel, kPlanThreads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  void* args[] = {const_cast<PlanArgs*>(&A)};
  e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(plan_kernel), dim3(num_sms), dim3(kPlanThreads), args,
                                  0, s);
  note_launches(1);
  return e;
}

}  // namespace cce

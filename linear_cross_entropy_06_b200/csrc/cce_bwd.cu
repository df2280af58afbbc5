// Backward: one persistent launch that recomputes the kept logit tiles, forms their bf16 gradient
// tiles, and runs the dC and dE MMAs on them, chunk by chunk of the vocabulary.
//
// mlx-cross-entropy README, "How it works" items 2 and 3 (recompute from the saved LSE, skip tiles
// whose softmax is below 2^-12, accumulate the gradients without [batch, tiles, D] buffers); Loss
// functions explainer, "How it works" item 2 (G = p - y, dE = G C, dC = G^T E); Cut Your Losses
// abstract (logits are recomputed blockwise and never stored).
//
// Work items, per vocabulary chunk c (its gradient tiles live in scratch buffer c mod kGradBuffers):
//   quad   up to four consecutive kept 64-column halves of row block b in the chunk (from one or
//          several of its listed tiles): S = E_b [C_h ...]^T (+ bias) over those halves (tcgen05
//          M=128 N=64 x halves K=D), then
//          G = scale_r (1 + 2 zl LSE_r) exp(S - LSE_r) - scale_r (1 - ls) [v = t_r] in fp32, rounded
//          to bf16 into a 128B-swizzled shared region (two halves at a time), one 16 KB bulk store
//          per half into its tile's slot of the scratch buffer; with a dbias output, the column sums
//          of the fp32 G are added into it.
//   dE     (row block b, 256-column slice s of D): sum over the kept halves h of the chunk's listed
//          tiles t of G_bth C_th[:, s] in TMEM, then one fp32 TMA reduce-add into dE_acc
//          (split-reduce over chunks).
//   dC     (vocabulary tile t, slice s): sum over the listed b of G_bt^T E_b[:, s] in TMEM (A = the
//          same G tile read MN-major, a skipped half read as zeros), plus the onehot terms of rows
//          whose target half in t was skipped and the label-smoothing term, written once by TMA
//          store: every listed tile of t lies in t's chunk, so dC needs no reduction.
//
// Scheduling: a global queue holds the items in the order quads(0), quads(1), dE/dC(0), quads(2),
// dE/dC(1), ..., quads(n-1), dE/dC(n-2), dE/dC(n-1): the dE/dC items of a chunk come one group of
// quads after the chunk's own quads, so their gradient halves are normally stored by the time they
// are claimed. CTAs claim items one at a time with an atomic counter, so a claimed item always
// belongs to a running CTA. Inside a chunk the quads are ordered by vocabulary tile and the dE and
// dC items by slice of D, so that the items running at the same time read the same C tiles and
// the same columns of C and E from L2. Dependencies point only to earlier items:
//   a dE item waits until every kept half of its row block in the chunk is stored, a dC item
//   until every kept half of its vocabulary tile is, and a quad of chunk c waits, before it
//   stores, until every dE/dC item of chunk c - kGradBuffers (the buffer's previous user) has
//   read it.
// Every such wait is bounded. Because items are claimed in order and the smallest unfinished item
// has no unfinished dependency, the queue always drains; and with no boundary between chunks the
// machine has a single tail per backward instead of one per chunk and kernel.
//
// Design (B200): one CTA per SM, 7 warps, 224 KB of shared memory.
//   warp 0      producer: per stage (at most 48 KB, 4 deep) either the E_b K-block of 64 and one
//               64 x 64 C box per half of the quad, or one K-half of a gradient tile (16 KB bulk
//               copy, or zeros for a skipped half) and the 64 x 256 operand slice (dE, dC).
//   warp 1      TMEM owner (two 256-column fp32 buffers); one lane issues tcgen05.mma M=128 N=256.
//   warps 2..5  write-out: G formation and bulk stores (quad), or TMEM -> swizzled staging -> TMA
//               store / reduce-add (dC / dE), while the MMA fills the other TMEM buffer.
//   warp 6      scheduler: claims and decodes items into an 8-deep shared ring, at most LOOKAHEAD
//               items ahead of the producer.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kBwdBM;
constexpr int BN = kBwdBN;
constexpr int BK = 64;
constexpr int SLICE = kGemmSlice;
constexpr int STAGES = 4;
constexpr int PART = 16384;              // 128 x 64 bf16: one K-block of 128 rows, or half a G tile
constexpr int X_BOX = 8192;              // 64 x 64 bf16
constexpr int STAGE_BYTES = 3 * PART;    // 48 KB
constexpr int TILE_BYTES = kGradTileBytes;
constexpr int REGION_BYTES = TILE_BYTES;  // two G halves (quad) or 4 x 8 KB staging (dE / dC)
constexpr int STG_WARP = 8192;
constexpr int RING = 8;
constexpr int NUM_THREADS = 224;
constexpr int TMEM_COLS = 512;

enum Kind : int { kQuad = 0, kDE = 1, kDC = 2, kEnd = 3 };

// A decoded work item, written by the scheduler into the shared ring (16-byte aligned: it is
// copied as int4).
struct alignas(16) WorkItem {
  int kind;
  int chunk;
  int key;         // quad, dE: row block b; dC: vocabulary tile t
  int s;           // dE, dC: slice of D; quad: its halves (1 to 4)
  int begin, end;  // dE, dC: list entries; quad: halves 0 and 1, each 2 t + h (-1 when absent)
  int slot0;       // quad: slot of half 0's tile in the chunk's buffer; dE, dC: the chunk's first slot
  int slot1;       // quad: slot of half 1's tile; dE: stages (kept halves of the entries)
  int dep_idx;     // counter this item waits on (-1: none): before its loads (dE, dC) or stores (quad)
  int dep_val;     // value the counter must reach
  int oh_begin;    // dC: rows whose target half in this vocabulary tile was skipped,
  int oh_end;      //     oh_rows[oh_begin:oh_end]; quad: halves 2 and 3
  int pad[4];      // quad: slots of halves 2 and 3
};
static_assert(sizeof(WorkItem) == 64, "ring entries are 64 bytes");

enum Bar : int {
  kFull = 0,
  kEmpty = kFull + STAGES,
  kAccFull = kEmpty + STAGES,
  kAccEmpty = kAccFull + 2,
  kDrain = kAccEmpty + 2,
  kRegion = kDrain + 1,  // the shared write-out region is free (one arrival per write-out warp)
  kGReady = kRegion + 1, // all 128 rows of a G tile are in the region
  kItemFull = kGReady + 1,
  kItemEmpty = kItemFull + RING,
  kItemTaken = kItemEmpty + RING,  // the producer has started the entry's item
  kNumBars = kItemTaken + RING
};

// The scheduler claims item k only once the producer has started item k - LOOKAHEAD: enough to
// hide the claim and decode latency, few enough that no CTA hoards claimed items at the end.
constexpr uint32_t LOOKAHEAD = 2;

constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + REGION_BYTES + kNumBars * 8 + RING * 64 + 16;
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB opt-in shared memory of an SM");

// S = E_b [C_h ...]^T over the quad's nh halves: N = 64 nh
__device__ __forceinline__ uint32_t idesc_quad(int nh) {
  constexpr uint32_t d1 = idesc_bf16(BM, 1 * kSubTile, false, false), d2 = idesc_bf16(BM, 2 * kSubTile, false, false),
                     d3 = idesc_bf16(BM, 3 * kSubTile, false, false), d4 = idesc_bf16(BM, 4 * kSubTile, false, false);
  return nh <= 1 ? d1 : nh == 2 ? d2 : nh == 3 ? d3 : d4;
}
constexpr uint32_t IDESC_DC = idesc_bf16(BN, SLICE, true, true);    // M = vocabulary (G^T, MN-major)
constexpr uint32_t IDESC_DE = idesc_bf16(BM, SLICE, false, true);   // M = rows (G, K-major)

// Consumers of one ring entry: producer lane, MMA lane, one lane per write-out warp.
constexpr uint32_t kRingConsumers = 1 + 1 + 4;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map), "r"(src),
               "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void read_item(const WorkItem* ring, int idx, WorkItem& it) {
  const int4* src = reinterpret_cast<const int4*>(ring + idx);
  int4* dst = reinterpret_cast<int4*>(&it);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = src[i];
}

// Half j (0..3) of a quad item: 2 t + h, and its tile's slot in the chunk's buffer.
__device__ __forceinline__ int quad_half(const WorkItem& it, int j) {
  return j == 0 ? it.begin : j == 1 ? it.end : j == 2 ? it.oh_begin : it.oh_end;
}
__device__ __forceinline__ int quad_slot(const WorkItem& it, int j) {
  return j == 0 ? it.slot0 : j == 1 ? it.slot1 : j == 2 ? it.pad[0] : it.pad[1];
}

// Queue group g -> (chunk, whether it holds the chunk's quads). The groups are quads(0), then
// quads(c), dE/dC(c - 1) for c = 1 .. n-1, then dE/dC(n - 1).
__device__ __forceinline__ int2 group_of(int g, int nchunks) {
  if (g == 0) return make_int2(0, 1);
  if (g == 2 * nchunks - 1) return make_int2(nchunks - 1, 0);
  const int pos = g - 1, c = pos / 2 + 1;
  return (pos & 1) == 0 ? make_int2(c, 1) : make_int2(c - 1, 0);
}

// Item w of the queue, in group g that starts at item g_begin -> its decoded form (the scheduler's
// only global reads).
__device__ __forceinline__ void decode_item(int w, int g, int g_begin, int nchunks, const BwdArgs& A,
                                            WorkItem& it) {
  const int2 gc = group_of(g, nchunks);
  const int c = gc.x, local = w - g_begin;
  const int t_begin = A.chunk_t[c];
  it.chunk = c;
  it.oh_begin = it.oh_end = 0;
  if (gc.y) {
    const int64_t pi = static_cast<int64_t>(A.pstart_t[t_begin]) + local;
    const int4 h = A.quad_h[pi];
    const int4 sl = A.quad_s[pi];
    it.kind = kQuad;
    it.key = A.quad_b[pi];
    it.begin = h.x;  // the halves, 2 t + h
    it.end = h.y;
    it.oh_begin = h.z;
    it.oh_end = h.w;
    it.s = (h.x >= 0 ? 1 : 0) + (h.y >= 0 ? 1 : 0) + (h.z >= 0 ? 1 : 0) + (h.w >= 0 ? 1 : 0);
    it.slot0 = sl.x;  // their tiles' slots
    it.slot1 = sl.y;
    it.pad[0] = sl.z;
    it.pad[1] = sl.w;
    if (c >= kGradBuffers) {  // the buffer's previous chunk must have been read by its dE / dC items
      const int prev = c - kGradBuffers;
      it.dep_idx = A.ctr_b_done + prev;
      it.dep_val = (A.nde[prev] + A.ndc[prev]) * A.S;
    } else {
      it.dep_idx = -1;
      it.dep_val = 0;
    }
  } else {
    // Only row blocks and vocabulary tiles with a listed tile in the chunk have items; the dC rows of
    // vocabulary tiles no row block lists are written by the streaming fill outside this kernel.
    const int S = A.S;
    const int nde = A.nde[c];
    it.slot0 = A.offsets_t[t_begin];
    it.slot1 = 0;
    if (local < nde * S) {  // slice-major: concurrent dE items read the same columns of C
      it.kind = kDE;
      it.key = A.de_list[static_cast<int64_t>(c) * A.nb + local % nde];
      // serpentine over chunks: a chunk starts on the slices of dE the previous one touched last
      it.s = (c & 1) ? S - 1 - local / nde : local / nde;
      const int2 r = A.rb_range[static_cast<int64_t>(c) * A.nb + it.key];
      it.begin = r.x;
      it.end = r.y;
      it.slot1 = A.hp_b[r.y] - A.hp_b[r.x];
      it.dep_idx = A.ctr_g_b + c * A.nb + it.key;
      it.dep_val = it.slot1;  // every kept half of the row block in the chunk is stored
    } else {  // slice-major too: concurrent dC items read the same columns of E
      const int v = local - nde * S;
      const int ndc = A.ndc[c];
      it.kind = kDC;
      it.key = A.vt_order[t_begin + v % ndc];
      it.s = v / ndc;
      it.begin = A.offsets_t[it.key];
      it.end = A.offsets_t[it.key + 1];
      it.dep_idx = A.ctr_g_t + it.key;
      it.dep_val = A.cnt_ht[it.key];  // every kept half of the vocabulary tile is stored
      it.oh_begin = A.oh_off[it.key];
      it.oh_end = A.oh_off[it.key + 1];
    }
    // test hook: the dE items of the first chunk wait for one gradient half more than the quads
    // store, so their bounded wait runs out
    if (A.inject_stall && c == 0 && it.kind == kDE) ++it.dep_val;
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmE128, const __grid_constant__ CUtensorMap tmC128,
               const __grid_constant__ CUtensorMap tmE64, const __grid_constant__ CUtensorMap tmC64,
               const __grid_constant__ CUtensorMap tmdC, const __grid_constant__ CUtensorMap tmdE,
               const __grid_constant__ BwdArgs A) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* region = base + STAGES * STAGE_BYTES;
  WorkItem* ring = reinterpret_cast<WorkItem*>(region + REGION_BYTES);  // 1024-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + RING);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int u = 0; u < STAGES; ++u) {
      mbar_init(bar(kFull + u), 1);
      mbar_init(bar(kEmpty + u), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(kAccFull + a), 1);
      mbar_init(bar(kAccEmpty + a), 128);
    }
    mbar_init(bar(kDrain), 1);
    mbar_init(bar(kRegion), 4);
    mbar_init(bar(kGReady), 128);
    for (int i = 0; i < RING; ++i) {
      mbar_init(bar(kItemFull + i), 1);
      mbar_init(bar(kItemEmpty + i), kRingConsumers);
      mbar_init(bar(kItemTaken + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  wait_for_previous_grid();  // the plan (and the zeroed counters) of the planning launch
  const WaitCtl wc{abort_flag, A.err, A.timeout_ns};
  const int num_kb = (A.D + BK - 1) / BK;
  auto buffer = [&](int chunk) { return A.gscratch + static_cast<size_t>(chunk % kGradBuffers) * A.buf_bytes; };

  if (warp == 6) {
    // ---------------- scheduler ----------------
    if (lane == 0) {
      // A planning launch that gave up (its bounded barrier wait ran out; the error word is set)
      // leaves the work lists unfinished: then no item is handed out at all.
      const bool planned = ld_relaxed(A.err) == 0;
      const int nchunks = planned ? *A.nchunks : 0;
      const int total = planned ? A.grp_start[2 * nchunks] : 0;
      int g = 0, g_begin = 0, g_end = A.grp_start[1];  // this CTA's claims only increase
      for (uint32_t k = 0;; ++k) {
        const int idx = static_cast<int>(k % RING);
        if (!mbar_wait(bar(kItemEmpty + idx), ((k / RING) & 1u) ^ 1u, wc)) break;
        if (k >= LOOKAHEAD) {
          const uint32_t j = k - LOOKAHEAD;
          if (!mbar_wait(bar(kItemTaken + j % RING), (j / RING) & 1u, wc)) break;
        }
        const int w = atomicAdd(A.qctr, 1);
        WorkItem it;
        if (w >= total) {
          it.kind = kEnd;
        } else {
          while (w >= g_end) {
            ++g;
            g_begin = g_end;
            g_end = A.grp_start[g + 1];
          }
          decode_item(w, g, g_begin, nchunks, A, it);
        }
        int4* dst = reinterpret_cast<int4*>(ring + idx);
        const int4* src = reinterpret_cast<const int4*>(&it);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = src[i];
        mbar_arrive(bar(kItemFull + idx));  // release: the entry is visible to the waiters
        if (it.kind == kEnd) break;
      }
    }
  } else if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES] = {0, 0, 0, 0};
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int idx = static_cast<int>(k % RING);
        if (!mbar_wait(bar(kItemFull + idx), (k / RING) & 1u, wc)) break;
        WorkItem it;
        read_item(ring, idx, it);
        mbar_arrive(bar(kItemEmpty + idx));
        mbar_arrive(bar(kItemTaken + idx));
        if (it.kind == kEnd) break;
        if (it.kind == kQuad) {
          if (it.s == 0) continue;  // no half: nothing to recompute
          const int rb = it.key * BM;
          const uint32_t stage_bytes = PART + static_cast<uint32_t>(it.s) * X_BOX;
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(bar(kEmpty + stage), phase ^ 1u, wc)) {
              ok = false;
              break;
            }
            const uint32_t dst = smem_u32(stages + stage * STAGE_BYTES);
            mbar_arrive_expect_tx(bar(kFull + stage), stage_bytes);
            tma_load_2d(dst, &tmE128, bar(kFull + stage), kb * BK, rb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // the quad's halves' C rows, in order
              if (j < it.s) {
                const int th = quad_half(it, j);
                const int vrow = (th >> 1) * BN + (th & 1) * kSubTile;
                tma_load_2d(dst + PART + j * X_BOX, &tmC128, bar(kFull + stage), kb * BK, vrow);
              }
            }
            ++issued[stage];
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          continue;
        }
        // dE / dC: every gradient tile this item reads must be stored
        if (it.begin < it.end && !wait_counter(A.counters + it.dep_idx, it.dep_val, wc)) break;
        const bool de = it.kind == kDE;
        const uint8_t* buf = buffer(it.chunk);
        const int x0 = it.s * SLICE;
        // (tile index of the other operand, slot in the chunk's buffer, kept halves of the tile)
        auto entry = [&](int i) {
          if (de) {
            const int2 en = A.entries_b[i];
            return make_int3(en.x, (en.y & kSlotMask) - it.slot0, en.y >> kSlotBits);
          }
          const int x = A.entries_t[i].x;
          return make_int3(x >> 4, i - it.slot0, flag_halves(x & 15));
        };
        const uint8_t* zero = static_cast<const uint8_t*>(A.zero_half);
        int3 os_next = it.begin < it.end ? entry(it.begin) : make_int3(0, 0, 0);
        for (int i = it.begin; i < it.end && ok; ++i) {
          const int3 os = os_next;
          if (i + 1 < it.end) os_next = entry(i + 1);
          const uint8_t* tile = buf + static_cast<size_t>(os.y) * TILE_BYTES;
          for (int h = 0; h < 2; ++h) {  // K-halves: 64 vocabulary columns (dE) or 64 rows (dC)
            if (de && !((os.z >> h) & 1)) continue;  // a skipped half adds nothing to dE
            if (!mbar_wait(bar(kEmpty + stage), phase ^ 1u, wc)) {
              ok = false;
              break;
            }
            const uint32_t dst = smem_u32(stages + stage * STAGE_BYTES);
            mbar_arrive_expect_tx(bar(kFull + stage), STAGE_BYTES);
            if (de) {  // G block h: rows 0..127, vocabulary 64h .. 64h + 63 (K-major A)
              bulk_load(dst, tile + h * PART, PART, bar(kFull + stage));
            } else {   // rows 64h .. 64h + 63 of both 64-column blocks (MN-major A = G^T); zeros for a
                       // skipped half
              bulk_load(dst, (os.z & 1) ? tile + h * (PART / 2) : zero, PART / 2, bar(kFull + stage));
              bulk_load(dst + PART / 2, (os.z & 2) ? tile + PART + h * (PART / 2) : zero, PART / 2,
                        bar(kFull + stage));
            }
            const int y = os.x * BM + 64 * h;  // K rows of the operand: C_t rows (dE), E_b rows (dC)
            if (A.slab3d) {
              tma_load_3d(dst + PART, de ? &tmC64 : &tmE64, bar(kFull + stage), 0, y, x0 / 64);
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c)
                tma_load_2d(dst + PART + c * X_BOX, de ? &tmC64 : &tmE64, bar(kFull + stage), x0 + 64 * c, y);
            }
            ++issued[stage];
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (*abort_flag) {
        for (int u = 0; u < STAGES; ++u)
          if (issued[u]) mbar_wait_drain(bar(kFull + u), (issued[u] - 1u) & 1u, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      bool ok = true, issued_any = false;
      for (uint32_t k = 0; ok; ++k) {
        const int idx = static_cast<int>(k % RING);
        if (!mbar_wait(bar(kItemFull + idx), (k / RING) & 1u, wc)) break;
        WorkItem it;
        read_item(ring, idx, it);
        mbar_arrive(bar(kItemEmpty + idx));
        if (it.kind == kEnd) break;
        const bool quad = it.kind == kQuad;
        if (quad ? it.s == 0 : it.begin == it.end) continue;  // no MMA for this item
        const int a = acc_iter & 1;
        if (!mbar_wait(bar(kAccEmpty + a), ((acc_iter >> 1) & 1u) ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(a * 2 * BN);
        const int nstage = quad ? num_kb : (it.kind == kDE ? it.slot1 : 2 * (it.end - it.begin));
        const uint32_t idesc = quad ? idesc_quad(it.s) : (it.kind == kDE ? IDESC_DE : IDESC_DC);
        for (int j = 0; j < nstage; ++j) {
          if (!mbar_wait(bar(kFull + stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t s0 = smem_u32(stages + stage * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 of the stage's 64 K values per MMA
            uint64_t adesc, bdesc;
            if (quad) {  // A = E_b K-block, B = the quad's halves' C rows (64 per half, rows of 128 bytes)
              adesc = sdesc_sw128(s0 + 32u * kk, 16, 1024);
              bdesc = sdesc_sw128(s0 + PART + 32u * kk, 16, 1024);
            } else {
              adesc = it.kind == kDE ? sdesc_sw128(s0 + 32u * kk, 16, 1024)
                                     : sdesc_sw128(s0 + 2048u * kk, PART / 2, 1024);
              bdesc = sdesc_sw128(s0 + PART + 2048u * kk, X_BOX, 1024);
            }
            tc_mma_bf16(d, adesc, bdesc, idesc, (j | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(bar(kEmpty + stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(bar(kAccFull + a));
        ++acc_iter;
      }
      if (*abort_flag && issued_any) {
        tc_commit(bar(kDrain));
        mbar_wait_drain(bar(kDrain), 0, 200000000ull);
      }
    }
  } else {
    // ---------------- write-out ----------------
    const int q = warp & 3;  // TMEM lane quarter of this warp (warps 2..5 -> 2, 3, 0, 1)
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    const uint32_t reg0 = smem_u32(region);
    const uint32_t stg = reg0 + static_cast<uint32_t>(q * STG_WARP);
    uint32_t acc_iter = 0, rphase = 0, gphase = 0;
    uint32_t img = 0;  // which of the two 4 KB staging images of this warp comes next
    bool region_shared = true;  // the last item used the whole region (a quad's G halves)
    bool ok = true;
    // Every lane waits (and acquires) itself; the vote makes the outcome warp-uniform, so the warp
    // stays converged for the .sync.aligned TMEM loads and takes one branch on failure.
    auto warp_wait = [&](uint32_t b, uint32_t parity) {
      const bool r = mbar_wait(b, parity, wc);
      return __all_sync(0xffffffffu, r ? 1 : 0) != 0;
    };
    // Every write-out warp's earlier bulk copies have read the region; then it may be rewritten.
    auto region_free = [&]() {
      if (lane == 0) {
        bulk_wait_group_read0();
        mbar_arrive(bar(kRegion));
      }
      const bool r = warp_wait(bar(kRegion), rphase & 1u);
      ++rphase;
      return r;
    };
    for (uint32_t k = 0; ok; ++k) {
      const int idx = static_cast<int>(k % RING);
      if (!warp_wait(bar(kItemFull + idx), (k / RING) & 1u)) break;
      WorkItem it;
      read_item(ring, idx, it);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kItemEmpty + idx));
      if (it.kind == kEnd) break;
      const int a = acc_iter & 1;

      if (it.kind == kQuad) {
        const int b = it.key;
        const int r = b * BM + row;
        const float lse_r = (r < A.N) ? A.lse[r] : 0.f;
        const float lse_l2 = lse_r * kLog2e;
        const float sc = (r < A.N) ? A.scale[r] : 0.f;
        const float sc_p = sc * fmaf(2.f * A.z_loss, lse_r, 1.f);  // softmax part: (1 + 2 zl LSE) p
        const float sc_y = sc * A.onehot_coef;                     // onehot part: (1 - ls) y
        // target in this problem's vocabulary coordinates (the shard's rows, for a vocabulary shard)
        const int64_t tg = (r < A.N) ? A.targets[r] - A.vocab_start : A.ignore_index - A.vocab_start;
        const bool tvalid = tg != A.ignore_index - A.vocab_start && tg >= 0 && tg < A.V;
        const bool mma = it.s != 0;
        if (mma) {
          if (!warp_wait(bar(kAccFull + a), (acc_iter >> 1) & 1u)) break;
          tc_fence_after();
        }
        // the chunk's buffer must no longer be read by the dE / dC items of chunk - 2
        if (leader && it.dep_idx >= 0 && !wait_counter(A.counters + it.dep_idx, it.dep_val, wc)) ok = false;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        uint8_t* buf = buffer(it.chunk);
        // rounds of up to two halves: the region holds two 64-column parts
        for (int j0 = 0; j0 < it.s && ok; j0 += 2) {
          if (!region_free()) {
            ok = false;
            break;
          }
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int j = j0 + jj;
            if (j >= it.s) break;
            const int th = quad_half(it, j);
            const int vb = (th >> 1) * BN + (th & 1) * kSubTile;  // the half's first vocabulary column
            const int64_t rel = tg - vb;
            const int tcol = (tvalid && rel >= 0 && rel < kSubTile) ? static_cast<int>(rel) : -1;  // -scale_r
            const uint32_t blk = reg0 + static_cast<uint32_t>(jj * PART);
#pragma unroll
            for (int c = 0; c < kSubTile / 32; ++c) {
              float v[32];
              const int col0 = vb + c * 32;
              tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(a * 2 * BN + j * kSubTile + c * 32), v);
              if (A.bias != nullptr) add_bias32(v, A.bias, col0, A.V);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = sc_p * exp2f(fmaf(v[e], kLog2e, -lse_l2));
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (c * 32 + e == tcol) v[e] -= sc_y;
                if (col0 + e >= A.V) v[e] = 0.f;
              }
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int ch = c * 4 + h;
                st_shared_v4(blk + swz(row, ch), pack_bf16x2(v[8 * h + 0], v[8 * h + 1]),
                             pack_bf16x2(v[8 * h + 2], v[8 * h + 3]), pack_bf16x2(v[8 * h + 4], v[8 * h + 5]),
                             pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
              }
              if (A.dbias != nullptr) {  // dbias += column sums of G (this warp's 32 rows), fp32
                const float cs = warp_column_sums32(v, lane);
                if (col0 + lane < A.V && cs != 0.f) atomicAdd(A.dbias + col0 + lane, cs);
              }
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(kGReady));
          if (warp == 2) {
            if (!warp_wait(bar(kGReady), gphase & 1u)) {
              ok = false;
            } else if (leader) {
              for (int jj = 0; jj < 2 && j0 + jj < it.s; ++jj) {  // each half into its tile's slot
                const int th = quad_half(it, j0 + jj);
                uint8_t* dst = buf + static_cast<size_t>(quad_slot(it, j0 + jj)) * TILE_BYTES + (th & 1) * PART;
                bulk_store(dst, reg0 + static_cast<uint32_t>(jj * PART), PART);
              }
              bulk_commit_group();
            }
          }
          ++gphase;
        }
        if (mma) {
          tc_fence_before();
          mbar_arrive(bar(kAccEmpty + a));
          ++acc_iter;
        }
        // publish the quad's halves to the dE / dC items that wait for them
        if (leader && ok) {
          bulk_wait_group0();
          fence_proxy_async_global();
          red_release_add(A.counters + A.ctr_g_b + it.chunk * A.nb + b, it.s);
          for (int j = 0; j < it.s; ++j) red_release_add(A.counters + A.ctr_g_t + (quad_half(it, j) >> 1), 1);
        }
        __syncwarp();
        if (*abort_flag) ok = false;
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        region_shared = true;
        continue;
      }

      // dE / dC
      const bool de = it.kind == kDE;
      const bool has = it.begin < it.end;
      // dC: the onehot terms -scale_r (1 - ls) E_r of the rows r whose target tile here was skipped
      // and whose target falls in this warp's 32 rows of the tile, in list order. The first two such
      // entries have this item's 256 columns of E_r loaded by the whole warp at once (16 bytes per
      // lane), before the accumulator is waited for; at each step the entry's owner lane takes its 64
      // columns by shuffles. Later entries (several rows targeting this warp's rows) are loaded by
      // their owner lane at each step.
      const int x_item = it.s * SLICE;
      int h_owner0 = -1, h_owner1 = -1;  // warp-uniform: the lane whose row gets held entry 0 / 1
      float h_coef0 = 0.f, h_coef1 = 0.f;
      uint4 h_cols0 = make_uint4(0, 0, 0, 0), h_cols1 = make_uint4(0, 0, 0, 0);  // columns x_item + 8 lane
      int oh_rest = -1;  // warp-uniform: first list entry handled step by step, or -1
      if (!de && it.oh_begin < it.oh_end) {
        const int64_t base_v = static_cast<int64_t>(it.key) * BN + q * 32 + A.vocab_start;
        const int64_t col = x_item + 8 * lane;
        int held = 0;
        for (int i0 = it.oh_begin; i0 < it.oh_end && oh_rest < 0; i0 += 32) {
          int r = 0, owner = -1;
          if (i0 + lane < it.oh_end) {
            r = A.oh_rows[i0 + lane];
            const int64_t o = A.targets[r] - base_v;
            owner = o >= 0 && o < 32 ? static_cast<int>(o) : -1;
          }
          for (unsigned m = __ballot_sync(0xffffffffu, owner >= 0); m != 0; m &= m - 1) {
            const int k = __ffs(m) - 1;
            if (held == 2) {
              oh_rest = i0 + k;
              break;
            }
            const int rk = __shfl_sync(0xffffffffu, r, k), ok = __shfl_sync(0xffffffffu, owner, k);
            const float ck = -A.scale[rk] * A.onehot_coef;
            const uint4 cols = col < A.D ? ld_global_nc_v4(A.E + static_cast<int64_t>(rk) * A.D + col)
                                         : make_uint4(0, 0, 0, 0);
            if (held == 0) {
              h_owner0 = ok;
              h_coef0 = ck;
              h_cols0 = cols;
            } else {
              h_owner1 = ok;
              h_coef1 = ck;
              h_cols1 = cols;
            }
            ++held;
          }
        }
      }
      if (has) {
        if (!warp_wait(bar(kAccFull + a), (acc_iter >> 1) & 1u)) break;
        tc_fence_after();
      }
      // every gradient tile of this item has been read into shared memory (the MMAs are done)
      if (leader) {
        fence_proxy_async_global();
        red_release_add(A.counters + A.ctr_b_done + it.chunk, 1);
      }
      if (de && !has) continue;  // nothing to add for this row block in this chunk
      // After a quad every warp's earlier bulk stores must have read the whole region; between dE / dC
      // items each warp only reuses its own staging images, which next_image() guards.
      if (region_shared && !region_free()) break;
      region_shared = false;
      const int rows_limit = de ? A.N : A.V;
      const int y = it.key * BM + q * 32;
      for (int p = 0; p < SLICE / 64; ++p) {
        const int x = x_item + 64 * p;
        if (x >= A.D) break;
        float v0[32], v1[32];
        if (has) {
          tmem_ld64(tmem_base + lane_off + static_cast<uint32_t>(a * SLICE + 64 * p), v0, v1);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v0[e] = v1[e] = 0.f;
        }
        auto add_vals = [&](const uint4 (&u8)[8], float coef) {  // u8: this step's 64 columns
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t w4[4] = {u8[k].x, u8[k].y, u8[k].z, u8[k].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              __nv_bfloat162 h;
              *reinterpret_cast<uint32_t*>(&h) = w4[j];
              float* dst = k < 4 ? v0 + 8 * k + 2 * j : v1 + 8 * (k - 4) + 2 * j;
              dst[0] = fmaf(coef, __low2float(h), dst[0]);
              dst[1] = fmaf(coef, __high2float(h), dst[1]);
            }
          }
        };
        auto add_held = [&](const uint4& cols, int owner, float coef) {  // lanes 8p .. 8p + 7 hold the step
          uint4 u8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            u8[k].x = __shfl_sync(0xffffffffu, cols.x, 8 * p + k);
            u8[k].y = __shfl_sync(0xffffffffu, cols.y, 8 * p + k);
            u8[k].z = __shfl_sync(0xffffffffu, cols.z, 8 * p + k);
            u8[k].w = __shfl_sync(0xffffffffu, cols.w, 8 * p + k);
          }
          if (lane == owner) add_vals(u8, coef);
        };
        if (h_owner0 >= 0) add_held(h_cols0, h_owner0, h_coef0);
        if (h_owner1 >= 0) add_held(h_cols1, h_owner1, h_coef1);
        if (oh_rest >= 0) {  // the rest of the list, each entry by its owner lane
          const int64_t my_v = static_cast<int64_t>(it.key) * BN + q * 32 + lane;
          for (int i = oh_rest; i < it.oh_end; ++i) {
            const int r = A.oh_rows[i];
            if (A.targets[r] - A.vocab_start != my_v) continue;
            uint4 u8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              u8[k] = x + 8 * k < A.D ? ld_global_nc_v4(A.E + static_cast<int64_t>(r) * A.D + x + 8 * k)
                                      : make_uint4(0, 0, 0, 0);
            add_vals(u8, -A.scale[r] * A.onehot_coef);
          }
        }
        if (!de && A.dc_add != nullptr) {  // the smoothing term, the same for every row of dC
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (x + e < A.D) v0[e] = fmaf(A.dc_coef, A.dc_add[x + e], v0[e]);
            if (x + 32 + e < A.D) v1[e] = fmaf(A.dc_coef, A.dc_add[x + 32 + e], v1[e]);
          }
        }
        if (y >= rows_limit) continue;  // this warp's 32 rows lie past the end of dE / dC
        // The warp's 8 KB of staging holds two 4 KB images used in turn; an image is rewritten once
        // the TMA operation issued from it two images earlier has read it, so one operation is
        // always in flight while the next image is written.
        auto next_image = [&]() {
          if (lane == 0) bulk_wait_group_read1();
          __syncwarp();
          return stg + 4096u * (img++ & 1u);
        };
        auto put_f32 = [&](const float (&v)[32], int xc) {  // 32 rows x 32 fp32 columns
          const uint32_t im = next_image();
#pragma unroll
          for (int h = 0; h < 8; ++h)
            st_shared_v4(im + swz(lane, h), __float_as_uint(v[4 * h]), __float_as_uint(v[4 * h + 1]),
                         __float_as_uint(v[4 * h + 2]), __float_as_uint(v[4 * h + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (de) tma_reduce_add_2d(&tmdE, im, xc, y);
            else tma_store_2d(&tmdC, im, xc, y);
            bulk_commit_group();
          }
        };
        if (!de && A.out_bf16) {  // 32 rows x 64 bf16 columns in one image
          const uint32_t im = next_image();
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const float* src = h < 4 ? v0 + 8 * h : v1 + 8 * (h - 4);
            st_shared_v4(im + swz(lane, h), pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                         pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmdC, im, x, y);
            bulk_commit_group();
          }
        } else {
          put_f32(v0, x);
          if (x + 32 < A.D) put_f32(v1, x + 32);
        }
      }
      if (has) {
        tc_fence_before();
        mbar_arrive(bar(kAccEmpty + a));
        ++acc_iter;
      }
    }
    // every store and reduce-add must be complete before the kernel ends
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_bwd(const BwdLaunch& L, bool after_kernel, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  if (after_kernel) {
    e = launch_after_previous(bwd_kernel, dim3(L.num_sms), dim3(NUM_THREADS), SMEM_BYTES, s, L.tmE128, L.tmC128,
                              L.tmE64, L.tmC64, L.tmdC, L.tmdE, L.args);
    if (e != cudaSuccess) return e;
  } else {
    bwd_kernel<<<L.num_sms, NUM_THREADS, SMEM_BYTES, s>>>(L.tmE128, L.tmC128, L.tmE64, L.tmC64, L.tmdC, L.tmdE,
                                                           L.args);
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

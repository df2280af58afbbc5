// Backward, step 1 of 3 per vocabulary chunk: the gradient tiles.
//
// For every listed tile (b, t) of the chunk: recompute S = E_b C_t^T (kept tiles), form
// G = scale_r * exp(S - LSE_r) - scale_r * [v = t_r] in fp32, round to bf16 into a 128B-swizzled
// shared-memory tile, and copy that tile (32 KB) to its slot of the chunk's gradient-tile scratch,
// from which the dC and dE kernels load it. Onehot-only tiles (skipped, but holding a target) get
// G = -scale_r * [v = t_r] without a recompute.
//
// mlx-cross-entropy README, "How it works" items 2 (recompute from the saved LSE, skip tiles below
// 2^-12); Loss functions explainer, "How it works" item 2 (gradient p - y); Cut Your Losses
// abstract (logits are recomputed blockwise, never stored).
//
// Two listed tiles of the same row block are recomputed together, as one 128 x 256 logit tile:
// E_b is loaded once for both vocabulary tiles and each MMA is M=128 x N=256, the forward's shape.
//
// Design (B200): one persistent CTA per SM, 6 warps, over pairs of consecutive listed tiles of a row
// block inside the chunk (the row-block lists are ordered by vocabulary tile).
//   warp 0      TMA producer: E_b, C_t1 and C_t2 K-blocks (bf16, 128B swizzle), 48 KB stages, 4 deep.
//   warp 1      TMEM (512 columns = two 256-column S buffers); one lane issues tcgen05.mma M=128 N=256.
//   warps 2..5  G formation (TMEM -> exp -> bf16 -> swizzled smem) and one bulk store per tile, while
//               the MMA recomputes the next pair into the other S buffer.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kBwdBM;
constexpr int BN = kBwdBN;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int HALF = 16384;            // 128 x 64 bf16
constexpr int STAGE_BYTES = 3 * HALF;  // E_b K-block | C_t1 K-block | C_t2 K-block
constexpr int G_BYTES = kGradTileBytes;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int NUM_BARRIERS = 2 * STAGES + 4 + 3;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + G_BYTES + NUM_BARRIERS * 8 + 16;
constexpr uint32_t IDESC_S = idesc_bf16(BM, 2 * BN, false, false);

static_assert(G_BYTES == BM * BN * 2, "gradient tile is 128 x 128 bf16");

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void bulk_store_32k(void* gdst, uint32_t src) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(src), "r"(G_BYTES)
               : "memory");
}

// Pair w of this chunk: its row block, and its one or two tiles (vocabulary tile, slot, kept?),
// from the plan's flat pair list (one 16-byte and one 8-byte load).
struct Pair {
  int b;
  int t[2], slot[2];
  bool kept[2], present[2];
  __device__ bool any_kept() const { return kept[0] || kept[1]; }
};

__device__ __forceinline__ Pair pair_at(int w, const int4* pair_desc, const int2* pair_slot) {
  const int4 d = pair_desc[w];
  const int2 sl = pair_slot[w];
  Pair p;
  p.b = d.x;
  p.t[0] = d.y;
  p.t[1] = d.z >= 0 ? d.z : d.y;
  p.present[0] = true;
  p.present[1] = d.z >= 0;
  p.kept[0] = (d.w & 1) != 0;
  p.kept[1] = (d.w & 2) != 0;
  p.slot[0] = sl.x;
  p.slot[1] = sl.y;
  return p;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_g_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC, int N, int D, int V,
                 const float* __restrict__ lse, const float* __restrict__ scale, const int64_t* __restrict__ targets,
                 int64_t ignore_index, const int* __restrict__ num_pairs_p, const int4* __restrict__ pair_desc,
                 const int2* __restrict__ pair_slot, uint8_t* __restrict__ gscratch, int* err, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* gbuf = base + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbuf + G_BYTES);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NUM_BARRIERS);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto sfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto sempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  const uint32_t gfree_bar = bar0 + 8u * (2 * STAGES + 5);   // leader: the smem G buffer may be rewritten
  const uint32_t gready_bar = bar0 + 8u * (2 * STAGES + 6);  // all 128 rows of G are in smem

  const int num_pairs = *num_pairs_p;
  if (num_pairs <= static_cast<int>(blockIdx.x)) return;  // uniform across the CTA, before any sync
  // Each role loads the next pair's descriptor before working on the current one.
  auto get_pair = [&](int w) { return pair_at(w < num_pairs ? w : static_cast<int>(blockIdx.x), pair_desc, pair_slot); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(sfull_bar(a), 1);
      mbar_init(sempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    mbar_init(gfree_bar, 1);
    mbar_init(gready_bar, 128);
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
  const WaitCtl wc{abort_flag, err, timeout_ns};
  const int num_kb = (D + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES] = {0, 0, 0, 0};
      bool ok = true;
      Pair nx = get_pair(blockIdx.x);
      for (int w = blockIdx.x; w < num_pairs && ok; w += gridDim.x) {
        const Pair p = nx;
        nx = get_pair(w + gridDim.x);
        if (!p.any_kept()) continue;  // onehot-only tiles need no recompute
        const int rb = p.b * BM;
        const int vb0 = p.t[0] * BN, vb1 = (p.present[1] ? p.t[1] : p.t[0]) * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + stage * STAGE_BYTES);
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          tma_load_2d(dst, &tmE, full_bar(stage), kb * BK, rb);
          tma_load_2d(dst + HALF, &tmC, full_bar(stage), kb * BK, vb0);
          tma_load_2d(dst + 2 * HALF, &tmC, full_bar(stage), kb * BK, vb1);
          ++issued[stage];
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(full_bar(s), (issued[s] - 1u) & 1u, 200000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t sidx = 0;
      bool ok = true, issued_any = false;
      Pair nx = get_pair(blockIdx.x);
      for (int w = blockIdx.x; w < num_pairs && ok; w += gridDim.x) {
        const Pair p = nx;
        nx = get_pair(w + gridDim.x);
        if (!p.any_kept()) continue;
        const int a = sidx & 1;
        if (!mbar_wait(sempty_bar(a), ((sidx >> 1) & 1u) ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * 2 * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stages + stage * STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // B = C_t1 and C_t2 rows: 256 rows of 128 bytes, contiguous
            tc_mma_bf16(d_tmem, sdesc_sw128(a0 + 32u * k, 16, 1024), sdesc_sw128(a0 + HALF + 32u * k, 16, 1024),
                        IDESC_S, (kb | k) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(sfull_bar(a));
        ++sidx;
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, 200000000ull);
      }
    }
  } else {
    // ---------------- epilogue: G tiles ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    const uint32_t g0 = smem_u32(gbuf);
    uint32_t sidx = 0, j = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < num_pairs && ok; w += gridDim.x) {
      const Pair p = get_pair(w);
      const int r = p.b * BM + row;
      const float lse_l2 = (r < N) ? lse[r] * kLog2e : 0.f;
      const float sc = (r < N) ? scale[r] : 0.f;
      const int64_t tg = (r < N) ? targets[r] : ignore_index;
      const bool tvalid = tg != ignore_index && tg >= 0 && tg < V;
      const int a = sidx & 1;
      if (p.any_kept()) {
        if (!mbar_wait(sfull_bar(a), (sidx >> 1) & 1u, wc)) break;
        tc_fence_after();
      }
      for (int k = 0; k < 2 && ok; ++k) {
        if (!p.present[k]) break;
        const int vb = p.t[k] * BN;
        const int64_t rel = tg - vb;
        const int tcol = (tvalid && rel >= 0 && rel < BN) ? static_cast<int>(rel) : -1;  // -scale_r goes here
        // The G buffer is free once the previous tile's store has read it (bounded mbarrier waits,
        // not a named barrier, so that an abort cannot hang here).
        if (leader) {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          mbar_arrive(gfree_bar);
        }
        if (!mbar_wait(gfree_bar, j & 1u, wc)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          if (p.kept[k]) {
            tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(a * 2 * BN + k * BN + c * 32), v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = sc * exp2f(fmaf(v[e], kLog2e, -lse_l2));
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0.f;
          }
          const int col0 = vb + c * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (c * 32 + e == tcol) v[e] -= sc;
            if (col0 + e >= V) v[e] = 0.f;
          }
          const uint32_t blk = g0 + static_cast<uint32_t>((c >> 1) * HALF);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int chunk = (c & 1) * 4 + h;
            st_shared_v4(blk + swz(row, chunk), pack_bf16x2(v[8 * h + 0], v[8 * h + 1]),
                         pack_bf16x2(v[8 * h + 2], v[8 * h + 3]), pack_bf16x2(v[8 * h + 4], v[8 * h + 5]),
                         pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(gready_bar);
        if (leader) {
          if (!mbar_wait(gready_bar, j & 1u, wc)) {
            ok = false;
            break;
          }
          bulk_store_32k(gscratch + static_cast<size_t>(p.slot[k]) * G_BYTES, g0);
          bulk_commit_group();
        }
        ++j;  // one gfree / gready phase per tile
      }
      if (p.any_kept()) {
        tc_fence_before();
        mbar_arrive(sempty_bar(a));
        ++sidx;
      }
    }
    // Every tile must be in global memory before the kernel ends (the next kernels read them).
    if (leader) bulk_wait_group0();
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

cudaError_t launch_bwd_g(const BwdGradTiles& L, int chunk, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_g_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = L.num_sms;  // CTAs past the chunk's pair count exit at once
  const int64_t first = static_cast<int64_t>(chunk) * L.pair_cap;
  bwd_g_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(
      L.tmE, L.tmC, L.N, L.D, L.V, L.lse, L.scale, L.targets, L.ignore_index,
      L.pair_off + static_cast<int64_t>(chunk) * (L.nb + 1) + L.nb, L.pair_desc + first, L.pair_slot + first,
      L.gscratch, L.err, L.timeout_ns);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

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
// Design (B200): one persistent CTA per SM, 6 warps.
//   warp 0      TMA producer: E_b and C_t K-blocks (bf16, 128B swizzle) into a 4-stage ring.
//   warp 1      TMEM (256 columns = two S buffers of 128); one lane issues tcgen05.mma M=128 N=128.
//   warps 2..5  G formation (TMEM -> exp -> bf16 -> swizzled smem), one bulk store per tile; the
//               two smem G buffers let the store of one tile overlap the formation of the next.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kBwdBM;
constexpr int BN = kBwdBN;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int HALF = 16384;            // 128 x 64 bf16
constexpr int STAGE_BYTES = 2 * HALF;  // E_b K-block | C_t K-block
constexpr int G_BYTES = kGradTileBytes;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 256;
constexpr int NUM_BARRIERS = 2 * STAGES + 4 + 3;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * G_BYTES + NUM_BARRIERS * 8 + 16;
constexpr uint32_t IDESC_S = idesc_bf16(BM, BN, false, false);

static_assert(G_BYTES == BM * BN * 2, "gradient tile is 128 x 128 bf16");

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void bulk_store_32k(void* gdst, uint32_t src) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(src), "r"(G_BYTES)
               : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_g_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC, int N, int D, int V,
                 const float* __restrict__ lse, const float* __restrict__ scale, const int64_t* __restrict__ targets,
                 int64_t ignore_index, const int2* __restrict__ entries_t, const int* __restrict__ offsets_t,
                 int chunk_t0, int chunk_t1, uint8_t* __restrict__ gscratch, int* err, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* gbuf = base + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbuf + 2 * G_BYTES);
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

  const int e0 = offsets_t[chunk_t0], e1 = offsets_t[chunk_t1];
  if (e1 - e0 <= static_cast<int>(blockIdx.x)) return;  // uniform across the CTA, before any sync

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
      for (int i = e0 + blockIdx.x; i < e1 && ok; i += gridDim.x) {
        const int2 en = entries_t[i];
        if ((en.x & 3) != 1) continue;  // onehot-only tiles need no recompute
        const int rb = (en.x >> 2) * BM, vb = en.y * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(stages + stage * STAGE_BYTES);
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          tma_load_2d(dst, &tmE, full_bar(stage), kb * BK, rb);
          tma_load_2d(dst + HALF, &tmC, full_bar(stage), kb * BK, vb);
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
      for (int i = e0 + blockIdx.x; i < e1 && ok; i += gridDim.x) {
        const int2 en = entries_t[i];
        if ((en.x & 3) != 1) continue;
        const int a = sidx & 1;
        if (!mbar_wait(sempty_bar(a), ((sidx >> 1) & 1u) ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stages + stage * STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
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
    uint32_t sidx = 0, j = 0;
    for (int i = e0 + blockIdx.x; i < e1; i += gridDim.x, ++j) {
      const int2 en = entries_t[i];
      const bool full = (en.x & 3) == 1;
      const int rb = (en.x >> 2) * BM, vb = en.y * BN;
      const int r = rb + row;
      const float lse_l2 = (r < N) ? lse[r] * kLog2e : 0.f;
      const float sc = (r < N) ? scale[r] : 0.f;
      int tcol = -1;  // target column inside this tile: G gets -scale_r there, in fp32, before rounding
      if (r < N) {
        const int64_t tg = targets[r];
        const int64_t rel = tg - vb;
        if (tg != ignore_index && tg >= 0 && tg < V && rel >= 0 && rel < BN) tcol = static_cast<int>(rel);
      }
      // The smem buffer of tile j was last stored two tiles ago: that store must have read it.
      // (mbarriers with bounded waits, not a named barrier, so that an abort cannot hang here.)
      if (leader) {
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        mbar_arrive(gfree_bar);
      }
      if (!mbar_wait(gfree_bar, j & 1u, wc)) break;
      const uint32_t g0 = smem_u32(gbuf + (j & 1) * G_BYTES);
      const int a = sidx & 1;
      if (full) {
        if (!mbar_wait(sfull_bar(a), (sidx >> 1) & 1u, wc)) break;
        tc_fence_after();
      }
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        if (full) {
          tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(a * BN + c * 32), v);
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = sc * exp2f(fmaf(v[k], kLog2e, -lse_l2));
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
        const int col0 = vb + c * 32;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          if (c * 32 + k == tcol) v[k] -= sc;
          if (col0 + k >= V) v[k] = 0.f;
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
      if (full) {
        tc_fence_before();
        mbar_arrive(sempty_bar(a));
        ++sidx;
      }
      fence_proxy_async_smem();
      mbar_arrive(gready_bar);
      if (leader) {
        if (!mbar_wait(gready_bar, j & 1u, wc)) break;
        bulk_store_32k(gscratch + static_cast<size_t>(i - e0) * G_BYTES, g0);
        bulk_commit_group();
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

cudaError_t launch_bwd_g(const BwdGradTiles& L, int chunk_t0, int chunk_t1, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_g_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = L.max_entries_per_chunk < L.num_sms ? L.max_entries_per_chunk : L.num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_g_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(L.tmE, L.tmC, L.N, L.D, L.V, L.lse, L.scale, L.targets,
                                                     L.ignore_index, L.entries_t, L.offsets_t, chunk_t0, chunk_t1,
                                                     L.gscratch, L.err, L.timeout_ns);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

// Forward of Cut Cross-Entropy on sm_100a: logit tiles z = E_b C_t^T on the tcgen05 tensor cores,
// reduced on the fly to a per-row maximum and sum of exponentials for every 128-wide vocabulary
// sub-tile. The [N, V] logits never leave the SM.
//
// mlx-cross-entropy README, "How it works" item 1: the matmul is tiled and each tile yields a
// local max and sum-exp that combine into a numerically stable log-sum-exp. Loss functions
// explainer, "How it works" item 1: LSE = m + log sum exp(z - m). The per-sub-tile maximum is
// also what the backward's tile skipping reads (mlx-cross-entropy README, item 2).
//
// Design (B200): one persistent CTA per SM, 6 warps.
//   warp 0      TMA producer: E and C tiles (bf16, 128B swizzle) into a 4-stage ring.
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma (M=128, N=256, K=16)
//               into one of two 256-column fp32 accumulators.
//   warps 2..5  epilogue: TMEM -> registers, per-row max / sum-exp over each 128-column sub-tile,
//               and the correct-token logit of rows whose target falls in the tile, while the MMA
//               fills the other accumulator.
// Tiles are visited row-block fastest within groups of 32 row blocks (see tile_coords), so the
// CTAs working at one time share a few C tiles and E stays in L2.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kFwdBM;
constexpr int BN = kFwdBN;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int NUM_BARRIERS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NUM_BARRIERS * 8 + 16;
constexpr uint32_t IDESC = idesc_bf16(BM, BN, false, false);

struct Smem {
  uint8_t* stage;  // STAGES x (A | B)
  uint64_t* bars;
  uint32_t* tmem_holder;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stage = base;
  s.bars = reinterpret_cast<uint64_t*>(base + STAGES * STAGE_BYTES);
  s.tmem_holder = reinterpret_cast<uint32_t*>(s.bars + NUM_BARRIERS);
  s.abort = reinterpret_cast<int*>(s.tmem_holder + 1);
  return s;
}

// Tile w -> (row block, vocabulary tile). Row blocks are taken in groups of kRowGroup (32 x 128
// rows: 8 MB of E per 1024 of D): row block fastest inside a group, then the next vocabulary tile,
// and the next group after the last vocabulary tile. The CTAs running at one time then share a
// few C tiles (read once from HBM per group) and at most one group of E rows, which stays in L2
// however large N is.
constexpr int kRowGroup = 32;

__device__ __forceinline__ void tile_coords(int w, int nb, int nt, int& b, int& t) {
  const int per_group = kRowGroup * nt;
  const int g = w / per_group, in = w - g * per_group;
  const int rows = min(kRowGroup, nb - g * kRowGroup);  // the last group may be short
  t = in / rows;
  b = g * kRowGroup + in % rows;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    fwd_lse_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC, int N, int D,
                   int V, int T, const __nv_bfloat16* __restrict__ bias, float* __restrict__ tile_max,
                   float* __restrict__ tile_sum, const int64_t* __restrict__ targets, int64_t vs,
                   int64_t ignore_index, float* __restrict__ zt, int* err, uint64_t timeout_ns, int inject_stall) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = smem_u32(sm.bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    *sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_holder), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_holder;

  const WaitCtl wc{sm.abort, err, timeout_ns};
  const int nb = (N + BM - 1) / BM;
  const int nt = (V + BN - 1) / BN;
  const int num_kb = (D + BK - 1) / BK;
  const int total = nb * nt;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // inject_stall (test hook): issue no loads at all, so the MMA warp's first bounded wait runs
    // out and the kernel reports kErrDeviceTimeout. Nothing is left in flight in that case.
    if (lane == 0 && !inject_stall) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES] = {0, 0, 0, 0};
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int b, t;
        tile_coords(tile, nb, nt, b, t);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(sm.stage + stage * STAGE_BYTES);
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          tma_load_2d(dst, &tmE, full_bar(stage), kb * BK, b * BM);
          tma_load_2d(dst + A_BYTES, &tmC, full_bar(stage), kb * BK, t * BN);
          ++issued[stage];
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let every load already issued land before the CTA can exit.
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) mbar_wait_drain(full_bar(s), (issued[s] - 1u) & 1u, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.stage + stage * STAGE_BYTES);
          const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            tc_mma_bf16(d_tmem, sdesc_sw128(a0 + 32u * k, 16, 1024), sdesc_sw128(b0 + 32u * k, 16, 1024), IDESC,
                        (kb | k) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && issued_any) {
        // No MMA may still be writing TMEM when it is released.
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, 200000000ull);
      }
    }
  } else {
    // ---------------- epilogue: per-row max and sum-exp of each 128-column sub-tile ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_in_tile = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int b, t;
      tile_coords(tile, nb, nt, b, t);
      if (!mbar_wait(tfull_bar(acc), acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int r = b * BM + row_in_tile;
      // The row's correct-token column inside this tile (-1: elsewhere, ignored, or no row)
      int tcol = -1;
      if (r < N) {
        const int64_t tl = targets[r] - vs;
        if (targets[r] != ignore_index && tl >= static_cast<int64_t>(t) * BN && tl < min(t * BN + BN, V))
          tcol = static_cast<int>(tl) - t * BN;
      }
#pragma unroll
      for (int sub = 0; sub < BN / kSubTile; ++sub) {
        float m = -INFINITY, s = 0.f;
#pragma unroll
        for (int c = 0; c < kSubTile / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + static_cast<uint32_t>(sub * kSubTile + c * 32), v);
          const int col0 = t * BN + sub * kSubTile + c * 32;
          if (bias != nullptr) add_bias32(v, bias, col0, V);
          // Cut Your Losses (abstract): of the logits only the correct token's is kept, picked here
          // from the same fp32 tile the log-sum-exp reads. Each row has one such column, so the branch
          // is rare.
          const int k = tcol - (sub * kSubTile + c * 32);
          const bool hit = k >= 0 && k < 32;
          if (__any_sync(0xffffffffu, hit)) {
            float z = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) z = i == k ? v[i] : z;
            if (hit) zt[r] = z;
          }
          if (col0 + 32 > V) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i >= V) v[i] = -INFINITY;
          }
          float cm = v[0];
#pragma unroll
          for (int i = 1; i < 32; ++i) cm = fmaxf(cm, v[i]);
          const float mn = fmaxf(m, cm);
          if (mn == -INFINITY) continue;  // every column so far is past V
          const float off = mn * kLog2e;
          float acc_s = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) acc_s += exp2f(fmaf(v[i], kLog2e, -off));
          s = s * exp2f(fmaf(m, kLog2e, -off)) + acc_s;
          m = mn;
        }
        const int j = t * (BN / kSubTile) + sub;
        if (r < N && j < T) {
          tile_max[static_cast<size_t>(j) * N + r] = m;
          tile_sum[static_cast<size_t>(j) * N + r] = s;
        }
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
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

cudaError_t launch_fwd_lse(const FwdLaunch& L, cudaStream_t s) {
  const int nb = (L.N + BM - 1) / BM;
  const int nt = (L.V + BN - 1) / BN;
  const long long total = static_cast<long long>(nb) * nt;
  if (total == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(fwd_lse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(total < L.num_sms ? total : L.num_sms);
  fwd_lse_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(L.tmE, L.tmC, L.N, L.D, L.V, L.T, L.bias, L.tile_max,
                                                       L.tile_sum, L.targets, L.vs, L.ignore_index, L.zt, L.err,
                                                       L.timeout_ns, L.inject_stall);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

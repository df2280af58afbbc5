// Backward of Cut Cross-Entropy on sm_100a: for every kept (row block b, vocabulary tile t)
// recompute S = E_b C_t^T, form G = scale_r * exp(S - LSE_r) in bf16 in shared memory, then issue
// dE_b += G C_t and dC_t += G^T E_b on the tensor cores in 64-column chunks of D and add each fp32
// chunk into the global accumulators with TMA reduce-add.
//
// mlx-cross-entropy README, "How it works" items 2 and 3 (recompute, skip tiles below 2^-12 using
// the forward's saved maxima, accumulate with atomics instead of [batch, tiles, D] buffers); Loss
// functions explainer, "How it works" item 2 (the logit gradient is p - y). The onehot "- y" of a
// kept tile is folded into G in fp32 before the bf16 rounding; for a skipped tile that holds a
// target it is added by a separate kernel, so it is never skipped. Cut Your Losses abstract (skip
// gradient elements below numerical precision).
//
// Design (B200): one persistent CTA per SM, 6 warps, walking the compacted list of kept tiles.
//   warp 0      TMA producer into a 3-stage ring of 32 KB stages: first the D/64 k-blocks of
//               (E_b, C_t) for the recompute, then the D/64 chunks of (C_t, E_b) for the gradients.
//   warp 1      TMEM (512 columns) and MMA issue:
//                 S       cols [0,128):   M=128 rows,  N=128 vocab, K=D    (A=E K-major, B=C K-major)
//                 dE chunk cols 128+128u: M=128 rows,  N=64 of D,  K=128 vocab (A=G K-major, B=C MN-major)
//                 dC chunk cols 192+128u: M=128 vocab, N=64 of D,  K=128 rows  (A=G MN-major, B=E MN-major)
//               with two gradient buffers u = 0, 1 so the flush of one overlaps the MMAs of the next.
//   warps 2..5  G formation (TMEM -> exp -> bf16 -> swizzled smem) and the flush (TMEM -> fp32
//               swizzled staging -> cp.reduce.async.bulk.tensor add).
// One G tile in 128B-swizzled layout serves as the K-major A of dE and, read MN-major, as the A of
// dC (G^T), so it is written once.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kBwdBM;  // rows per tile
constexpr int BN = kBwdBN;  // vocabulary columns per tile
constexpr int BK = 64;      // K block of the recompute
constexpr int DC = 64;      // D columns per gradient chunk
constexpr int STAGES = 3;
constexpr int HALF = 16384;            // one 128 x 64 bf16 operand tile
constexpr int STAGE_BYTES = 2 * HALF;  // recompute: E | C ; gradient: C chunk | E chunk
constexpr int G_BYTES = BM * BN * 2;   // 2 blocks of 128 rows x 64 vocab
constexpr int STG_WARP = 4 * 4096;     // per epilogue warp: dE (2 boxes of 32x32 fp32) + dC (2 boxes)
constexpr int STG_BYTES = 4 * STG_WARP;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int NUM_BARRIERS = 2 * STAGES + 2 + 4 + 1;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + G_BYTES + STG_BYTES + NUM_BARRIERS * 8 + 16;

constexpr uint32_t IDESC_S = idesc_bf16(BM, BN, false, false);
constexpr uint32_t IDESC_DE = idesc_bf16(BM, DC, false, true);
constexpr uint32_t IDESC_DC = idesc_bf16(BN, DC, true, true);

struct Smem {
  uint8_t* stage;
  uint8_t* g;
  uint8_t* stg;
  uint64_t* bars;
  uint32_t* tmem_holder;
  int* abort;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stage = base;
  s.g = base + STAGES * STAGE_BYTES;
  s.stg = s.g + G_BYTES;
  s.bars = reinterpret_cast<uint64_t*>(s.stg + STG_BYTES);
  s.tmem_holder = reinterpret_cast<uint32_t*>(s.bars + NUM_BARRIERS);
  s.abort = reinterpret_cast<int*>(s.tmem_holder + 1);
  return s;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of 128-byte row `row` in a 128B-swizzled block.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <bool kDirectRed>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_grad_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmdE, const __grid_constant__ CUtensorMap tmdC, int N,
                    int D, int V, const float* __restrict__ lse, const float* __restrict__ scale,
                    const int64_t* __restrict__ targets, int64_t ignore_index, const int2* __restrict__ tiles,
                    const int* __restrict__ num_tiles_ptr, uint32_t l2_hints, float* __restrict__ dE_acc,
                    float* __restrict__ dC_acc, int* err, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = smem_u32(sm.bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t sfull_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t gfull_bar = bar0 + 8u * (2 * STAGES + 1);
  auto gradfull_bar = [&](int u) { return bar0 + 8u * (2 * STAGES + 2 + u); };
  auto gradempty_bar = [&](int u) { return bar0 + 8u * (2 * STAGES + 4 + u); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 6);

  const int num_tiles = *num_tiles_ptr;
  if (num_tiles <= static_cast<int>(blockIdx.x)) return;  // uniform across the CTA, before any sync

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(sfull_bar, 1);
    mbar_init(gfull_bar, 128);
    for (int u = 0; u < 2; ++u) {
      mbar_init(gradfull_bar(u), 1);
      mbar_init(gradempty_bar(u), 128);
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
  const int num_kb = (D + BK - 1) / BK;
  const int num_dc = (D + DC - 1) / DC;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES] = {0, 0, 0};
      bool ok = true;
      const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
      const bool keepE = (l2_hints & kL2KeepE) != 0, streamC = (l2_hints & kL2StreamC) != 0;
      auto load_E = [&](uint32_t dst, uint32_t bar, int x, int y) {
        if (keepE) tma_load_2d_hint(dst, &tmE, bar, x, y, pol_last);
        else tma_load_2d(dst, &tmE, bar, x, y);
      };
      auto load_C = [&](uint32_t dst, uint32_t bar, int x, int y) {
        if (streamC) tma_load_2d_hint(dst, &tmC, bar, x, y, pol_first);
        else tma_load_2d(dst, &tmC, bar, x, y);
      };
      for (int i = blockIdx.x; i < num_tiles && ok; i += gridDim.x) {
        const int2 bt = tiles[i];
        const int rb = bt.x * BM, vb = bt.y * BN;
        for (int step = 0; step < num_kb + num_dc; ++step) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(sm.stage + stage * STAGE_BYTES);
          mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          if (step < num_kb) {  // recompute operands: E_b | C_t, K block `step`
            load_E(dst, full_bar(stage), step * BK, rb);
            load_C(dst + HALF, full_bar(stage), step * BK, vb);
          } else {  // gradient operands: C_t | E_b, D chunk `c`
            const int c = step - num_kb;
            load_C(dst, full_bar(stage), c * DC, vb);
            load_E(dst + HALF, full_bar(stage), c * DC, rb);
          }
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
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t tile_iter = 0, gc = 0;
      bool ok = true, issued_any = false;
      const uint32_t g0 = smem_u32(sm.g);
      for (int i = blockIdx.x; i < num_tiles && ok; i += gridDim.x, ++tile_iter) {
        // Recompute S. The previous tile's G was formed before its gradient MMAs were issued, so
        // the S columns are free again.
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sm.stage + stage * STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            tc_mma_bf16(tmem_base, sdesc_sw128(a0 + 32u * k, 16, 1024), sdesc_sw128(a0 + HALF + 32u * k, 16, 1024),
                        IDESC_S, (kb | k) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(sfull_bar);
        // G must be in shared memory before the gradient MMAs read it.
        if (!mbar_wait(gfull_bar, tile_iter & 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < num_dc; ++c, ++gc) {
          const int u = gc & 1;
          if (!mbar_wait(gradempty_bar(u), ((gc >> 1) & 1u) ^ 1u, wc) || !mbar_wait(full_bar(stage), phase, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t cchunk = smem_u32(sm.stage + stage * STAGE_BYTES);
          const uint32_t echunk = cchunk + HALF;
          const uint32_t d_de = tmem_base + 128u + 128u * u;
          const uint32_t d_dc = d_de + 64u;
#pragma unroll
          for (int k = 0; k < BN / 16; ++k) {  // dE_b[:, chunk] += G[:, 16k..] * C_t[16k.., chunk]
            const uint64_t a = sdesc_sw128(g0 + (k >> 2) * HALF + 32u * (k & 3), 16, 1024);
            const uint64_t bd = sdesc_sw128(cchunk + 2048u * k, HALF, 1024);
            tc_mma_bf16(d_de, a, bd, IDESC_DE, k != 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < BM / 16; ++k) {  // dC_t[:, chunk] += G^T[:, 16k..] * E_b[16k.., chunk]
            const uint64_t a = sdesc_sw128(g0 + 2048u * k, HALF, 1024);
            const uint64_t bd = sdesc_sw128(echunk + 2048u * k, HALF, 1024);
            tc_mma_bf16(d_dc, a, bd, IDESC_DC, k != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          tc_commit(gradfull_bar(u));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, 200000000ull);
      }
    }
  } else {
    // ---------------- epilogue: G formation and gradient flush ----------------
    const int q = warp & 3;
    const int row = q * 32 + lane;  // TMEM lane = tile row (dE) = tile vocab row (dC)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t g0 = smem_u32(sm.g);
    const uint32_t stg = smem_u32(sm.stg + q * STG_WARP);
    const uint64_t pol_last = policy_evict_last(), pol_first = policy_evict_first();
    const bool keep_dE = (l2_hints & kL2KeepdE) != 0, stream_dC = (l2_hints & kL2StreamdC) != 0;
    auto add_dE = [&](uint32_t src, int x, int y) {
      if (keep_dE) tma_reduce_add_2d_hint(&tmdE, src, x, y, pol_last);
      else tma_reduce_add_2d(&tmdE, src, x, y);
    };
    auto add_dC = [&](uint32_t src, int x, int y) {
      if (stream_dC) tma_reduce_add_2d_hint(&tmdC, src, x, y, pol_first);
      else tma_reduce_add_2d(&tmdC, src, x, y);
    };
    uint32_t tile_iter = 0, gc = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < num_tiles && ok; i += gridDim.x, ++tile_iter) {
      const int2 bt = tiles[i];
      const int r = bt.x * BM + row;
      const float lse_l2 = (r < N) ? lse[r] * kLog2e : 0.f;
      const float sc = (r < N) ? scale[r] : 0.f;
      // Column of this row's target inside the tile, or -1: there G gets the onehot term -scale_r
      // in fp32, before rounding, so p_t - 1 does not lose its digits when p_t is close to 1.
      int tcol = -1;
      if (r < N) {
        const int64_t tg = targets[r];
        const int64_t rel = tg - static_cast<int64_t>(bt.y) * BN;
        if (tg != ignore_index && tg >= 0 && tg < V && rel >= 0 && rel < BN) tcol = static_cast<int>(rel);
      }
      if (!mbar_wait(sfull_bar, tile_iter & 1u, wc)) break;
      tc_fence_after();
      // G[row, :] = scale_r * exp(S[row, :] - LSE_r), bf16, 128B-swizzled, two 64-column blocks.
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(c * 32), v);
        const int col0 = bt.y * BN + c * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float gval = sc * exp2f(fmaf(v[j], kLog2e, -lse_l2));
          if (c * 32 + j == tcol) gval -= sc;
          v[j] = (col0 + j < V) ? gval : 0.f;
        }
        const uint32_t blk = g0 + static_cast<uint32_t>((c >> 1) * HALF);
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // four 16-byte chunks of 8 bf16
          const int chunk = (c & 1) * 4 + h;
          st_shared_v4(blk + swz(row, chunk), pack_bf16x2(v[8 * h + 0], v[8 * h + 1]),
                       pack_bf16x2(v[8 * h + 2], v[8 * h + 3]), pack_bf16x2(v[8 * h + 4], v[8 * h + 5]),
                       pack_bf16x2(v[8 * h + 6], v[8 * h + 7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(gfull_bar);

      for (int c = 0; c < num_dc; ++c, ++gc) {
        const int u = gc & 1;
        if (!mbar_wait(gradfull_bar(u), (gc >> 1) & 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_de = tmem_base + lane_off + 128u + 128u * u;
        if constexpr (kDirectRed) {
          // Registers -> L2 with red.global.add.v2.f32: the 16x256b load shape gives four threads
          // 8 consecutive columns of one row, so every warp instruction adds whole 32-byte sectors.
          float a0[32], a1[32], b0[32], b1[32];
          tmem_ld16x256b_x8(t_de, a0);
          tmem_ld16x256b_x8(t_de + (16u << 16), a1);
          tmem_ld16x256b_x8(t_de + 64u, b0);
          tmem_ld16x256b_x8(t_de + 64u + (16u << 16), b1);
          tc_fence_before();
          mbar_arrive(gradempty_bar(u));
          const int t0 = lane & 3, t1 = lane >> 2;
          const int rE = bt.x * BM + q * 32 + t1, rC = bt.y * BN + q * 32 + t1;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int col = c * DC + 8 * k + 2 * t0;
            if (col >= D) continue;
#pragma unroll
            for (int g = 0; g < 4; ++g) {  // rows +0, +8 (first 16 lanes), +16, +24 (second 16 lanes)
              const float* src_e = g < 2 ? a0 : a1;
              const float* src_c = g < 2 ? b0 : b1;
              const int reg = 4 * k + 2 * (g & 1);
              const int roff = (g >> 1) * 16 + (g & 1) * 8;
              if (rE + roff < N)
                red_add_v2(dE_acc + static_cast<size_t>(rE + roff) * D + col, src_e[reg], src_e[reg + 1]);
              if (rC + roff < V)
                red_add_v2(dC_acc + static_cast<size_t>(rC + roff) * D + col, src_c[reg], src_c[reg + 1]);
            }
          }
          continue;
        }
        float e0[32], e1[32], c0[32], c1[32];
        tmem_ld32(t_de, e0);
        tmem_ld32(t_de + 32u, e1);
        tmem_ld32(t_de + 64u, c0);
        tmem_ld32(t_de + 96u, c1);
        tc_fence_before();
        mbar_arrive(gradempty_bar(u));
        // The staging buffer of this warp is free once its previous reduce has read it.
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        const float* parts[4] = {e0, e1, c0, c1};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const uint32_t box = stg + p * 4096u;
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const float* x = parts[p] + 4 * h;
            st_shared_v4(box + swz(lane, h), __float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                         __float_as_uint(x[3]));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // Boxes that start past the end of a tensor hold nothing to add; they are not issued.
          const int x = c * DC;
          const int ye = bt.x * BM + q * 32, yc = bt.y * BN + q * 32;
          if (ye < N) {
            add_dE(stg, x, ye);
            if (x + 32 < D) add_dE(stg + 4096u, x + 32, ye);
          }
          if (yc < V) {
            add_dC(stg + 8192u, x, yc);
            if (x + 32 < D) add_dC(stg + 12288u, x + 32, yc);
          }
          bulk_commit_group();
        }
      }
    }
    // Every reduce must have completed before the kernel ends (later kernels read the sums).
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

cudaError_t launch_bwd_grad(const BwdLaunch& L, cudaStream_t s) {
  const long long nb = (L.N + BM - 1) / BM;
  const long long nt = (L.V + BN - 1) / BN;
  const long long max_tiles = nb * nt;
  if (max_tiles == 0) return cudaSuccess;
  auto kernel = L.direct_red ? bwd_grad_kernel<true> : bwd_grad_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(max_tiles < L.num_sms ? max_tiles : L.num_sms);
  kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(L.tmE, L.tmC, L.tmdE, L.tmdC, L.N, L.D, L.V, L.lse, L.scale, L.targets,
                                               L.ignore_index, L.tiles, L.num_tiles, L.l2_hints, L.dE_acc, L.dC_acc,
                                               L.err, L.timeout_ns);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

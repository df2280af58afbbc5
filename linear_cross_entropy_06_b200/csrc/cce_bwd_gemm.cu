// Backward, step 2 of 2 per vocabulary chunk: the gradient MMAs, from bf16 gradient tiles in shared
// memory, with fp32 accumulation in TMEM. One launch per chunk runs both kinds of work item (dE
// items first: they are the longer ones), so the chunk has a single tail.
//
//   dC mode  work item (vocabulary tile t, 256-column slice s of D):
//            dC[t rows, s cols] = sum over listed b of G_bt^T E_b[:, s]     (written directly; every
//            listed tile of t is in this chunk, so no reduction is needed)
//   dE mode  work item (row block b, slice s):
//            dE[b rows, s cols] += sum over listed t in the chunk of G_bt C_t[:, s]
//            (one fp32 TMA reduce-add per item and chunk: split-reduce over vocabulary chunks)
//
// mlx-cross-entropy README, "How it works" item 3 (gradients accumulated without intermediate
// [batch, tiles, D] buffers); Loss functions explainer, "How it works" item 2 (dE = G C and
// dC = G^T E with G = p - y). The gradient tiles come from the recompute kernel (cce_bwd_g.cu).
//
// Design (B200): one persistent CTA per SM, 6 warps.
//   warp 0      producer: per listed tile, two 48 KB stages, one per 64-wide half of the MMA's K:
//               16 KB of the gradient tile (bulk copy from the chunk scratch) and the 64 x 256
//               operand slice (four TMA boxes of 64 x 64, 128B swizzle) into a 4-stage ring.
//   warp 1      TMEM: two 256-column fp32 accumulators; one lane issues tcgen05.mma M=128 N=256
//               K=16, four per stage (dC: A = G read MN-major as G^T; dE: A = G K-major; B = the
//               slice, MN-major). The shape and the 48 KB per 512 cycles match the forward kernel.
//   warps 2..5  write-out: TMEM -> registers -> swizzled staging -> TMA store (dC, bf16 or fp32)
//               or TMA reduce-add (dE, fp32), while the MMA fills the other accumulator.
#include "cce_device.cuh"
#include "cce_internal.h"

namespace cce {
namespace {

constexpr int BM = kBwdBM;
constexpr int BN = kBwdBN;
constexpr int SLICE = kGemmSlice;  // 256 columns of D per work item
constexpr int STAGES = 4;
constexpr int G_PART = 16384;       // one K-half of the gradient tile
constexpr int X_BOX = 8192;         // 64 rows x 64 bf16
constexpr int STAGE_BYTES = G_PART + 4 * X_BOX;
constexpr int TILE_BYTES = kGradTileBytes;
constexpr int STG_WARP = 8192;    // per epilogue warp: 32 rows x 64 columns of fp32 (or bf16 + unused)
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr int NUM_BARRIERS = 2 * STAGES + 4 + 1;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 4 * STG_WARP + NUM_BARRIERS * 8 + 16;

constexpr uint32_t IDESC_DC = idesc_bf16(BN, SLICE, true, true);   // M = vocab (G^T, MN-major), N = 256 of D
constexpr uint32_t IDESC_DE = idesc_bf16(BM, SLICE, false, true);  // M = rows (G, K-major), N = 256 of D

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

struct ItemRange {
  bool de;                 // dE item (row block key) or dC item (vocabulary tile key)
  int key, s, begin, end;  // entries [begin, end) of the key's list
};

// Items [0, nb * S) are dE items (row block w / S, slice w % S); the rest are dC items (vocabulary
// tile chunk_t0 + (w - nb S) / S). Each gets the range of its list entries inside this chunk: for
// a row block, the plan's range of its entries_b inside the chunk; for a vocabulary tile, all of
// its entries_t (every listed tile of a vocabulary tile lies in the tile's chunk).
__device__ __forceinline__ ItemRange item_in_chunk(int w, int S, int nb, int chunk_t0, const int2* rb_range,
                                                   const int* offsets_t) {
  ItemRange it;
  it.de = w < nb * S;
  if (it.de) {
    it.key = w / S;
    it.s = w % S;
    const int2 r = rb_range[it.key];
    it.begin = r.x;
    it.end = r.y;
  } else {
    const int v = w - nb * S;
    it.key = chunk_t0 + v / S;
    it.s = v % S;
    it.begin = offsets_t[it.key];
    it.end = offsets_t[it.key + 1];
  }
  return it;
}

// Entry i of the item's list -> (tile index of the "other" operand, slot of its gradient tile).
__device__ __forceinline__ int2 entry_of(bool de, const int2* entries_b, const int2* entries_t, int i,
                                         int slot_base) {
  if (de) {
    const int2 en = entries_b[i];
    return make_int2(en.x, en.y - slot_base);  // (vocabulary tile t, slot)
  }
  const int2 en = entries_t[i];
  return make_int2(en.x >> 2, i - slot_base);  // (row block b, slot)
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmC,
                    const __grid_constant__ CUtensorMap tmdC, const __grid_constant__ CUtensorMap tmdE, int N, int D,
                    int V, const int2* __restrict__ entries_t, const int* __restrict__ offsets_t,
                    const int2* __restrict__ entries_b, const int2* __restrict__ rb_range,
                    const int* __restrict__ chunk_t, int chunk, int nb, const uint8_t* __restrict__ gscratch,
                    int out_bf16, int* err, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* stg_all = base + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg_all + 4 * STG_WARP);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NUM_BARRIERS);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int u) { return bar0 + 8u * u; };
  auto empty_bar = [&](int u) { return bar0 + 8u * (STAGES + u); };
  auto accfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto accempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);

  const int S = (D + SLICE - 1) / SLICE;
  const int chunk_t0 = chunk_t[chunk], chunk_t1 = chunk_t[chunk + 1];
  if (chunk_t0 >= chunk_t1) return;  // empty chunk
  const int num_items = (nb + chunk_t1 - chunk_t0) * S;
  if (num_items <= static_cast<int>(blockIdx.x)) return;
  // Each role loads the next item's range before working on the current one.
  auto item = [&](int w) {
    return item_in_chunk(w < num_items ? w : static_cast<int>(blockIdx.x), S, nb, chunk_t0, rb_range, offsets_t);
  };
  const int slot_base = offsets_t[chunk_t0];

  if (threadIdx.x == 0) {
    for (int u = 0; u < STAGES; ++u) {
      mbar_init(full_bar(u), 1);
      mbar_init(empty_bar(u), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accfull_bar(a), 1);
      mbar_init(accempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
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

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES] = {0, 0, 0, 0};
      bool ok = true;
      ItemRange nx = item(blockIdx.x);
      for (int w = blockIdx.x; w < num_items && ok; w += gridDim.x) {
        const ItemRange it = nx;
        nx = item(w + gridDim.x);
        const int x0 = it.s * SLICE;
        int2 os_next = it.begin < it.end ? entry_of(it.de, entries_b, entries_t, it.begin, slot_base) : make_int2(0, 0);
        for (int i = it.begin; i < it.end && ok; ++i) {
          const int2 os = os_next;
          if (i + 1 < it.end) os_next = entry_of(it.de, entries_b, entries_t, i + 1, slot_base);
          const uint8_t* tile = gscratch + static_cast<size_t>(os.y) * TILE_BYTES;
          for (int h = 0; h < 2; ++h) {  // K-halves: 64 rows (dC) or 64 vocabulary columns (dE)
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, wc)) {
              ok = false;
              break;
            }
            const uint32_t dst = smem_u32(stages + stage * STAGE_BYTES);
            mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
            if (it.de) {  // G block h: rows 0..127, vocabulary 64h .. 64h + 63 (K-major A)
              bulk_load(dst, tile + h * G_PART, G_PART, full_bar(stage));
            } else {  // rows 64h .. 64h + 63 of both 64-column vocabulary blocks (MN-major A = G^T)
              bulk_load(dst, tile + h * (G_PART / 2), G_PART / 2, full_bar(stage));
              bulk_load(dst + G_PART / 2, tile + G_PART + h * (G_PART / 2), G_PART / 2, full_bar(stage));
            }
            const int y = os.x * BM + 64 * h;  // K rows of the operand: E_b rows (dC), C_t rows (dE)
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_2d(dst + G_PART + c * X_BOX, it.de ? &tmC : &tmE, full_bar(stage), x0 + 64 * c, y);
            ++issued[stage];
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      if (!ok) {
        for (int u = 0; u < STAGES; ++u)
          if (issued[u]) mbar_wait_drain(full_bar(u), (issued[u] - 1u) & 1u, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      bool ok = true, issued_any = false;
      ItemRange nx = item(blockIdx.x);
      for (int w = blockIdx.x; w < num_items && ok; w += gridDim.x) {
        const ItemRange it = nx;
        nx = item(w + gridDim.x);
        if (it.begin == it.end) continue;  // nothing to accumulate (dC writes zeros without TMEM)
        const int a = acc_iter & 1;
        if (!mbar_wait(accempty_bar(a), ((acc_iter >> 1) & 1u) ^ 1u, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(a * SLICE);
        for (int i = it.begin; i < it.end && ok; ++i) {
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(full_bar(stage), phase, wc)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t g0 = smem_u32(stages + stage * STAGE_BYTES);
            const uint32_t x0 = g0 + G_PART;
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // 16 of the 64 K values per MMA
              const uint64_t adesc = it.de ? sdesc_sw128(g0 + 32u * k, 16, 1024)
                                           : sdesc_sw128(g0 + 2048u * k, G_PART / 2, 1024);
              const uint64_t bdesc = sdesc_sw128(x0 + 2048u * k, X_BOX, 1024);
              tc_mma_bf16(d, adesc, bdesc, it.de ? IDESC_DE : IDESC_DC, (i > it.begin || h > 0 || k > 0) ? 1u : 0u);
            }
            issued_any = true;
            tc_commit(empty_bar(stage));
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        tc_commit(accfull_bar(a));
        ++acc_iter;
      }
      if (!ok && issued_any) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, 200000000ull);
      }
    }
  } else {
    // ---------------- write-out ----------------
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t stg = smem_u32(stg_all + q * STG_WARP);
    uint32_t acc_iter = 0;
    for (int w = blockIdx.x; w < num_items; w += gridDim.x) {
      const ItemRange it = item(w);
      const bool has = it.begin < it.end;
      if (it.de && !has) continue;  // nothing to add for this row block in this chunk
      const int rows_limit = it.de ? N : V;
      const int a = acc_iter & 1;
      if (has) {
        if (!mbar_wait(accfull_bar(a), (acc_iter >> 1) & 1u, wc)) break;
        tc_fence_after();
      }
      const int y = it.key * BM + q * 32;
      for (int p = 0; p < SLICE / 64; ++p) {
        const int x = it.s * SLICE + 64 * p;
        if (x >= D) break;
        float v0[32], v1[32];
        if (has) {
          tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(a * SLICE + 64 * p), v0);
          tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(a * SLICE + 64 * p + 32), v1);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v0[k] = v1[k] = 0.f;
        }
        // This warp's staging is free once its previous TMA op has read it.
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        if (!it.de && out_bf16) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const float* src = h < 4 ? v0 + 8 * h : v1 + 8 * (h - 4);
            st_shared_v4(stg + swz(lane, h), pack_bf16x2(src[0], src[1]), pack_bf16x2(src[2], src[3]),
                         pack_bf16x2(src[4], src[5]), pack_bf16x2(src[6], src[7]));
          }
        } else {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            st_shared_v4(stg + swz(lane, h), __float_as_uint(v0[4 * h]), __float_as_uint(v0[4 * h + 1]),
                         __float_as_uint(v0[4 * h + 2]), __float_as_uint(v0[4 * h + 3]));
            st_shared_v4(stg + 4096u + swz(lane, h), __float_as_uint(v1[4 * h]), __float_as_uint(v1[4 * h + 1]),
                         __float_as_uint(v1[4 * h + 2]), __float_as_uint(v1[4 * h + 3]));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && y < rows_limit) {
          if (!it.de && out_bf16) {
            tma_store_2d(&tmdC, stg, x, y);
          } else if (!it.de) {
            tma_store_2d(&tmdC, stg, x, y);
            if (x + 32 < D) tma_store_2d(&tmdC, stg + 4096u, x + 32, y);
          } else {
            tma_reduce_add_2d(&tmdE, stg, x, y);
            if (x + 32 < D) tma_reduce_add_2d(&tmdE, stg + 4096u, x + 32, y);
          }
          bulk_commit_group();
        }
      }
      if (has) {
        tc_fence_before();
        mbar_arrive(accempty_bar(a));
        ++acc_iter;
      }
    }
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

cudaError_t launch_bwd_gemm(const BwdGemm& L, int chunk, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = L.num_sms;  // CTAs past the chunk's item count exit at once
  bwd_gemm_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(
      L.tmE, L.tmC, L.tmdC, L.tmdE, L.N, L.D, L.V, L.entries_t, L.offsets_t, L.entries_b,
      L.rb_range + static_cast<int64_t>(chunk) * L.nb, L.chunk_t, chunk, L.nb, L.gscratch, L.dC_bf16, L.err,
      L.timeout_ns);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace cce

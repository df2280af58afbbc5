// cce_forward_noalloc: the forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or an allocator of their own at the point where they
// compute the loss: an embedding host that hands this library only fixed, pre-registered buffers
// for inputs and outputs and owns all other device memory itself, or a runtime whose allocator
// must not be re-entered from inside a loss callback (it may hold its own lock there, or account
// every byte against a fixed budget). For them this entry point keeps its scratch (per-sub-tile
// exp sums, target logits, per-row losses and the device error word) in one file-scope device
// array of kNoAllocScratchBytes, which every GPU that loads the library holds until the process
// exits. The caller passes inputs and outputs only.
//
// It launches the same kernels as cce_forward(); only where the scratch lives differs. A device
// error (a target outside [0, V), a bounded wait that ran out) cannot be returned by this call,
// which does not wait for the GPU; the final kernel then writes the loss as NaN instead.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "cce.h"
#include "cce_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = CCE_NOALLOC_SCRATCH_BYTES;
constexpr size_t kHeader = 256;
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode_fn = nullptr;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

cce_status fail(cce_status s, const char* msg) {
  cce::set_last_error(msg);
  return s;
}

// Device address of the scratch array for the current device. The first call on a device looks
// it up (with that device current) and caches it.
cce_status scratch_for_current_device(void** out, int* num_sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(CCE_ERR_CUDA, "cce_forward_noalloc: no usable current CUDA device");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return fail(CCE_ERR_UNSUPPORTED, "cce_forward_noalloc: device is not sm_100 (B200)");
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(CCE_ERR_CUDA, "cce_forward_noalloc: cudaDeviceGetAttribute failed");
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(CCE_ERR_CUDA, "cce_forward_noalloc: cudaGetSymbolAddress failed");
    g_scratch_addr[dev] = ptr;
  }
  if (g_encode_fn == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return fail(CCE_ERR_CUDA, "cce_forward_noalloc: cuTensorMapEncodeTiled unavailable");
    g_encode_fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_scratch_addr[dev];
  return CCE_OK;
}

cce_status encode(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  if (g_encode_fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return fail(CCE_ERR_CUDA, "cce_forward_noalloc: cuTensorMapEncodeTiled failed");
  return CCE_OK;
}

}  // namespace

extern "C" cce_status cce_forward_noalloc(const cce_problem* p, const void* E, const void* C, const void* bias,
                                          const int64_t* targets, float* loss, float* lse, float* tile_max,
                                          int64_t* count, cce_stream_t stream) {
  cce::set_last_error("");
  if (p == nullptr || p->N < 0 || p->D < 8 || p->D % 8 != 0 || p->V < 1 || p->reduction < 0 || p->reduction > 2 ||
      p->reserved != 0 || p->N >= (int64_t(1) << 31) - 256 || p->V >= (int64_t(1) << 31) - 256 ||
      p->D >= (int64_t(1) << 24) || !(p->label_smoothing >= 0.f && p->label_smoothing <= 1.f) ||
      !(p->z_loss >= 0.f && p->z_loss < INFINITY) || p->vocab_start != 0 ||
      (p->vocab_total != 0 && p->vocab_total != p->V))
    return fail(CCE_ERR_INVALID_ARG, "cce_forward_noalloc: invalid problem (or a vocabulary shard)");
  const int64_t N = p->N, D = p->D, V = p->V;
  const int64_t T = (V + cce::kSubTile - 1) / cce::kSubTile;
  if (C == nullptr || loss == nullptr || count == nullptr ||
      (N > 0 && (E == nullptr || targets == nullptr || lse == nullptr || tile_max == nullptr)))
    return fail(CCE_ERR_INVALID_ARG, "cce_forward_noalloc: a required pointer is NULL");
  if ((reinterpret_cast<uintptr_t>(E) | reinterpret_cast<uintptr_t>(C) | reinterpret_cast<uintptr_t>(bias)) & 15u)
    return fail(CCE_ERR_INVALID_ARG, "cce_forward_noalloc: E, C and bias must be 16-byte aligned");
  // Same layout as the forward workspace: header (error word, finish counter) | tile_sum [T, N] |
  // zt [N] (correct-token logits) | csum [D + 1] (label smoothing) | per-block loss sums and counts
  // of the finish kernel.
  const size_t nblk = static_cast<size_t>(N > 0 ? (N + cce::kFinishRows - 1) / cce::kFinishRows : 1);
  const size_t off_sum = kHeader;
  const size_t off_zt = up(off_sum + sizeof(float) * static_cast<size_t>(T * N));
  const size_t off_csum = up(off_zt + sizeof(float) * static_cast<size_t>(N));
  const size_t off_bsum = up(off_csum + sizeof(float) * static_cast<size_t>(D + 1));
  const size_t off_bcnt = up(off_bsum + sizeof(double) * nblk);
  const size_t need = up(off_bcnt + sizeof(long long) * nblk);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "cce_forward_noalloc: this problem needs %zu bytes of scratch, more than the %zu bytes the library "
             "holds for allocation-free calls (about ceil(V/64) * N * 4 bytes); use cce_forward with a workspace",
             need, kNoAllocScratchBytes);
    return fail(CCE_ERR_UNSUPPORTED, msg);
  }
  void* base = nullptr;
  int num_sms = 0;
  cce_status st = scratch_for_current_device(&base, &num_sms);
  if (st != CCE_OK) return st;
  char* b = static_cast<char*>(base);
  int* err = reinterpret_cast<int*>(b);
  int* done = err + 1;
  float* tile_sum = reinterpret_cast<float*>(b + off_sum);
  float* zt = reinterpret_cast<float*>(b + off_zt);
  float* csum = reinterpret_cast<float*>(b + off_csum);
  const bool smooth = p->label_smoothing > 0.f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* Cb = static_cast<const __nv_bfloat16*>(C);
  const auto* Bb = static_cast<const __nv_bfloat16*>(bias);

  // The array keeps the previous call's contents: the error word and the finish kernel's counter must
  // start at zero; every other scratch value is written before it is read.
  if (cudaMemsetAsync(err, 0, kHeader, s) != cudaSuccess) return fail(CCE_ERR_CUDA, "cce_forward_noalloc: memset");
  if (N > 0) {
    cce::FwdLaunch L{};
    if ((st = encode(&L.tmE, E, N, D, cce::kFwdBM)) != CCE_OK) return st;
    if ((st = encode(&L.tmC, C, V, D, cce::kFwdBN)) != CCE_OK) return st;
    L.N = static_cast<int>(N);
    L.D = static_cast<int>(D);
    L.V = static_cast<int>(V);
    L.T = static_cast<int>(T);
    L.tile_max = tile_max;
    L.tile_sum = tile_sum;
    L.targets = targets;
    L.vs = 0;
    L.ignore_index = p->ignore_index;
    L.zt = zt;
    L.err = err;
    L.timeout_ns = cce::wait_timeout_ns();
    L.num_sms = num_sms;
    L.inject_stall = 0;
    L.bias = Bb;
    if ((smooth && cce::launch_weighted_colsum(Cb, V, D, nullptr, Bb, csum, s) != cudaSuccess) ||
        cce::launch_fwd_lse(L, s) != cudaSuccess)
      return fail(CCE_ERR_CUDA, "cce_forward_noalloc: kernel launch failed");
  }
  cce::FwdFinish F{};
  F.tile_max = tile_max;
  F.tile_sum = tile_sum;
  F.N = N;
  F.T = T;
  F.D = D;
  F.V = V;
  F.vs = 0;
  F.vtot = V;
  F.ignore_index = p->ignore_index;
  F.E = static_cast<const __nv_bfloat16*>(E);
  F.targets = targets;
  F.zt = zt;
  F.csum = smooth ? csum : nullptr;
  F.label_smoothing = p->label_smoothing;
  F.z_loss = p->z_loss;
  F.lse = lse;
  F.loss = loss;
  F.reduction = p->reduction;
  F.count = count;
  F.block_sums = reinterpret_cast<double*>(b + off_bsum);
  F.block_counts = reinterpret_cast<long long*>(b + off_bcnt);
  F.done = done;
  F.err = err;
  if (cce::launch_fwd_finish(F, N > 0, s) != cudaSuccess)
    return fail(CCE_ERR_CUDA, "cce_forward_noalloc: kernel launch failed");
  return CCE_OK;
}

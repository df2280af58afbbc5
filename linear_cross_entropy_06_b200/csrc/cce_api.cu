// The C ABI of libcce.so (declared in include/cce.h): argument checks, workspace carving, TMA
// descriptor encoding and the launch sequence of each call. Host code only.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>

#include "cce.h"
#include "cce_internal.h"

namespace {

constexpr int32_t kVersion = 500;  // 0.5.0: the skip rule on 128 x 64 units (saved maxima per 64 columns)
constexpr size_t kHeaderBytes = 256;
constexpr size_t kAlign = 256;

thread_local std::string g_last_error;
thread_local int64_t g_launches = 0;
thread_local cudaEvent_t g_fwd_ev[2] = {nullptr, nullptr};
thread_local cudaEvent_t g_bwd_ev[2] = {nullptr, nullptr};

cce_status fail(cce_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

cce_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CCE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Layout of the area at the start of every workspace (zeroed by every call).
struct WsHeader {
  int err;   // device error word
  int done;  // blocks of the forward's finish kernel that are done
  int bar;   // grid barrier counter of the backward's planning launch
};

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Size of the whole vocabulary: the classifier's rows, or vocab_total for a shard of it.
int64_t vocab_total(const cce_problem* p) { return p->vocab_total > 0 ? p->vocab_total : p->V; }

bool sharded(const cce_problem* p) { return p->vocab_total > 0 && p->vocab_total != p->V; }

// Output dtypes of cce_backward's out_fp32 argument (CCE_OUT_*).
bool de_fp32(int32_t out) { return out == CCE_OUT_FP32 || out == CCE_OUT_DE_FP32; }
bool dc_fp32(int32_t out) { return out == CCE_OUT_FP32; }

bool problem_ok(const cce_problem* p, bool set_error) {
  auto bad = [&](const char* msg) {
    if (set_error) fail(CCE_ERR_INVALID_ARG, "%s", msg);
    return false;
  };
  if (p == nullptr) return bad("problem is NULL");
  if (p->N < 0) return bad("N must be >= 0");
  if (p->D < 8 || p->D % 8 != 0) return bad("D must be a positive multiple of 8");
  if (p->V < 1) return bad("V must be >= 1");
  if (p->reduction < 0 || p->reduction > 2) return bad("reduction must be 0 (none), 1 (mean) or 2 (sum)");
  if (p->reserved != 0) return bad("reserved must be 0");
  if (!(p->label_smoothing >= 0.f && p->label_smoothing <= 1.f)) return bad("label_smoothing must be in [0, 1]");
  if (!(p->z_loss >= 0.f && p->z_loss < INFINITY)) return bad("z_loss must be finite and >= 0");
  if (p->vocab_total < 0) return bad("vocab_total must be >= 0");
  if (p->vocab_total == 0 && p->vocab_start != 0) return bad("vocab_start must be 0 when vocab_total is 0");
  if (p->vocab_total > 0 && (p->vocab_start < 0 || p->vocab_start > p->vocab_total - p->V))
    return bad("a vocabulary shard needs 0 <= vocab_start and vocab_start + V <= vocab_total");
  if (p->vocab_total >= (int64_t(1) << 31) - 256) return bad("vocab_total too large");
  // Kernel indices are 32-bit for rows and tiles; keep every count well inside that.
  if (p->N >= (int64_t(1) << 31) - 256 || p->V >= (int64_t(1) << 31) - 256 || p->D >= (int64_t(1) << 24))
    return bad("N, V or D too large");
  // (a tile's gradient slot shares a 32-bit word with its kept halves)
  if (ceil_div(p->N, cce::kBwdBM) * ceil_div(p->V, cce::kBwdBN) >= (int64_t(1) << cce::kSlotBits))
    return bad("too many backward tiles");
  return true;
}

struct FwdWs {
  WsHeader* hdr;
  float* tile_sum;           // [T, N]
  float* zt;                 // [N]: correct-token logits picked by the forward kernel
  float* csum;               // [D + 1]: column sums of C and the bias sum (label smoothing only)
  double* block_sums;        // [ceil(N / 32)]: per-block loss sums of the finish kernel
  long long* block_counts;   // [ceil(N / 32)]
  size_t bytes;
};

FwdWs carve_fwd(const cce_problem* p, void* base) {
  const int64_t T = ceil_div(p->V, cce::kSubTile);
  const size_t nblk = static_cast<size_t>(std::max<int64_t>(ceil_div(p->N, cce::kFinishRows), 1));
  FwdWs w{};
  size_t off = kHeaderBytes;
  char* b = static_cast<char*>(base);
  w.hdr = reinterpret_cast<WsHeader*>(b);
  w.tile_sum = reinterpret_cast<float*>(b + off);
  off = align_up(off + sizeof(float) * static_cast<size_t>(T * p->N));
  w.zt = reinterpret_cast<float*>(b + off);
  off = align_up(off + sizeof(float) * static_cast<size_t>(p->N));
  w.csum = reinterpret_cast<float*>(b + off);
  off = align_up(off + sizeof(float) * static_cast<size_t>(p->D + 1));
  w.block_sums = reinterpret_cast<double*>(b + off);
  off = align_up(off + sizeof(double) * nblk);
  w.block_counts = reinterpret_cast<long long*>(b + off);
  off = align_up(off + sizeof(long long) * nblk);
  w.bytes = off;
  return w;
}

// The finish kernel's arguments common to the whole-vocabulary and the shard forward.
cce::FwdFinish finish_args(const cce_problem* p, const FwdWs& w, const void* E, const int64_t* targets,
                           const float* tile_max, bool smooth) {
  cce::FwdFinish F{};
  F.tile_max = tile_max;
  F.tile_sum = w.tile_sum;
  F.N = p->N;
  F.T = ceil_div(p->V, cce::kSubTile);
  F.D = p->D;
  F.V = p->V;
  F.vs = p->vocab_start;
  F.vtot = vocab_total(p);
  F.ignore_index = p->ignore_index;
  F.E = static_cast<const __nv_bfloat16*>(E);
  F.targets = targets;
  F.zt = w.zt;
  F.csum = smooth ? w.csum : nullptr;
  F.label_smoothing = p->label_smoothing;
  F.z_loss = p->z_loss;
  F.reduction = p->reduction;
  F.block_sums = w.block_sums;
  F.block_counts = w.block_counts;
  F.done = &w.hdr->done;
  F.err = &w.hdr->err;
  return F;
}

// Workspace of the backward: the tile plan and work lists, the queue counters, two gradient-tile
// buffers (one vocabulary chunk each) and the fp32 dE accumulator. dC needs no accumulator: each
// vocabulary tile's rows are summed in TMEM and written once.
struct SplitWs {
  WsHeader* hdr;
  float* scale;
  cce::BwdPlan plan;
  int* sync;         // [1 + nchunks * nb + nt + nchunks]: queue position, then the counters
  size_t sync_bytes;
  uint8_t* gscratch; // kGradBuffers * buf_bytes
  size_t buf_bytes;
  float* dE_acc;
  float* dbias_acc;  // [V] fp32 (absent when dbias is written in fp32)
  float* csum;       // [D + 1]: column sums of C (label smoothing only)
  float* wsum;       // [D + 1]: sum_r scale_r E_r and sum_r scale_r (label smoothing only)
  void* zero_half;   // [kZeroHalfBytes]: zeros read in place of a skipped half
  size_t bytes;
};

SplitWs carve_split(const cce_problem* p, int32_t out_fp32, void* base) {
  const int64_t nb = ceil_div(p->N, cce::kBwdBM), nt = ceil_div(p->V, cce::kBwdBN);
  const int64_t tiles = nb * nt;
  SplitWs w{};
  char* b = static_cast<char*>(base);
  size_t off = kHeaderBytes;
  auto take = [&](size_t bytes) {
    char* ptr = b + off;
    off = align_up(off + bytes);
    return ptr;
  };
  w.hdr = reinterpret_cast<WsHeader*>(b);
  w.scale = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(p->N)));
  w.plan.nb = static_cast<int>(nb);
  w.plan.nt = static_cast<int>(nt);
  w.plan.flags = reinterpret_cast<uint8_t*>(take(static_cast<size_t>(tiles)));
  w.plan.rank = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(tiles)));
  w.plan.cnt_t = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.offsets_t = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt + 1)));
  w.plan.entries_t = reinterpret_cast<int2*>(take(sizeof(int2) * static_cast<size_t>(tiles)));
  w.plan.cnt_b = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nb)));
  w.plan.offsets_b = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nb + 1)));
  w.plan.entries_b = reinterpret_cast<int2*>(take(sizeof(int2) * static_cast<size_t>(tiles)));
  w.plan.pos_b = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(tiles)));
  w.plan.cnt_hb = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nb)));
  w.plan.off_hb = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nb + 1)));
  w.plan.hp_b = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(tiles + 1)));
  w.zero_half = take(cce::kZeroHalfBytes);
  w.plan.kept_total = reinterpret_cast<int*>(take(2 * sizeof(int)));
  w.plan.n_empty = w.plan.kept_total + 1;
  // A chunk spans at most kChunkCBytes of C (the trade-off between dE's split-reduce passes and
  // re-reads of C), and the gradient tiles of kGradBuffers chunks, at most nb per vocabulary tile,
  // fit in the scratch budget; at least one vocabulary tile per chunk.
  const int64_t vt_bytes = static_cast<int64_t>(cce::kBwdBN) * p->D * 2;
  const int64_t per_vtile = std::max<int64_t>(nb, 1) * cce::kGradTileBytes;
  const int64_t budget = std::max(cce::kGradScratchMin, nb * cce::kGradScratchPerRowBlock);
  const int64_t chunk_vt =
      std::max<int64_t>(1, std::min({nt, cce::kChunkCBytes / vt_bytes, budget / cce::kGradBuffers / per_vtile}));
  w.plan.chunk_vt = static_cast<int>(chunk_vt);
  w.plan.nchunks = static_cast<int>(ceil_div(nt, chunk_vt));
  w.plan.chunk_c_tiles = std::max<int64_t>(1, cce::kChunkCBytes / vt_bytes);
  w.plan.chunk_g_tiles = static_cast<int64_t>(nb) * chunk_vt;
  w.plan.nchunks_dev = reinterpret_cast<int*>(take(sizeof(int)));
  w.plan.chunk_of = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.chunk_t = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(w.plan.nchunks + 1)));
  w.plan.rb_range = reinterpret_cast<int2*>(take(sizeof(int2) * static_cast<size_t>(w.plan.nchunks) * nb));
  w.plan.pstart_t = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt + 1)));
  // a row block with k kept halves (at most 2 per listed tile) in a chunk forms ceil(k / 4) quads there
  const size_t quads = static_cast<size_t>(tiles / 2 + static_cast<int64_t>(w.plan.nchunks) * nb + 1);
  w.plan.quad_b = reinterpret_cast<int*>(take(sizeof(int) * quads));
  w.plan.quad_h = reinterpret_cast<int4*>(take(sizeof(int4) * quads));
  w.plan.quad_s = reinterpret_cast<int4*>(take(sizeof(int4) * quads));
  w.plan.cnt_ht = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.S = static_cast<int>(ceil_div(p->D, cce::kGemmSlice));
  w.plan.grp_size = reinterpret_cast<int*>(take(sizeof(int) * 2 * static_cast<size_t>(w.plan.nchunks)));
  w.plan.grp_start = reinterpret_cast<int*>(take(sizeof(int) * (2 * static_cast<size_t>(w.plan.nchunks) + 1)));
  w.plan.vt_order = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.ndc = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(w.plan.nchunks)));
  w.plan.de_list = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(w.plan.nchunks) * nb));
  w.plan.nde = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(w.plan.nchunks)));
  w.plan.empty_list = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.oh_cnt = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.oh_cur = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt)));
  w.plan.oh_off = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(nt + 1)));
  w.plan.oh_rows = reinterpret_cast<int*>(take(sizeof(int) * static_cast<size_t>(std::max<int64_t>(p->N, 1))));
  w.sync_bytes = sizeof(int) * static_cast<size_t>(1 + w.plan.nchunks * nb + nt + w.plan.nchunks);
  w.sync = reinterpret_cast<int*>(take(w.sync_bytes));
  w.buf_bytes = static_cast<size_t>(nb * chunk_vt) * cce::kGradTileBytes;
  w.gscratch = reinterpret_cast<uint8_t*>(take(cce::kGradBuffers * w.buf_bytes));
  if (!de_fp32(out_fp32)) w.dE_acc = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(p->N * p->D)));
  if (!dc_fp32(out_fp32)) w.dbias_acc = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(p->V)));
  w.csum = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(p->D + 1)));
  w.wsum = reinterpret_cast<float*>(take(sizeof(float) * static_cast<size_t>(p->D + 1)));
  w.bytes = off;
  return w;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// ---------------------------------------------------------------------------------------------
// Device checks and TMA descriptors
// ---------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cce_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return fail(CCE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  return CCE_OK;
}

cce_status check_device(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(CCE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev, major,
                minor);
  e = cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  return CCE_OK;
}

// 2-D row-major tensor [rows, cols] with contiguous rows, box [box_rows, box_cols], 128B swizzle.
cce_status make_map(CUtensorMap* map, CUtensorMapDataType dtype, size_t elem, const void* ptr, int64_t rows,
                    int64_t cols, uint32_t box_cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CCE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return CCE_OK;
}

#define CCE_TRY(expr)                                \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_, #expr); \
  } while (0)

#define CCE_CHECK(expr)            \
  do {                             \
    cce_status s_ = (expr);        \
    if (s_ != CCE_OK) return s_;   \
  } while (0)


// The backward: plan the tiles and work lists, then one persistent launch (cce_bwd.cu) forms the
// gradient tiles chunk by chunk and runs the dC and dE MMAs from them.
cce_status backward_split(const cce_problem* p, const void* E, const void* C, const void* bias, const int64_t* targets,
                          const float* lse, const float* tile_max, const int64_t* count, const float* grad_out,
                          float filter_eps, void* dE, void* dC, void* dbias, int32_t out_fp32,
                          int64_t* filtered_tiles, void* workspace, size_t workspace_bytes, cudaStream_t s) {
  const SplitWs w = carve_split(p, out_fp32, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CCE_ERR_WORKSPACE, "backward workspace is %zu bytes, needs %zu", workspace_bytes, w.bytes);
  int num_sms = 0;
  CCE_CHECK(check_device(&num_sms));
  CCE_CHECK(get_encoder());
  const int64_t N = p->N, D = p->D, V = p->V, T = ceil_div(V, cce::kSubTile);
  const bool e32 = de_fp32(out_fp32), c32 = dc_fp32(out_fp32);
  const int64_t vs = p->vocab_start, vtot = vocab_total(p);
  float* dE_acc = e32 ? static_cast<float*>(dE) : w.dE_acc;
  float* dbias_acc = dbias == nullptr ? nullptr : (c32 ? static_cast<float*>(dbias) : w.dbias_acc);

  CCE_TRY(cudaMemsetAsync(w.hdr, 0, sizeof(WsHeader), s));
  if (N == 0) {  // no rows: dC = 0 (and dbias = 0)
    CCE_TRY(cce::launch_fill_zero(dC, V * D * (c32 ? 4 : 2), s));
    if (dbias != nullptr) CCE_TRY(cce::launch_fill_zero(dbias, V * (c32 ? 4 : 2), s));
    return cudaMemsetAsync(filtered_tiles, 0, sizeof(int64_t), s) == cudaSuccess ? CCE_OK
                                                                                  : fail(CCE_ERR_CUDA, "memset");
  }
  {
    cce::PlanArgs PA{};
    PA.sync = w.sync;
    PA.sync_ints = static_cast<int64_t>(w.sync_bytes / sizeof(int));
    PA.P = w.plan;
    PA.tile_max = tile_max;
    PA.lse = lse;
    PA.targets = targets;
    PA.count = count;
    PA.grad_out = grad_out;
    PA.N = N;
    PA.D = D;
    PA.V = V;
    PA.T = T;
    PA.vs = vs;
    PA.vtot = vtot;
    PA.ignore_index = p->ignore_index;
    PA.reduction = p->reduction;
    PA.filter_on = filter_eps > 0.f ? 1 : 0;
    PA.ln_eps = PA.filter_on ? logf(filter_eps) : -INFINITY;
    PA.scale = w.scale;
    PA.onehot_coef = 1.f - p->label_smoothing;
    PA.dE_acc = dE_acc;
    PA.dbias_acc = dbias_acc;
    PA.zero_half = w.zero_half;
    PA.filtered_tiles = filtered_tiles;
    PA.bar = &w.hdr->bar;
    PA.err = &w.hdr->err;
    PA.timeout_ns = cce::wait_timeout_ns();
    // Failure-detection test hook: CCE_TEST_INJECT_STALL=3 makes the planning launch's first grid
    // barrier wait run out (reported as CCE_ERR_DEVICE_TIMEOUT; the backward then hands out no work).
    const char* stall = std::getenv("CCE_TEST_INJECT_STALL");
    PA.inject_stall = (stall != nullptr && stall[0] == '3') ? 1 : 0;
    CCE_TRY(cce::launch_bwd_plan(PA, num_sms, s));
  }
  // Label smoothing: the ls / V part of every row's target is a rank-one term, added exactly:
  // dE_r -= scale_r (ls / V) sum_v C_v, dC_v -= (ls / V) sum_r scale_r E_r, dbias_v -= (ls / V) sum_r scale_r.
  const bool smooth = p->label_smoothing > 0.f;
  const float ls_v = p->label_smoothing / static_cast<float>(vtot);
  const auto* Eb = static_cast<const __nv_bfloat16*>(E);
  if (smooth) {
    CCE_TRY(cce::launch_weighted_colsum(static_cast<const __nv_bfloat16*>(C), V, D, nullptr, nullptr, w.csum, s));
    CCE_TRY(cce::launch_weighted_colsum(Eb, N, D, w.scale, nullptr, w.wsum, s));
  }

  cce::BwdLaunch L{};
  CCE_CHECK(make_map(&L.tmE128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, D, 64, cce::kBwdBM));
  CCE_CHECK(make_map(&L.tmC128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, V, D, 64, cce::kSubTile));
  // The dE / dC items load a 64-row x 256-column operand slice per stage. With D a multiple of 256
  // it is one 3-D TMA load (64 columns x 64 rows x 4 column blocks: the same shared-memory image as
  // four 64 x 64 boxes); otherwise four 2-D boxes (the last slice of D may be partial).
  const bool slab3d = D % 256 == 0;
  if (slab3d) {
    auto map3 = [&](CUtensorMap* m, const void* ptr, int64_t rows) {
      cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(D / 64)};
      cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, 128};
      cuuint32_t box[3] = {64, 64, 4};
      cuuint32_t estr[3] = {1, 1, 1};
      CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      return r == CUDA_SUCCESS ? CCE_OK
                               : fail(CCE_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", static_cast<int>(r));
    };
    CCE_CHECK(map3(&L.tmE64, E, N));
    CCE_CHECK(map3(&L.tmC64, C, V));
  } else {
    CCE_CHECK(make_map(&L.tmE64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, D, 64, 64));
    CCE_CHECK(make_map(&L.tmC64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, V, D, 64, 64));
  }
  CCE_CHECK(make_map(&L.tmdE, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dE_acc, N, D, 32, 32));
  if (c32) CCE_CHECK(make_map(&L.tmdC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, dC, V, D, 32, 32));
  else CCE_CHECK(make_map(&L.tmdC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dC, V, D, 64, 32));
  cce::BwdArgs& A = L.args;
  A.N = static_cast<int>(N);
  A.D = static_cast<int>(D);
  A.V = static_cast<int>(V);
  A.nb = w.plan.nb;
  A.nt = w.plan.nt;
  A.S = w.plan.S;
  A.nchunks = w.plan.nchunks_dev;
  A.out_bf16 = c32 ? 0 : 1;
  A.slab3d = slab3d ? 1 : 0;
  A.ignore_index = p->ignore_index;
  A.vocab_start = vs;
  A.buf_bytes = w.buf_bytes;
  A.lse = lse;
  A.scale = w.scale;
  A.targets = targets;
  A.bias = static_cast<const __nv_bfloat16*>(bias);
  A.dbias = dbias_acc;
  A.z_loss = p->z_loss;
  A.onehot_coef = 1.f - p->label_smoothing;
  A.dc_add = smooth ? w.wsum : nullptr;
  A.dc_coef = -ls_v;
  A.E = Eb;
  A.oh_off = w.plan.oh_off;
  A.oh_rows = w.plan.oh_rows;
  A.grp_start = w.plan.grp_start;
  A.vt_order = w.plan.vt_order;
  A.ndc = w.plan.ndc;
  A.de_list = w.plan.de_list;
  A.nde = w.plan.nde;
  A.chunk_t = w.plan.chunk_t;
  A.pstart_t = w.plan.pstart_t;
  A.quad_b = w.plan.quad_b;
  A.quad_h = w.plan.quad_h;
  A.quad_s = w.plan.quad_s;
  A.cnt_ht = w.plan.cnt_ht;
  A.rb_range = w.plan.rb_range;
  A.offsets_t = w.plan.offsets_t;
  A.entries_t = w.plan.entries_t;
  A.entries_b = w.plan.entries_b;
  A.hp_b = w.plan.hp_b;
  A.zero_half = w.zero_half;
  A.gscratch = w.gscratch;
  A.qctr = w.sync;
  A.counters = w.sync + 1;
  A.ctr_g_b = 0;
  A.ctr_g_t = w.plan.nchunks * w.plan.nb;
  A.ctr_b_done = A.ctr_g_t + w.plan.nt;
  A.err = &w.hdr->err;
  A.timeout_ns = cce::wait_timeout_ns();
  // Failure-detection test hook: CCE_TEST_INJECT_STALL=2 makes the backward's dE items of the first
  // chunk wait for a gradient tile that is never stored (reported as CCE_ERR_DEVICE_TIMEOUT).
  const char* stall = std::getenv("CCE_TEST_INJECT_STALL");
  A.inject_stall = (stall != nullptr && stall[0] == '2') ? 1 : 0;
  L.num_sms = num_sms;

  if (g_bwd_ev[0] && g_bwd_ev[1]) CCE_TRY(cudaEventRecord(g_bwd_ev[0], s));
  // launches that overlap the previous kernel's tail, unless a timing event sits between them
  const bool timed = g_bwd_ev[0] && g_bwd_ev[1];
  CCE_TRY(cce::launch_bwd(L, !timed, s));
  if (g_bwd_ev[0] && g_bwd_ev[1]) CCE_TRY(cudaEventRecord(g_bwd_ev[1], s));
  // the rest: dC rows of vocabulary tiles no row block lists, then dE's last terms and conversion,
  // and dbias
  cce::BwdFinalize F{};
  F.N = N;
  F.D = D;
  F.V = V;
  F.vs = vs;
  F.ignore_index = p->ignore_index;
  F.nt = w.plan.nt;
  F.flags = w.plan.flags;
  F.empty_list = w.plan.empty_list;
  F.n_empty = w.plan.n_empty;
  F.oh_off = w.plan.oh_off;
  F.oh_rows = w.plan.oh_rows;
  F.targets = targets;
  F.scale = w.scale;
  F.onehot_coef = 1.f - p->label_smoothing;
  F.ls_v = ls_v;
  F.E = Eb;
  F.C = static_cast<const __nv_bfloat16*>(C);
  F.csum = smooth ? w.csum : nullptr;
  F.wsum = smooth ? w.wsum : nullptr;
  F.dE_acc = dE_acc;
  F.dE_out = e32 ? nullptr : dE;
  F.dC = dC;
  F.dc_bf16 = c32 ? 0 : 1;
  F.dbias_acc = dbias_acc;
  F.dbias_out = (dbias != nullptr && !c32) ? dbias : nullptr;
  CCE_TRY(cce::launch_empty_tiles(F, num_sms, !timed, s));
  CCE_TRY(cce::launch_bwd_finalize(F, num_sms, s));
  return CCE_OK;
}

}  // namespace

namespace cce {
void note_launches(int n) { g_launches += n; }
uint64_t wait_timeout_ns() {
  const char* s = std::getenv("CCE_WAIT_TIMEOUT_MS");
  double ms = s ? std::atof(s) : 4000.0;
  if (!(ms > 0)) ms = 4000.0;
  return static_cast<uint64_t>(ms * 1e6);
}
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace cce

extern "C" {

void cce_set_kernel_events(void* fwd_start, void* fwd_stop, void* bwd_start, void* bwd_stop) {
  g_fwd_ev[0] = static_cast<cudaEvent_t>(fwd_start);
  g_fwd_ev[1] = static_cast<cudaEvent_t>(fwd_stop);
  g_bwd_ev[0] = static_cast<cudaEvent_t>(bwd_start);
  g_bwd_ev[1] = static_cast<cudaEvent_t>(bwd_stop);
}

int64_t cce_kernel_launch_count(void) { return g_launches; }


int32_t cce_version(void) { return kVersion; }

const char* cce_status_string(cce_status s) {
  switch (s) {
    case CCE_OK: return "ok";
    case CCE_ERR_INVALID_ARG: return "invalid argument";
    case CCE_ERR_UNSUPPORTED: return "unsupported device or size";
    case CCE_ERR_WORKSPACE: return "workspace too small";
    case CCE_ERR_TARGET_RANGE: return "target outside [0, V) and not ignore_index";
    case CCE_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case CCE_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* cce_last_error_message(void) { return g_last_error.c_str(); }

int64_t cce_tile_max_len(const cce_problem* p) {
  if (!problem_ok(p, false)) return -1;
  return ceil_div(p->V, cce::kSubTile) * p->N;
}

void cce_backward_tile_shape(int32_t* tile_rows, int32_t* tile_cols) {
  if (tile_rows) *tile_rows = cce::kBwdBM;
  if (tile_cols) *tile_cols = cce::kSubTile;
}

size_t cce_forward_workspace_size(const cce_problem* p) {
  if (!problem_ok(p, false)) return 0;
  return carve_fwd(p, nullptr).bytes;
}

size_t cce_backward_workspace_size(const cce_problem* p, int32_t out_fp32) {
  if (!problem_ok(p, false) || out_fp32 < CCE_OUT_BF16 || out_fp32 > CCE_OUT_DE_FP32) return 0;
  return carve_split(p, out_fp32, nullptr).bytes;
}

cce_status cce_forward(const cce_problem* p, const void* E, const void* C, const void* bias, const int64_t* targets,
                       float* loss, float* lse, float* tile_max, int64_t* count, void* workspace,
                       size_t workspace_bytes, cce_stream_t stream) {
  g_last_error.clear();
  if (!problem_ok(p, true)) return CCE_ERR_INVALID_ARG;
  if (sharded(p))
    return fail(CCE_ERR_INVALID_ARG, "a vocabulary shard's loss needs every shard: use cce_forward_partial and "
                                     "cce_forward_merge");
  const bool has_rows = p->N > 0;
  if (C == nullptr || loss == nullptr || count == nullptr || workspace == nullptr ||
      (has_rows && (E == nullptr || targets == nullptr || lse == nullptr || tile_max == nullptr)))
    return fail(CCE_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(E) || !aligned16(C) || !aligned16(bias) || !aligned16(workspace))
    return fail(CCE_ERR_INVALID_ARG, "E, C, bias and workspace must be 16-byte aligned");
  const FwdWs w = carve_fwd(p, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CCE_ERR_WORKSPACE, "forward workspace is %zu bytes, needs %zu", workspace_bytes, w.bytes);
  int num_sms = 0;
  CCE_CHECK(check_device(&num_sms));
  CCE_CHECK(get_encoder());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = p->N, D = p->D, V = p->V, T = ceil_div(V, cce::kSubTile);
  const auto* Cb = static_cast<const __nv_bfloat16*>(C);
  const auto* Bb = static_cast<const __nv_bfloat16*>(bias);

  CCE_TRY(cudaMemsetAsync(w.hdr, 0, sizeof(WsHeader), s));
  const bool smooth = p->label_smoothing > 0.f;
  if (has_rows) {
    cce::FwdLaunch L{};
    L.bias = Bb;
    CCE_CHECK(make_map(&L.tmE, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, D, 64, cce::kFwdBM));
    CCE_CHECK(make_map(&L.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, V, D, 64, cce::kFwdBN));
    L.N = static_cast<int>(N);
    L.D = static_cast<int>(D);
    L.V = static_cast<int>(V);
    L.T = static_cast<int>(T);
    L.tile_max = tile_max;
    L.tile_sum = w.tile_sum;
    L.targets = targets;
    L.vs = 0;
    L.ignore_index = p->ignore_index;
    L.zt = w.zt;
    L.err = &w.hdr->err;
    L.timeout_ns = cce::wait_timeout_ns();
    L.num_sms = num_sms;
    // Failure-detection test hook: CCE_TEST_INJECT_STALL=1 makes the forward's bounded wait run out
    // (reported as CCE_ERR_DEVICE_TIMEOUT by cce_check_device_error; the outputs are undefined).
    const char* stall = std::getenv("CCE_TEST_INJECT_STALL");
    L.inject_stall = (stall != nullptr && stall[0] == '1') ? 1 : 0;
    if (smooth) CCE_TRY(cce::launch_weighted_colsum(Cb, V, D, nullptr, Bb, w.csum, s));
    if (g_fwd_ev[0] && g_fwd_ev[1]) CCE_TRY(cudaEventRecord(g_fwd_ev[0], s));
    CCE_TRY(cce::launch_fwd_lse(L, s));
    if (g_fwd_ev[0] && g_fwd_ev[1]) CCE_TRY(cudaEventRecord(g_fwd_ev[1], s));
  }
  cce::FwdFinish F = finish_args(p, w, E, targets, tile_max, smooth);
  F.lse = lse;
  F.loss = loss;
  F.count = count;
  // overlap the finish's launch with the tensor-core kernel's tail, unless a timing event sits between
  CCE_TRY(cce::launch_fwd_finish(F, has_rows && !(g_fwd_ev[0] && g_fwd_ev[1]), s));
  return CCE_OK;
}

cce_status cce_backward(const cce_problem* p, const void* E, const void* C, const void* bias, const int64_t* targets,
                        const float* lse, const float* tile_max, const int64_t* count, const float* grad_out,
                        float filter_eps, void* dE, void* dC, void* dbias, int32_t out_fp32,
                        int64_t* filtered_tiles, void* workspace, size_t workspace_bytes, cce_stream_t stream) {
  g_last_error.clear();
  if (!problem_ok(p, true)) return CCE_ERR_INVALID_ARG;
  const bool has_rows = p->N > 0;
  if (C == nullptr || dC == nullptr || count == nullptr || filtered_tiles == nullptr || workspace == nullptr ||
      (has_rows && (E == nullptr || targets == nullptr || lse == nullptr || tile_max == nullptr || dE == nullptr ||
                    grad_out == nullptr)))
    return fail(CCE_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(E) || !aligned16(C) || !aligned16(bias) || !aligned16(dE) || !aligned16(dC) ||
      !aligned16(dbias) || !aligned16(workspace))
    return fail(CCE_ERR_INVALID_ARG, "E, C, bias, dE, dC, dbias and workspace must be 16-byte aligned");
  if (std::isnan(filter_eps)) return fail(CCE_ERR_INVALID_ARG, "filter_eps is NaN");
  if (out_fp32 < CCE_OUT_BF16 || out_fp32 > CCE_OUT_DE_FP32)
    return fail(CCE_ERR_INVALID_ARG, "out_fp32 must be CCE_OUT_BF16, CCE_OUT_FP32 or CCE_OUT_DE_FP32");
  return backward_split(p, E, C, bias, targets, lse, tile_max, count, grad_out, filter_eps, dE, dC, dbias, out_fp32,
                        filtered_tiles, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

cce_status cce_forward_partial(const cce_problem* p, const void* E, const void* C, const void* bias,
                               const int64_t* targets, float* partial, float* tile_max, void* workspace,
                               size_t workspace_bytes, cce_stream_t stream) {
  g_last_error.clear();
  if (!problem_ok(p, true)) return CCE_ERR_INVALID_ARG;
  const int64_t N = p->N, D = p->D, V = p->V, T = ceil_div(V, cce::kSubTile);
  if (C == nullptr || workspace == nullptr ||
      (N > 0 && (E == nullptr || targets == nullptr || partial == nullptr || tile_max == nullptr)))
    return fail(CCE_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(E) || !aligned16(C) || !aligned16(bias) || !aligned16(workspace))
    return fail(CCE_ERR_INVALID_ARG, "E, C, bias and workspace must be 16-byte aligned");
  const FwdWs w = carve_fwd(p, workspace);
  if (workspace_bytes < w.bytes)
    return fail(CCE_ERR_WORKSPACE, "forward workspace is %zu bytes, needs %zu", workspace_bytes, w.bytes);
  int num_sms = 0;
  CCE_CHECK(check_device(&num_sms));
  CCE_CHECK(get_encoder());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CCE_TRY(cudaMemsetAsync(w.hdr, 0, sizeof(WsHeader), s));
  if (N == 0) return CCE_OK;
  const auto* Cb = static_cast<const __nv_bfloat16*>(C);
  const auto* Bb = static_cast<const __nv_bfloat16*>(bias);
  const bool smooth = p->label_smoothing > 0.f;
  cce::FwdLaunch L{};
  L.bias = Bb;
  CCE_CHECK(make_map(&L.tmE, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, E, N, D, 64, cce::kFwdBM));
  CCE_CHECK(make_map(&L.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, V, D, 64, cce::kFwdBN));
  L.N = static_cast<int>(N);
  L.D = static_cast<int>(D);
  L.V = static_cast<int>(V);
  L.T = static_cast<int>(T);
  L.tile_max = tile_max;
  L.tile_sum = w.tile_sum;
  L.targets = targets;
  L.vs = p->vocab_start;
  L.ignore_index = p->ignore_index;
  L.zt = w.zt;
  L.err = &w.hdr->err;
  L.timeout_ns = cce::wait_timeout_ns();
  L.num_sms = num_sms;
  L.inject_stall = 0;
  if (smooth) CCE_TRY(cce::launch_weighted_colsum(Cb, V, D, nullptr, Bb, w.csum, s));
  if (g_fwd_ev[0] && g_fwd_ev[1]) CCE_TRY(cudaEventRecord(g_fwd_ev[0], s));
  CCE_TRY(cce::launch_fwd_lse(L, s));
  if (g_fwd_ev[0] && g_fwd_ev[1]) CCE_TRY(cudaEventRecord(g_fwd_ev[1], s));
  // partial rows: the shard's log-sum-exp, correct-token logit and logit sum (0 without smoothing)
  cce::FwdFinish F = finish_args(p, w, E, targets, tile_max, smooth);
  F.lse = partial;
  F.zt_out = partial + N;
  F.zs_out = partial + 2 * N;
  CCE_TRY(cce::launch_fwd_finish(F, !(g_fwd_ev[0] && g_fwd_ev[1]), s));  // N > 0: the tensor-core kernel ran
  return CCE_OK;
}

cce_status cce_forward_merge(const cce_problem* p, const float* partials, int32_t shards, const int64_t* targets,
                             float* loss, float* lse, int64_t* count, cce_stream_t stream) {
  g_last_error.clear();
  if (!problem_ok(p, true)) return CCE_ERR_INVALID_ARG;
  if (sharded(p)) return fail(CCE_ERR_INVALID_ARG, "cce_forward_merge takes the whole problem, not a shard");
  if (shards < 1) return fail(CCE_ERR_INVALID_ARG, "shards must be >= 1");
  if (loss == nullptr || count == nullptr ||
      (p->N > 0 && (partials == nullptr || targets == nullptr || lse == nullptr)))
    return fail(CCE_ERR_INVALID_ARG, "a required pointer is NULL");
  int num_sms = 0;
  CCE_CHECK(check_device(&num_sms));
  CCE_TRY(cce::launch_shard_merge(partials, shards, targets, p->N, p->V, p->ignore_index, p->label_smoothing,
                                  p->z_loss, p->reduction, loss, lse, count, reinterpret_cast<cudaStream_t>(stream)));
  return CCE_OK;
}

cce_status cce_backward_skip_map(const cce_problem* p, const void* workspace, size_t workspace_bytes,
                                 uint8_t* skipped, cce_stream_t stream) {
  g_last_error.clear();
  if (!problem_ok(p, true)) return CCE_ERR_INVALID_ARG;
  if (workspace == nullptr || (p->N > 0 && skipped == nullptr))
    return fail(CCE_ERR_INVALID_ARG, "a required pointer is NULL");
  // The tile flags sit at the same place in both workspace layouts; the smaller one bounds them.
  const SplitWs w = carve_split(p, 1, const_cast<void*>(workspace));
  if (workspace_bytes < w.bytes)
    return fail(CCE_ERR_WORKSPACE, "backward workspace is %zu bytes, needs %zu", workspace_bytes, w.bytes);
  if (p->N == 0) return CCE_OK;
  CCE_TRY(cce::launch_skip_map(w.plan.flags, w.plan.nb, w.plan.nt, ceil_div(p->V, cce::kSubTile), skipped,
                               reinterpret_cast<cudaStream_t>(stream)));
  return CCE_OK;
}

cce_status cce_check_device_error(void* workspace, cce_stream_t stream) {
  if (workspace == nullptr) return fail(CCE_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int err = 0;
  e = cudaMemcpy(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  if (err != 0) {
    const int zero = 0;
    cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice);
    const cce_status st = static_cast<cce_status>(err);
    return fail(st, "device reported: %s", cce_status_string(st));
  }
  return CCE_OK;
}

}  // extern "C"

// api.cu -- the extern "C" boundary of libsvq (declared in include/svq.h):
// argument validation, workspace sizing, the device status word, dispatch to
// the kernel launchers.  No entry point allocates or frees memory.
#include <cuda_runtime.h>

#include <mutex>

#include <cstdint>
#include <cstring>

#include "layout.cuh"
#include "svq.h"
#include "gemm_params.h"
#include "moe_params.h"
#include "svq_internal.h"
#include "calib.h"

namespace {

__device__ int g_status_word;   // set by kernels whose bounded waits run out

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SVQ_OK : SVQ_ERR_CUDA; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int check_matrix(const svq_matrix* W) {
  if (!W) return SVQ_ERR_INVALID_ARG;
  if (W->b_d < 1 || W->b_d > 10) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (W->K % 8 != 0 || !svq::layout_supported(W->N, W->K)) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!W->packed || !W->codebook) return SVQ_ERR_INVALID_ARG;
  if (W->radius_lut) {
    // per-row radius table: at most 16 levels (b_r <= 4)
    if (10 - W->b_d > svq::kLutMaxBits) return SVQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(W->radius_lut, 2)) return SVQ_ERR_INVALID_ARG;
  } else {
    if (!W->radius_scale || !W->radius_offset) return SVQ_ERR_INVALID_ARG;
    if (!aligned(W->radius_scale, 2) || !aligned(W->radius_offset, 2)) return SVQ_ERR_INVALID_ARG;
  }
  if (!aligned(W->packed, 16) || !aligned(W->codebook, 16) || (W->perm && !aligned(W->perm, 4)))
    return SVQ_ERR_INVALID_ARG;
  return SVQ_OK;
}

svq::GemvMatDesc desc_of(const svq_matrix& W, const uint16_t* x, void* y) {
  svq::GemvMatDesc d;
  d.N = W.N; d.K = W.K; d.b_d = W.b_d;
  d.packed = W.packed; d.codebook = W.codebook; d.scale = W.radius_scale; d.offset = W.radius_offset;
  d.perm = W.perm; d.lut = W.radius_lut; d.x = x; d.y = y;
  return d;
}

int plan_group(const svq_matrix* mats, int n_mats, int M, svq::GemvPlan* plan,
               svq::GemvMatDesc* descs, const uint16_t* const* x, void* const* y) {
  if (!mats || n_mats < 1 || n_mats > svq::kGemvMaxMats) return SVQ_ERR_INVALID_ARG;
  if (M < 1 || M > 16) return SVQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_mats; ++i) {
    const int st = check_matrix(&mats[i]);
    if (st != SVQ_OK) return st;
    // one grouped launch: every matrix with a radius table, or none
    if ((mats[i].radius_lut != nullptr) != (mats[0].radius_lut != nullptr)) return SVQ_ERR_INVALID_ARG;
    descs[i] = desc_of(mats[i], x ? x[i] : nullptr, y ? y[i] : nullptr);
  }
  const int sms = num_sms();
  if (sms <= 0) return SVQ_ERR_CUDA;
  // The plan depends only on the shapes, M and the SM count: keep the last few
  // (a decode loop calls the same layers over and over).
  struct Key {
    int sms, M, n, dims[3 * svq::kGemvMaxMats];
    bool operator==(const Key& o) const {
      if (sms != o.sms || M != o.M || n != o.n) return false;
      for (int i = 0; i < 3 * n; ++i)
        if (dims[i] != o.dims[i]) return false;
      return true;
    }
  };
  struct Entry {
    Key key;
    svq::GemvPlan plan;
    bool used;
  };
  static Entry cache[32];
  static int next_slot = 0;
  static std::mutex mu;
  Key key{};
  key.sms = sms; key.M = M; key.n = n_mats;
  for (int i = 0; i < n_mats; ++i) {
    // b_d, plus 16 when the matrix carries a radius table (its shared memory differs)
    key.dims[3 * i] = mats[i].N; key.dims[3 * i + 1] = mats[i].K;
    key.dims[3 * i + 2] = mats[i].b_d + (mats[i].radius_lut ? 16 : 0);
  }
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.used && e.key == key) {
        *plan = e.plan;
        return SVQ_OK;
      }
  }
  if (!svq::plan_gemv(descs, n_mats, M, sms, plan)) return SVQ_ERR_UNSUPPORTED_SHAPE;
  std::lock_guard<std::mutex> lock(mu);
  cache[next_slot] = Entry{key, *plan, true};
  next_slot = (next_slot + 1) % 32;
  return SVQ_OK;
}

// Scratch for svq_linear_gemv_noalloc: split-K partial sums and completion
// counters of one call.  Every GPU that loads the library holds these bytes
// until the process exits.
constexpr size_t kNoAllocScratchBytes = 1u << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for the current device, looked up (and
// the scratch zero-filled on `stream`) on the first call per device.  In host
// code the array's name is only a host-side stand-in; kernels must be given the
// address returned by cudaGetSymbolAddress.
void* noalloc_scratch(cudaStream_t stream) {
  static void* ptr[64] = {nullptr};
  static std::mutex mu;                          // first calls from several host threads
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    // Completion counters must start at zero; every completed call leaves them zero.
    if (cudaMemsetAsync(p, 0, kNoAllocScratchBytes, stream) != cudaSuccess) return nullptr;
    ptr[dev] = p;
  }
  return ptr[dev];
}

int* status_word() {
  static int* ptr[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int*>(p);
  }
  return ptr[dev];
}

}  // namespace

extern "C" {

const char* svq_status_string(int status) {
  switch (status) {
    case SVQ_OK: return "ok";
    case SVQ_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad enum or batch size)";
    case SVQ_ERR_UNSUPPORTED_SHAPE:
      return "unsupported shape (needs K % 8 == 0, 1 <= b_d <= 10; radius tables b_r <= 4; MoE K % 128 == 0 and N % 4 == 0)";
    case SVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case SVQ_ERR_CUDA: return "CUDA runtime error";
    case SVQ_ERR_TIMEOUT: return "a kernel's bounded wait timed out";
    default: return "unknown status";
  }
}

int svq_version(void) { return 100; }

size_t svq_packed_bytes(int N, int K) {
  if (!svq::layout_supported(N, K)) return 0;
  return svq::packed_bytes(N, K);
}

size_t svq_canonical_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % 8) return 0;
  return (size_t)N * (((size_t)(K / 8) * 18 + 7) / 8);
}

int svq_repack(const uint8_t* canonical, int N, int K, int b_d, void* packed_out, svq_stream_t stream) {
  if (!canonical || !packed_out) return SVQ_ERR_INVALID_ARG;
  if (b_d < 1 || b_d > 10 || !svq::layout_supported(N, K)) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(packed_out, 16)) return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_repack(canonical, N, K, b_d, packed_out, (cudaStream_t)stream));
}

int svq_unpack_fields(const void* packed, int N, int K, int b_d, uint8_t* signs, uint16_t* idx,
                      uint16_t* code, svq_stream_t stream) {
  if (!packed || !signs || !idx || !code) return SVQ_ERR_INVALID_ARG;
  if (b_d < 1 || b_d > 10 || !svq::layout_supported(N, K)) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(packed, 16) || !aligned(idx, 2) || !aligned(code, 2)) return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_unpack(packed, N, K, b_d, signs, idx, code, (cudaStream_t)stream));
}

int svq_dequantize(const svq_matrix* W, int out_dtype, void* w_out, svq_stream_t stream) {
  const int st = check_matrix(W);
  if (st != SVQ_OK) return st;
  if (!w_out || !aligned(w_out, 16)) return SVQ_ERR_INVALID_ARG;
  if (out_dtype != SVQ_F16 && out_dtype != SVQ_BF16) return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_dequant(W->packed, W->N, W->K, W->b_d, W->codebook, W->radius_scale,
                                         W->radius_offset, W->radius_lut, out_dtype == SVQ_BF16, (uint16_t*)w_out,
                                         (cudaStream_t)stream));
}

int svq_linear_gemv_batched_workspace_size(const svq_matrix* mats, int n_mats, int M, size_t* bytes) {
  if (!bytes) return SVQ_ERR_INVALID_ARG;
  svq::GemvPlan plan;
  svq::GemvMatDesc descs[svq::kGemvMaxMats];
  const int st = plan_group(mats, n_mats, M, &plan, descs, nullptr, nullptr);
  if (st != SVQ_OK) return st;
  *bytes = plan.ws_total;
  return SVQ_OK;
}

int svq_linear_gemv_workspace_size(const svq_matrix* W, int M, size_t* bytes) {
  return svq_linear_gemv_batched_workspace_size(W, 1, M, bytes);
}

int svq_workspace_init(void* workspace, size_t bytes, svq_stream_t stream) {
  if (bytes == 0) return SVQ_OK;
  if (!workspace) return SVQ_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, bytes, (cudaStream_t)stream));
}

// Checks and plans a grouped GEMV call (nothing is enqueued).
static int prepare_batched(const svq_matrix* mats, int n_mats, const uint16_t* const* x, int M, void* const* y,
                           int y_dtype, void* workspace, size_t workspace_bytes, svq::GemvPlan* plan,
                           svq::GemvMatDesc* descs) {
  if (!x || !y) return SVQ_ERR_INVALID_ARG;
  if (y_dtype != SVQ_F16 && y_dtype != SVQ_F32) return SVQ_ERR_INVALID_ARG;
  if (n_mats < 1 || n_mats > svq::kGemvMaxMats) return SVQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_mats; ++i) {
    if (!x[i] || !y[i]) return SVQ_ERR_INVALID_ARG;
    if (!aligned(x[i], 2) || !aligned(y[i], y_dtype == SVQ_F32 ? 4 : 2)) return SVQ_ERR_INVALID_ARG;
  }
  const int st = plan_group(mats, n_mats, M, plan, descs, x, y);
  if (st != SVQ_OK) return st;
  if (plan->ws_total > 0 && (!workspace || workspace_bytes < plan->ws_total || !aligned(workspace, 256)))
    return SVQ_ERR_WORKSPACE;
  return SVQ_OK;
}

int svq_linear_gemv_batched(const svq_matrix* mats, int n_mats, const uint16_t* const* x, int M,
                            void* const* y, int y_dtype, void* workspace, size_t workspace_bytes,
                            svq_stream_t stream) {
  svq::GemvPlan plan;
  svq::GemvMatDesc descs[svq::kGemvMaxMats];
  const int st = prepare_batched(mats, n_mats, x, M, y, y_dtype, workspace, workspace_bytes, &plan, descs);
  if (st != SVQ_OK) return st;
  return cuda_status(svq::launch_gemv(descs, plan, y_dtype == SVQ_F32, workspace, (cudaStream_t)stream));
}

int svq_linear_gemv_batched_host(const svq_matrix* mats, int n_mats, const uint16_t* x_host, uint16_t* x_dev,
                                 int M, void* y_host, void* y_dev, int y_dtype, void* workspace,
                                 size_t workspace_bytes, svq_stream_t stream) {
  if (!mats || !x_host || !x_dev || !y_host || !y_dev) return SVQ_ERR_INVALID_ARG;
  if (n_mats < 1 || n_mats > svq::kGemvMaxMats || M < 1) return SVQ_ERR_INVALID_ARG;
  if (y_dtype != SVQ_F16 && y_dtype != SVQ_F32) return SVQ_ERR_INVALID_ARG;
  const size_t ysz = y_dtype == SVQ_F32 ? 4 : 2;
  const uint16_t* xs[svq::kGemvMaxMats];
  void* ys[svq::kGemvMaxMats];
  size_t xo = 0, yo = 0;                             // elements of x, bytes of y
  for (int i = 0; i < n_mats; ++i) {
    if (mats[i].N < 1 || mats[i].K < 1) return SVQ_ERR_INVALID_ARG;
    xs[i] = x_dev + xo;
    ys[i] = reinterpret_cast<char*>(y_dev) + yo;
    xo += (size_t)M * mats[i].K;
    yo += (size_t)M * mats[i].N * ysz;
  }
  svq::GemvPlan plan;
  svq::GemvMatDesc descs[svq::kGemvMaxMats];
  // every check passes before anything is enqueued
  const int st = prepare_batched(mats, n_mats, xs, M, ys, y_dtype, workspace, workspace_bytes, &plan, descs);
  if (st != SVQ_OK) return st;
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xo * 2, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_status(e);
  e = svq::launch_gemv(descs, plan, y_dtype == SVQ_F32, workspace, s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(cudaMemcpyAsync(y_host, y_dev, yo, cudaMemcpyDeviceToHost, s));
}

int svq_linear_gemv(const svq_matrix* W, const uint16_t* x, int M, void* y, int y_dtype, void* workspace,
                    size_t workspace_bytes, svq_stream_t stream) {
  void* yy[1] = {y};
  const uint16_t* xx[1] = {x};
  if (!x || !y) return SVQ_ERR_INVALID_ARG;
  return svq_linear_gemv_batched(W, 1, xx, M, yy, y_dtype, workspace, workspace_bytes, stream);
}

int svq_linear_gemv_noalloc(const svq_matrix* W, const uint16_t* x, int M, void* y, int y_dtype,
                            svq_stream_t stream) {
  if (!x || !y) return SVQ_ERR_INVALID_ARG;
  if (y_dtype != SVQ_F16 && y_dtype != SVQ_F32) return SVQ_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(y, y_dtype == SVQ_F32 ? 4 : 2)) return SVQ_ERR_INVALID_ARG;
  svq::GemvPlan plan;
  svq::GemvMatDesc descs[1];
  const uint16_t* xx[1] = {x};
  void* yy[1] = {y};
  const int st = plan_group(W, 1, M, &plan, descs, xx, yy);
  if (st != SVQ_OK) return st;
  if (plan.ws_total > kNoAllocScratchBytes) return SVQ_ERR_WORKSPACE;
  void* scratch = noalloc_scratch((cudaStream_t)stream);
  if (!scratch) return SVQ_ERR_CUDA;
  return cuda_status(svq::launch_gemv(descs, plan, y_dtype == SVQ_F32, scratch, (cudaStream_t)stream));
}

int svq_linear_gemm_workspace_size(const svq_matrix* W, int M, size_t* bytes) {
  if (!bytes) return SVQ_ERR_INVALID_ARG;
  const int st = check_matrix(W);
  if (st != SVQ_OK) return st;
  if (M < 1) return SVQ_ERR_INVALID_ARG;
  const int sms = num_sms();
  if (sms <= 0) return SVQ_ERR_CUDA;
  *bytes = svq::plan_gemm(W->N, W->K, M, sms).ws_bytes;
  return SVQ_OK;
}

int svq_linear_gemm(const svq_matrix* W, const uint16_t* x, int x_dtype, int M, void* y, int y_dtype,
                    void* workspace, size_t workspace_bytes, svq_stream_t stream) {
  const int st = check_matrix(W);
  if (st != SVQ_OK) return st;
  if (!x || !y || M < 1) return SVQ_ERR_INVALID_ARG;
  if (x_dtype != SVQ_BF16 && x_dtype != SVQ_F16) return SVQ_ERR_INVALID_ARG;
  if (y_dtype != SVQ_BF16 && y_dtype != SVQ_F32) return SVQ_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(y, 16)) return SVQ_ERR_INVALID_ARG;
  if (!W->perm && !aligned(x, 16)) return SVQ_ERR_INVALID_ARG;     // read directly by TMA
  const int sms = num_sms();
  if (sms <= 0) return SVQ_ERR_CUDA;
  const svq::GemmPlan g = svq::plan_gemm(W->N, W->K, M, sms);
  if (!workspace || workspace_bytes < g.ws_bytes || !aligned(workspace, 256)) return SVQ_ERR_WORKSPACE;
  int* status = status_word();
  if (!status) return SVQ_ERR_CUDA;
  svq::GemmMatDesc d;
  d.N = W->N; d.K = W->K; d.b_d = W->b_d; d.M = M;
  d.packed = W->packed; d.codebook = W->codebook; d.scale = W->radius_scale; d.offset = W->radius_offset;
  d.lut = W->radius_lut;
  d.perm = W->perm; d.x = x; d.x_bf16 = x_dtype == SVQ_BF16; d.y = y; d.y_f32 = y_dtype == SVQ_F32;
  return cuda_status(svq::launch_gemm(d, g, workspace, status, (cudaStream_t)stream));
}

int svq_moe_grouped_gemv_workspace_size(int n_mats, int n_items, int N, int accumulate, size_t* bytes) {
  if (!bytes || n_mats < 1 || n_items < 0 || N < 1) return SVQ_ERR_INVALID_ARG;
  *bytes = svq::moe_workspace_layout(n_mats, n_items, N, accumulate ? 1 : 0).total;
  return SVQ_OK;
}

int svq_moe_grouped_gemv(const svq_matrix* mats, int n_mats, int N, int K, int max_b_d, const svq_group_item* items,
                         int n_items, int max_items_per_matrix, const void* x, int x_mode, int n_x_rows, float* y,
                         int n_out_rows, int accumulate, void* workspace, size_t workspace_bytes,
                         svq_stream_t stream) {
  if (!mats || !items || !x || !y || n_mats < 1 || n_items < 1 || n_out_rows < 1 || n_x_rows < 1)
    return SVQ_ERR_INVALID_ARG;
  // the grouped MoE kernel takes only shapes that need no padding
  if (max_b_d < 1 || max_b_d > 10 || !svq::layout_supported(N, K) || N % 4 != 0 || K % 128 != 0)
    return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (n_mats > 16384 || max_items_per_matrix < 1) return SVQ_ERR_INVALID_ARG;
  if (x_mode != SVQ_X_F16 && x_mode != SVQ_X_SWIGLU_F32) return SVQ_ERR_INVALID_ARG;
  if (!aligned(mats, 8) || !aligned(items, 4) || !aligned(y, 4) || !aligned(x, x_mode == SVQ_X_F16 ? 2 : 4))
    return SVQ_ERR_INVALID_ARG;
  const int mt = max_items_per_matrix == 1 ? 1 : (max_items_per_matrix == 2 ? 2 : 4);
  if (svq::moe_smem_bytes(max_b_d, K, mt, n_mats, n_items) > 220 * 1024) return SVQ_ERR_UNSUPPORTED_SHAPE;
  const svq::MoeWorkspace w = svq::moe_workspace_layout(n_mats, n_items, N, accumulate ? 1 : 0);
  if (!workspace || workspace_bytes < w.total || !aligned(workspace, 256)) return SVQ_ERR_WORKSPACE;
  const int sms = num_sms();
  int* status = status_word();
  if (sms <= 0 || !status) return SVQ_ERR_CUDA;
  char* b = reinterpret_cast<char*>(workspace);
  svq::MoeKParams p;
  p.mats = mats; p.n_mats = n_mats; p.N = N; p.K = K; p.max_b_d = max_b_d;
  p.items = items; p.n_items = n_items; p.x = x; p.x_mode = x_mode; p.n_x_rows = n_x_rows; p.y = y;
  p.n_out_rows = n_out_rows; p.accumulate = accumulate ? 1 : 0;
  p.offsets = reinterpret_cast<int*>(b + w.offsets);
  p.cursor = reinterpret_cast<int*>(b + w.cursor);
  p.sorted = reinterpret_cast<int*>(b + w.sorted);
  p.active = reinterpret_cast<int*>(b + w.active);
  p.n_active = reinterpret_cast<int*>(b + w.n_active);
  p.costpre = reinterpret_cast<int*>(b + w.costpre);
  p.mt = mt;
  p.local_route = svq::moe_local_route(n_mats, n_items) ? 1 : 0;
  p.item_out = accumulate ? reinterpret_cast<float*>(b + w.item_out) : nullptr;
  p.status = status;
  return cuda_status(svq::launch_moe(p, mt, n_out_rows, sms, (cudaStream_t)stream));
}

int svq_rmsnorm_permute(const uint16_t* h, int h_dtype, const uint16_t* gamma, float eps, int M, int K,
                        const int32_t* const* perms, uint16_t* const* outs, int n_out, svq_stream_t stream) {
  if (h_dtype != SVQ_F16 && h_dtype != SVQ_BF16) return SVQ_ERR_INVALID_ARG;
  if (n_out < 1 || n_out > svq::kMaxProducerOuts || !outs) return SVQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || eps > 3.0e38f) return SVQ_ERR_INVALID_ARG;   // rejects NaN and infinity
  if (M < 0 || M > 65535) return SVQ_ERR_INVALID_ARG;
  if (K < 8 || K % 8 != 0) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVQ_OK;                     // nothing to read or write
  if (!h || !gamma || !aligned(h, 16) || !aligned(gamma, 16)) return SVQ_ERR_INVALID_ARG;
  for (int g = 0; g < n_out; ++g) {
    if (!outs[g] || !aligned(outs[g], 16)) return SVQ_ERR_INVALID_ARG;
    if (perms && perms[g] && !aligned(perms[g], 4)) return SVQ_ERR_INVALID_ARG;
  }
  return cuda_status(svq::launch_rmsnorm_permute(h, h_dtype == SVQ_BF16, gamma, eps, M, K, perms, outs, n_out,
                                                 (cudaStream_t)stream));
}

int svq_swiglu_permute(const float* gate, const float* up, int M, int I, const int32_t* perm, uint16_t* x,
                       svq_stream_t stream) {
  if (M < 0 || M > 65535) return SVQ_ERR_INVALID_ARG;
  if (I < 8 || I % 8 != 0) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVQ_OK;                     // nothing to read or write
  if (!gate || !up || !x || !aligned(gate, 16) || !aligned(up, 16) || !aligned(x, 16)) return SVQ_ERR_INVALID_ARG;
  if (perm && !aligned(perm, 4)) return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_swiglu_permute(gate, up, M, I, perm, x, (cudaStream_t)stream));
}

int svq_esg(const float* x_cal, int T, int K, double gamma, double* energy, int32_t* perm, float* weights,
            svq_stream_t stream) {
  if (T < 1 || K < 8 || K % 8 != 0) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!x_cal || !energy || !perm) return SVQ_ERR_INVALID_ARG;
  if (!aligned(x_cal, 4) || !aligned(energy, 8) || !aligned(perm, 4) || (weights && !aligned(weights, 4)))
    return SVQ_ERR_INVALID_ARG;
  if (!(gamma == gamma)) return SVQ_ERR_INVALID_ARG;               // NaN exponent
  return cuda_status(svq::launch_esg(x_cal, T, K, gamma, energy, perm, weights, (cudaStream_t)stream));
}

int svq_radius_grid(const float* W, int N, int K, const int32_t* perm, int b_d, uint16_t* scale, uint16_t* offset,
                    svq_stream_t stream) {
  if (N < 1 || K < 8 || K % 8 != 0 || b_d < 1 || b_d > 10) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!W || !scale || !offset) return SVQ_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(scale, 2) || !aligned(offset, 2) || (perm && !aligned(perm, 4)))
    return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_radius_grid(W, N, K, perm, b_d, scale, offset, (cudaStream_t)stream));
}

int svq_encode(const float* W, int N, int K, int b_d, const int32_t* perm, const float* weights,
               const uint16_t* codebook, const uint16_t* scale, const uint16_t* offset, const uint16_t* radius_lut,
               uint8_t* canonical, double* row_err, svq_stream_t stream) {
  if (N < 1 || K < 8 || K % 8 != 0 || b_d < 1 || b_d > 10) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (radius_lut && 10 - b_d > svq::kLutMaxBits) return SVQ_ERR_UNSUPPORTED_SHAPE;
  if (!W || !codebook || !canonical || (!radius_lut && (!scale || !offset))) return SVQ_ERR_INVALID_ARG;
  if (!aligned(W, 4) || !aligned(codebook, 2) || (scale && !aligned(scale, 2)) || (offset && !aligned(offset, 2)) ||
      (radius_lut && !aligned(radius_lut, 2)) || (perm && !aligned(perm, 4)) || (weights && !aligned(weights, 4)) ||
      (row_err && !aligned(row_err, 8)))
    return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_encode(W, N, K, b_d, perm, weights, codebook, scale, offset, radius_lut, canonical,
                                        row_err, (cudaStream_t)stream));
}

int svq_abs_select(const double* row_err, int n_cand, int N, double* totals, int32_t* best, svq_stream_t stream) {
  if (n_cand < 1 || n_cand > svq::kAbsMaxCandidates || N < 1) return SVQ_ERR_INVALID_ARG;
  if (!row_err || !best || !aligned(row_err, 8) || !aligned(best, 4) || (totals && !aligned(totals, 8)))
    return SVQ_ERR_INVALID_ARG;
  return cuda_status(svq::launch_abs_select(row_err, n_cand, N, totals, best, (cudaStream_t)stream));
}

unsigned svq_debug_set_wait_polls(unsigned polls) { return svq::set_wait_polls(polls); }

int svq_get_device_status(svq_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SVQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return SVQ_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) return SVQ_ERR_CUDA;
  return v;
}

}  // extern "C"

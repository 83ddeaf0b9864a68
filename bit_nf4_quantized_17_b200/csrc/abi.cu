// C ABI of libqlora.so: argument checks on the host, then kernel launches on
// the caller's stream.  See include/qlora.h for the contract of each call.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "internal.cuh"
#include "kernels.cuh"
#include "linear.cuh"
#include "tc_ptx.cuh"

using namespace qlora;

namespace qlora {

static constexpr int64_t kMaxElems = int64_t(1) << 36;

static bool pow2_in(int32_t v, int32_t lo, int32_t hi) {
  return v >= lo && v <= hi && (v & (v - 1)) == 0;
}

const LevelTable* level_table(int32_t table) {
  static LevelTable tabs[2];
  static qlora_status ok[2];
  static std::once_flag once;
  std::call_once(once, [] {
    ok[0] = make_level_table(QLORA_TABLE_NF4, &tabs[0]);
    ok[1] = make_level_table(QLORA_TABLE_UNIFORM, &tabs[1]);
  });
  if (table < 0 || table > 1 || ok[table] != QLORA_OK) return nullptr;
  return &tabs[table];
}

qlora_status check_nf4_shape(const qlora_nf4& q) {
  if (q.rows < 1 || q.cols < 1 || q.rows > kMaxElems / q.cols) return QLORA_ERR_SHAPE;
  if (!pow2_in(q.blocksize, 64, 1024)) return QLORA_ERR_UNSUPPORTED;
  if (q.dq_blocksize != 0 && !pow2_in(q.dq_blocksize, 64, 1024)) return QLORA_ERR_UNSUPPORTED;
  if (q.table != QLORA_TABLE_NF4 && q.table != QLORA_TABLE_UNIFORM) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

qlora_status check_nf4_ptrs(const qlora_nf4& q) {
  if (!q.codes || !q.factors) return QLORA_ERR_NULL;
  if (q.dq_blocksize && (!q.scale_codes || !q.mean)) return QLORA_ERR_NULL;
  if (!aligned16(q.codes) || !aligned16(q.factors)) return QLORA_ERR_ALIGN;
  if (q.dq_blocksize && (!aligned16(q.scale_codes) || !aligned16(q.mean))) return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

}  // namespace qlora

namespace {
std::atomic<uint64_t> g_launches{0};

// State of qlora_timing_begin/end: event pairs, the kind of each, how many used.
struct Timing {
  std::mutex mu;
  std::atomic<bool> on{false};
  uint32_t mask = 0;
  std::vector<cudaEvent_t> ev;  // 2 per launch: start, stop
  std::vector<int> kind;
  int used = 0;
  bool open = false;  // a start was recorded, its stop not yet
};
Timing g_timing;
}  // namespace

namespace {
std::mutex g_setup_mu;
std::map<std::tuple<int, const void*, int>, int> g_setup;  // (device, kernel, tag) -> value
constexpr int kSmemTag = -1;
}  // namespace

bool qlora::cached_value(const void* func, int tag, int* value) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  const auto it = g_setup.find(std::make_tuple(dev, func, tag));
  if (it == g_setup.end()) return false;
  *value = it->second;
  return true;
}

void qlora::store_value(const void* func, int tag, int value) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  g_setup[std::make_tuple(dev, func, tag)] = value;
}

qlora_status qlora::ensure_smem(const void* func, int bytes) {
  int have = 0;
  if (cached_value(func, kSmemTag, &have) && have >= bytes) return QLORA_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  store_value(func, kSmemTag, bytes);
  return QLORA_OK;
}

void qlora::count_launch(unsigned n) {
  g_launches.fetch_add(n, std::memory_order_relaxed);
  // every launch is followed by after_launch, which reads the thread's last
  // error: clear one left by an unrelated earlier call so that it reports this launch
  (void)cudaGetLastError();
}

namespace {
// Record a timing event.  Inside a stream capture the record must be external
// to become a graph node that records the event when the graph runs; outside
// a capture the plain record is used.  A failed record leaves no error behind
// for the launch checks to report: the launch is not timed, nothing else.
bool record_timing_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  const cudaError_t e = (cs == cudaStreamCaptureStatusActive)
                            ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                            : cudaEventRecord(ev, s);
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e == cudaSuccess;
}
}  // namespace

void qlora::timing_mark(int kind, cudaStream_t s, bool start) {
  if (!g_timing.on.load(std::memory_order_acquire)) return;
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (!g_timing.on.load() || !(g_timing.mask >> kind & 1u)) return;
  const int cap = static_cast<int>(g_timing.kind.size());
  if (start) {
    if (g_timing.used >= cap) return;
    if (record_timing_event(g_timing.ev[2 * g_timing.used], s)) {
      g_timing.kind[g_timing.used] = kind;
      g_timing.open = true;
    }
  } else if (g_timing.open) {
    g_timing.open = false;
    if (record_timing_event(g_timing.ev[2 * g_timing.used + 1], s)) ++g_timing.used;
  }
}

qlora_status qlora::after_launch(const char* kernel, cudaStream_t s) {
  static const bool sync_check = [] {
    const char* e = std::getenv("QLORA_SYNC_CHECK");
    return e && e[0] == '1';
  }();
  cudaError_t e = cudaPeekAtLastError();
  if (e == cudaSuccess && sync_check) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    if (sync_check) std::fprintf(stderr, "qlora: %s: %s\n", kernel, cudaGetErrorString(e));
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

namespace {

size_t quantize_workspace(int64_t n, int32_t bs, int32_t dq) {
  const int64_t nb = ceil_div(n, bs);
  return dq ? 512 + static_cast<size_t>(ceil_div(4 * nb, 256) * 256) : 512;
}

}  // namespace

namespace {
// One CTA waits on an mbarrier that nothing completes, with the library's
// bounded wait, and reports the timeout the way the real kernels do.
__global__ void timeout_selftest_kernel(long long limit, DeviceStatus* st) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (!ptx::mbar_wait(&bar, 0, limit, &abort_flag) && threadIdx.x == 0)
    report(st, QLORA_ERR_DEVICE_TIMEOUT, 900u);
}
}  // namespace

extern "C" {

const char* qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "a required pointer is NULL";
    case QLORA_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case QLORA_ERR_SHAPE: return "a size is out of range or sizes disagree";
    case QLORA_ERR_UNSUPPORTED: return "request not supported by this build";
    case QLORA_ERR_NONFINITE: return "non-finite weight met while quantising";
    case QLORA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case QLORA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

qlora_status qlora_levels(int32_t table, float levels_out[16]) {
  if (!levels_out) return QLORA_ERR_NULL;
  const LevelTable* t = level_table(table);
  if (!t) return QLORA_ERR_UNSUPPORTED;
  std::memcpy(levels_out, t->level, sizeof(float) * 16);
  return QLORA_OK;
}

qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int32_t blocksize, int32_t dq_blocksize,
                             size_t* codes_bytes, size_t* scale_codes_bytes, size_t* factors_bytes,
                             size_t* mean_bytes, size_t* workspace_bytes) {
  qlora_nf4 q{};
  q.rows = rows;
  q.cols = cols;
  q.blocksize = blocksize;
  q.dq_blocksize = dq_blocksize;
  qlora_status st = check_nf4_shape(q);
  if (st != QLORA_OK) return st;
  const int64_t n = rows * cols;
  const int64_t nb = ceil_div(n, blocksize);
  const int64_t ng = dq_blocksize ? ceil_div(nb, dq_blocksize) : 0;
  if (codes_bytes) *codes_bytes = static_cast<size_t>(ceil_div(n, 2));
  if (scale_codes_bytes) *scale_codes_bytes = dq_blocksize ? static_cast<size_t>(nb) : 0;
  if (factors_bytes) *factors_bytes = static_cast<size_t>(4 * (dq_blocksize ? ng : nb));
  if (mean_bytes) *mean_bytes = dq_blocksize ? 4 : 0;
  if (workspace_bytes) *workspace_bytes = quantize_workspace(n, blocksize, dq_blocksize);
  return QLORA_OK;
}

qlora_status qlora_quantize(const void* W, int32_t w_dtype, const qlora_nf4* q, void* workspace,
                            size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx("qlora_quantize");
  if (!q || !W || !workspace) return QLORA_ERR_NULL;
  qlora_status st = check_nf4_shape(*q);
  if (st != QLORA_OK) return st;
  if ((st = check_nf4_ptrs(*q)) != QLORA_OK) return st;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(W) || !aligned16(workspace)) return QLORA_ERR_ALIGN;
  if (workspace_bytes < quantize_workspace(q->rows * q->cols, q->blocksize, q->dq_blocksize))
    return QLORA_ERR_WORKSPACE;
  const LevelTable* t = level_table(q->table);
  if (!t) return QLORA_ERR_UNSUPPORTED;
  return launch_quantize(W, w_dtype, *q, *t, workspace, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_dequantize(const qlora_nf4* q, void* W_out, int32_t out_dtype, void* stream) {
  const NvtxRange nvtx("qlora_dequantize");
  if (!q || !W_out) return QLORA_ERR_NULL;
  qlora_status st = check_nf4_shape(*q);
  if (st != QLORA_OK) return st;
  if ((st = check_nf4_ptrs(*q)) != QLORA_OK) return st;
  if (out_dtype != QLORA_F32 && out_dtype != QLORA_BF16) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(W_out)) return QLORA_ERR_ALIGN;
  const LevelTable* t = level_table(q->table);
  if (!t) return QLORA_ERR_UNSUPPORTED;
  return launch_dequantize(*q, *t, W_out, out_dtype, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_adamw(float* param, void* param_bf16, const float* grad, float* m, float* v,
                         int64_t n, int32_t step, float lr, float beta1, float beta2, float eps,
                         float weight_decay, float grad_scale, void* stream) {
  const NvtxRange nvtx("qlora_adamw");
  if (n < 0 || step < 1) return QLORA_ERR_SHAPE;
  if (n == 0) return QLORA_OK;
  if (!param || !grad || !m || !v) return QLORA_ERR_NULL;
  if (!aligned16(param) || !aligned16(grad) || !aligned16(m) || !aligned16(v) ||
      !aligned16(param_bf16))
    return QLORA_ERR_ALIGN;  // (a NULL param_bf16 counts as aligned)
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f) ||
      !(lr >= 0.0f))
    return QLORA_ERR_UNSUPPORTED;
  return launch_adamw(param, param_bf16, grad, m, v, n, step, lr, beta1, beta2, eps, weight_decay,
                      grad_scale, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_paged_alloc(size_t bytes, void** ptr) {
  if (!ptr) return QLORA_ERR_NULL;
  *ptr = nullptr;
  if (bytes == 0) return QLORA_ERR_SHAPE;
  void* p = nullptr;
  if (cudaMallocManaged(&p, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(p);
    return QLORA_ERR_CUDA;
  }
  *ptr = p;
  return QLORA_OK;
}

qlora_status qlora_paged_prefetch(void* ptr, size_t bytes, int32_t to_device, void* stream) {
  if (!ptr) return QLORA_ERR_NULL;
  if (bytes == 0) return QLORA_ERR_SHAPE;
  int dev = cudaCpuDeviceId;
  if (to_device && cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemPrefetchAsync(ptr, bytes, dev, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

qlora_status qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  return cudaFree(ptr) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_merge(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                         float alpha, void* W_out, void* stream) {
  const NvtxRange nvtx("qlora_merge");
  if (!W || !A || !B || !W_out) return QLORA_ERR_NULL;
  qlora_status st = check_nf4_shape(*W);
  if (st != QLORA_OK) return st;
  if ((st = check_nf4_ptrs(*W)) != QLORA_OK) return st;
  if (W->cols % W->blocksize != 0) return QLORA_ERR_UNSUPPORTED;
  if (r < 1 || r > 256) return QLORA_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(W_out)) return QLORA_ERR_ALIGN;
  const LevelTable* t = level_table(W->table);
  if (!t) return QLORA_ERR_UNSUPPORTED;
  return launch_merge(*W, *t, A, B, r, alpha, W_out, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_merge_dense(const void* W_in, int64_t rows, int64_t cols, const void* A,
                               const void* B, int32_t r, float alpha, void* W_out, void* stream) {
  const NvtxRange nvtx("qlora_merge_dense");
  if (!W_in || !A || !B || !W_out) return QLORA_ERR_NULL;
  if (rows < 1 || cols < 1 || cols % 8 != 0 || r < 1 || r > 256 || rows > (int64_t(1) << 22))
    return QLORA_ERR_SHAPE;
  if (!aligned16(W_in) || !aligned16(A) || !aligned16(B) || !aligned16(W_out))
    return QLORA_ERR_ALIGN;
  return launch_merge_dense(W_in, rows, cols, A, B, r, alpha, W_out,
                            static_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_workspace(int64_t M, int64_t N, int64_t K, int32_t r, size_t* fwd_bytes,
                                    size_t* bwd_bytes) {
  if (M < 0 || N < 1 || K < 1 || r < 1 || r > 256) return QLORA_ERR_SHAPE;
  LinearPlan p = plan_linear(M, N, K, r);
  if (fwd_bytes) *fwd_bytes = p.fwd_workspace;
  if (bwd_bytes) *bwd_bytes = p.bwd_workspace;
  return QLORA_OK;
}

static qlora_status check_linear(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                                 int64_t M, const void* X, const void* workspace,
                                 size_t workspace_bytes, bool bwd) {
  if (!W || !A || !B || !workspace || (M > 0 && !X)) return QLORA_ERR_NULL;
  qlora_status st = check_nf4_shape(*W);
  if (st != QLORA_OK) return st;
  if ((st = check_nf4_ptrs(*W)) != QLORA_OK) return st;
  // blocks never straddle rows, so every 64-weight k-tile lies in one block
  if (W->cols % W->blocksize != 0) return QLORA_ERR_UNSUPPORTED;
  if (r < 1 || r > 256 || M < 0) return QLORA_ERR_SHAPE;
  if (!aligned16(A) || !aligned16(B) || !aligned16(X) || !aligned16(workspace))
    return QLORA_ERR_ALIGN;  // (a NULL X with M = 0 counts as aligned)
  LinearPlan p = plan_linear(M, W->rows, W->cols, r);
  if (workspace_bytes < (bwd ? p.bwd_workspace : p.fwd_workspace)) return QLORA_ERR_WORKSPACE;
  if (!level_table(W->table)) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                              float alpha, const void* X, int64_t M, void* Y, float* U_save,
                              void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx("qlora_linear_fwd");
  qlora_status st = check_linear(W, A, B, r, M, X, workspace, workspace_bytes, false);
  if (st != QLORA_OK) return st;
  if (M == 0) return QLORA_OK;
  if (!Y) return QLORA_ERR_NULL;
  if (!aligned16(Y) || (U_save && !aligned16(U_save))) return QLORA_ERR_ALIGN;
  return linear_forward(*W, *level_table(W->table), A, B, r, alpha, X, M, Y, U_save, workspace,
                        static_cast<cudaStream_t>(stream), LoraOpts{r, nullptr, nullptr, nullptr, 1.0f});
}

qlora_status qlora_linear_bwd(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                              float alpha, const void* X, const float* U, const void* dY,
                              int64_t M, void* dX, float* dA, float* dB, int32_t accumulate,
                              void* workspace, size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx("qlora_linear_bwd");
  qlora_status st = check_linear(W, A, B, r, M, X, workspace, workspace_bytes, true);
  if (st != QLORA_OK) return st;
  if ((M > 0 && !dY) || !dA || !dB) return QLORA_ERR_NULL;
  if (!aligned16(dY) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)) ||
      (U && !aligned16(U)))
    return QLORA_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    if (accumulate) return QLORA_OK;
    // no tokens: the gradients of A and B are zero
    if (cudaMemsetAsync(dA, 0, sizeof(float) * r * W->cols, s) != cudaSuccess ||
        cudaMemsetAsync(dB, 0, sizeof(float) * r * W->rows, s) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  return linear_backward(*W, *level_table(W->table), A, B, r, alpha, X, U, dY, M, dX, dA, dB,
                         accumulate != 0, workspace, s, LoraOpts{r, nullptr, nullptr, nullptr, 1.0f});
}

static qlora_status check_multi(const qlora_nf4* W, int32_t n_adapters, int32_t r,
                                const int32_t* adapter, int64_t M) {
  if (n_adapters < 1 || r < 1 || static_cast<int64_t>(n_adapters) * r > 256) return QLORA_ERR_SHAPE;
  if (M > 0 && !adapter) return QLORA_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(adapter) % 4 != 0) return QLORA_ERR_ALIGN;
  if (!linear_multi_supported(M, W->rows, W->cols, n_adapters * r)) return QLORA_ERR_UNSUPPORTED;
  return QLORA_OK;
}

static qlora_status opts_of(const qlora_adapter_opts* x, const qlora_nf4* W, int32_t r, int64_t M,
                            LoraOpts* o, int32_t* rt) {
  const int32_t n = x ? x->n_adapters : 1;
  if (n < 1 || r < 1 || static_cast<int64_t>(n) * r > 256) return QLORA_ERR_SHAPE;
  *rt = n * r;
  *o = LoraOpts{r, nullptr, nullptr, nullptr, 1.0f};
  if (!x) return QLORA_OK;
  if (x->adapter || n > 1) {
    qlora_status st = check_multi(W, n, r, x->adapter, M);
    if (st != QLORA_OK) return st;
    o->seg = x->adapter;
  }
  if (x->keep_mask) {
    if (!(x->dropout_p >= 0.0f && x->dropout_p < 1.0f)) return QLORA_ERR_UNSUPPORTED;
    if (M > 0 && !x->x_drop) return QLORA_ERR_NULL;
    if (!aligned16(x->x_drop)) return QLORA_ERR_ALIGN;
    if (!linear_multi_supported(M, W->rows, W->cols, *rt)) return QLORA_ERR_UNSUPPORTED;
    o->mask = x->keep_mask;
    o->x_drop = x->x_drop;
    o->keep = 1.0f / (1.0f - x->dropout_p);
  }
  return QLORA_OK;
}

qlora_status qlora_linear_fwd_ex(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                                 float alpha, const qlora_adapter_opts* opts, const void* X,
                                 int64_t M, void* Y, float* U_save, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx("qlora_linear_fwd_ex");
  if (!W) return QLORA_ERR_NULL;
  LoraOpts o{};
  int32_t rt = 0;
  qlora_status st = opts_of(opts, W, r, M, &o, &rt);
  if (st != QLORA_OK) return st;
  if ((st = check_linear(W, A, B, rt, M, X, workspace, workspace_bytes, false)) != QLORA_OK)
    return st;
  if (M == 0) return QLORA_OK;
  if (!Y) return QLORA_ERR_NULL;
  if (!aligned16(Y) || (U_save && !aligned16(U_save))) return QLORA_ERR_ALIGN;
  return linear_forward(*W, *level_table(W->table), A, B, rt, alpha, X, M, Y, U_save, workspace,
                        static_cast<cudaStream_t>(stream), o);
}

qlora_status qlora_linear_bwd_ex(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                                 float alpha, const qlora_adapter_opts* opts, const void* X,
                                 const float* U, const void* dY, int64_t M, void* dX, float* dA,
                                 float* dB, int32_t accumulate, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  const NvtxRange nvtx("qlora_linear_bwd_ex");
  if (!W) return QLORA_ERR_NULL;
  LoraOpts o{};
  int32_t rt = 0;
  qlora_status st = opts_of(opts, W, r, M, &o, &rt);
  if (st != QLORA_OK) return st;
  if ((st = check_linear(W, A, B, rt, M, X, workspace, workspace_bytes, true)) != QLORA_OK)
    return st;
  if ((M > 0 && !dY) || !dA || !dB) return QLORA_ERR_NULL;
  if (!aligned16(dY) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)) ||
      (U && !aligned16(U)))
    return QLORA_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {
    if (accumulate) return QLORA_OK;
    if (cudaMemsetAsync(dA, 0, sizeof(float) * rt * W->cols, s) != cudaSuccess ||
        cudaMemsetAsync(dB, 0, sizeof(float) * rt * W->rows, s) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  return linear_backward(*W, *level_table(W->table), A, B, rt, alpha, X, U, dY, M, dX, dA, dB,
                         accumulate != 0, workspace, s, o);
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4* W, const void* A, const void* B,
                                    int32_t n_adapters, int32_t r, float alpha,
                                    const int32_t* adapter, const void* X, int64_t M, void* Y,
                                    float* U_save, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  qlora_adapter_opts x{};
  x.n_adapters = n_adapters;
  x.adapter = adapter;
  if (M > 0 && !adapter) return QLORA_ERR_NULL;
  return qlora_linear_fwd_ex(W, A, B, r, alpha, &x, X, M, Y, U_save, workspace, workspace_bytes,
                             stream);
}

qlora_status qlora_linear_bwd_multi(const qlora_nf4* W, const void* A, const void* B,
                                    int32_t n_adapters, int32_t r, float alpha,
                                    const int32_t* adapter, const void* X, const float* U,
                                    const void* dY, int64_t M, void* dX, float* dA, float* dB,
                                    int32_t accumulate, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  qlora_adapter_opts x{};
  x.n_adapters = n_adapters;
  x.adapter = adapter;
  if (M > 0 && !adapter) return QLORA_ERR_NULL;
  return qlora_linear_bwd_ex(W, A, B, r, alpha, &x, X, U, dY, M, dX, dA, dB, accumulate,
                             workspace, workspace_bytes, stream);
}

qlora_status qlora_selftest_timeout(int64_t limit_cycles, void* workspace, void* stream) {
  if (!workspace) return QLORA_ERR_NULL;
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 32)) return QLORA_ERR_SHAPE;
  if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  count_launch();
  timeout_selftest_kernel<<<1, 32, 0, s>>>(static_cast<long long>(limit_cycles),
                                           static_cast<DeviceStatus*>(workspace));
  return after_launch("timeout_selftest", s);
}

qlora_status qlora_check(void* workspace, void* stream) {
  if (!workspace) return QLORA_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
  DeviceStatus h{};
  if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return QLORA_ERR_CUDA;
  if (h.code != 0u) {
    if (cudaMemset(workspace, 0, sizeof(h)) != cudaSuccess) return QLORA_ERR_CUDA;
    return static_cast<qlora_status>(h.code);
  }
  return QLORA_OK;
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

qlora_status qlora_timing_begin(uint32_t kind_mask, int32_t max_launches) {
  if (max_launches < 1 || max_launches > 65536) return QLORA_ERR_SHAPE;
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (g_timing.on.load()) return QLORA_ERR_UNSUPPORTED;
  g_timing.ev.assign(2 * static_cast<size_t>(max_launches), nullptr);
  for (auto& e : g_timing.ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (auto& d : g_timing.ev)
        if (d) cudaEventDestroy(d);
      g_timing.ev.clear();
      return QLORA_ERR_CUDA;
    }
  }
  g_timing.kind.assign(static_cast<size_t>(max_launches), -1);
  g_timing.mask = kind_mask;
  g_timing.used = 0;
  g_timing.open = false;
  g_timing.on.store(true, std::memory_order_release);
  return QLORA_OK;
}

qlora_status qlora_timing_end(float* ms, int32_t* launches) {
  std::lock_guard<std::mutex> lock(g_timing.mu);
  if (!g_timing.on.load()) return QLORA_ERR_UNSUPPORTED;
  g_timing.on.store(false, std::memory_order_release);
  float total[QLORA_KERNEL_KINDS] = {};
  int32_t count[QLORA_KERNEL_KINDS] = {};
  qlora_status st = QLORA_OK;
  for (int i = 0; i < g_timing.used && st == QLORA_OK; ++i) {
    float t = 0.0f;
    if (cudaEventSynchronize(g_timing.ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_timing.ev[2 * i], g_timing.ev[2 * i + 1]) != cudaSuccess) {
      st = QLORA_ERR_CUDA;
      break;
    }
    const int k = g_timing.kind[i];
    if (k >= 0 && k < QLORA_KERNEL_KINDS) {
      total[k] += t;
      ++count[k];
    }
  }
  for (auto& e : g_timing.ev) cudaEventDestroy(e);
  g_timing.ev.clear();
  g_timing.kind.clear();
  for (int k = 0; k < QLORA_KERNEL_KINDS; ++k) {
    if (ms) ms[k] = total[k];
    if (launches) launches[k] = count[k];
  }
  return st;
}

}  // extern "C"

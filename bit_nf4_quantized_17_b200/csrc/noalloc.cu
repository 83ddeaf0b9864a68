// qlora_quantize_noalloc: quantisation for callers that cannot allocate.
//
// qlora_quantize needs a caller-provided workspace for its reductions (the
// global maximum and fixed-point sum of the block scales, and one fp32
// absmax per block).  Some callers cannot allocate that workspace: code whose
// device memory is owned by a pool that has already reserved the GPU (where
// a fresh cudaMalloc fails or fragments the pool), and loops that cannot
// afford the device-wide synchronisation that cudaMalloc/cudaFree imply.
// This entry point runs the same kernels with the workspace in a fixed
// array that lives in the library's own device memory.
//
// Limits and sharing:
//   * the array holds 512 bytes of reduction words plus one fp32 per block,
//     for at most kMaxBlocks blocks (2^20, i.e. 64 Mi weights at blocksize
//     64); larger double-quantised tensors are refused with
//     QLORA_ERR_WORKSPACE.  Without double quantisation the block absmax
//     goes straight to q->factors and only the 512-byte header is used, so
//     that case has no size limit beyond qlora_quantize's own;
//   * every GPU that loads the library keeps its own copy of the array
//     (4 MiB + 512 B) until the process exits;
//   * all calls on a device share it: two calls whose work overlaps on the
//     GPU (different streams, no ordering between them) race and corrupt each
//     other's result.  Calls on one stream are ordered and safe;
//   * each call clears the words that must start at zero (status, maximum,
//     sum); the per-block values are fully rewritten before they are read.
// The first call on a device looks up the array's device address with
// cudaGetSymbolAddress (with that device current); make that first call
// before any stream capture.
#include <mutex>

#include "internal.cuh"

namespace qlora {
namespace {

constexpr int64_t kMaxBlocks = int64_t(1) << 20;
constexpr size_t kHeaderBytes = 512;
constexpr size_t kScratchBytes = kHeaderBytes + sizeof(float) * kMaxBlocks;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_quantize_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_quantize_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace qlora

extern "C" qlora_status qlora_quantize_noalloc(const void* W, int32_t w_dtype,
                                               const qlora_nf4* q, uint32_t* status_out,
                                               void* stream) {
  using namespace qlora;
  const NvtxRange nvtx("qlora_quantize_noalloc");
  if (!q || !W) return QLORA_ERR_NULL;
  qlora_status st = check_nf4_shape(*q);
  if (st != QLORA_OK) return st;
  if ((st = check_nf4_ptrs(*q)) != QLORA_OK) return st;
  if (w_dtype != QLORA_F32 && w_dtype != QLORA_BF16) return QLORA_ERR_UNSUPPORTED;
  if (!aligned16(W) || (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u)))
    return QLORA_ERR_ALIGN;
  // the per-block absmax lives in the array only with double quantisation
  if (q->dq_blocksize != 0 && ceil_div(q->rows * q->cols, q->blocksize) > kMaxBlocks)
    return QLORA_ERR_WORKSPACE;
  const LevelTable* table = level_table(q->table);
  if (!table) return QLORA_ERR_UNSUPPORTED;

  void* scratch = scratch_on_current_device();
  if (!scratch) return QLORA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: clear the status word and
  // the reduction words (the quantiser clears the latter again itself)
  if (cudaMemsetAsync(scratch, 0, kHeaderBytes, s) != cudaSuccess) return QLORA_ERR_CUDA;
  st = launch_quantize(W, w_dtype, *q, *table, scratch, s);
  if (st != QLORA_OK) return st;
  if (status_out &&
      cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) !=
          cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

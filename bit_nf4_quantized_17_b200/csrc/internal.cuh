// Internal declarations shared by the translation units of libqlora.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qlora.h"

#include <nvtx3/nvToolsExt.h>

namespace qlora {

// First 256 bytes of every workspace: a status word written by kernels that
// detect an error on the device, read (and cleared) by qlora_check().
constexpr size_t kStatusBytes = 256;
struct DeviceStatus {
  unsigned int code;    // qlora_status, first error wins
  unsigned int detail;  // kernel-specific detail (e.g. which wait gave up)
};

#ifdef __CUDACC__
__device__ __forceinline__ void report(DeviceStatus* st, unsigned int code,
                                       unsigned int detail) {
  if (st && atomicCAS(&st->code, 0u, code) == 0u) st->detail = detail;
}
#endif

// Level table and decision thresholds handed to kernels by value.
// thr[k] is the largest fp32 not above the exact midpoint of levels k, k+1,
// so that, for fp32 x, (x > thr[k]) == (x > exact midpoint).
struct LevelTable {
  float level[16];
  float thr[16];  // 15 used
};

// tables.cpp
qlora_status make_level_table(int32_t table, LevelTable* out);

// abi.cu: the argument checks every call on a quantised weight shares.
// check_nf4_shape: sizes, block sizes and table; check_nf4_ptrs: the device
// arrays present and 16-byte aligned.  level_table: the library's level and
// threshold table of QLORA_TABLE_NF4 / QLORA_TABLE_UNIFORM (nullptr otherwise).
qlora_status check_nf4_shape(const qlora_nf4& q);
qlora_status check_nf4_ptrs(const qlora_nf4& q);
const LevelTable* level_table(int32_t table);

// An NVTX range around an ABI call, so that profiles show the library's calls
// (free when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// abi.cu: every kernel launch site calls this once per launch.
void count_launch(unsigned n = 1);
// Per-device, thread-safe launch setup.  ensure_smem raises `func`'s dynamic
// shared-memory limit on the current device to at least `bytes` (once per
// device).  cached_value / store_value keep a per-device integer for `func`
// under `tag` (resident CTA or cluster counts measured once).
qlora_status ensure_smem(const void* func, int bytes);
bool cached_value(const void* func, int tag, int* value);
void store_value(const void* func, int tag, int value);

// abi.cu: kernel timing hook.  A launch site of a timed kind calls it with
// start = true just before its launch and start = false just after; both are
// no-ops unless qlora_timing_begin enabled that kind.
void timing_mark(int kind, cudaStream_t s, bool start);

// abi.cu: status of the launch just enqueued.  With the environment variable
// QLORA_SYNC_CHECK=1 the stream is synchronised after every launch and a
// failing kernel is named on stderr (a debugging aid; off by default).
qlora_status after_launch(const char* kernel, cudaStream_t s);

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// quantize.cu
qlora_status launch_quantize(const void* W, int32_t w_dtype, const qlora_nf4& q,
                             const LevelTable& t, void* workspace, cudaStream_t s);
qlora_status launch_dequantize(const qlora_nf4& q, const LevelTable& t, void* out,
                               int32_t out_dtype, cudaStream_t s);

// adamw.cu: one AdamW step over n fp32 parameters (and their bf16 copy)
qlora_status launch_adamw(float* p, void* p16, const float* g, float* m, float* v, int64_t n,
                          int32_t step, float lr, float beta1, float beta2, float eps,
                          float weight_decay, float grad_scale, cudaStream_t s);

// merge.cu: W_out = bf16(dequant(W) + (alpha / r) B A)
qlora_status launch_merge(const qlora_nf4& q, const LevelTable& t, const void* A, const void* B,
                          int32_t r, float alpha, void* out, cudaStream_t s);
// merge.cu: W_out = bf16(W_in + (alpha / r) B A) for a dense bf16 W_in (may alias W_out)
qlora_status launch_merge_dense(const void* W_in, int64_t rows, int64_t cols, const void* A,
                                const void* B, int32_t r, float alpha, void* out, cudaStream_t s);
// The same two updates with the rank-r product on the tensor cores
// (merge_tc.cu), for r a multiple of 8 up to 256 and cols a multiple of 64.
struct QView;
bool merge_tc_eligible(int64_t cols, int32_t r);
qlora_status launch_merge_tc(const QView& w, const LevelTable& t, const void* A, const void* B,
                             int32_t r, float alpha, void* out, cudaStream_t s);
qlora_status launch_merge_dense_tc(const void* W_in, int64_t rows, int64_t cols, const void* A,
                                   const void* B, int32_t r, float alpha, void* out,
                                   cudaStream_t s);

// Everything a linear-layer kernel needs to read a quantised W.
struct QView {
  const uint8_t* codes;
  const int8_t* scale_codes;
  const float* factors;
  const float* mean;
  int64_t rows, cols;
  int32_t dq_shift;  // log2(dq_blocksize); -1 without double quantisation
  int32_t bs_shift;  // log2(blocksize / 64): 64-weight k-tile t of a row lies in block t >> bs_shift
};

#ifdef __CUDACC__
__device__ __forceinline__ float block_scale(const QView& w, int64_t b, float mu) {
  if (w.dq_shift < 0) return __ldg(w.factors + b);
  float q = static_cast<float>(__ldg(w.scale_codes + b));
  float f = __ldg(w.factors + (b >> w.dq_shift));
  return __fadd_rn(__fmul_rn(q, f), mu);
}
#endif

}  // namespace qlora

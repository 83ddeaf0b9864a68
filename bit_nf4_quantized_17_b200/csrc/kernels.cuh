// Launch interfaces of the linear-layer kernels.
#pragma once

#include "internal.cuh"

namespace qlora {

// How a contraction operand is stored.  Element (i, k): i runs over the
// operand's own output dimension, k over the contraction.
enum OperandKind {
  OP_BF16_K = 0,   // bf16, address i*ld + k
  OP_BF16_MN = 1,  // bf16, address k*ld + i
  OP_F32_K = 2,    // fp32, address i*ld + k
  OP_F32_MN = 3,   // fp32, address k*ld + i
  OP_NF4_K = 4,    // quantised W read as W[i][k]
  OP_NF4_MN = 5,   // quantised W read as W[k][i]
};

struct Operand {
  const void* ptr;
  int64_t ld;
  QView w;
};

inline Operand dense(const void* p, int64_t ld) { return Operand{p, ld, QView{}}; }
inline Operand quantised(const QView& w) { return Operand{nullptr, 0, w}; }

// gemm_simt.cu: C = alpha * opA . opB^T (+ cin), any shape.
qlora_status simt_gemm(int kind_a, const Operand& a, int kind_b, const Operand& b, int64_t m,
                       int64_t n, int64_t k, float alpha, const float* cin, void* c,
                       int64_t ldc, bool c_bf16, const LevelTable& t, cudaStream_t s);

// gemm_tc.cu: tcgen05 / TMEM / TMA kernels.
enum BMode { B_TMA_K = 0, B_DQ_K = 1, B_DQ_MN = 2 };

// Columns of one half of a [hi | lo] LoRA operand buffer: r rounded up to 64.
inline int32_t lora_span(int32_t r) { return (r + 63) / 64 * 64; }
// Rows of one half of a transposed [hi ; lo] LoRA operand: r rounded up to 16.
inline int32_t lora_rows(int32_t r) { return (r + 15) / 16 * 16; }

int tc_split_count(int64_t m_tiles, int64_t k_tiles);

// Shape of a fused launch: mt 128-row accumulators per CTA (1 or 2) and the
// number of contraction splits (1 = bf16 output written directly; more =
// fp32 partials out[z] of M x n_out, summed by splitk_reduce).
struct FusedShape {
  int mt;
  int splits;
};
FusedShape fused_shape(int64_t M, int64_t n_out, int64_t kt_total);

// Y = X W^T + sU B^T, W dequantised on load; sU (M x 2*lora_span(r) bf16) holds
// hi = bf16(s X A^T) in columns [0, r) and lo = bf16(s X A^T - hi) from column
// lora_span(r), zero elsewhere.
qlora_status tc_fused_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                              const void* sU, const void* B, int32_t r, void* out,
                              const FusedShape& f, DeviceStatus* st, cudaStream_t s);
// dX = dY W + sV A, W dequantised on load; sV laid out like sU, for s dY B.
qlora_status tc_fused_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                            const void* sV, const void* A, int32_t r, void* out,
                            const FusedShape& f, DeviceStatus* st, cudaStream_t s);
// The same two products on CTA pairs (gemm_tc2.cu): a 512 x 256 output tile
// per pair, each CTA dequantising half of the W tile.  Used for one split
// with more than 256 tokens; bf16 output only.
bool tc2_eligible(int64_t M, const FusedShape& f);
qlora_status tc2_fused_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                               const void* sU, const void* B, int32_t r, void* Y,
                               DeviceStatus* st, cudaStream_t s);
qlora_status tc2_fused_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                             const void* sV, const void* A, int32_t r, void* dX,
                             DeviceStatus* st, cudaStream_t s);
// Forward for M <= 16 tokens with the dequantised W in TMEM as the MMA's A
// operand (gemm_tc_decode.cu): Y^T = W X^T + B (sU)^T into `out` (M x N bf16);
// with splits > 1 the CTAs of a row tile form a cluster and sum their
// contraction splits in shared memory, in split order.
int tc_decode_splits(int64_t M, int64_t N, int64_t K);
qlora_status tc_decode_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                               const void* sU, const void* B, int32_t r, void* out, int splits,
                               DeviceStatus* st, cudaStream_t s);
// Dequant GEMV for the dX product of one or two tokens on the CUDA cores
// (gemv_small.cu): partials part[c][m][k] of dY W + s V A (V fp32), one per
// cluster of row chunks; *parts (at most gemv_dgrad_parts(M, K), the
// workspace bound) is the number written, to be summed by splitk_reduce.
bool gemv_eligible(int64_t M, int64_t K, int32_t r);
int gemv_dgrad_parts(int64_t M, int64_t K);
qlora_status gemv_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                        const float* V, const void* A, int32_t r, float s, float* part,
                        int* parts, cudaStream_t st);
// part[z] (m_rows x n_cols fp32) = A . B^T over split z of the contraction; B has
// b_rows rows, read as n_cols (rows past b_rows are zero).
qlora_status tc_lora_gemm(const void* A, bool a_mn, int64_t m_rows, int64_t kdim, int64_t ld_a,
                          const void* B, int64_t ld_b, int32_t b_rows, int32_t n_cols,
                          float* part, int splits, DeviceStatus* st, cudaStream_t s);

struct ReduceArgs;
// gemm_rank.cu: the same product as tc_lora_gemm followed by splitk_reduce,
// in one launch: the contraction split over the CTAs of a cluster, the fp32
// partials summed in distributed shared memory in split order, the sums
// written to the outputs of `out` (its part, splits and pcols are ignored;
// cols and lo index the n_cols partial columns).  n_cols a multiple of 16 in
// [16, 256], cols and lo multiples of 4 with cols + lo <= n_cols
// (tc_rank_eligible); otherwise QLORA_ERR_UNSUPPORTED.
bool tc_rank_eligible(int32_t n_cols, int32_t cols, int32_t lo);
int tc_rank_splits(int64_t m_tiles, int64_t k_tiles);
// b_mn: B stored with its n_cols columns contiguous (element (j, k) at
// k * ld_b + j, b_rows = n_cols); needs n_cols % 64 == 0.
qlora_status tc_rank_gemm(const void* A, bool a_mn, int64_t m_rows, int64_t kdim, int64_t ld_a,
                          const void* B, bool b_mn, int64_t ld_b, int32_t b_rows, int32_t n_cols,
                          const ReduceArgs& out, DeviceStatus* st, cudaStream_t s);

struct ReduceArgs {
  const float* part;
  int splits;
  int64_t rows;
  int cols, pcols, lo;
  float* o1;
  int64_t ld1;
  bool trans1;
  float a1;
  bool acc1;
  void* o2;
  int64_t ld2;
  float a2;
  int o2_lo;
  void* o3;
  int64_t ld3;
  float a3;
  int o3_lo;
  int o2_pad;  // > 0: also write zeros to o2 columns [cols, o2_lo) and [o2_lo + cols, 2 o2_lo)
  // adapter mask: when set, output (i, j) is kept only if seg[i] == j / seg_cols
  // (row i = a token, its columns [a seg_cols, (a + 1) seg_cols) = adapter a)
  const int32_t* seg;
  int seg_cols;
};
qlora_status splitk_reduce(const ReduceArgs& a, cudaStream_t s);
qlora_status transpose_to_bf16(const void* in, bool in_f32, int64_t rows, int cols, int64_t ld_in,
                               void* out, int64_t ld_out, int lo_rows, cudaStream_t s);

// lora_decode.cu: U = X A^T and V = dY B for M <= 16 tokens in one launch each
// (cluster-reduced, deterministic).  Outputs for token m < M, rank column j:
//   o1[m ld1 + j] = a1 v (j < r),  o2[m ld2 + j] = hi(a2 v), o2[m ld2 + j + o2_lo] =
//   lo(a2 v) (j < r; zeros for r <= j < o2_lo), v masked to 0 when seg[m] != j / seg_cols.
struct RankOut {
  int32_t r;
  float* o1;
  int64_t ld1;
  float a1;
  __nv_bfloat16* o2;
  int64_t ld2;
  float a2;
  int32_t o2_lo;
  const int32_t* seg;
  int32_t seg_cols;
};
qlora_status rank_down(const void* X, const void* A, int M, int64_t K, int32_t span,
                       const RankOut& o, cudaStream_t s);
qlora_status rank_v(const void* dY, const void* B, int M, int64_t N, int32_t span,
                    const RankOut& o, cudaStream_t s);

// dropout.cu: X_drop = X (.) D (mask bit (k % 8) of byte m K / 8 + k / 8 keeps
// X[m][k]; K a multiple of 8), and dX[m][k] += D[m][k] scale (V A)[m][k] in place.
qlora_status dropout_apply(const void* X, const uint8_t* mask, int64_t M, int64_t K, void* X_drop,
                           cudaStream_t s);
qlora_status dropout_dx(void* dX, const float* V, int64_t ldv, const void* A, const uint8_t* mask,
                        int64_t M, int64_t K, int32_t r, float scale, cudaStream_t s);

// lora_small.cu: dA and dB for M <= 16 tokens (CUDA cores); r a multiple of 8.
constexpr int kSmallM = 16;
qlora_status small_grad_b(const void* dY, const float* U, int M, int64_t N, int r, float sc,
                          bool accumulate, float* dB, cudaStream_t s);
qlora_status small_grad_a(const float* V, const void* X, int M, int64_t K, int r, float sc,
                          bool accumulate, float* dA, cudaStream_t s);

}  // namespace qlora

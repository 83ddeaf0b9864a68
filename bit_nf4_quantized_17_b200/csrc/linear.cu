// Forward and backward pass of the QLoRA linear layer.
//
// Forward ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", 2; "QLoRA技术从入门
// 到精通", 3(2)):   U = X A^T,  Y = X W^T + s U B^T,  s = alpha / r.
// Backward (same pages, 6 and 3(3)): V = dY B, dX = dY W + s V A,
// dB = s dY^T U, dA = s V^T X; no gradient for W.
#include "kernels.cuh"
#include "linear.cuh"

namespace qlora {
namespace {

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

QView view_of(const qlora_nf4& W) {
  return QView{W.codes, W.scale_codes, W.factors, W.mean, W.rows, W.cols,
               W.dq_blocksize ? __builtin_ctz(W.dq_blocksize) : -1};
}

float lora_scale(float alpha, int32_t r) { return alpha / static_cast<float>(r); }

}  // namespace

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int32_t r) {
  LinearPlan p;
  const size_t mr = align256(sizeof(float) * M * r);
  p.fwd_workspace = kStatusBytes + mr + align256(sizeof(float) * M * N);
  p.bwd_workspace = kStatusBytes + 2 * mr + align256(sizeof(float) * M * K);
  return p;
}

qlora_status linear_forward(const qlora_nf4& W, const LevelTable& t, const void* A,
                            const void* B, int32_t r, float alpha, const void* X, int64_t M,
                            void* Y, float* U_save, void* workspace, cudaStream_t s) {
  const int64_t N = W.rows, K = W.cols;
  char* ws = static_cast<char*>(workspace) + kStatusBytes;
  float* u = U_save ? U_save : reinterpret_cast<float*>(ws);
  ws += align256(sizeof(float) * M * r);
  float* y0 = reinterpret_cast<float*>(ws);
  const QView w = view_of(W);
  qlora_status st;
  // U = X A^T
  st = simt_gemm(OP_BF16_K, dense(X, K), OP_BF16_K, dense(A, K), M, r, K, 1.0f, nullptr, u, r,
                 false, t, s);
  if (st != QLORA_OK) return st;
  // Y0 = X W^T (W dequantised on the fly)
  st = simt_gemm(OP_BF16_K, dense(X, K), OP_NF4_K, quantised(w), M, N, K, 1.0f, nullptr, y0, N,
                 false, t, s);
  if (st != QLORA_OK) return st;
  // Y = bf16(Y0 + s U B^T)
  return simt_gemm(OP_F32_K, dense(u, r), OP_BF16_K, dense(B, r), M, N, r, lora_scale(alpha, r),
                   y0, Y, N, true, t, s);
}

qlora_status linear_backward(const qlora_nf4& W, const LevelTable& t, const void* A,
                             const void* B, int32_t r, float alpha, const void* X,
                             const float* U, const void* dY, int64_t M, void* dX, float* dA,
                             float* dB, bool accumulate, void* workspace, cudaStream_t s) {
  const int64_t N = W.rows, K = W.cols;
  const float sc = lora_scale(alpha, r);
  char* ws = static_cast<char*>(workspace) + kStatusBytes;
  float* u = reinterpret_cast<float*>(ws);
  ws += align256(sizeof(float) * M * r);
  float* v = reinterpret_cast<float*>(ws);
  ws += align256(sizeof(float) * M * r);
  float* dx0 = reinterpret_cast<float*>(ws);
  const QView w = view_of(W);
  qlora_status st;
  if (!U) {
    st = simt_gemm(OP_BF16_K, dense(X, K), OP_BF16_K, dense(A, K), M, r, K, 1.0f, nullptr, u, r,
                   false, t, s);
    if (st != QLORA_OK) return st;
    U = u;
  }
  // V = dY B      (B is N x r: element (j, n) = B[n][j])
  st = simt_gemm(OP_BF16_K, dense(dY, N), OP_BF16_MN, dense(B, r), M, r, N, 1.0f, nullptr, v, r,
                 false, t, s);
  if (st != QLORA_OK) return st;
  if (dX) {
    // dX0 = dY W    (element (k, n) of the second operand = W[n][k])
    st = simt_gemm(OP_BF16_K, dense(dY, N), OP_NF4_MN, quantised(w), M, K, N, 1.0f, nullptr,
                   dx0, K, false, t, s);
    if (st != QLORA_OK) return st;
    // dX = bf16(dX0 + s V A)   (A is r x K: element (k, j) = A[j][k])
    st = simt_gemm(OP_F32_K, dense(v, r), OP_BF16_MN, dense(A, K), M, K, r, sc, dx0, dX, K,
                   true, t, s);
    if (st != QLORA_OK) return st;
  }
  // dB = s dY^T U (+ dB)   element (n, m) of dY^T = dY[m][n]; element (j, m) of U^T = U[m][j]
  st = simt_gemm(OP_BF16_MN, dense(dY, N), OP_F32_MN, dense(U, r), N, r, M, sc,
                 accumulate ? dB : nullptr, dB, r, false, t, s);
  if (st != QLORA_OK) return st;
  // dA = s V^T X (+ dA)
  return simt_gemm(OP_F32_MN, dense(v, r), OP_BF16_MN, dense(X, K), r, K, M, sc,
                   accumulate ? dA : nullptr, dA, K, false, t, s);
}

}  // namespace qlora

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

}  // namespace qlora

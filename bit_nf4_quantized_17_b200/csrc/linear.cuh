// Forward / backward orchestration of the QLoRA linear layer.
#pragma once

#include "internal.cuh"

namespace qlora {

struct LinearPlan {
  size_t fwd_workspace;
  size_t bwd_workspace;
};

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int32_t r);

// Options of the adapter branch.
//  - Several adapters: r = n_adapters * r_adapter (A and B stacked along the
//    rank); seg[m] is the adapter of token m, and the reductions that produce
//    U and V zero the columns of the other adapters, so every later step (the
//    fused GEMMs' LoRA stages, dA, dB) sees only each token's own adapter.
//    One adapter: seg == nullptr and r_adapter == r.  The scale is
//    alpha / r_adapter.
//  - LoRA dropout: the adapter branch reads x_drop = X (.) D instead of X,
//    keep = 1 / (1 - p), and the LoRA part of dX is masked by D (mask != nullptr).
//    Without dropout x_drop = X, keep = 1 and mask = nullptr.
struct LoraOpts {
  int32_t r_adapter;
  const int32_t* seg;
  const void* x_drop;
  const uint8_t* mask;
  float keep;
};

bool linear_multi_supported(int64_t M, int64_t N, int64_t K, int32_t r);

qlora_status linear_forward(const qlora_nf4& W, const LevelTable& t, const void* A,
                            const void* B, int32_t r, float alpha, const void* X, int64_t M,
                            void* Y, float* U_save, void* workspace, cudaStream_t s,
                            const LoraOpts& o);

qlora_status linear_backward(const qlora_nf4& W, const LevelTable& t, const void* A,
                             const void* B, int32_t r, float alpha, const void* X,
                             const float* U, const void* dY, int64_t M, void* dX, float* dA,
                             float* dB, bool accumulate, void* workspace, cudaStream_t s,
                             const LoraOpts& o);

}  // namespace qlora

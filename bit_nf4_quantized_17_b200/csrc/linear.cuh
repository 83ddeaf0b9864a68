// Forward / backward orchestration of the QLoRA linear layer.
#pragma once

#include "internal.cuh"

namespace qlora {

struct LinearPlan {
  size_t fwd_workspace;
  size_t bwd_workspace;
};

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int32_t r);

qlora_status linear_forward(const qlora_nf4& W, const LevelTable& t, const void* A,
                            const void* B, int32_t r, float alpha, const void* X, int64_t M,
                            void* Y, float* U_save, void* workspace, cudaStream_t s);

qlora_status linear_backward(const qlora_nf4& W, const LevelTable& t, const void* A,
                             const void* B, int32_t r, float alpha, const void* X,
                             const float* U, const void* dY, int64_t M, void* dX, float* dA,
                             float* dB, bool accumulate, void* workspace, cudaStream_t s);

}  // namespace qlora

// LoRA dropout on the adapter input.
//
// The adapter branch reads a dropped-out copy of its input while the frozen
// base reads X itself ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section
// 4.3, lora_dropout; "QLoRA 量化微调", the LoRA dropout of the training
// recipe).  With a keep mask D (one bit per element of X, drawn by the caller)
// and keep probability 1 - p:
//   X~ = D (.) X / (1 - p),  U = X~ A^T,  Y = X W^T + s U B^T
//   dX = dY W + s D (.) (V A) / (1 - p),  dA = s V^T X~,  dB = s dY^T U
// Two kernels serve it: the masked copy X (.) D (exact in bf16: each element is
// kept or zeroed, the 1 / (1 - p) goes into the scalars of the GEMMs that read
// it), and the masked rank-r update of dX, added after the base product.
#include "internal.cuh"
#include "kernels.cuh"

namespace qlora {
namespace {

// X_drop = X (.) D: 8 elements per thread (16 bytes of X, one mask byte)
__global__ void __launch_bounds__(256)
dropout_apply_kernel(const uint4* __restrict__ X, const uint8_t* __restrict__ mask, int64_t n8,
                     uint4* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint4 v = X[i];
    const uint32_t m = mask[i];
    // 16-bit lanes: keep lane e when bit e of the mask byte is set
    auto keep2 = [&](uint32_t w, int e) {
      const uint32_t lo = (m >> e) & 1u ? 0x0000ffffu : 0u;
      const uint32_t hi = (m >> (e + 1)) & 1u ? 0xffff0000u : 0u;
      return w & (lo | hi);
    };
    v.x = keep2(v.x, 0);
    v.y = keep2(v.y, 2);
    v.z = keep2(v.z, 4);
    v.w = keep2(v.w, 6);
    out[i] = v;
  }
}

constexpr int kCols = 256;  // columns of dX per CTA: 32 lanes x 8
constexpr int kRows = 64;   // rows of dX per CTA: 8 warps x 8

// dX[m][k] = bf16(dX[m][k] + D[m][k] scale sum_j V[m][j] A[j][k]) over a
// 64 x 256 tile; A's 256 columns staged in shared memory as bf16, V rows read
// as warp-uniform broadcasts.  fp32 accumulation in rank order.
__global__ void __launch_bounds__(256)
dropout_dx_kernel(__nv_bfloat16* __restrict__ dX, const float* __restrict__ V, int64_t ldv,
                  const __nv_bfloat16* __restrict__ A, const uint8_t* __restrict__ mask,
                  int64_t M, int64_t K, int r, float scale) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* as = reinterpret_cast<__nv_bfloat16*>(smem);  // r x kCols
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kCols;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kRows;
  const int ncols = static_cast<int>(K - k0 < kCols ? K - k0 : kCols);  // a multiple of 8
  for (int e = threadIdx.x; e < r * (kCols / 8); e += blockDim.x) {
    const int j = e / (kCols / 8), c = 8 * (e % (kCols / 8));
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (c < ncols) v = *reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k0 + c);
    *reinterpret_cast<uint4*>(as + j * kCols + c) = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = 8 * lane;
  if (c >= ncols) return;
  const int64_t k = k0 + c;
  for (int i = 0; i < kRows / 8; ++i) {
    const int64_t m = m0 + warp + 8 * i;
    if (m >= M) break;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float* vrow = V + m * ldv;
    for (int j = 0; j < r; ++j) {
      const float v = __ldg(vrow + j);
      const uint4 a = *reinterpret_cast<const uint4*>(as + j * kCols + c);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = fmaf(v, __uint_as_float(w[q] << 16), acc[2 * q]);
        acc[2 * q + 1] = fmaf(v, __uint_as_float(w[q] & 0xffff0000u), acc[2 * q + 1]);
      }
    }
    const uint32_t mb = mask[(m * K + k) >> 3];
    uint4* dst = reinterpret_cast<uint4*>(dX + m * K + k);
    uint4 d = *dst;
    uint32_t dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float lo = __uint_as_float(dw[q] << 16), hi = __uint_as_float(dw[q] & 0xffff0000u);
      if ((mb >> (2 * q)) & 1u) lo = __fadd_rn(lo, __fmul_rn(scale, acc[2 * q]));
      if ((mb >> (2 * q + 1)) & 1u) hi = __fadd_rn(hi, __fmul_rn(scale, acc[2 * q + 1]));
      const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
      dw[q] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *dst = make_uint4(dw[0], dw[1], dw[2], dw[3]);
  }
}

}  // namespace

qlora_status dropout_apply(const void* X, const uint8_t* mask, int64_t M, int64_t K, void* X_drop,
                           cudaStream_t s) {
  const int64_t n8 = M * K / 8;
  if (n8 == 0) return QLORA_OK;
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(n8, 256), 148 * 8));
  count_launch();
  dropout_apply_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(X), mask, n8,
                                            static_cast<uint4*>(X_drop));
  return after_launch("dropout_apply", s);
}

qlora_status dropout_dx(void* dX, const float* V, int64_t ldv, const void* A, const uint8_t* mask,
                        int64_t M, int64_t K, int32_t r, float scale, cudaStream_t s) {
  const size_t smem = sizeof(__nv_bfloat16) * static_cast<size_t>(r) * kCols;
  const qlora_status cs = ensure_smem(reinterpret_cast<const void*>(dropout_dx_kernel),
                                      static_cast<int>(sizeof(__nv_bfloat16) * 256 * kCols));
  if (cs != QLORA_OK) return cs;
  const dim3 grid(static_cast<unsigned>(ceil_div(K, kCols)), static_cast<unsigned>(ceil_div(M, kRows)));
  if (grid.y > 65535) return QLORA_ERR_SHAPE;
  count_launch();
  dropout_dx_kernel<<<grid, 256, smem, s>>>(static_cast<__nv_bfloat16*>(dX), V, ldv,
                                            static_cast<const __nv_bfloat16*>(A), mask, M, K, r,
                                            scale);
  return after_launch("dropout_dx", s);
}

}  // namespace qlora

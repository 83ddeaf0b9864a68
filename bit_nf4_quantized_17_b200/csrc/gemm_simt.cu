// General-shape fallback contraction on CUDA cores.
//
//   C[i][j] = alpha * sum_k  opA(i, k) * opB(j, k)  (+ Cin[i][j])
//
// Each operand is read through an accessor: bf16 or fp32 stored with the
// contraction index contiguous (K-major) or the other index contiguous
// (MN-major), or the quantised weight read as W[i][k] (forward) or W[k][i]
// (backward), dequantised element by element as level[idx] * s_b.  fp32
// accumulation.  This path serves the shapes the tensor-core kernels do not
// take (odd r, tiny M) and is the reference the faster kernels are tested
// against on the device.
#include "internal.cuh"
#include "kernels.cuh"

namespace qlora {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <int KIND>
__device__ __forceinline__ float load_operand(const Operand& o, int64_t i, int64_t k,
                                              int64_t extent_i, int64_t extent_k,
                                              const float* lv, float mu) {
  if (i >= extent_i || k >= extent_k) return 0.0f;
  if constexpr (KIND == OP_BF16_K) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(o.ptr)[i * o.ld + k]);
  } else if constexpr (KIND == OP_BF16_MN) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(o.ptr)[k * o.ld + i]);
  } else if constexpr (KIND == OP_F32_K) {
    return static_cast<const float*>(o.ptr)[i * o.ld + k];
  } else if constexpr (KIND == OP_F32_MN) {
    return static_cast<const float*>(o.ptr)[k * o.ld + i];
  } else {
    // quantised weight, blocks of 64: element (row, col) of W
    const int64_t row = (KIND == OP_NF4_K) ? i : k;
    const int64_t col = (KIND == OP_NF4_K) ? k : i;
    const int64_t e = row * o.w.cols + col;
    const uint8_t byte = __ldg(o.w.codes + (e >> 1));
    const int idx = (e & 1) ? (byte >> 4) : (byte & 15);
    // the product uses the dequantised weight rounded to bf16
    return __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[idx], block_scale(o.w, e >> (6 + o.w.bs_shift), mu))));
  }
}

template <int KA, int KB>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(Operand a, Operand b, int64_t m, int64_t n, int64_t k, float alpha,
                 const float* cin, void* c, int64_t ldc, int c_bf16, LevelTable tab) {
  __shared__ float as[TK][TM + 4];
  __shared__ float bs[TK][TN + 4];
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = tab.level[threadIdx.x];
  const float mu_a = (KA >= OP_NF4_K && a.w.dq_shift >= 0) ? __ldg(a.w.mean) : 0.0f;
  const float mu_b = (KB >= OP_NF4_K && b.w.dq_shift >= 0) ? __ldg(b.w.mean) : 0.0f;
  __syncthreads();
  const int64_t i0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * TN;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < k; k0 += TK) {
    for (int t = threadIdx.x; t < TM * TK; t += 256) {
      const int ii = t % TM, kk = t / TM;
      as[kk][ii] = load_operand<KA>(a, i0 + ii, k0 + kk, m, k, lv, mu_a);
      bs[kk][ii] = load_operand<KB>(b, j0 + ii, k0 + kk, n, k, lv, mu_b);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        av[u] = as[kk][ty + 16 * u];
        bv[u] = bs[kk][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = i0 + ty + 16 * u;
    if (i >= m) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = j0 + tx + 16 * v;
      if (j >= n) continue;
      float val = alpha * acc[u][v];
      if (cin) val += cin[i * ldc + j];
      if (c_bf16)
        static_cast<__nv_bfloat16*>(c)[i * ldc + j] = __float2bfloat16_rn(val);
      else
        static_cast<float*>(c)[i * ldc + j] = val;
    }
  }
}

template <int KA, int KB>
void launch(const Operand& a, const Operand& b, int64_t m, int64_t n, int64_t k, float alpha,
            const float* cin, void* c, int64_t ldc, bool c_bf16, const LevelTable& t,
            cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(ceil_div(n, TN)), static_cast<unsigned>(ceil_div(m, TM)));
  count_launch();
  simt_gemm_kernel<KA, KB><<<grid, 256, 0, s>>>(a, b, m, n, k, alpha, cin, c, ldc, c_bf16 ? 1 : 0, t);
}

}  // namespace

qlora_status simt_gemm(int kind_a, const Operand& a, int kind_b, const Operand& b, int64_t m,
                       int64_t n, int64_t k, float alpha, const float* cin, void* c,
                       int64_t ldc, bool c_bf16, const LevelTable& t, cudaStream_t s) {
  if (m <= 0 || n <= 0) return QLORA_OK;
#define QLORA_CASE(KA, KB) \
  if (kind_a == KA && kind_b == KB) { launch<KA, KB>(a, b, m, n, k, alpha, cin, c, ldc, c_bf16, t, s); } else
  QLORA_CASE(OP_BF16_K, OP_BF16_K)
  QLORA_CASE(OP_BF16_K, OP_BF16_MN)
  QLORA_CASE(OP_BF16_K, OP_NF4_K)
  QLORA_CASE(OP_BF16_K, OP_NF4_MN)
  QLORA_CASE(OP_F32_K, OP_BF16_K)
  QLORA_CASE(OP_F32_K, OP_BF16_MN)
  QLORA_CASE(OP_BF16_MN, OP_F32_MN)
  QLORA_CASE(OP_F32_MN, OP_BF16_MN)
  { return QLORA_ERR_UNSUPPORTED; }
#undef QLORA_CASE
  return after_launch("simt_gemm", s);
}

}  // namespace qlora

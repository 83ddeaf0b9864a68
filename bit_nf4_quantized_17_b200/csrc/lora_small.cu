// LoRA gradients for decode-sized batches (M <= 16 tokens).
//
// With so few tokens dA and dB of the rank-r branch ("LoRA 与 QLoRA：把大模型
// 微调拆成可负担的工程", 2: h = W x + (alpha/r) B A x) are rank-M outer
// products, bound by writing dA and dB:
//
//   grad_b        dB[n][j] = s sum_m dY[m][n] U[m][j]   (+ dB)
//   grad_a        dA[j][k] = s sum_m V[m][j] X[m][k]    (+ dA)
#include "internal.cuh"
#include "kernels.cuh"

namespace qlora {
namespace {

constexpr int kMaxM = 16;

// dB[n][j..j+3] = s sum_m dY[m][n] U[m][j..j+3]  (+ dB); one thread per 4 ranks of a row
template <int MM>
__global__ void __launch_bounds__(256)
grad_b_kernel(const __nv_bfloat16* __restrict__ dY, const float* __restrict__ U, int M, int64_t N,
              int r, float s, int accumulate, float* __restrict__ dB) {
  __shared__ __align__(16) float us[kMaxM * 256];
  for (int e = threadIdx.x; e < M * r; e += 256) us[e] = U[e];
  __syncthreads();
  const int q4 = r / 4;
  const int64_t total = N * q4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t n = e / q4;
    const int j = 4 * static_cast<int>(e - n * q4);
    float dy[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m) dy[m] = (m < M) ? __bfloat162float(dY[m * N + n]) : 0.0f;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      if (m >= M) break;
      const float4 u = *reinterpret_cast<const float4*>(&us[m * r + j]);
      v.x = fmaf(dy[m], u.x, v.x);
      v.y = fmaf(dy[m], u.y, v.y);
      v.z = fmaf(dy[m], u.z, v.z);
      v.w = fmaf(dy[m], u.w, v.w);
    }
    float4* dst = reinterpret_cast<float4*>(dB + n * r + j);
    float4 o = make_float4(s * v.x, s * v.y, s * v.z, s * v.w);
    if (accumulate) {
      const float4 d = *dst;
      o = make_float4(d.x + o.x, d.y + o.y, d.z + o.z, d.w + o.w);
    }
    *dst = o;
  }
}

// dA[j][k..k+7] = s sum_m V[m][j] X[m][k..k+7]  (+ dA); one thread per 8 columns of a rank
template <int MM>
__global__ void __launch_bounds__(256)
grad_a_kernel(const float* __restrict__ V, const __nv_bfloat16* __restrict__ X, int M, int64_t K,
              int r, float s, int accumulate, float* __restrict__ dA) {
  __shared__ float vs[kMaxM * 256];
  for (int e = threadIdx.x; e < M * r; e += 256) vs[e] = V[e];
  __syncthreads();
  const int64_t k8 = K / 8;
  const int64_t total = static_cast<int64_t>(r) * k8;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int j = static_cast<int>(e / k8);
    const int64_t k = 8 * (e - static_cast<int64_t>(j) * k8);
    uint4 xr[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m)
      xr[m] = (m < M) ? *reinterpret_cast<const uint4*>(X + m * K + k) : make_uint4(0u, 0u, 0u, 0u);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      if (m >= M) break;
      const float v = vs[m * r + j];
      const uint32_t w[4] = {xr[m].x, xr[m].y, xr[m].z, xr[m].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] = fmaf(v, __uint_as_float(w[q] << 16), acc[2 * q]);
        acc[2 * q + 1] = fmaf(v, __uint_as_float(w[q] & 0xffff0000u), acc[2 * q + 1]);
      }
    }
    float4* dst = reinterpret_cast<float4*>(dA + static_cast<int64_t>(j) * K + k);
    float4 o0 = make_float4(s * acc[0], s * acc[1], s * acc[2], s * acc[3]);
    float4 o1 = make_float4(s * acc[4], s * acc[5], s * acc[6], s * acc[7]);
    if (accumulate) {
      const float4 d0 = dst[0], d1 = dst[1];
      o0 = make_float4(d0.x + o0.x, d0.y + o0.y, d0.z + o0.z, d0.w + o0.w);
      o1 = make_float4(d1.x + o1.x, d1.y + o1.y, d1.z + o1.z, d1.w + o1.w);
    }
    dst[0] = o0;
    dst[1] = o1;
  }
}

int grid_cap(int64_t items) {
  const int64_t g = ceil_div(items, 256);
  return static_cast<int>(g < 148 * 8 ? (g < 1 ? 1 : g) : 148 * 8);
}

}  // namespace

qlora_status small_grad_b(const void* dY, const float* U, int M, int64_t N, int r, float sc,
                          bool accumulate, float* dB, cudaStream_t s) {
  if (M > kMaxM || r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  const int g = grid_cap(N * (r / 4));
  const auto* y = static_cast<const __nv_bfloat16*>(dY);
  const int acc = accumulate ? 1 : 0;
  count_launch();
  if (M == 1) grad_b_kernel<1><<<g, 256, 0, s>>>(y, U, M, N, r, sc, acc, dB);
  else if (M <= 4) grad_b_kernel<4><<<g, 256, 0, s>>>(y, U, M, N, r, sc, acc, dB);
  else grad_b_kernel<16><<<g, 256, 0, s>>>(y, U, M, N, r, sc, acc, dB);
  return after_launch("small_grad_b", s);
}

qlora_status small_grad_a(const float* V, const void* X, int M, int64_t K, int r, float sc,
                          bool accumulate, float* dA, cudaStream_t s) {
  if (M > kMaxM || K % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  const int g = grid_cap(r * (K / 8));
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const int acc = accumulate ? 1 : 0;
  count_launch();
  if (M == 1) grad_a_kernel<1><<<g, 256, 0, s>>>(V, x, M, K, r, sc, acc, dA);
  else if (M <= 4) grad_a_kernel<4><<<g, 256, 0, s>>>(V, x, M, K, r, sc, acc, dA);
  else grad_a_kernel<16><<<g, 256, 0, s>>>(V, x, M, K, r, sc, acc, dA);
  return after_launch("small_grad_a", s);
}

}  // namespace qlora

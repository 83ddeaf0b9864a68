// LoRA-side contractions for decode-sized batches (M <= 16 tokens).
//
// With so few tokens the rank-r branch ("LoRA 与 QLoRA：把大模型微调拆成可负担
// 的工程", 2: h = W x + (alpha/r) B A x) is a handful of short reductions and
// rank-M outer products, bound by reading A and B and writing dA and dB:
//
//   down_partial  part[z][m][j] = sum_{k in chunk z} X[m][k] A[j][k]    (U = X A^T)
//   v_partial     part[z][m][j] = sum_{n in chunk z} dY[m][n] B[n][j]   (V = dY B)
//   grad_b        dB[n][j] = s sum_m dY[m][n] U[m][j]   (+ dB)
//   grad_a        dA[j][k] = s sum_m V[m][j] X[m][k]    (+ dA)
//
// The partials are summed in a fixed order by splitk_reduce (deterministic).
#include "internal.cuh"
#include "kernels.cuh"

namespace qlora {
namespace {

constexpr int kMaxM = 16;
constexpr int kChunk = 64;

// One CTA per chunk of 64 k; warp w handles ranks j = w, w + 8, ...; lanes
// stride over k; X chunk staged in shared memory.
__global__ void __launch_bounds__(256)
down_partial_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A,
                    int M, int64_t K, int r, int r16, float* __restrict__ part) {
  __shared__ float xs[kMaxM][kChunk];
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kChunk;
  const int kc = static_cast<int>((K - k0) < kChunk ? (K - k0) : kChunk);
  for (int e = threadIdx.x; e < M * kChunk; e += 256) {
    const int m = e / kChunk, k = e % kChunk;
    xs[m][k] = (k < kc) ? __bfloat162float(X[m * K + k0 + k]) : 0.0f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* out = part + static_cast<int64_t>(blockIdx.x) * M * r16;
  for (int j = warp; j < r; j += 8) {
    float acc[kMaxM];
#pragma unroll
    for (int m = 0; m < kMaxM; ++m) acc[m] = 0.0f;
    const __nv_bfloat16* arow = A + j * K + k0;
    for (int k = lane; k < kc; k += 32) {
      const float a = __bfloat162float(arow[k]);
#pragma unroll
      for (int m = 0; m < kMaxM; ++m)
        if (m < M) acc[m] = fmaf(xs[m][k], a, acc[m]);
    }
#pragma unroll
    for (int m = 0; m < kMaxM; ++m) {
      if (m >= M) break;
      float v = acc[m];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) out[m * r16 + j] = v;
    }
  }
}

// One CTA per chunk of 64 rows n (dY chunk staged in shared memory); thread t
// covers rank j = t % r and row lane t / r; the row lanes are summed in
// shared memory.
__global__ void __launch_bounds__(256)
v_partial_kernel(const __nv_bfloat16* __restrict__ dY, const __nv_bfloat16* __restrict__ B,
                 int M, int64_t N, int r, int r16, float* __restrict__ part) {
  __shared__ float ys[kMaxM][kChunk];
  __shared__ float red[256][kMaxM + 1];
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kChunk;
  const int nc = static_cast<int>((N - n0) < kChunk ? (N - n0) : kChunk);
  for (int e = threadIdx.x; e < M * kChunk; e += 256) {
    const int m = e / kChunk, n = e % kChunk;
    ys[m][n] = (n < nc) ? __bfloat162float(dY[m * N + n0 + n]) : 0.0f;
  }
  __syncthreads();
  const int lanes = 256 / r;
  const int j = threadIdx.x % r, nl = threadIdx.x / r;
  float acc[kMaxM];
#pragma unroll
  for (int m = 0; m < kMaxM; ++m) acc[m] = 0.0f;
  if (nl < lanes) {
    for (int n = nl; n < nc; n += lanes) {
      const float b = __bfloat162float(B[(n0 + n) * r + j]);
#pragma unroll
      for (int m = 0; m < kMaxM; ++m)
        if (m < M) acc[m] = fmaf(ys[m][n], b, acc[m]);
    }
  }
#pragma unroll
  for (int m = 0; m < kMaxM; ++m) red[threadIdx.x][m] = acc[m];
  __syncthreads();
  float* out = part + static_cast<int64_t>(blockIdx.x) * M * r16;
  for (int e = threadIdx.x; e < M * r; e += 256) {
    const int m = e / r, jj = e % r;
    float v = 0.0f;
    for (int l = 0; l < lanes; ++l) v += red[l * r + jj][m];
    out[m * r16 + jj] = v;
  }
}

// dB[n][j] = s sum_m dY[m][n] U[m][j]  (+ dB)
__global__ void __launch_bounds__(256)
grad_b_kernel(const __nv_bfloat16* __restrict__ dY, const float* __restrict__ U, int M, int64_t N,
              int r, float s, int accumulate, float* __restrict__ dB) {
  __shared__ float us[kMaxM * 256];
  for (int e = threadIdx.x; e < M * r; e += 256) us[e] = U[e];
  __syncthreads();
  const int64_t total = N * r;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t n = e / r;
    const int j = static_cast<int>(e - n * r);
    float v = 0.0f;
    for (int m = 0; m < M; ++m) v = fmaf(__bfloat162float(dY[m * N + n]), us[m * r + j], v);
    dB[e] = accumulate ? dB[e] + s * v : s * v;
  }
}

// dA[j][k] = s sum_m V[m][j] X[m][k]  (+ dA)
__global__ void __launch_bounds__(256)
grad_a_kernel(const float* __restrict__ V, const __nv_bfloat16* __restrict__ X, int M, int64_t K,
              int r, float s, int accumulate, float* __restrict__ dA) {
  __shared__ float vs[kMaxM * 256];
  for (int e = threadIdx.x; e < M * r; e += 256) vs[e] = V[e];
  __syncthreads();
  const int64_t total = static_cast<int64_t>(r) * K;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int j = static_cast<int>(e / K);
    const int64_t k = e - static_cast<int64_t>(j) * K;
    float v = 0.0f;
    for (int m = 0; m < M; ++m) v = fmaf(vs[m * r + j], __bfloat162float(X[m * K + k]), v);
    dA[e] = accumulate ? dA[e] + s * v : s * v;
  }
}

int grid_cap(int64_t items) {
  const int64_t g = ceil_div(items, 256);
  return static_cast<int>(g < 148 * 8 ? (g < 1 ? 1 : g) : 148 * 8);
}

}  // namespace

int small_chunks(int64_t len) { return static_cast<int>(ceil_div(len, kChunk)); }

qlora_status small_down_partial(const void* X, const void* A, int M, int64_t K, int r,
                                float* part, cudaStream_t s) {
  if (M > kMaxM) return QLORA_ERR_UNSUPPORTED;
  count_launch();
  down_partial_kernel<<<small_chunks(K), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(X), static_cast<const __nv_bfloat16*>(A), M, K, r,
      lora_rows(r), part);
  return after_launch("small_down_partial", s);
}

qlora_status small_v_partial(const void* dY, const void* B, int M, int64_t N, int r, float* part,
                             cudaStream_t s) {
  if (M > kMaxM) return QLORA_ERR_UNSUPPORTED;
  count_launch();
  v_partial_kernel<<<small_chunks(N), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(dY),
                                                   static_cast<const __nv_bfloat16*>(B), M, N, r,
                                                   lora_rows(r), part);
  return after_launch("small_v_partial", s);
}

qlora_status small_grad_b(const void* dY, const float* U, int M, int64_t N, int r, float sc,
                          bool accumulate, float* dB, cudaStream_t s) {
  if (M > kMaxM) return QLORA_ERR_UNSUPPORTED;
  count_launch();
  grad_b_kernel<<<grid_cap(N * r), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(dY), U, M, N, r,
                                                sc, accumulate ? 1 : 0, dB);
  return after_launch("small_grad_b", s);
}

qlora_status small_grad_a(const float* V, const void* X, int M, int64_t K, int r, float sc,
                          bool accumulate, float* dA, cudaStream_t s) {
  if (M > kMaxM) return QLORA_ERR_UNSUPPORTED;
  count_launch();
  grad_a_kernel<<<grid_cap(K * r), 256, 0, s>>>(V, static_cast<const __nv_bfloat16*>(X), M, K, r,
                                                sc, accumulate ? 1 : 0, dA);
  return after_launch("small_grad_a", s);
}

}  // namespace qlora

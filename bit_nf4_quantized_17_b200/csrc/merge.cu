// Merging a trained adapter into a restored 16-bit weight, and the same
// update on a dense bf16 weight.
//
// After training, B A has the shape of W and can be added to it ("LoRA 与
// QLoRA：把大模型微调拆成可负担的工程", section 3); the 4-bit storage cannot
// take the update, so the sum goes into a restored bf16 weight:
//
//   W_merged[n][k] = bf16( fp32(level[idx] * s_hat) + s sum_j B[n][j] A[j][k] )
//
// The dense form adds the update to a bf16 weight instead,
// bf16(W_in + s B A): with -alpha it takes a merged adapter out again
// (unmerge), or moves a merged weight from one adapter to another.
//
// One CTA per 64 x 128 tile of W: the rank-r product is accumulated in fp32
// registers over 32-rank chunks of A and B staged in shared memory (each
// thread 4 rows x 8 columns), then the tile's codes are dequantised, the
// update added and the result rounded once to bf16.  CUDA cores: the update
// has only r multiply-adds per weight.
#include "internal.cuh"

namespace qlora {
namespace {

constexpr int kRows = 64, kCols = 128, kRankChunk = 32;

// DENSE = false: the base is the NF4 weight `w`; true: the bf16 matrix `win`
// (w.rows x w.cols; it may be `out` itself: each element is read, then written,
// by the same thread).
template <bool DENSE>
__global__ void __launch_bounds__(256)
merge_kernel(QView w, LevelTable tab, const __nv_bfloat16* win, const __nv_bfloat16* __restrict__ A,
             const __nv_bfloat16* __restrict__ B, int r, float s, __nv_bfloat16* out) {
  __shared__ __align__(16) float as[kRankChunk][kCols];
  __shared__ float bs[kRows][kRankChunk + 1];
  __shared__ float lv[16];
  const int64_t N = w.rows, K = w.cols;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kCols;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;  // rows 4 ty .., columns 8 tx ..
  if (threadIdx.x == 0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];  // constant indices: no local copy
  }
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[i][c] = 0.0f;

  for (int j0 = 0; j0 < r; j0 += kRankChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kRankChunk * kCols; e += 256) {
      const int jj = e / kCols, c = e % kCols;
      const int64_t k = k0 + c;
      as[jj][c] = (j0 + jj < r && k < K) ? __bfloat162float(A[(j0 + jj) * K + k]) : 0.0f;
    }
    for (int e = threadIdx.x; e < kRows * kRankChunk; e += 256) {
      const int i = e / kRankChunk, jj = e % kRankChunk;
      const int64_t n = n0 + i;
      bs[i][jj] = (j0 + jj < r && n < N) ? __bfloat162float(B[n * r + j0 + jj]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kRankChunk; ++jj) {
      const float4 a0 = *reinterpret_cast<const float4*>(&as[jj][8 * tx]);
      const float4 a1 = *reinterpret_cast<const float4*>(&as[jj][8 * tx + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float b = bs[4 * ty + i][jj];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[i][c] = fmaf(b, a[c], acc[i][c]);
      }
    }
  }
  __syncthreads();

  const float mu = (!DENSE && w.dq_shift >= 0) ? __ldg(w.mean) : 0.0f;
  const int64_t k = k0 + 8 * tx;
  if (k >= K) return;  // K is a multiple of 64: a thread's 8 columns are all in or all out
  const int64_t nb_row = K >> (6 + w.bs_shift);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = n0 + 4 * ty + i;
    if (n >= N) break;
    float base[8];
    if constexpr (DENSE) {
      const uint4 v = *reinterpret_cast<const uint4*>(win + n * K + k);
      const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        base[2 * c] = __uint_as_float(vw[c] << 16);
        base[2 * c + 1] = __uint_as_float(vw[c] & 0xffff0000u);
      }
    } else {
      const uint32_t codes = __ldg(reinterpret_cast<const uint32_t*>(w.codes + (n * K + k) / 2));
      const float sc = block_scale(w, n * nb_row + (k >> (6 + w.bs_shift)), mu);
#pragma unroll
      for (int c = 0; c < 8; ++c) base[c] = __fmul_rn(lv[(codes >> (4 * c)) & 15u], sc);
    }
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const float w0 = base[c];
      const float w1 = base[c + 1];
      const __nv_bfloat162 h = __floats2bfloat162_rn(__fadd_rn(w0, __fmul_rn(s, acc[i][c])),
                                                     __fadd_rn(w1, __fmul_rn(s, acc[i][c + 1])));
      o[c / 2] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(out + n * K + k) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

qlora_status launch_merge(const qlora_nf4& q, const LevelTable& t, const void* A, const void* B,
                          int32_t r, float alpha, void* out, cudaStream_t s) {
  QView w{q.codes, q.scale_codes, q.factors, q.mean, q.rows, q.cols,
          q.dq_blocksize ? __builtin_ctz(q.dq_blocksize) : -1, __builtin_ctz(q.blocksize) - 6};
  const dim3 grid(static_cast<unsigned>(ceil_div(q.cols, kCols)),
                  static_cast<unsigned>(ceil_div(q.rows, kRows)));
  if (grid.y > 65535) return QLORA_ERR_SHAPE;
  count_launch();
  timing_mark(QLORA_KERNEL_MERGE, s, true);
  merge_kernel<false><<<grid, 256, 0, s>>>(w, t, nullptr, static_cast<const __nv_bfloat16*>(A),
                                           static_cast<const __nv_bfloat16*>(B), r,
                                           alpha / static_cast<float>(r),
                                           static_cast<__nv_bfloat16*>(out));
  timing_mark(QLORA_KERNEL_MERGE, s, false);
  return after_launch("merge", s);
}

qlora_status launch_merge_dense(const void* W_in, int64_t rows, int64_t cols, const void* A,
                                const void* B, int32_t r, float alpha, void* out, cudaStream_t s) {
  QView w{};
  w.rows = rows;
  w.cols = cols;
  const dim3 grid(static_cast<unsigned>(ceil_div(cols, kCols)), static_cast<unsigned>(ceil_div(rows, kRows)));
  if (grid.y > 65535) return QLORA_ERR_SHAPE;
  LevelTable unused{};
  count_launch();
  timing_mark(QLORA_KERNEL_MERGE, s, true);
  merge_kernel<true><<<grid, 256, 0, s>>>(w, unused, static_cast<const __nv_bfloat16*>(W_in),
                                          static_cast<const __nv_bfloat16*>(A),
                                          static_cast<const __nv_bfloat16*>(B), r,
                                          alpha / static_cast<float>(r),
                                          static_cast<__nv_bfloat16*>(out));
  timing_mark(QLORA_KERNEL_MERGE, s, false);
  return after_launch("merge_dense", s);
}

}  // namespace qlora

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
// This file holds the CUDA-core form, for the shapes the tensor-core kernel
// (merge_tc.cu) does not take: r not a multiple of 8, or cols not a multiple
// of 64 (dense form).  One CTA per 64 x 128 tile of W: the rank-r product is
// accumulated in fp32
// registers over chunks of up to 32 ranks of A and B staged in shared memory
// (each thread 4 rows x 8 columns, paired fp32 multiply-adds), then the tile's
// codes are dequantised, the update added and the result rounded once to bf16.
// CUDA cores: the update has only r multiply-adds per weight.
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
  __shared__ __align__(16) float bs[kRankChunk][kRows];  // B transposed: a thread's 4 rows in one read
  __shared__ float lv[16];
  const int64_t N = w.rows, K = w.cols;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kCols;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;  // rows 4 ty .., columns 8 tx ..
  if (threadIdx.x == 0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];  // constant indices: no local copy
  }
  // acc[i][c] holds columns 2c, 2c + 1 of row i: paired fp32 multiply-adds
  float2 acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = make_float2(0.0f, 0.0f);

  for (int j0 = 0; j0 < r; j0 += kRankChunk) {
    const int nj = min(kRankChunk, r - j0);
    __syncthreads();
    // A rows j0 .. j0 + nj - 1, columns k0 .. k0 + 127: 8 bf16 (16 bytes) per load
    for (int e = threadIdx.x; e < nj * (kCols / 8); e += 256) {
      const int jj = e / (kCols / 8), c8 = 8 * (e % (kCols / 8));
      const int64_t k = k0 + c8;
      float4 lo = make_float4(0.0f, 0.0f, 0.0f, 0.0f), hi = lo;
      if (k < K) {  // K is a multiple of 64: the 8 columns are all in or all out
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(A + (j0 + jj) * K + k));
        lo = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
        hi = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                         __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
      }
      *reinterpret_cast<float4*>(&as[jj][c8]) = lo;
      *reinterpret_cast<float4*>(&as[jj][c8 + 4]) = hi;
    }
    for (int e = threadIdx.x; e < kRows * nj; e += 256) {
      const int i = e / nj, jj = e % nj;
      const int64_t n = n0 + i;
      bs[jj][i] = (n < N) ? __bfloat162float(B[n * r + j0 + jj]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < nj; ++jj) {
      const float4 a0 = *reinterpret_cast<const float4*>(&as[jj][8 * tx]);
      const float4 a1 = *reinterpret_cast<const float4*>(&as[jj][8 * tx + 4]);
      const float2 a[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w),
                           make_float2(a1.x, a1.y), make_float2(a1.z, a1.w)};
      const float4 b4 = *reinterpret_cast<const float4*>(&bs[jj][4 * ty]);
      const float b[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 bb = make_float2(b[i], b[i]);
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = __ffma2_rn(bb, a[c], acc[i][c]);
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
      const __nv_bfloat162 h = __floats2bfloat162_rn(__fadd_rn(w0, __fmul_rn(s, acc[i][c / 2].x)),
                                                     __fadd_rn(w1, __fmul_rn(s, acc[i][c / 2].y)));
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
  if (merge_tc_eligible(q.cols, r)) return launch_merge_tc(w, t, A, B, r, alpha, out, s);
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
  if (merge_tc_eligible(cols, r))
    return launch_merge_dense_tc(W_in, rows, cols, A, B, r, alpha, out, s);
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

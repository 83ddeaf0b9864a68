// Dequant GEMV kernels for one or two tokens.
//
// With M <= 2 the products Y = X W^T + s U B^T and dX = dY W + s V A are
// matrix-vector products: every weight is used M times, so the work is
// reading the 4-bit codes and turning each into its bf16 compute weight
// bf16(fp32(level[idx] * s_hat)) ("QLoRA技术从入门到精通", 3(2): restore a
// block to BF16 and multiply).  Here that happens in registers on the CUDA
// cores, with the same per-block byte tables and byte permutes as the
// tensor-core kernels, and nothing passes through shared memory but the
// activation vector:
//
//   gemv_fwd    a group of P warps per W row (lanes over 64-weight blocks);
//               the LoRA term s U B^T (U in fp32) joins the same warp sum
//   gemv_dgrad  lanes own 32 consecutive output columns and stream W rows;
//               each CTA sums its warps in a fixed order and writes one fp32
//               partial row per token, summed by splitk_reduce; CTAs of the
//               first row chunk add s V A
//
// Accumulation is fp32 in a fixed order, so results are deterministic.
#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

namespace qlora {
namespace {

using tc::block_tables;
using tc::expand8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRedStride = 32 * 33;  // one warp's 1024 column sums, padded

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// x (MM tokens) lives in shared memory as fp32 in a block-interleaved layout:
// element e of 64-weight block b of token m at ((m * 16 + e / 4) * nb + b) * 4
// + e % 4, so that lanes reading the same 4 elements of consecutive blocks
// hit consecutive 16-byte words.
__device__ __forceinline__ int xs_index(int m, int b, int e, int nb) {
  return ((m * 16 + (e >> 2)) * nb + b) * 4 + (e & 3);
}

template <int MM>
__global__ void __launch_bounds__(kThreads)
gemv_fwd_kernel(QView w, LevelTable tab, const __nv_bfloat16* __restrict__ X,
                const float* __restrict__ U, const __nv_bfloat16* __restrict__ B, int r, float s,
                int P, int iters, __nv_bfloat16* __restrict__ Y) {
  extern __shared__ __align__(16) float xs[];  // MM * K fp32, then MM * r fp32 (s U), then kWarps * MM
  const int64_t N = w.rows;
  const int K = static_cast<int>(w.cols), nb = K / 64;
  float* us = xs + MM * K;
  float* red = us + MM * r;
  // 8 consecutive elements (16 bytes) per load; K % 64 == 0, so no vector
  // straddles a token row or a block, and 4-aligned groups stay together
  for (int i = threadIdx.x; i < MM * K / 8; i += kThreads) {
    const int m = (8 * i) / K, k = 8 * i - m * K;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K + k));
    const int b = k >> 6, e = k & 63;
    *reinterpret_cast<float4*>(xs + xs_index(m, b, e, nb)) =
        make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    *reinterpret_cast<float4*>(xs + xs_index(m, b, e + 4, nb)) =
        make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
  for (int i = threadIdx.x; i < MM * r; i += kThreads) us[i] = s * U[i];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp % P;                       // this warp's share of the row's blocks
  const int groups = kWarps / P;                // row groups per CTA
  const int64_t rg = static_cast<int64_t>(blockIdx.x) * groups + warp / P;
  const int64_t n_groups = static_cast<int64_t>(gridDim.x) * groups;
  float lv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];
  const float mu = (w.dq_shift >= 0) ? __ldg(w.mean) : 0.0f;

  // This lane's work items are (row, block) pairs: blocks lane + 32 q,
  // + 32 P, ... of rows rg, rg + n_groups, ...  The codes and raw scale of the
  // next item are loaded before the current one is processed.
  const int b_first = lane + 32 * q;
  struct Item {
    uint4 c0, c1;
    float q, f;
  };
  auto load = [&](int64_t n, int b, Item& x) {
    if (n < N && b < nb) {
      const uint8_t* cp = w.codes + n * (K / 2) + b * 32;
      x.c0 = __ldg(reinterpret_cast<const uint4*>(cp));
      x.c1 = __ldg(reinterpret_cast<const uint4*>(cp + 16));
      const int64_t blk = n * nb + b;
      if (w.dq_shift < 0) {
        x.q = 1.0f;
        x.f = __ldg(w.factors + blk);
      } else {
        x.q = static_cast<float>(__ldg(w.scale_codes + blk));
        x.f = __ldg(w.factors + (blk >> w.dq_shift));
      }
    }
  };
  Item cur{};
  load(rg, b_first, cur);

  // every warp of the CTA runs `iters` row slots (the CTA synchronises per slot)
  for (int it = 0; it < iters; ++it) {
    const int64_t n = rg + static_cast<int64_t>(it) * n_groups;
    float acc[MM];
#pragma unroll
    for (int m = 0; m < MM; ++m) acc[m] = 0.0f;
    if (n < N) {
      for (int b = b_first; b < nb;) {
        int bn = b + 32 * P;
        int64_t nn = n;
        if (bn >= nb) {
          bn = b_first;
          nn = n + n_groups;
        }
        Item nxt{};
        load(nn, bn, nxt);
        const float sc = (w.dq_shift < 0) ? cur.f : __fadd_rn(__fmul_rn(cur.q, cur.f), mu);
        uint32_t L[4], H[4];
        block_tables(lv, sc, L, H);
        const uint32_t words[8] = {cur.c0.x, cur.c0.y, cur.c0.z, cur.c0.w,
                                   cur.c1.x, cur.c1.y, cur.c1.z, cur.c1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = expand8(words[j], L, H);  // weights 8j .. 8j + 7 of the block
#pragma unroll
          for (int m = 0; m < MM; ++m) {
            const float4 x0 = *reinterpret_cast<const float4*>(xs + xs_index(m, b, 8 * j, nb));
            const float4 x1 = *reinterpret_cast<const float4*>(xs + xs_index(m, b, 8 * j + 4, nb));
            float a = acc[m];
            a = fmaf(bf16_lo(v.x), x0.x, a);
            a = fmaf(bf16_hi(v.x), x0.y, a);
            a = fmaf(bf16_lo(v.y), x0.z, a);
            a = fmaf(bf16_hi(v.y), x0.w, a);
            a = fmaf(bf16_lo(v.z), x1.x, a);
            a = fmaf(bf16_hi(v.z), x1.y, a);
            a = fmaf(bf16_lo(v.w), x1.z, a);
            a = fmaf(bf16_hi(v.w), x1.w, a);
            acc[m] = a;
          }
        }
        cur = nxt;
        if (nn != n) break;  // the prefetched item starts the next row slot
        b = bn;
      }
      if (q == 0) {
        // the LoRA term of this output: sum_j (s U[m][j]) B[n][j]
        for (int j = lane; j < r; j += 32) {
          const float bj = __bfloat162float(B[n * r + j]);
#pragma unroll
          for (int m = 0; m < MM; ++m) acc[m] = fmaf(us[m * r + j], bj, acc[m]);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MM; ++m) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
    }
    if (P == 1) {
      if (n < N && lane == 0)
#pragma unroll
        for (int m = 0; m < MM; ++m) Y[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(acc[m]);
    } else {
      // the P warps of a row group add their sums in a fixed order
      if (lane == 0)
#pragma unroll
        for (int m = 0; m < MM; ++m) red[warp * MM + m] = acc[m];
      __syncthreads();
      if (q == 0 && lane == 0 && n < N) {
#pragma unroll
        for (int m = 0; m < MM; ++m) {
          float t = 0.0f;
          for (int i = 0; i < P; ++i) t += red[(warp + i) * MM + m];
          Y[static_cast<int64_t>(m) * N + n] = __float2bfloat16_rn(t);
        }
      }
      __syncthreads();
    }
  }
}

// CTA c of k-group g: rows [c N / C, (c + 1) N / C), output columns
// [1024 g, 1024 g + 1024); lane l of every warp owns columns 1024 g + 32 l ..
// + 31 (half of one 64-weight block), warp w takes every 8th row of the chunk.
template <int MM>
__global__ void __launch_bounds__(kThreads)
gemv_dgrad_kernel(QView w, LevelTable tab, const __nv_bfloat16* __restrict__ dY,
                  const float* __restrict__ V, const __nv_bfloat16* __restrict__ A, int r, float s,
                  int n_kgroups, float* __restrict__ part) {
  extern __shared__ float red[];  // kWarps * MM * kRedStride fp32
  const int64_t N = w.rows;
  const int K = static_cast<int>(w.cols), nb = K / 64;
  const int g = blockIdx.x % n_kgroups;
  const int c = blockIdx.x / n_kgroups;
  const int C = gridDim.x / n_kgroups;
  const int64_t n_lo = static_cast<int64_t>(c) * N / C, n_hi = static_cast<int64_t>(c + 1) * N / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = 1024 * g + 32 * lane;
  const bool active = k0 < K;
  const int b = k0 >> 6;
  float lv[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];
  const float mu = (w.dq_shift >= 0) ? __ldg(w.mean) : 0.0f;
  float acc[MM][32];
#pragma unroll
  for (int m = 0; m < MM; ++m)
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[m][e] = 0.0f;
  if (active) {
    // the next row's codes, raw scale and dY values are loaded before this row is processed
    struct Row {
      uint4 cw;
      float q, f;
      float dy[MM];
    };
    auto load = [&](int64_t n, Row& x) {
      if (n < n_hi) {
        x.cw = __ldg(reinterpret_cast<const uint4*>(w.codes + n * (K / 2) + k0 / 2));
        const int64_t blk = n * nb + b;
        if (w.dq_shift < 0) {
          x.q = 1.0f;
          x.f = __ldg(w.factors + blk);
        } else {
          x.q = static_cast<float>(__ldg(w.scale_codes + blk));
          x.f = __ldg(w.factors + (blk >> w.dq_shift));
        }
#pragma unroll
        for (int m = 0; m < MM; ++m) x.dy[m] = __bfloat162float(dY[static_cast<int64_t>(m) * N + n]);
      }
    };
    Row cur{};
    load(n_lo + warp, cur);
    for (int64_t n = n_lo + warp; n < n_hi; n += kWarps) {
      Row nxt{};
      load(n + kWarps, nxt);
      const uint4 cw = cur.cw;
      float dy[MM];
#pragma unroll
      for (int m = 0; m < MM; ++m) dy[m] = cur.dy[m];
      const float sc = (w.dq_shift < 0) ? cur.f : __fadd_rn(__fmul_rn(cur.q, cur.f), mu);
      cur = nxt;
      uint32_t L[4], H[4];
      block_tables(lv, sc, L, H);
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = expand8(words[j], L, H);  // columns k0 + 8j .. + 7
        const float wv[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                             bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
        for (int m = 0; m < MM; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[m][8 * j + e] = fmaf(wv[e], dy[m], acc[m][8 * j + e]);
      }
    }
  }
  // the 8 warps' sums, added in a fixed order; column 32 l + e of a warp at
  // l * 33 + e (the padding keeps both the stores and the loads conflict-free)
#pragma unroll
  for (int m = 0; m < MM; ++m)
#pragma unroll
    for (int e = 0; e < 32; ++e) red[(warp * MM + m) * kRedStride + lane * 33 + e] = acc[m][e];
  __syncthreads();
  for (int i = threadIdx.x; i < MM * 1024; i += kThreads) {
    const int m = i / 1024, kk = i - m * 1024;
    const int k = 1024 * g + kk;
    if (k >= K) continue;
    float t = 0.0f;
    for (int wi = 0; wi < kWarps; ++wi) t += red[(wi * MM + m) * kRedStride + (kk >> 5) * 33 + (kk & 31)];
    // the LoRA term s sum_j V[m][j] A[j][k], ranks spread over the row chunks:
    // chunk c adds ranks c, c + C, ...
    float l = 0.0f;
    for (int j = c; j < r; j += C)
      l = fmaf(V[m * r + j], __bfloat162float(A[static_cast<int64_t>(j) * K + k]), l);
    t = fmaf(s, l, t);
    part[(static_cast<int64_t>(c) * MM + m) * K + k] = t;
  }
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return sms;
}

}  // namespace

bool gemv_eligible(int64_t M, int64_t K, int32_t r) {
  return M >= 1 && M <= 2 && K % 64 == 0 && r <= 256 && K <= (int64_t(1) << 20);
}

int gemv_dgrad_chunks(int64_t M, int64_t K) {
  (void)M;
  const int64_t nkg = ceil_div(K, 1024);
  const int64_t target = 3 * 148;
  int64_t c = target / nkg;
  if (c < 1) c = 1;
  return static_cast<int>(c);
}

// CTAs of `kernel` that fit on the device at once with `smem` bytes each.
int resident_grid(const void* kernel, size_t smem) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  return per_sm * device_sms();
}

qlora_status gemv_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                          const float* U, const void* B, int32_t r, float s, void* Y,
                          cudaStream_t st) {
  const int64_t N = w.rows, K = w.cols, nb = K / 64;
  const size_t smem = sizeof(float) * (M * K + M * r + kWarps * M);
  const void* kernel = M == 1 ? reinterpret_cast<const void*>(gemv_fwd_kernel<1>)
                              : reinterpret_cast<const void*>(gemv_fwd_kernel<2>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return QLORA_ERR_CUDA;
  const int grid = resident_grid(kernel, smem);
  const int64_t warps = static_cast<int64_t>(grid) * kWarps;
  // P warps per row: the fewest row slots x blocks per lane
  int best_p = 1;
  int64_t best = -1;
  for (int p = 1; p <= kWarps; p *= 2) {
    const int64_t slots = ceil_div(N, warps / p);
    const int64_t cost = slots * ceil_div(nb, 32 * p);
    if (best < 0 || cost < best) {
      best = cost;
      best_p = p;
    }
  }
  const int iters = static_cast<int>(ceil_div(N, warps / best_p));
  count_launch();
  if (M == 1) {
    timing_mark(QLORA_KERNEL_FUSED_FWD, st, true);
    gemv_fwd_kernel<1><<<grid, kThreads, smem, st>>>(
        w, t, static_cast<const __nv_bfloat16*>(X), U, static_cast<const __nv_bfloat16*>(B), r, s,
        best_p, iters, static_cast<__nv_bfloat16*>(Y));
  } else {
    timing_mark(QLORA_KERNEL_FUSED_FWD, st, true);
    gemv_fwd_kernel<2><<<grid, kThreads, smem, st>>>(
        w, t, static_cast<const __nv_bfloat16*>(X), U, static_cast<const __nv_bfloat16*>(B), r, s,
        best_p, iters, static_cast<__nv_bfloat16*>(Y));
  }
  timing_mark(QLORA_KERNEL_FUSED_FWD, st, false);
  return after_launch("gemv_fwd", st);
}

qlora_status gemv_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                        const float* V, const void* A, int32_t r, float s, float* part,
                        cudaStream_t st) {
  const int64_t K = w.cols;
  const int nkg = static_cast<int>(ceil_div(K, 1024));
  const int C = gemv_dgrad_chunks(M, K);
  const size_t smem = sizeof(float) * kWarps * M * kRedStride;
  count_launch();
  if (M == 1) {
    if (cudaFuncSetAttribute(gemv_dgrad_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    timing_mark(QLORA_KERNEL_FUSED_DGRAD, st, true);
    gemv_dgrad_kernel<1><<<nkg * C, kThreads, smem, st>>>(
        w, t, static_cast<const __nv_bfloat16*>(dY), V, static_cast<const __nv_bfloat16*>(A), r, s,
        nkg, part);
  } else {
    if (cudaFuncSetAttribute(gemv_dgrad_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return QLORA_ERR_CUDA;
    timing_mark(QLORA_KERNEL_FUSED_DGRAD, st, true);
    gemv_dgrad_kernel<2><<<nkg * C, kThreads, smem, st>>>(
        w, t, static_cast<const __nv_bfloat16*>(dY), V, static_cast<const __nv_bfloat16*>(A), r, s,
        nkg, part);
  }
  timing_mark(QLORA_KERNEL_FUSED_DGRAD, st, false);
  return after_launch("gemv_dgrad", st);
}

}  // namespace qlora

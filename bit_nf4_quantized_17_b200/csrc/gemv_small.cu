// Dequant GEMV for the dX product of one or two tokens.
//
// With M <= 2 the product dX = dY W + s V A is a vector-matrix product: every
// weight is used M times, so the work is reading the 4-bit codes and turning
// each into its bf16 compute weight
// bf16(fp32(level[idx] * s_hat)) ("QLoRA技术从入门到精通", 3(2): restore a
// block to BF16 and multiply).  Here that happens in registers on the CUDA
// cores, with the same per-block byte tables and byte permutes as the
// tensor-core kernels: lanes own 32 consecutive output columns and stream W
// rows; each CTA sums its warps in a fixed order, the 8 CTAs of a cluster
// (consecutive row chunks of one column group) sum their rows in shared
// memory, and each cluster writes one fp32 partial row per token, summed by
// splitk_reduce; the LoRA term s V A is spread over the row chunks.
//
// Accumulation is fp32 in a fixed order, so results are deterministic.
#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

using tc::block_tables;
using tc::expand8;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRedStride = 32 * 33;  // one warp's 1024 column sums, padded
constexpr int kCluster = 8;          // row chunks summed in shared memory

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// CTA c of k-group g (blockIdx.x = g C + c): rows [c N / C, (c + 1) N / C),
// output columns [1024 g, 1024 g + 1024); lane l of every warp owns columns
// 1024 g + 32 l .. + 31 (half of one 64-weight block), warp w takes every 8th
// row of the chunk.
template <int MM>
__global__ void __launch_bounds__(kThreads)
gemv_dgrad_kernel(QView w, LevelTable tab, const __nv_bfloat16* __restrict__ dY,
                  const float* __restrict__ V, const __nv_bfloat16* __restrict__ A, int r, float s,
                  int n_kgroups, float* __restrict__ part) {
  extern __shared__ float red[];  // kWarps * MM * kRedStride fp32, then the MM x 1024 CTA sums
  float* csum = red;
  const int64_t N = w.rows;
  const int K = static_cast<int>(w.cols), nb = K >> (6 + w.bs_shift);  // blocks per row
  const int C = gridDim.x / n_kgroups;
  const int g = blockIdx.x / C;
  const int c = blockIdx.x % C;
  const int64_t n_lo = static_cast<int64_t>(c) * N / C, n_hi = static_cast<int64_t>(c + 1) * N / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = 1024 * g + 32 * lane;
  const bool active = k0 < K;
  const int b = k0 >> (6 + w.bs_shift);  // this lane's block within the row
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
  // V is the output of the launch before this one, which lets this grid
  // start early (programmatic dependent launch): the row loop above reads only
  // dY and W
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int kPer = MM * 1024 / kThreads;  // column sums per thread
  float tv[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = threadIdx.x + u * kThreads;
    const int m = i / 1024, kk = i - m * 1024;
    const int k = 1024 * g + kk;
    float t = 0.0f;
    if (k < K) {
      for (int wi = 0; wi < kWarps; ++wi)
        t += red[(wi * MM + m) * kRedStride + (kk >> 5) * 33 + (kk & 31)];
      // the LoRA term s sum_j V[m][j] A[j][k], ranks spread over the row chunks:
      // chunk c adds ranks c, c + C, ...
      float l = 0.0f;
      for (int j = c; j < r; j += C)
        l = fmaf(V[m * r + j], __bfloat162float(A[static_cast<int64_t>(j) * K + k]), l);
      t = fmaf(s, l, t);
    }
    tv[u] = t;
  }
  __syncthreads();  // every warp has read `red`: its space now holds the CTA sums
#pragma unroll
  for (int u = 0; u < kPer; ++u) csum[threadIdx.x + u * kThreads] = tv[u];
  // the cluster's CTAs (row chunks c0 .. c0 + 7) summed in chunk order; CTA q
  // of the cluster writes the q-th eighth of the sums
  ptx::cluster_sync();
  {
    const int cl = c / kCluster;
    const int q0 = static_cast<int>(ptx::cluster_ctarank());
    constexpr int kShare = MM * 1024 / kCluster;
    for (int i = q0 * kShare + threadIdx.x; i < (q0 + 1) * kShare; i += kThreads) {
      const int m = i / 1024, kk = i - m * 1024;
      const int k = 1024 * g + kk;
      float x[kCluster];
#pragma unroll
      for (int q = 0; q < kCluster; ++q) x[q] = ptx::ld_cluster_f32(ptx::cluster_addr(&csum[i], q));
      float t = 0.0f;
#pragma unroll
      for (int q = 0; q < kCluster; ++q) t += x[q];
      if (k < K) part[(static_cast<int64_t>(cl) * MM + m) * K + k] = t;
    }
  }
  ptx::cluster_sync();
}


}  // namespace

bool gemv_eligible(int64_t M, int64_t K, int32_t r) {
  return M >= 1 && M <= 2 && K % 64 == 0 && r <= 256 && K <= (int64_t(1) << 20);
}

namespace {
// Upper bound of the row chunks per column group: about three CTAs per SM, a
// multiple of the cluster size.
int max_chunks(int64_t K) {
  const int64_t nkg = ceil_div(K, 1024);
  int64_t c = (3 * 148) / nkg / kCluster * kCluster;
  if (c < kCluster) c = kCluster;
  return static_cast<int>(c);
}
}  // namespace

int gemv_dgrad_parts(int64_t M, int64_t K) {
  (void)M;
  return max_chunks(K) / kCluster;
}

qlora_status gemv_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                        const float* V, const void* A, int32_t r, float s, float* part,
                        int* parts, cudaStream_t st) {
  const int64_t K = w.cols;
  const int nkg = static_cast<int>(ceil_div(K, 1024));
  const size_t smem = sizeof(float) * kWarps * M * kRedStride;
  auto kernel = (M == 1) ? gemv_dgrad_kernel<1> : gemv_dgrad_kernel<2>;
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the V launch
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // as many row chunks as keep every cluster resident at once (one wave),
  // within the workspace's bound
  const void* fn = reinterpret_cast<const void*>(kernel);
  const qlora_status cs = ensure_smem(fn, static_cast<int>(smem));
  if (cs != QLORA_OK) return cs;
  int res = 0;
  if (!cached_value(fn, 0, &res)) {
    cfg.gridDim = dim3(kCluster, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&res, kernel, &cfg) != cudaSuccess || res < 1) {
      (void)cudaGetLastError();
      res = 1;
    }
    store_value(fn, 0, res);
  }
  int C = (res / nkg) * kCluster;
  if (C > max_chunks(K)) C = max_chunks(K);
  if (C < kCluster) C = kCluster;
  *parts = C / kCluster;
  cfg.gridDim = dim3(static_cast<unsigned>(nkg * C), 1, 1);
  const auto* y = static_cast<const __nv_bfloat16*>(dY);
  const auto* a = static_cast<const __nv_bfloat16*>(A);
  count_launch();
  timing_mark(QLORA_KERNEL_FUSED_DGRAD, st, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, w, t, y, V, a, r, s, nkg, part);
  timing_mark(QLORA_KERNEL_FUSED_DGRAD, st, false);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  return after_launch("gemv_dgrad", st);
}

}  // namespace qlora

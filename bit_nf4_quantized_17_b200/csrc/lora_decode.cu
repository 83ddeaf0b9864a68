// The rank-r products of the adapter branch for decode-sized batches
// (M <= 16 tokens), each in one launch:
//
//   U = X A^T   (X: M x K, A: r x K)    U[m][j] = sum_k X[m][k] A[j][k]
//   V = dY B    (dY: M x N, B: N x r)   V[m][j] = sum_n dY[m][n] B[n][j]
//
// ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", 2: h = W x + (alpha/r) B A x;
// V = dY B is the first factor of dX, dA of the backward pass.)  With so few
// tokens both are reads of A or B (at most 2 MB) with a short contraction per
// output, so the work is spread over a grid of (contraction chunk, 8-rank
// block) CTAs; the CTAs of one rank block form a thread-block cluster, and the
// first CTA of the cluster sums the chunk partials from the others' shared
// memory in chunk order - deterministic, no partials in global memory, no
// second launch - and writes the outputs the callers need: fp32 (U_save, V),
// bf16 hi/lo pairs (the scaled operand of the fused GEMMs' LoRA stage, its
// padding columns zeroed), each token masked to its own adapter's columns.
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 256;
constexpr int kSub = 512;      // contraction elements staged in shared memory at a time
constexpr int kMaxChunks = 8;  // CTAs per cluster (portable cluster size)

__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
  }
}

// The warp's sums of N values per lane (N a power of two), stored to dst[0..N)
// by a reduce-scatter butterfly: at offset o every lane keeps one half of its
// values and adds the partner's copy of that half, so lane l ends with the
// elements [l N/32, (l + 1) N/32) (N >= 32) after N - N/32 shuffles instead of
// 5 N; smaller N finish with a plain butterfly.  Fixed order: deterministic.
template <int N>
__device__ __forceinline__ void warp_sum_store(float (&a)[N], int lane, float* dst) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n >= 2) {
      const bool upper = (lane & o) != 0;
      const int h = n / 2;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < h) {
          const float send = upper ? a[i] : a[i + h];
          const float keep = upper ? a[i + h] : a[i];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n = h;
    } else {
      a[0] += __shfl_xor_sync(0xffffffffu, a[0], o);
    }
  }
  if (N >= 32) {
#pragma unroll
    for (int i = 0; i < (N >= 32 ? N / 32 : 1); ++i) dst[lane * (N / 32) + i] = a[i];
  } else if (lane % (32 / N) == 0) {
    dst[lane / (32 / N)] = a[0];
  }
}

// Write rank column j of token m from the cluster sum v (rank 0 of the cluster).
__device__ __forceinline__ void store_rank(const RankOut& o, int m, int j, float v) {
  if (j < o.r) {
    if (o.seg && __ldg(o.seg + m) != j / o.seg_cols) v = 0.0f;
    if (o.o1) o.o1[static_cast<int64_t>(m) * o.ld1 + j] = o.a1 * v;
    if (o.o2) {
      const float x = o.a2 * v;
      const __nv_bfloat16 h = __float2bfloat16_rn(x);
      o.o2[static_cast<int64_t>(m) * o.ld2 + j] = h;
      o.o2[static_cast<int64_t>(m) * o.ld2 + j + o.o2_lo] = __float2bfloat16_rn(x - __bfloat162float(h));
    }
  } else if (o.o2 && j < o.o2_lo) {
    // padding columns [r, o2_lo) of both halves: they meet zero columns in the MMA
    o.o2[static_cast<int64_t>(m) * o.ld2 + j] = __float2bfloat16_rn(0.0f);
    o.o2[static_cast<int64_t>(m) * o.ld2 + j + o.o2_lo] = __float2bfloat16_rn(0.0f);
  }
}

// Sum the per-CTA partials red[w][m] (JB ranks x MM tokens) over the cluster's
// CTAs in rank order and store; CTA q of the cluster writes the items
// t = q, q + nrank, ... of the 8 MM, and every CTA keeps its shared memory
// until the others have read it.
template <int MM, int JB>
__device__ __forceinline__ void cluster_finish(const float (&red)[JB][MM], const RankOut& o, int M,
                                               int jb) {
  ptx::cluster_sync();
  const int nrank = static_cast<int>(gridDim.x);  // the cluster spans the grid's x dimension
  for (int t = static_cast<int>(ptx::cluster_ctarank()) + nrank * static_cast<int>(threadIdx.x);
       t < JB * MM; t += nrank * static_cast<int>(blockDim.x)) {
    const int w = t / MM, m = t % MM;
    float x[kMaxChunks];
#pragma unroll
    for (int q = 0; q < kMaxChunks; ++q)
      x[q] = (q < nrank) ? ptx::ld_cluster_f32(ptx::cluster_addr(&red[w][m], q)) : 0.0f;
    float v = 0.0f;
#pragma unroll
    for (int q = 0; q < kMaxChunks; ++q)
      if (q < nrank) v += x[q];
    if (m < M) store_rank(o, m, JB * jb + w, v);
  }
  ptx::cluster_sync();
}

// U = X A^T.  CTA (c, jb): contraction chunk c of `len` elements, ranks
// 8 jb .. 8 jb + 7 (one per warp); lanes take 8 consecutive k per step.
template <int MM>
__global__ void __launch_bounds__(kThreads)
rank_down_kernel(const __nv_bfloat16* __restrict__ X, const __nv_bfloat16* __restrict__ A, int M,
                 int64_t K, int len, RankOut o) {
  // the decode forward that follows may start now: it reads this launch's
  // output only after its own grid-dependency wait
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ __align__(16) float xs[MM][kSub];
  __shared__ float red[8][MM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jb = blockIdx.y;
  const int j = 8 * jb + warp;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * len;
  const int64_t c1 = (c0 + len < K) ? c0 + len : K;
  float acc[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) acc[m] = 0.0f;
  for (int64_t s0 = c0; s0 < c1; s0 += kSub) {
    const int n = static_cast<int>((c1 - s0) < kSub ? (c1 - s0) : kSub);  // a multiple of 8
    __syncthreads();
    for (int e = threadIdx.x; e < MM * (kSub / 8); e += kThreads) {
      const int m = e / (kSub / 8), k = 8 * (e % (kSub / 8));
      float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (m < M && k < n) bf16x8_to_f32(*reinterpret_cast<const uint4*>(X + m * K + s0 + k), f);
      *reinterpret_cast<float4*>(&xs[m][k]) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4*>(&xs[m][k + 4]) = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncthreads();
    if (j < o.r) {
      for (int k = 8 * lane; k < n; k += 256) {
        float a[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + s0 + k), a);
#pragma unroll
        for (int m = 0; m < MM; ++m) {
          const float4 x0 = *reinterpret_cast<const float4*>(&xs[m][k]);
          const float4 x1 = *reinterpret_cast<const float4*>(&xs[m][k + 4]);
          float t = acc[m];
          t = fmaf(x0.x, a[0], t);
          t = fmaf(x0.y, a[1], t);
          t = fmaf(x0.z, a[2], t);
          t = fmaf(x0.w, a[3], t);
          t = fmaf(x1.x, a[4], t);
          t = fmaf(x1.y, a[5], t);
          t = fmaf(x1.z, a[6], t);
          t = fmaf(x1.w, a[7], t);
          acc[m] = t;
        }
      }
    }
  }
  warp_sum_store<MM>(acc, lane, red[warp]);
  cluster_finish<MM, 8>(red, o, M, jb);
}

// V = dY B.  CTA (c, jb): rows [c len, (c + 1) len) of B, rank columns
// JB jb .. JB jb + JB - 1 (2 JB bytes of each row); thread t takes rows t,
// t + 256, ..., loading kAhead rows (B and the tokens' dY values) before using
// them.  Wide token counts take 4-rank blocks: half the accumulators per
// thread, twice the CTAs.
template <int MM>
__global__ void __launch_bounds__(kThreads)
rank_v_kernel(const __nv_bfloat16* __restrict__ dY, const __nv_bfloat16* __restrict__ B, int M,
              int64_t N, int len, RankOut o) {
  // the dX kernel that follows may start now: it reads V only after its own
  // grid-dependency wait
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int JB = MM >= 8 ? 4 : 8;
  constexpr int kAhead = MM >= 8 ? 2 : 4;
  __shared__ float wred[8][MM * JB];
  __shared__ float red[JB][MM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jb = blockIdx.y;
  const bool real = JB * jb < o.r;  // r is a multiple of 8: a block is all ranks or all padding
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * len;
  const int64_t c1 = (c0 + len < N) ? c0 + len : N;
  float acc[MM * JB];  // [m][q]
#pragma unroll
  for (int e = 0; e < MM * JB; ++e) acc[e] = 0.0f;
  if (real) {
    for (int64_t n0 = c0 + threadIdx.x; n0 < c1; n0 += kAhead * kThreads) {
      float bf[kAhead][JB];
      float dy[kAhead][MM];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const int64_t n = n0 + static_cast<int64_t>(u) * kThreads;
        const bool in = n < c1;
        if constexpr (JB == 8) {
          const uint4 v = in ? *reinterpret_cast<const uint4*>(B + n * o.r + 8 * jb)
                             : make_uint4(0u, 0u, 0u, 0u);
          bf16x8_to_f32(v, bf[u]);
        } else {
          const uint2 v = in ? *reinterpret_cast<const uint2*>(B + n * o.r + 4 * jb)
                             : make_uint2(0u, 0u);
          bf[u][0] = __uint_as_float(v.x << 16);
          bf[u][1] = __uint_as_float(v.x & 0xffff0000u);
          bf[u][2] = __uint_as_float(v.y << 16);
          bf[u][3] = __uint_as_float(v.y & 0xffff0000u);
        }
#pragma unroll
        for (int m = 0; m < MM; ++m) dy[u][m] = (in && m < M) ? __bfloat162float(dY[m * N + n]) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
#pragma unroll
        for (int m = 0; m < MM; ++m)
#pragma unroll
          for (int q = 0; q < JB; ++q) acc[JB * m + q] = fmaf(dy[u][m], bf[u][q], acc[JB * m + q]);
    }
  }
  // sum over the CTA's threads: the lanes of each warp, then the 8 warps in order
  warp_sum_store<MM * JB>(acc, lane, wred[warp]);
  __syncthreads();
  for (int t = threadIdx.x; t < JB * MM; t += kThreads) {
    const int q = t / MM, m = t % MM;
    float v = 0.0f;
    for (int w = 0; w < 8; ++w) v += wred[w][JB * m + q];
    red[q][m] = v;
  }
  cluster_finish<MM, JB>(red, o, M, jb);
}

int tokens_pad(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

template <typename KernelT>
qlora_status launch_cluster(KernelT kernel, int chunks, int jblocks, cudaStream_t s,
                            const void* a0, const void* a1, int M, int64_t L, int len,
                            const RankOut& o) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(jblocks), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(chunks);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<const __nv_bfloat16*>(a0),
                                           static_cast<const __nv_bfloat16*>(a1), M, L, len, o);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

// Contraction of `L` elements split into at most kMaxChunks chunks of a
// multiple of 64 elements, at least 512 each.
void chunking(int64_t L, int* chunks, int* len) {
  int64_t c = ceil_div(L, 512);
  if (c > kMaxChunks) c = kMaxChunks;
  if (c < 1) c = 1;
  int64_t l = ceil_div(ceil_div(L, c), 64) * 64;
  *chunks = static_cast<int>(ceil_div(L, l));
  *len = static_cast<int>(l);
}

}  // namespace

qlora_status rank_down(const void* X, const void* A, int M, int64_t K, int32_t span,
                       const RankOut& o, cudaStream_t s) {
  if (M < 1 || M > kSmallM || K % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  int chunks, len;
  chunking(K, &chunks, &len);
  const int jblocks = ceil_div(span, 8);
  qlora_status st;
  switch (tokens_pad(M)) {
    case 1: st = launch_cluster(rank_down_kernel<1>, chunks, jblocks, s, X, A, M, K, len, o); break;
    case 2: st = launch_cluster(rank_down_kernel<2>, chunks, jblocks, s, X, A, M, K, len, o); break;
    case 4: st = launch_cluster(rank_down_kernel<4>, chunks, jblocks, s, X, A, M, K, len, o); break;
    case 8: st = launch_cluster(rank_down_kernel<8>, chunks, jblocks, s, X, A, M, K, len, o); break;
    default: st = launch_cluster(rank_down_kernel<16>, chunks, jblocks, s, X, A, M, K, len, o);
  }
  if (st != QLORA_OK) return st;
  return after_launch("rank_down", s);
}

qlora_status rank_v(const void* dY, const void* B, int M, int64_t N, int32_t span,
                    const RankOut& o, cudaStream_t s) {
  if (M < 1 || M > kSmallM || o.r % 8 != 0) return QLORA_ERR_UNSUPPORTED;
  int chunks, len;
  chunking(N, &chunks, &len);
  const int jblocks = ceil_div(span, tokens_pad(M) >= 8 ? 4 : 8);  // the kernel's JB
  qlora_status st;
  switch (tokens_pad(M)) {
    case 1: st = launch_cluster(rank_v_kernel<1>, chunks, jblocks, s, dY, B, M, N, len, o); break;
    case 2: st = launch_cluster(rank_v_kernel<2>, chunks, jblocks, s, dY, B, M, N, len, o); break;
    case 4: st = launch_cluster(rank_v_kernel<4>, chunks, jblocks, s, dY, B, M, N, len, o); break;
    case 8: st = launch_cluster(rank_v_kernel<8>, chunks, jblocks, s, dY, B, M, N, len, o); break;
    default: st = launch_cluster(rank_v_kernel<16>, chunks, jblocks, s, dY, B, M, N, len, o);
  }
  if (st != QLORA_OK) return st;
  return after_launch("rank_v", s);
}

}  // namespace qlora

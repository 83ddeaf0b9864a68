// Quantise, double-quantise and dequantise kernels.
//
// Steps ("QLoRA技术从入门到精通", 3(1) 基座模型初始化量化): per block of
// `blocksize` consecutive weights, scale = absmax; x = w / scale in [-1, 1];
// index of the nearest table level; two indices per byte; then the fp32
// block scales are quantised again to 8 bits (双重量化).  Dequantisation is
// level[idx] * scale (same page, 3(2) 前向传播).
//
// Launch sequence of qlora_quantize (all on the caller's stream):
//   1. memset of the reduction words in the workspace
//   2. quantize_blocks_kernel   one warp per block: warp-shuffle absmax,
//                               IEEE division, 4-step branch-free search of
//                               the decision thresholds, nibble packing; CTA
//                               max of the scales -> one atomicMax per CTA
//   3. scale_sum_kernel         fixed-point sum of the scales (integer
//                               atomics: the result is order-independent)
//   4. dq_groups_kernel         one CTA per group: centred scales, group
//                               absmax, factor, int8 codes, and the mean
// Without double quantisation only step 2 runs and writes absmax to
// `factors`.
#include <cuda_bf16.h>

#include "internal.cuh"

namespace qlora {
namespace {

constexpr int kMeanFracBits = 32;

__device__ __forceinline__ int nearest_index(float x, const float* thr) {
  int i = (x > thr[7]) ? 8 : 0;
  i += (x > thr[i + 3]) ? 4 : 0;
  i += (x > thr[i + 1]) ? 2 : 0;
  i += (x > thr[i]) ? 1 : 0;
  return i;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ void load_pair(const T* __restrict__ w, int64_t e, int64_t n,
                                          float& a, float& b) {
  if (e + 1 < n) {
    if constexpr (sizeof(T) == 4) {
      float2 v = __ldg(reinterpret_cast<const float2*>(w + e));
      a = v.x;
      b = v.y;
    } else {
      __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(w + e);
      a = __low2float(v);
      b = __high2float(v);
    }
  } else {
    a = (e < n) ? to_f32(w[e]) : 0.0f;
    b = 0.0f;
  }
}

template <typename T, int BS>
__global__ void __launch_bounds__(256)
quantize_blocks_kernel(const T* __restrict__ w, int64_t n, LevelTable tab,
                       uint8_t* __restrict__ codes, float* __restrict__ absmax,
                       unsigned int* __restrict__ gmax_bits, DeviceStatus* st) {
  constexpr int kPairs = BS / 64;  // element pairs per lane per block
  __shared__ float thr[16];
  __shared__ unsigned int cta_max;
  if (threadIdx.x < 16) thr[threadIdx.x] = tab.thr[threadIdx.x];
  if (threadIdx.x == 0) cta_max = 0u;
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t nb = (n + BS - 1) / BS;
  float seen_max = 0.0f;
  bool nonfinite = false;

  for (int64_t b = warp; b < nb; b += nwarps) {
    const int64_t base = b * BS;
    float v[2 * kPairs];
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      load_pair(w, base + 64 * j + 2 * lane, n, v[2 * j], v[2 * j + 1]);
      nonfinite |= !isfinite(v[2 * j]) || !isfinite(v[2 * j + 1]);
      a = fmaxf(a, fmaxf(fabsf(v[2 * j]), fabsf(v[2 * j + 1])));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
      const int64_t e = base + 64 * j + 2 * lane;
      if (e >= n) continue;
      float x0 = (a > 0.0f) ? __fdiv_rn(v[2 * j], a) : 0.0f;
      float x1 = (a > 0.0f) ? __fdiv_rn(v[2 * j + 1], a) : 0.0f;
      int i0 = nearest_index(x0, thr);
      int i1 = (e + 1 < n) ? nearest_index(x1, thr) : 0;
      codes[e >> 1] = static_cast<uint8_t>(i0 | (i1 << 4));
    }
    if (lane == 0) absmax[b] = a;
    seen_max = fmaxf(seen_max, a);
  }
  if (nonfinite) report(st, QLORA_ERR_NONFINITE, 1u);
  // scales are >= 0, so their fp32 bit patterns order like unsigned integers
  atomicMax(&cta_max, __float_as_uint(seen_max));
  __syncthreads();
  if (threadIdx.x == 0 && cta_max != 0u) atomicMax(gmax_bits, cta_max);
}

// t_b = floor(s_b * 2^(32 - E)) summed exactly in 64-bit integers.
__global__ void __launch_bounds__(256)
scale_sum_kernel(const float* __restrict__ absmax, int64_t nb,
                 const unsigned int* __restrict__ gmax_bits,
                 unsigned long long* __restrict__ sum) {
  const float smax = __uint_as_float(*gmax_bits);
  if (smax == 0.0f) return;
  int e;
  frexpf(smax, &e);
  const double scale = ldexp(1.0, kMeanFracBits - e);
  unsigned long long acc = 0ull;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nb;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    acc += static_cast<unsigned long long>(__dmul_rn(static_cast<double>(absmax[b]), scale));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  __shared__ unsigned long long part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0ull;
    for (int i = 0; i < (blockDim.x >> 5); ++i) t += part[i];
    if (t) atomicAdd(sum, t);
  }
}

__device__ __forceinline__ float scale_mean(const unsigned int* gmax_bits,
                                            const unsigned long long* sum, int64_t nb) {
  const float smax = __uint_as_float(*gmax_bits);
  if (smax == 0.0f) return 0.0f;
  int e;
  frexpf(smax, &e);
  double m = __dmul_rn(__ull2double_rn(*sum), ldexp(1.0, e - kMeanFracBits));
  return __double2float_rn(__ddiv_rn(m, static_cast<double>(nb)));
}

// One CTA of dq threads per group of dq consecutive block scales.
__global__ void dq_groups_kernel(const float* __restrict__ absmax, int64_t nb,
                                 const unsigned int* __restrict__ gmax_bits,
                                 const unsigned long long* __restrict__ sum,
                                 int8_t* __restrict__ qcodes, float* __restrict__ factors,
                                 float* __restrict__ mean_out) {
  __shared__ float red[32];
  const float mu = scale_mean(gmax_bits, sum, nb);
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const bool valid = b < nb;
  const float c = valid ? __fsub_rn(absmax[b], mu) : 0.0f;
  float a = fabsf(c);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, off));
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float f = __fdiv_rn(red[0], 127.0f);
  if (valid) {
    int q = 0;
    if (f > 0.0f) {
      float r = rintf(__fdiv_rn(c, f));
      r = fminf(fmaxf(r, -127.0f), 127.0f);
      q = static_cast<int>(r);
    }
    qcodes[b] = static_cast<int8_t>(q);
  }
  if (threadIdx.x == 0) {
    factors[blockIdx.x] = f;
    if (blockIdx.x == 0) *mean_out = mu;
  }
}

// Eight weights per thread; blocks are >= 64 weights, so the eight share a scale.
template <typename T>
__global__ void __launch_bounds__(256)
dequantize_kernel(QView w, int32_t bs_shift, LevelTable tab, T* __restrict__ out) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = tab.level[threadIdx.x];
  __syncthreads();
  const int64_t n = w.rows * w.cols;
  const int64_t groups = (n + 7) >> 3;
  const float mu = (w.dq_shift >= 0) ? __ldg(w.mean) : 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < groups;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e0 = i << 3;
    const bool full = e0 + 8 <= n;
    uint32_t c;
    if (full) {
      c = __ldg(reinterpret_cast<const uint32_t*>(w.codes) + i);
    } else {
      c = 0u;
      for (int j = 0; j < 4 && e0 + 2 * j < n; ++j)
        c |= static_cast<uint32_t>(w.codes[(e0 >> 1) + j]) << (8 * j);
    }
    const float sc = block_scale(w, e0 >> bs_shift, mu);
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = __fmul_rn(lv[(c >> (4 * j)) & 15u], sc);
    if constexpr (sizeof(T) == 4) {
      if (full) {
        float4* o = reinterpret_cast<float4*>(out + e0);
        o[0] = make_float4(v[0], v[1], v[2], v[3]);
        o[1] = make_float4(v[4], v[5], v[6], v[7]);
      } else {
        for (int j = 0; j < 8 && e0 + j < n; ++j) out[e0 + j] = v[j];
      }
    } else {
      if (full) {
        __align__(16) __nv_bfloat162 h[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        *reinterpret_cast<uint4*>(out + e0) = *reinterpret_cast<uint4*>(h);
      } else {
        for (int j = 0; j < 8 && e0 + j < n; ++j) out[e0 + j] = __float2bfloat16_rn(v[j]);
      }
    }
  }
}

int grid_for(int64_t work_items, int per_cta, int max_ctas) {
  int64_t g = ceil_div(work_items, per_cta);
  if (g < 1) g = 1;
  if (g > max_ctas) g = max_ctas;
  return static_cast<int>(g);
}

template <typename T>
void launch_blocks(int bs, const T* w, int64_t n, const LevelTable& t, uint8_t* codes,
                   float* absmax, unsigned int* gmax, DeviceStatus* st, cudaStream_t s) {
  const int64_t nb = ceil_div(n, bs);
  const int grid = grid_for(nb, 8, 148 * 16);
  count_launch();
  timing_mark(QLORA_KERNEL_QUANTIZE, s, true);
  switch (bs) {
    case 64: quantize_blocks_kernel<T, 64><<<grid, 256, 0, s>>>(w, n, t, codes, absmax, gmax, st); break;
    case 128: quantize_blocks_kernel<T, 128><<<grid, 256, 0, s>>>(w, n, t, codes, absmax, gmax, st); break;
    case 256: quantize_blocks_kernel<T, 256><<<grid, 256, 0, s>>>(w, n, t, codes, absmax, gmax, st); break;
    case 512: quantize_blocks_kernel<T, 512><<<grid, 256, 0, s>>>(w, n, t, codes, absmax, gmax, st); break;
    default: quantize_blocks_kernel<T, 1024><<<grid, 256, 0, s>>>(w, n, t, codes, absmax, gmax, st); break;
  }
  timing_mark(QLORA_KERNEL_QUANTIZE, s, false);
}

}  // namespace

// Workspace of qlora_quantize: [status 256 B][gmax u32 @256][sum u64 @264][absmax fp32[nb] @512]
qlora_status launch_quantize(const void* W, int32_t w_dtype, const qlora_nf4& q,
                             const LevelTable& t, void* workspace, cudaStream_t s) {
  char* ws = static_cast<char*>(workspace);
  auto* st = reinterpret_cast<DeviceStatus*>(ws);
  auto* gmax = reinterpret_cast<unsigned int*>(ws + 256);
  auto* sum = reinterpret_cast<unsigned long long*>(ws + 264);
  float* absmax = q.dq_blocksize ? reinterpret_cast<float*>(ws + 512) : q.factors;
  const int64_t n = q.rows * q.cols;
  const int64_t nb = ceil_div(n, q.blocksize);
  if (cudaMemsetAsync(ws + 256, 0, 16, s) != cudaSuccess) return QLORA_ERR_CUDA;
  if (w_dtype == QLORA_F32)
    launch_blocks(q.blocksize, static_cast<const float*>(W), n, t, q.codes, absmax, gmax, st, s);
  else
    launch_blocks(q.blocksize, static_cast<const __nv_bfloat16*>(W), n, t, q.codes, absmax, gmax,
                  st, s);
  if (after_launch("quantize_blocks", s) != QLORA_OK) return QLORA_ERR_CUDA;
  if (q.dq_blocksize) {
    count_launch(2);
    scale_sum_kernel<<<grid_for(nb, 256, 148 * 8), 256, 0, s>>>(absmax, nb, gmax, sum);
    if (after_launch("scale_sum", s) != QLORA_OK) return QLORA_ERR_CUDA;
    const int64_t ng = ceil_div(nb, q.dq_blocksize);
    dq_groups_kernel<<<static_cast<unsigned>(ng), q.dq_blocksize, 0, s>>>(
        absmax, nb, gmax, sum, q.scale_codes, q.factors, q.mean);
    if (after_launch("dq_groups", s) != QLORA_OK) return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

qlora_status launch_dequantize(const qlora_nf4& q, const LevelTable& t, void* out,
                               int32_t out_dtype, cudaStream_t s) {
  QView w{q.codes, q.scale_codes, q.factors, q.mean, q.rows, q.cols,
          q.dq_blocksize ? __builtin_ctz(q.dq_blocksize) : -1};
  const int bs_shift = __builtin_ctz(q.blocksize);
  const int64_t n = q.rows * q.cols;
  const int grid = grid_for(ceil_div(n, 8), 256, 148 * 8);
  count_launch();
  if (out_dtype == QLORA_F32)
    dequantize_kernel<float><<<grid, 256, 0, s>>>(w, bs_shift, t, static_cast<float*>(out));
  else
    dequantize_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(w, bs_shift, t,
                                                          static_cast<__nv_bfloat16*>(out));
  return after_launch("dequantize", s);
}

}  // namespace qlora

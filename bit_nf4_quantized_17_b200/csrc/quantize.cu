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
//   2. quantize_blocks_kernel   16 (or 32) weights per thread, one block per
//                               4..32 lanes: shuffle absmax, nearest level by
//                               a cell lookup (IEEE division where the lookup
//                               cannot decide), nibble packing; CTA max of
//                               the scales -> one atomicMax per CTA
//   3. scale_sum_kernel         fixed-point sum of the scales (integer
//                               atomics: the result is order-independent)
//   4. dq_groups_kernel         one CTA per group: centred scales, group
//                               absmax, factor, int8 codes, and the mean
// Without double quantisation only step 2 runs and writes absmax to
// `factors`.
#include <cuda_bf16.h>

#include <cstring>

#include "internal.cuh"

namespace qlora {
namespace {

constexpr int kMeanFracBits = 32;

// Nearest-level search.  The index of x = RN(w / s) is the number of
// decision thresholds below it (ties go to the lower level).  The quantiser
// finds it without dividing for almost every weight:
//   x' = RN(w * RN(1/s)) lies within 1.5e-7 of x (|x| <= 1 and s a normal
//   float: two roundings of relative size 2^-24 each, plus the rounding of x);
//   c = round(32 x') + 32 picks one of 65 cells of width 1/32 covering
//   [-1, 1] (computed exactly by one FMA into the low mantissa bits of
//   1.5 * 2^23); every gap between thresholds of the two tables is wider than
//   a cell (NF4: 0.046, uniform: 0.133), so a cell widened by kCellPad on each
//   side holds at most one threshold t_c (2.0 when it holds none);
//   index = (number of thresholds below the widened cell) + (x' > t_c).
// The comparison of x' with t_c agrees with that of x whenever
// |x' - t_c| > kNear; otherwise, and for blocks whose scale is 0, subnormal,
// huge or not finite, the chunk is redone with IEEE division and a comparison
// against every threshold.
//
// Arithmetic form (mostly FMA-pipe work, pairs of weights in the paired fp32
// instructions): the cell's bits, c + 1.5 * 2^23, times the table's row pitch
// are its shared-memory address less a constant, one integer multiply-add;
// step = sat((x' - t_c) * 2^126) is 1.0 or 0.0 outside the near band;
// 2^23 + count + step has the index in its low mantissa bits, and an integer
// multiply-add places those bits at the weight's nibble (the constant 2^23
// bits cancel: see kPackBias).
constexpr int kCells = 65;
constexpr double kCellPad = 1e-6;
constexpr float kNear = 1e-6f;
// 32-bit words of the float 2^23 (+ index), shifted to nibbles 0 and 1, summed
// mod 2^32 (higher nibbles shift the constant out): 0x4B000000 + 0xB0000000.
constexpr uint32_t kPackBias = 0xFB000000u;

struct CellLut {
  float2 e[kCells];  // x: t_c, y: 2^23 + number of thresholds below the cell
};

bool make_cell_lut(const LevelTable& tab, CellLut* out) {
  for (int c = 0; c < kCells; ++c) {
    const double lo = (c - 32 - 0.5) / 32.0 - kCellPad;
    const double hi = (c - 32 + 0.5) / 32.0 + kCellPad;
    int below = 0, inside = -1, n_inside = 0;
    for (int k = 0; k < 15; ++k) {
      const double t = tab.thr[k];
      if (t < lo) {
        ++below;
      } else if (t <= hi) {
        inside = k;
        ++n_inside;
      }
    }
    if (n_inside > 1) return false;
    out->e[c].x = n_inside ? tab.thr[inside] : 2.0f;
    out->e[c].y = 8388608.0f + static_cast<float>(below);
  }
  return true;
}

// Raw words of E consecutive weights at e0 (bf16: two per 32-bit word, the
// even element in the low half); zeros at and beyond n.
template <typename T, int E>
struct Raw {
  static constexpr int kWords = sizeof(T) == 4 ? E : E / 2;
  uint32_t u[kWords];
};

template <typename T, int E>
__device__ __forceinline__ void load_raw(const T* __restrict__ w, int64_t e0, int64_t n,
                                         Raw<T, E>& r) {
  if (e0 + E <= n) {
#pragma unroll
    for (int i = 0; i < Raw<T, E>::kWords / 4; ++i) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(w + e0) + i);
      r.u[4 * i] = q.x;
      r.u[4 * i + 1] = q.y;
      r.u[4 * i + 2] = q.z;
      r.u[4 * i + 3] = q.w;
    }
  } else {
    const uint32_t* wb = reinterpret_cast<const uint32_t*>(w);
#pragma unroll
    for (int i = 0; i < Raw<T, E>::kWords; ++i) {
      uint32_t x = 0u;
      if constexpr (sizeof(T) == 4) {
        if (e0 + i < n) x = wb[e0 + i];
      } else {
        const uint16_t* h = reinterpret_cast<const uint16_t*>(w);
        if (e0 + 2 * i < n) x = h[e0 + 2 * i];
        if (e0 + 2 * i + 1 < n) x |= static_cast<uint32_t>(h[e0 + 2 * i + 1]) << 16;
      }
      r.u[i] = x;
    }
  }
}

template <typename T, int E>
__device__ __forceinline__ void unpack_raw(const Raw<T, E>& r, float* v) {
#pragma unroll
  for (int i = 0; i < Raw<T, E>::kWords; ++i) {
    if constexpr (sizeof(T) == 4) {
      v[i] = __uint_as_float(r.u[i]);
    } else {
      v[2 * i] = __uint_as_float(r.u[i] << 16);
      v[2 * i + 1] = __uint_as_float(r.u[i] & 0xffff0000u);
    }
  }
}

// max(a, |b|), NaN if either is NaN
__device__ __forceinline__ float max_abs_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(fabsf(b)));
  return r;
}

// One thread per E consecutive weights (16-byte loads), BS / E threads per
// block, all within one warp: the block absmax is a shuffle reduction over
// those threads.  Codes go out as one 8- or 16-byte store per thread; the
// first thread of each block writes its scale.  The next chunk's words are
// loaded before the current one is processed.
template <typename T, int BS>
__global__ void __launch_bounds__(256)
quantize_blocks_kernel(const T* __restrict__ w, int64_t n, LevelTable tab, CellLut cells,
                       uint8_t* __restrict__ codes, float* __restrict__ absmax,
                       unsigned int* __restrict__ gmax_bits, DeviceStatus* st) {
  constexpr int E = BS <= 512 ? 16 : 32;  // weights per thread
  constexpr int TPB = BS / E;             // threads per block: 4 .. 32
  constexpr int W = E / 8;                // 32-bit words of codes per thread
  // cell table replicated per lane (entry c of lane l at c * 32 + l): a warp's
  // 8-byte reads take the minimum two shared-memory wavefronts
  __shared__ float2 lut[kCells * 32];
  __shared__ unsigned int cta_max;
  for (int i = threadIdx.x; i < kCells * 32; i += blockDim.x) lut[i] = cells.e[i >> 5];
  if (threadIdx.x == 0) cta_max = 0u;
  __syncthreads();

  const int lane = threadIdx.x & 31;
  // address of entry c of this lane's copy: bits(1.5 * 2^23 + c) * 256 + lut_bias
  // (mod 2^32), since bits(1.5 * 2^23) * 256 = 0x4B400000 * 256 = 0x40000000 mod 2^32
  const uint32_t lut_bias = static_cast<uint32_t>(__cvta_generic_to_shared(lut + lane)) - 0x40000000u;
  const int64_t n_chunks = (n + E - 1) / E;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float seen = 0.0f;  // largest finite scale
  bool nonfinite = false;

  // the trip count is the same for every lane of a warp (shuffles inside)
  int64_t wc = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  Raw<T, E> cur;
  if (wc < n_chunks) load_raw<T, E>(w, (wc + lane) * E, n, cur);
  for (; wc < n_chunks; wc += stride) {
    const int64_t e0 = (wc + lane) * E;
    Raw<T, E> nxt;
    if (wc + stride < n_chunks) load_raw<T, E>(w, (wc + stride + lane) * E, n, nxt);
    float v[E];
    unpack_raw<T, E>(cur, v);
    float a = 0.0f;
#pragma unroll
    for (int j = 0; j < E; ++j) a = max_abs_nan(a, v[j]);
#pragma unroll
    for (int off = 1; off < TPB; off <<= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, a, off);
      asm("max.NaN.f32 %0, %0, %1;" : "+f"(a) : "f"(o));
    }
    const float s = a;
    const bool finite = s <= 3.402823466e38f;  // false for inf and NaN
    nonfinite |= !finite;
    if (finite) seen = fmaxf(seen, s);

    uint32_t packed[W];
    bool exact = !(s >= 0x1p-126f && s < 0x1p126f);
    if (!exact) {
      // |v| <= s (s is the block's absmax, finite) and s normal: |x'| <= 1 + 2^-23,
      // so f = RN(32 x' + 1.5 * 2^23 + 32) is an integer in [0, 64] above
      // 1.5 * 2^23 and every table read stays inside this lane's 65 entries
      const float r = __frcp_rn(s);
      const float2 r2 = make_float2(r, r);
      float near = 1.0f;
#pragma unroll
      for (int i = 0; i < W; ++i) packed[i] = 0u - kPackBias;
#pragma unroll
      for (int j = 0; j < E; j += 2) {
        const float2 xp = __fmul2_rn(make_float2(v[j], v[j + 1]), r2);
        const float2 f = __ffma2_rn(xp, make_float2(32.0f, 32.0f),
                                    make_float2(12582944.0f, 12582944.0f));  // 1.5 * 2^23 + 32
        float xq[2] = {xp.x, xp.y};
        const uint32_t fb[2] = {__float_as_uint(f.x), __float_as_uint(f.y)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float tc, below;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                       : "=f"(tc), "=f"(below)
                       : "r"(fb[h] * 256u + lut_bias));
          const float d = __fsub_rn(xq[h], tc);
          near = fminf(near, fabsf(d));
          const float step = __saturatef(__fmul_rn(d, 0x1p126f));
          const float im = __fadd_rn(below, step);  // 2^23 + index
          packed[(j + h) >> 3] += __float_as_uint(im) * (1u << (4 * ((j + h) & 7)));
        }
      }
      exact = near <= kNear;
    }
    if (exact) {
      // IEEE division and every threshold (a zero block gives x = 0)
#pragma unroll
      for (int i = 0; i < W; ++i) packed[i] = 0u;
#pragma unroll
      for (int j = 0; j < E; ++j) {
        const float x = (s > 0.0f) ? __fdiv_rn(v[j], s) : 0.0f;
        uint32_t idx = 0u;
#pragma unroll
        for (int k = 0; k < 15; ++k) idx += (x > tab.thr[k]) ? 1u : 0u;
        packed[j >> 3] |= idx << (4 * (j & 7));
      }
    }
    if (e0 + E <= n) {
      if constexpr (W == 2) {
        *reinterpret_cast<uint2*>(codes + e0 / 2) = make_uint2(packed[0], packed[1]);
      } else {
        *reinterpret_cast<uint4*>(codes + e0 / 2) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    } else if (e0 < n) {
      // ragged end: bytes that hold a weight; the nibble after the last weight is 0
#pragma unroll
      for (int b = 0; b < E / 2; ++b) {
        if (e0 + 2 * b >= n) break;
        uint32_t byte = (packed[b >> 2] >> (8 * (b & 3))) & 0xffu;
        if (e0 + 2 * b + 1 >= n) byte &= 0x0fu;
        codes[e0 / 2 + b] = static_cast<uint8_t>(byte);
      }
    }
    if ((lane & (TPB - 1)) == 0 && e0 < n) absmax[e0 / BS] = s;
    cur = nxt;
  }
  if (nonfinite) report(st, QLORA_ERR_NONFINITE, 1u);
  // scales are >= 0, so their fp32 bit patterns order like unsigned integers
  atomicMax(&cta_max, __float_as_uint(seen));
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
qlora_status launch_blocks(int bs, const T* w, int64_t n, const LevelTable& t, uint8_t* codes,
                           float* absmax, unsigned int* gmax, DeviceStatus* st, cudaStream_t s) {
  CellLut cells;
  if (!make_cell_lut(t, &cells)) return QLORA_ERR_UNSUPPORTED;
  const int64_t chunks = ceil_div(n, bs <= 512 ? 16 : 32);
  // persistent grid: as many CTAs as fit on the device at once
  const void* fn = bs == 64    ? reinterpret_cast<const void*>(quantize_blocks_kernel<T, 64>)
                   : bs == 128 ? reinterpret_cast<const void*>(quantize_blocks_kernel<T, 128>)
                   : bs == 256 ? reinterpret_cast<const void*>(quantize_blocks_kernel<T, 256>)
                   : bs == 512 ? reinterpret_cast<const void*>(quantize_blocks_kernel<T, 512>)
                               : reinterpret_cast<const void*>(quantize_blocks_kernel<T, 1024>);
  int resident = 0;
  if (!cached_value(fn, 0, &resident)) {
    int dev = 0, sms = 148, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 256, 0) != cudaSuccess ||
        per_sm < 1)
      return QLORA_ERR_CUDA;
    resident = sms * per_sm;
    store_value(fn, 0, resident);
  }
  const int grid = grid_for(chunks, 256, resident);
  count_launch();
  timing_mark(QLORA_KERNEL_QUANTIZE, s, true);
  switch (bs) {
    case 64: quantize_blocks_kernel<T, 64><<<grid, 256, 0, s>>>(w, n, t, cells, codes, absmax, gmax, st); break;
    case 128: quantize_blocks_kernel<T, 128><<<grid, 256, 0, s>>>(w, n, t, cells, codes, absmax, gmax, st); break;
    case 256: quantize_blocks_kernel<T, 256><<<grid, 256, 0, s>>>(w, n, t, cells, codes, absmax, gmax, st); break;
    case 512: quantize_blocks_kernel<T, 512><<<grid, 256, 0, s>>>(w, n, t, cells, codes, absmax, gmax, st); break;
    default: quantize_blocks_kernel<T, 1024><<<grid, 256, 0, s>>>(w, n, t, cells, codes, absmax, gmax, st); break;
  }
  timing_mark(QLORA_KERNEL_QUANTIZE, s, false);
  return QLORA_OK;
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
  const qlora_status ls =
      (w_dtype == QLORA_F32)
          ? launch_blocks(q.blocksize, static_cast<const float*>(W), n, t, q.codes, absmax, gmax,
                          st, s)
          : launch_blocks(q.blocksize, static_cast<const __nv_bfloat16*>(W), n, t, q.codes,
                          absmax, gmax, st, s);
  if (ls != QLORA_OK) return ls;
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
          q.dq_blocksize ? __builtin_ctz(q.dq_blocksize) : -1, __builtin_ctz(q.blocksize) - 6};
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

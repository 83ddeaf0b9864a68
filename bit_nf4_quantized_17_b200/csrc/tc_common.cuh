// Pieces shared by the fused dequant GEMM kernels (gemm_tc.cu, gemm_tc2.cu):
// the in-register dequantisation of 4-bit codes into bf16 operands, and the
// TMA tensor-map builder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace qlora {

// 2-D tensor map over a row-major matrix of `outer` rows x `inner` elements
// (bf16 or bytes), row stride `ld` elements, box box_inner x box_outer,
// optionally 128-byte swizzled.
bool make_map(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
              uint64_t ld, uint32_t box_inner, uint32_t box_outer, bool swizzle);

namespace tc {

static __device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Expand 8 nibbles (weights k..k+7, nibble j = weight k+j) into 8 bf16 values
// T[idx] using the byte tables L (low bytes of T[0..15]) and H (high bytes).
static __device__ __forceinline__ uint4 expand8(uint32_t x, const uint32_t (&L)[4],
                                         const uint32_t (&H)[4]) {
  const uint32_t sel = x & 0x77777777u;                          // byte index within a half table
  const uint32_t msel = ((x >> 1) & 0x44444444u) | 0x32103210u;  // pick the half by bit 3
  uint4 out;
  {
    const uint32_t lo = __byte_perm(__byte_perm(L[0], L[1], sel), __byte_perm(L[2], L[3], sel), msel);
    const uint32_t hi = __byte_perm(__byte_perm(H[0], H[1], sel), __byte_perm(H[2], H[3], sel), msel);
    out.x = __byte_perm(lo, hi, 0x5140);
    out.y = __byte_perm(lo, hi, 0x7362);
  }
  {
    const uint32_t s2 = sel >> 16, m2 = msel >> 16;
    const uint32_t lo = __byte_perm(__byte_perm(L[0], L[1], s2), __byte_perm(L[2], L[3], s2), m2);
    const uint32_t hi = __byte_perm(__byte_perm(H[0], H[1], s2), __byte_perm(H[2], H[3], s2), m2);
    out.z = __byte_perm(lo, hi, 0x5140);
    out.w = __byte_perm(lo, hi, 0x7362);
  }
  return out;
}

// The 16 dequantised values of one block, bf16(fp32(level[k] * s)), as byte tables.
static __device__ __forceinline__ void block_tables(const float (&lv)[16], float s, uint32_t (&L)[4],
                                             uint32_t (&H)[4]) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) P[j] = pack_bf16x2(__fmul_rn(lv[2 * j], s), __fmul_rn(lv[2 * j + 1], s));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    L[j] = __byte_perm(P[2 * j], P[2 * j + 1], 0x6420);
    H[j] = __byte_perm(P[2 * j], P[2 * j + 1], 0x7531);
  }
}

// The outputs of a reduced rank-r product v at row i, column j:
//   o1  fp32  a1 * v, at [i][j] or transposed [j][i], optionally added to o1
//   o2  bf16  hi = bf16(a2 v) at [i][j] and, if o2_lo > 0, lo = bf16(a2 v - hi) at [i][j + o2_lo]
//   o3  bf16  the same pair transposed: hi at [j][i], lo at [j + o3_lo][i]
// hi + lo carries a2 v to about 16 significant bits through bf16 tensor-core operands.
static __device__ __forceinline__ void reduce_store(float v, int64_t i, int j, float* o1,
                                                    int64_t ld1, int trans1, float a1, int acc1,
                                                    __nv_bfloat16* o2, int64_t ld2, float a2,
                                                    int o2_lo, __nv_bfloat16* o3, int64_t ld3,
                                                    float a3, int o3_lo) {
  if (o1) {
    float* dst = trans1 ? o1 + j * ld1 + i : o1 + i * ld1 + j;
    *dst = acc1 ? *dst + a1 * v : a1 * v;
  }
  if (o2) {
    const float x = a2 * v;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    o2[i * ld2 + j] = h;
    if (o2_lo) o2[i * ld2 + j + o2_lo] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
  if (o3) {
    const float x = a3 * v;
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    o3[j * ld3 + i] = h;
    if (o3_lo) o3[(j + o3_lo) * ld3 + i] = __float2bfloat16_rn(x - __bfloat162float(h));
  }
}

}  // namespace tc
}  // namespace qlora

// AdamW step over the adapter parameters, in one pass.
//
// Only A and B are trained ("QLoRA技术从入门到精通", 3(3): the optimiser
// updates only the adapter weights); their optimiser states may live in
// paged (managed) memory ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", 6.3) -
// the kernel takes plain pointers, so managed allocations work unchanged.
// The rule is AdamW (Adam with decoupled weight decay), per element:
//   g' = grad_scale g
//   m  = beta1 m + (1 - beta1) g'          v = beta2 v + (1 - beta2) g'^2
//   p  = p - lr (m / bc1 / (sqrt(v / bc2) + eps) + weight_decay p)
// with bc1 = 1 - beta1^t, bc2 = 1 - beta2^t (computed on the host in double),
// and the bf16 copy of p that the linear layer reads written in the same pass.
// fp32 master parameters and moments; 16-byte vectors with a scalar tail.
#include <cmath>

#include "internal.cuh"

namespace qlora {
namespace {

struct AdamwArgs {
  float lr, b1, b2, eps, wd, inv_bc1, inv_bc2, gs;
};

__device__ __forceinline__ void adamw_one(float& p, float& m, float& v, float g,
                                          const AdamwArgs& a) {
  g *= a.gs;
  m = fmaf(a.b1, m, (1.0f - a.b1) * g);
  v = fmaf(a.b2, v, (1.0f - a.b2) * g * g);
  const float mh = m * a.inv_bc1;
  const float vh = v * a.inv_bc2;
  p = p - a.lr * (__fdiv_rn(mh, __fsqrt_rn(vh) + a.eps) + a.wd * p);
}

__global__ void __launch_bounds__(256)
adamw_kernel(float* __restrict__ p, __nv_bfloat16* __restrict__ p16, const float* __restrict__ g,
             float* __restrict__ m, float* __restrict__ v, int64_t n, AdamwArgs a) {
  const int64_t n4 = n / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += stride) {
    float4 pp = reinterpret_cast<float4*>(p)[i];
    float4 mm = reinterpret_cast<float4*>(m)[i];
    float4 vv = reinterpret_cast<float4*>(v)[i];
    const float4 gg = reinterpret_cast<const float4*>(g)[i];
    adamw_one(pp.x, mm.x, vv.x, gg.x, a);
    adamw_one(pp.y, mm.y, vv.y, gg.y, a);
    adamw_one(pp.z, mm.z, vv.z, gg.z, a);
    adamw_one(pp.w, mm.w, vv.w, gg.w, a);
    reinterpret_cast<float4*>(p)[i] = pp;
    reinterpret_cast<float4*>(m)[i] = mm;
    reinterpret_cast<float4*>(v)[i] = vv;
    if (p16) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(pp.x, pp.y), hi = __floats2bfloat162_rn(pp.z, pp.w);
      reinterpret_cast<uint2*>(p16)[i] =
          make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
  }
  // the last n % 4 elements
  const int64_t t = 4 * n4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < n) {
    float pp = p[t], mm = m[t], vv = v[t];
    adamw_one(pp, mm, vv, g[t], a);
    p[t] = pp;
    m[t] = mm;
    v[t] = vv;
    if (p16) p16[t] = __float2bfloat16_rn(pp);
  }
}

}  // namespace

qlora_status launch_adamw(float* p, void* p16, const float* g, float* m, float* v, int64_t n,
                          int32_t step, float lr, float beta1, float beta2, float eps,
                          float weight_decay, float grad_scale, cudaStream_t s) {
  AdamwArgs a;
  a.lr = lr;
  a.b1 = beta1;
  a.b2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  a.inv_bc1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta1), step)));
  a.inv_bc2 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta2), step)));
  a.gs = grad_scale;
  int64_t blocks = ceil_div(n / 4 > 0 ? n / 4 : 1, 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  count_launch();
  adamw_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      p, static_cast<__nv_bfloat16*>(p16), g, m, v, n, a);
  return after_launch("adamw", s);
}

}  // namespace qlora

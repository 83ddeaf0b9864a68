// Forward and backward pass of the QLoRA linear layer.
//
// Forward ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", 2; "QLoRA技术从入门
// 到精通", 3(2)):   U = X A^T,  Y = X W^T + s U B^T,  s = alpha / r.
// Backward (same pages, 6 and 3(3)): V = dY B, dX = dY W + s V A,
// dB = s dY^T U, dA = s V^T X; no gradient for W.
//
// Tensor-core paths (tcgen05), taken when d_out % 8 == 0 and r % 8 == 0 (TMA
// needs 16-byte row strides):
//   M <= 16   forward   U = X A^T in one cluster-reduced launch (U_save, sU),
//                       then the decode kernel with W in TMEM; its contraction
//                       splits are summed in their cluster             2 launches
//             backward  V = dY B in one launch (V, sV); dX by the CUDA-core GEMV
//                       (M <= 2, clustered row chunks + one reduce) or by the
//                       single-CTA fused kernel (split + reduce); dB, dA on a
//                       second stream that joins back
//   M > 16    forward   U = X A^T (one cluster-reduced launch: U fp32, sU bf16)
//                       -> fused dequant GEMM (CTA pairs for large M) with the
//                       LoRA term as extra K stages                       2 launches
//             backward  V = dY B (one launch: sV, V^T; B read in place), fused
//                       dX GEMM on the caller's stream; U^T, dB, dA (one
//                       launch each) on a second stream that joins back   5 launches
//             (ranks above 128 keep the split-K GEMM + reduce pairs for dB, dA)
// Every kernel that reads U or V right after the launch that makes it (the
// fused GEMMs, the decode kernel, the dX GEMV) is launched as its programmatic
// dependent: it reads them only after a grid-dependency wait, late in the
// kernel, so it starts while the U / V launch still runs.
// Several adapters per batch and LoRA dropout use the same kernels (LoraOpts).
// Other shapes take the CUDA-core contraction of gemm_simt.cu.
#include <algorithm>

#include "kernels.cuh"
#include "linear.cuh"

namespace qlora {
namespace {

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

QView view_of(const qlora_nf4& W) {
  return QView{W.codes, W.scale_codes, W.factors, W.mean, W.rows, W.cols,
               W.dq_blocksize ? __builtin_ctz(W.dq_blocksize) : -1,
               __builtin_ctz(W.blocksize) - 6};
}

float lora_scale(float alpha, int32_t r) { return alpha / static_cast<float>(r); }

bool use_tc(int64_t M, int64_t N, int64_t K, int32_t r) {
  (void)K;
  return M >= 1 && M < (int64_t(1) << 30) && N % 8 == 0 && r % 8 == 0;
}

int64_t pad8(int64_t v) { return (v + 7) / 8 * 8; }

struct TcSplits {
  int u, v, db, da;
};

TcSplits tc_splits(int64_t M, int64_t N, int64_t K) {
  TcSplits s;
  s.u = tc_split_count(ceil_div(M, 128), K / 64);
  s.v = tc_split_count(ceil_div(M, 128), ceil_div(N, 64));
  s.db = tc_split_count(ceil_div(N, 128), ceil_div(M, 64));
  s.da = tc_split_count(ceil_div(K, 128), ceil_div(M, 64));
  return s;
}

// Workspace regions of the tensor-core path (byte offsets; the status word is first).
//   forward   sU [hi | lo] (M x 2*span bf16) | split-K partials
//   backward  U^T [hi ; lo] (2*r16 x M8 bf16) | B^T (r x N bf16) | sV [hi | lo] |
//             V^T [hi ; lo] | V (M x r fp32) | split-K partials
struct TcLayout {
  size_t su, part_f, fused_f, ut, bt, sv, vt, v32, part_b, fused_b, fwd_end, bwd_end;
};

TcLayout tc_layout(int64_t M, int64_t N, int64_t K, int32_t r) {
  const TcSplits sp = tc_splits(M, N, K);
  const int64_t r16 = lora_rows(r), span = lora_span(r), mp = pad8(M);
  TcLayout L{};
  L.su = kStatusBytes;
  L.part_f = L.su + align256(2 * M * 2 * span);
  L.fused_f = L.part_f + align256(sizeof(float) * sp.u * M * r16);
  const FusedShape ff = fused_shape(M, N, K / 64);
  L.fwd_end = L.fused_f + (ff.splits > 1 ? align256(sizeof(float) * ff.splits * M * N) : 0);
  L.ut = kStatusBytes;
  L.bt = L.ut + align256(2 * 2 * r16 * mp);
  L.sv = L.bt + align256(2 * r * N);
  L.vt = L.sv + align256(2 * M * 2 * span);
  L.v32 = L.vt + align256(2 * 2 * r16 * mp);  // V in fp32, for the dropout-masked dX term
  L.part_b = L.v32 + align256(sizeof(float) * M * r);
  const int64_t part = std::max(std::max(sp.u * M * r16, sp.v * M * r16),
                                std::max(sp.db * N * 2 * r16, sp.da * K * 2 * r16));
  L.fused_b = L.part_b + align256(sizeof(float) * part);
  const FusedShape fb = fused_shape(M, K, ceil_div(N, 64));
  L.bwd_end = L.fused_b + (fb.splits > 1 ? align256(sizeof(float) * fb.splits * M * K) : 0);
  return L;
}

// Workspace of the decode-sized path (M <= 16, tensor-core conditions):
//   forward   sU [hi | lo]
//   backward  sV [hi | lo] | V (fp32) | U (fp32, when recomputed) | fused partials
struct SmallLayout {
  size_t su, fwd_end, sv, v, u, fused_b, bwd_end;
};

SmallLayout small_layout(int64_t M, int64_t N, int64_t K, int32_t r) {
  const int64_t span = lora_span(r);
  SmallLayout L{};
  L.su = kStatusBytes;
  L.fwd_end = L.su + align256(2 * M * 2 * span);
  L.sv = kStatusBytes;
  L.v = L.sv + align256(2 * M * 2 * span);
  L.u = L.v + align256(sizeof(float) * M * r);
  L.fused_b = L.u + align256(sizeof(float) * M * r);
  const FusedShape fb = fused_shape(M, K, ceil_div(N, 64));
  const size_t fused_parts = fb.splits > 1 ? sizeof(float) * fb.splits * M * K : 0;
  const size_t gemv_parts =
      gemv_eligible(M, K, r) ? sizeof(float) * gemv_dgrad_parts(M, K) * M * K : 0;
  L.bwd_end = L.fused_b + align256(std::max(fused_parts, gemv_parts));
  return L;
}

bool use_small(int64_t M) { return M <= kSmallM; }

// A second stream for the part of the backward pass that does not feed the
// fused dX kernel (dB, dA): launched after V is ready, it runs on the SMs that
// kernel leaves idle in its last wave.  One per host thread and device; the
// caller's stream waits for it before the call returns, so every call stays
// ordered on the caller's stream (and can be captured in a CUDA graph).
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

qlora_status side_stream(SideStream** out) {
  constexpr int kMaxDevices = 64;
  thread_local SideStream per_device[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  SideStream& x = per_device[dev];
  if (!x.stream) {
    if (cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess ||
        cudaStreamCreateWithFlags(&x.stream, cudaStreamNonBlocking) != cudaSuccess)
      return QLORA_ERR_CUDA;
  }
  *out = &x;
  return QLORA_OK;
}

ReduceArgs reduce_args(const float* part, int splits, int64_t rows, int cols, int pcols) {
  ReduceArgs a{};
  a.part = part;
  a.splits = splits;
  a.rows = rows;
  a.cols = cols;
  a.pcols = pcols;
  return a;
}

// A rank-r product and its outputs: one cluster-reduced launch where the
// partial tile fits (n_cols <= 256), else the split-K GEMM into `part` and
// the reduction launch.
qlora_status rank_product(const void* A, bool a_mn, int64_t m_rows, int64_t kdim, int64_t ld_a,
                          const void* B, int64_t ld_b, int32_t b_rows, int32_t n_cols,
                          float* part, int splits, const ReduceArgs& out, DeviceStatus* st,
                          cudaStream_t s) {
  if (tc_rank_eligible(n_cols, out.cols, out.lo))
    return tc_rank_gemm(A, a_mn, m_rows, kdim, ld_a, B, false, ld_b, b_rows, n_cols, out, st, s);
  qlora_status e = tc_lora_gemm(A, a_mn, m_rows, kdim, ld_a, B, ld_b, b_rows, n_cols, part,
                                splits, st, s);
  if (e != QLORA_OK) return e;
  ReduceArgs ra = out;
  ra.part = part;
  ra.splits = splits;
  ra.pcols = n_cols;
  return splitk_reduce(ra, s);
}

}  // namespace

LinearPlan plan_linear(int64_t M, int64_t N, int64_t K, int32_t r) {
  LinearPlan p;
  if (use_tc(M, N, K, r) && use_small(M)) {
    SmallLayout L = small_layout(M, N, K, r);
    p.fwd_workspace = L.fwd_end;
    p.bwd_workspace = L.bwd_end;
    return p;
  }
  if (use_tc(M, N, K, r)) {
    TcLayout L = tc_layout(M, N, K, r);
    p.fwd_workspace = L.fwd_end;
    p.bwd_workspace = L.bwd_end;
    return p;
  }
  const size_t mr = align256(sizeof(float) * M * r);
  p.fwd_workspace = kStatusBytes + mr + align256(sizeof(float) * M * N);
  p.bwd_workspace = kStatusBytes + 2 * mr + align256(sizeof(float) * M * K);
  return p;
}

#define QLORA_TRY(x)                      \
  do {                                    \
    qlora_status _st = (x);               \
    if (_st != QLORA_OK) return _st;      \
  } while (0)

bool linear_multi_supported(int64_t M, int64_t N, int64_t K, int32_t r) {
  return use_tc(M > 0 ? M : 1, N, K, r);  // (M = 0 is a no-op on every path)
}

qlora_status linear_forward(const qlora_nf4& W, const LevelTable& t, const void* A,
                            const void* B, int32_t r, float alpha, const void* X, int64_t M,
                            void* Y, float* U_save, void* workspace, cudaStream_t s,
                            const LoraOpts& o) {
  const int64_t N = W.rows, K = W.cols;
  const QView w = view_of(W);
  char* ws = static_cast<char*>(workspace);
  auto* st = reinterpret_cast<DeviceStatus*>(ws);
  const float sc = lora_scale(alpha, o.r_adapter);
  const int32_t* seg = o.seg;
  const int32_t r_adapter = o.r_adapter;
  if ((seg || o.mask) && !linear_multi_supported(M, N, K, r)) return QLORA_ERR_UNSUPPORTED;
  // the adapter branch's input: X, or its dropped-out copy X (.) D
  const void* xl = X;
  if (o.mask) {
    QLORA_TRY(dropout_apply(X, o.mask, M, K, const_cast<void*>(o.x_drop), s));
    xl = o.x_drop;
  }
  if (use_tc(M, N, K, r) && use_small(M)) {
    const SmallLayout L = small_layout(M, N, K, r);
    const int32_t span = lora_span(r);
    char* su = ws + L.su;
    // U = X A^T -> U_save (fp32) and sU = s U as bf16 hi + lo, one launch
    const RankOut ro{r, U_save, r, o.keep, reinterpret_cast<__nv_bfloat16*>(su), 2 * span,
                     sc * o.keep, span, seg, r_adapter};
    QLORA_TRY(rank_down(xl, A, static_cast<int>(M), K, span, ro, s));
    // Y = X W^T + sU B^T with W in TMEM as the MMA's A operand; the splits of
    // the contraction are summed inside their cluster
    return tc_decode_forward(w, t, X, M, su, B, r, Y, tc_decode_splits(M, N, K), st, s);
  }
  if (use_tc(M, N, K, r)) {
    const TcLayout L = tc_layout(M, N, K, r);
    const TcSplits sp = tc_splits(M, N, K);
    const int32_t r16 = lora_rows(r), span = lora_span(r);
    char* su = ws + L.su;
    float* part = reinterpret_cast<float*>(ws + L.part_f);
    // U = X A^T (split-K over d_in) -> U_save (fp32) and sU = s U as bf16 hi + lo
    ReduceArgs ra = reduce_args(part, sp.u, M, r, r16);
    ra.seg = seg;  // U / V: each token keeps only its adapter's columns
    ra.seg_cols = r_adapter;
    ra.o1 = U_save;
    ra.ld1 = r;
    ra.a1 = o.keep;
    ra.o2 = su;
    ra.ld2 = 2 * span;
    ra.a2 = sc * o.keep;
    ra.o2_lo = span;
    ra.o2_pad = 1;  // the padding columns meet zero B columns in the MMA: written as zeros
    QLORA_TRY(rank_product(xl, false, M, K, K, A, K, r, r16, part, sp.u, ra, st, s));
    // Y = X W^T + sU B^T in one kernel (split over d_in, then summed, when the
    // output alone would leave SMs idle)
    const FusedShape f = fused_shape(M, N, K / 64);
    if (f.splits == 1) return tc_fused_forward(w, t, X, M, su, B, r, Y, f, st, s);
    float* fpart = reinterpret_cast<float*>(ws + L.fused_f);
    QLORA_TRY(tc_fused_forward(w, t, X, M, su, B, r, fpart, f, st, s));
    ReduceArgs ry = reduce_args(fpart, f.splits, M, static_cast<int>(N), static_cast<int>(N));
    ry.o2 = Y;
    ry.ld2 = N;
    ry.a2 = 1.0f;
    return splitk_reduce(ry, s);
  }
  char* p = ws + kStatusBytes;
  float* u = U_save ? U_save : reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * M * r);
  float* y0 = reinterpret_cast<float*>(p);
  // U = X A^T
  QLORA_TRY(simt_gemm(OP_BF16_K, dense(X, K), OP_BF16_K, dense(A, K), M, r, K, 1.0f, nullptr, u,
                      r, false, t, s));
  // Y0 = X W^T (W dequantised on the fly)
  QLORA_TRY(simt_gemm(OP_BF16_K, dense(X, K), OP_NF4_K, quantised(w), M, N, K, 1.0f, nullptr, y0,
                      N, false, t, s));
  // Y = bf16(Y0 + s U B^T)
  return simt_gemm(OP_F32_K, dense(u, r), OP_BF16_K, dense(B, r), M, N, r, sc, y0, Y, N, true, t,
                   s);
}

qlora_status linear_backward(const qlora_nf4& W, const LevelTable& t, const void* A,
                             const void* B, int32_t r, float alpha, const void* X,
                             const float* U, const void* dY, int64_t M, void* dX, float* dA,
                             float* dB, bool accumulate, void* workspace, cudaStream_t s,
                             const LoraOpts& o) {
  const int64_t N = W.rows, K = W.cols;
  const float sc = lora_scale(alpha, o.r_adapter);
  const int32_t* seg = o.seg;
  const int32_t r_adapter = o.r_adapter;
  if ((seg || o.mask) && !linear_multi_supported(M, N, K, r)) return QLORA_ERR_UNSUPPORTED;
  // with dropout the adapter branch saw X (.) D: dA and a recomputed U read it,
  // the LoRA stage of the dX GEMM is switched off (sV = 0) and the masked
  // term D (.) s V A / (1 - p) is added to dX afterwards
  const void* xl = o.mask ? o.x_drop : X;
  const float sc_dx = o.mask ? 0.0f : sc;
  const QView w = view_of(W);
  char* ws = static_cast<char*>(workspace);
  auto* st = reinterpret_cast<DeviceStatus*>(ws);
  if (use_tc(M, N, K, r) && use_small(M)) {
    const SmallLayout L = small_layout(M, N, K, r);
    const int32_t span = lora_span(r);
    const int m = static_cast<int>(M);
    char* sv = ws + L.sv;
    float* v = reinterpret_cast<float*>(ws + L.v);
    const bool gemv = gemv_eligible(M, K, r);
    // V = dY B -> V (fp32) and, for the tensor-core kernel, sV = s V as [hi | lo]
    const RankOut rv{r, v, r, 1.0f, gemv ? nullptr : reinterpret_cast<__nv_bfloat16*>(sv),
                     2 * span, sc_dx, span, seg, r_adapter};
    QLORA_TRY(rank_v(dY, B, m, N, span, rv, s));
    if (!U) {
      float* u = reinterpret_cast<float*>(ws + L.u);
      const RankOut ru{r, u, r, o.keep, nullptr, 0, 0.0f, 0, seg, r_adapter};
      QLORA_TRY(rank_down(xl, A, m, K, span, ru, s));
      U = u;
    }
    // dB and dA on the side stream, dX on the caller's (as for large M): they
    // share only inputs, all ready once V (and U) are
    SideStream* ss = nullptr;
    QLORA_TRY(side_stream(&ss));
    const cudaStream_t s2 = ss->stream;
    if (cudaEventRecord(ss->fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(s2, ss->fork, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    auto main_work = [&]() -> qlora_status {
      if (dX && gemv) {
        // dX = dY W + s V A: CTA partials of the dequant GEMV, summed in order
        float* fpart = reinterpret_cast<float*>(ws + L.fused_b);
        int parts = 0;
        QLORA_TRY(gemv_dgrad(w, t, dY, M, v, A, r, sc_dx, fpart, &parts, s));
        ReduceArgs rx = reduce_args(fpart, parts, M, static_cast<int>(K),
                                    static_cast<int>(K));
        rx.o2 = dX;
        rx.ld2 = K;
        rx.a2 = 1.0f;
        QLORA_TRY(splitk_reduce(rx, s));
      } else if (dX) {
        const FusedShape f = fused_shape(M, K, ceil_div(N, 64));
        if (f.splits == 1) {
          QLORA_TRY(tc_fused_dgrad(w, t, dY, M, sv, A, r, dX, f, st, s));
        } else {
          float* fpart = reinterpret_cast<float*>(ws + L.fused_b);
          QLORA_TRY(tc_fused_dgrad(w, t, dY, M, sv, A, r, fpart, f, st, s));
          ReduceArgs rx = reduce_args(fpart, f.splits, M, static_cast<int>(K), static_cast<int>(K));
          rx.o2 = dX;
          rx.ld2 = K;
          rx.a2 = 1.0f;
          QLORA_TRY(splitk_reduce(rx, s));
        }
      }
      if (dX && o.mask) QLORA_TRY(dropout_dx(dX, v, r, A, o.mask, M, K, r, sc * o.keep, s));
      return QLORA_OK;
    };
    auto side_work = [&]() -> qlora_status {
      QLORA_TRY(small_grad_b(dY, U, m, N, r, sc, accumulate, dB, s2));
      return small_grad_a(v, xl, m, K, r, sc * o.keep, accumulate, dA, s2);
    };
    // the dX kernel is enqueued first so that it takes the SMs
    const qlora_status st_main = main_work();
    const qlora_status st_side = side_work();
    // join on every path, so that nothing of this call runs past it on the side stream
    const bool joined = cudaEventRecord(ss->join, s2) == cudaSuccess &&
                        cudaStreamWaitEvent(s, ss->join, 0) == cudaSuccess;
    if (st_side != QLORA_OK) return st_side;
    if (st_main != QLORA_OK) return st_main;
    return joined ? QLORA_OK : QLORA_ERR_CUDA;
  }
  if (use_tc(M, N, K, r)) {
    const TcLayout L = tc_layout(M, N, K, r);
    const TcSplits sp = tc_splits(M, N, K);
    const int64_t mp = pad8(M);
    const int32_t r16 = lora_rows(r), span = lora_span(r);
    char* ut = ws + L.ut;
    char* bt = ws + L.bt;
    char* sv = ws + L.sv;
    char* vt = ws + L.vt;
    float* part = reinterpret_cast<float*>(ws + L.part_b);
    // V = dY B -> sV = s V as [hi | lo] and V^T as [hi ; lo].  B (N x r, its
    // r columns contiguous) is read in place as an MN-major operand, in boxes
    // of 64 columns (the MMA is lora_span(r) wide; columns past r read as 0);
    // its rows are a multiple of 16 bytes on this path (r % 8 == 0).  The B^T
    // form below (both operands K-major) is kept for any shape the rank
    // kernel would refuse
    const bool v_direct = r % 8 == 0 && tc_rank_eligible(span, r, 0);
    if (!v_direct) QLORA_TRY(transpose_to_bf16(B, false, N, r, r, bt, N, 0, s));
    {
      ReduceArgs ra = reduce_args(part, sp.v, M, r, r16);
      ra.seg = seg;  // U / V: each token keeps only its adapter's columns
      ra.seg_cols = r_adapter;
      ra.o2 = sv;
      ra.ld2 = 2 * span;
      ra.a2 = sc_dx;
      ra.o2_lo = span;
      ra.o2_pad = 1;
      if (o.mask) {
        ra.o1 = reinterpret_cast<float*>(ws + L.v32);
        ra.ld1 = r;
        ra.a1 = 1.0f;
      }
      ra.o3 = vt;
      ra.ld3 = mp;
      ra.a3 = 1.0f;
      ra.o3_lo = r16;
      if (v_direct) {
        QLORA_TRY(tc_rank_gemm(dY, false, M, N, N, B, true, r, r, span, ra, st, s));
      } else {
        QLORA_TRY(rank_product(dY, false, M, N, N, bt, N, r, r16, part, sp.v, ra, st, s));
      }
    }
    // dB and dA on the side stream, dX on the caller's: they share only
    // inputs, and the side stream reuses `part` after V's reduction
    SideStream* ss = nullptr;
    QLORA_TRY(side_stream(&ss));
    const cudaStream_t s2 = ss->stream;
    if (cudaEventRecord(ss->fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(s2, ss->fork, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    auto side_work = [&]() -> qlora_status {
      // U^T as bf16 hi (rows [0, r)) + lo (rows [r16, r16 + r)), from the saved U or X A^T
      if (U) {
        QLORA_TRY(transpose_to_bf16(U, true, M, r, r, ut, mp, r16, s2));
      } else {
        ReduceArgs ra = reduce_args(part, sp.u, M, r, r16);
        ra.seg = seg;  // U / V: each token keeps only its adapter's columns
        ra.seg_cols = r_adapter;
        ra.o3 = ut;
        ra.ld3 = mp;
        ra.a3 = o.keep;
        ra.o3_lo = r16;
        QLORA_TRY(rank_product(xl, false, M, K, K, A, K, r, r16, part, sp.u, ra, st, s2));
      }
      // dB = s dY^T U: rows d_out, contraction over tokens, hi and lo columns summed
      {
        ReduceArgs ra = reduce_args(part, sp.db, N, r, 2 * r16);
        ra.lo = r16;
        ra.o1 = dB;
        ra.ld1 = r;
        ra.a1 = sc;
        ra.acc1 = accumulate;
        QLORA_TRY(rank_product(dY, true, N, M, N, ut, mp, 2 * r16, 2 * r16, part, sp.db, ra, st,
                               s2));
      }
      // dA = s V^T X: rows d_in, stored transposed as r x d_in
      ReduceArgs ra = reduce_args(part, sp.da, K, r, 2 * r16);
      ra.lo = r16;
      ra.o1 = dA;
      ra.ld1 = K;
      ra.trans1 = true;
      ra.a1 = sc * o.keep;
      ra.acc1 = accumulate;
      return rank_product(xl, true, K, M, K, vt, mp, 2 * r16, 2 * r16, part, sp.da, ra, st, s2);
    };
    auto main_work = [&]() -> qlora_status {
      // dX = dY W + sV A in one kernel (split over d_out when needed)
      if (!dX) return QLORA_OK;
      const FusedShape f = fused_shape(M, K, ceil_div(N, 64));
      if (f.splits == 1) {
        QLORA_TRY(tc_fused_dgrad(w, t, dY, M, sv, A, r, dX, f, st, s));
      } else {
        float* fpart = reinterpret_cast<float*>(ws + L.fused_b);
        QLORA_TRY(tc_fused_dgrad(w, t, dY, M, sv, A, r, fpart, f, st, s));
        ReduceArgs rx = reduce_args(fpart, f.splits, M, static_cast<int>(K), static_cast<int>(K));
        rx.o2 = dX;
        rx.ld2 = K;
        rx.a2 = 1.0f;
        QLORA_TRY(splitk_reduce(rx, s));
      }
      if (!o.mask) return QLORA_OK;
      return dropout_dx(dX, reinterpret_cast<const float*>(ws + L.v32), r, A, o.mask, M, K, r,
                        sc * o.keep, s);
    };
    // the fused kernel is enqueued first so that its first wave takes the SMs
    const qlora_status st_main = main_work();
    const qlora_status st_side = side_work();
    // join on every path, so that nothing of this call runs past it on the side stream
    const bool joined = cudaEventRecord(ss->join, s2) == cudaSuccess &&
                        cudaStreamWaitEvent(s, ss->join, 0) == cudaSuccess;
    if (st_side != QLORA_OK) return st_side;
    if (st_main != QLORA_OK) return st_main;
    return joined ? QLORA_OK : QLORA_ERR_CUDA;
  }
  char* p = ws + kStatusBytes;
  float* u = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * M * r);
  float* v = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * M * r);
  float* dx0 = reinterpret_cast<float*>(p);
  if (!U) {
    QLORA_TRY(simt_gemm(OP_BF16_K, dense(X, K), OP_BF16_K, dense(A, K), M, r, K, 1.0f, nullptr, u,
                        r, false, t, s));
    U = u;
  }
  // V = dY B      (B is N x r: element (j, n) = B[n][j])
  QLORA_TRY(simt_gemm(OP_BF16_K, dense(dY, N), OP_BF16_MN, dense(B, r), M, r, N, 1.0f, nullptr, v,
                      r, false, t, s));
  if (dX) {
    // dX0 = dY W    (element (k, n) of the second operand = W[n][k])
    QLORA_TRY(simt_gemm(OP_BF16_K, dense(dY, N), OP_NF4_MN, quantised(w), M, K, N, 1.0f, nullptr,
                        dx0, K, false, t, s));
    // dX = bf16(dX0 + s V A)   (A is r x K: element (k, j) = A[j][k])
    QLORA_TRY(simt_gemm(OP_F32_K, dense(v, r), OP_BF16_MN, dense(A, K), M, K, r, sc, dx0, dX, K,
                        true, t, s));
  }
  // dB = s dY^T U (+ dB)   element (n, m) of dY^T = dY[m][n]; element (j, m) of U^T = U[m][j]
  QLORA_TRY(simt_gemm(OP_BF16_MN, dense(dY, N), OP_F32_MN, dense(U, r), N, r, M, sc,
                      accumulate ? dB : nullptr, dB, r, false, t, s));
  // dA = s V^T X (+ dA)
  return simt_gemm(OP_F32_MN, dense(v, r), OP_BF16_MN, dense(X, K), r, K, M, sc,
                   accumulate ? dA : nullptr, dA, K, false, t, s);
}

}  // namespace qlora

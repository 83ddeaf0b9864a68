// Forward dequant GEMM for decode-sized batches (M <= 16 tokens), with the
// dequantised W as the MMA's A operand in tensor memory.
//
// Y^T = W X^T + B (s U)^T: the 128 W rows of a CTA are the MMA's M rows, the
// tokens (padded to 16) its N columns.  Each dequant thread owns one W row
// (one TMEM lane): it expands the 64 codes of a k-tile into bf16 compute
// weights bf16(fp32(level[idx] * s_hat)) ("QLoRA技术从入门到精通", 3(2):
// restore a block to BF16 and multiply) and writes them straight into TMEM
// with tcgen05.st, two k values per 32-bit column - no shared-memory round
// trip for W, which at decode sizes is the whole cost besides the dequant
// arithmetic itself.  The MMA (tcgen05.mma kind::f16, A from TMEM, M = 128,
// N = 16) reads the token tile from shared memory (TMA, 128B swizzle).  The
// LoRA term runs as extension stages with both operands in shared memory
// (B's rows as A, sU as B): each stage holds a 64-rank B tile once and both
// the hi and lo halves of sU, and the first two are loaded early, so the
// term adds no load latency after the main loop.  The contraction is split over CTAs when the
// rows alone give too few; the splits of a row tile form a thread-block
// cluster and sum their fp32 tiles in shared memory, in split order, before
// the one bf16 store of Y.
//
// Roles (320 threads, two CTAs per SM): warp 0 TMA producer (up to 8 stages
// of token tile + codes in flight), warp 1 TMEM owner and MMA issuer, warps
// 2-9 two dequant groups of four warps (group g takes k-tiles i % 2 == g and
// writes one of 4 TMEM slots, freed by the commit of their MMAs; warp w writes
// TMEM lanes 32 (w % 4) .. + 31, so warps 2-5 and 6-9 each cover all 128
// lanes), group 0 drains the accumulator.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

using tc::block_tables;
using tc::expand8;

constexpr int kThreads = 320;
constexpr int kStages = 8;  // shared-memory stages (TMA in flight)
constexpr int kSlots = 4;   // TMEM slots for the dequantised W of a k-tile
constexpr int kXBytes = 2048;                    // 16 token rows x 64 bf16 (128B swizzle)
constexpr int kCodeBytes = 4096;                 // 128 W rows x 32 bytes
constexpr int kStageBytes = kXBytes + kCodeBytes;
constexpr int kExtABytes = 16384;                // 128 rows of B x 64 ranks
constexpr int kExtUBytes = 2048;                 // 16 tokens x 64 ranks of sU (its hi or lo half)
constexpr int kExtSlotBytes = kExtABytes + 2 * kExtUBytes;  // B tile, sU hi, sU lo
constexpr int kExtSlots = 2;                     // extension stages in flight
constexpr int kRedBytes = 16 * 128 * 4;          // this CTA's fp32 output tile (cluster reduce)
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kExtSlots * kExtSlotBytes + kRedBytes + 256;
constexpr uint32_t kTmemCols = 256;              // D: [0, 16); A slot a: [32 + 32 a, 64 + 32 a)
constexpr long long kTimeoutCycles = 4000000000ll;

struct DecArgs {
  int32_t m, n;
  int32_t k_tiles, kt_total;  // main k-tiles per split, in all
  int32_t k2_half, k2_last_steps;  // 64-rank extension stages, MMA steps of the last
  QView w;
  int32_t kblocks;
  int64_t nblocks;
  __nv_bfloat16* out;  // Y, M x N
  int64_t out_elems;
  int32_t cluster;  // > 1: the splits of a row tile form a cluster and sum in shared memory
  DeviceStatus* st;
};

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, bf16 inputs, fp32 accumulation
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 2)
tc_decode_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmU2,
                     const DecArgs p, const LevelTable tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // [kStages x (X | codes)] [kExtSlots x (B tile | sU hi | sU lo)] [output tile] [barriers]
  uint8_t* ext = smem + kStages * kStageBytes;
  float* red = reinterpret_cast<float*>(ext + kExtSlots * kExtSlotBytes);  // [16 tokens][128 rows]
  uint64_t* full = reinterpret_cast<uint64_t*>(ext + kExtSlots * kExtSlotBytes + kRedBytes);
  uint64_t* empty = full + kStages;   // the stage's MMAs are done
  uint64_t* afull = empty + kStages;  // the slot holds the k-tile's W rows
  uint64_t* aempty = afull + kSlots;  // the slot's MMAs are done
  uint64_t* ext_full = aempty + kSlots;       // [kExtSlots]
  uint64_t* ext_empty = ext_full + kExtSlots;  // [kExtSlots]
  uint64_t* accum = ext_empty + kExtSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * 128;
  const int kt0 = blockIdx.y * p.k_tiles;
  const int kn = min(p.k_tiles, p.kt_total - kt0);
  // extension stages (64 ranks each) on the last split, which has the fewest
  // main k-tiles when they do not divide evenly
  const int k2 = (blockIdx.y == gridDim.y - 1) ? p.k2_half : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kSlots; ++a) {
      ptx::mbar_init(&afull[a], 4);  // the four warps of the group
      ptx::mbar_init(&aempty[a], 1);
    }
    for (int e = 0; e < kExtSlots; ++e) {
      ptx::mbar_init(&ext_full[e], 1);
      ptx::mbar_init(&ext_empty[e], 1);
    }
    ptx::mbar_init(accum, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmX);
    ptx::prefetch_tmap(&tmC);
    if (k2) {
      ptx::prefetch_tmap(&tmB2);
      ptx::prefetch_tmap(&tmU2);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    // extension stage h: B columns [64 h, 64 h + 64) of this CTA's rows and the
    // same 64 ranks of sU's hi and lo halves.  sU comes from the launch before
    // this one, which lets this grid start early (programmatic dependent
    // launch): the main loop reads only X and W, and the producer waits for
    // that launch to finish only halfway through it, before the first
    // extension loads, so they have landed when the main loop ends.
    auto issue_ext = [&](int h) {
      const int e = h % kExtSlots;
      uint8_t* xb = ext + e * kExtSlotBytes;
      ptx::mbar_arrive_expect_tx(&ext_full[e], kExtSlotBytes);
      ptx::tma_load_2d(&tmB2, &ext_full[e], xb, h * 64, n0);
      ptx::tma_load_2d(&tmU2, &ext_full[e], xb + kExtABytes, h * 64, 0);
      ptx::tma_load_2d(&tmU2, &ext_full[e], xb + kExtABytes + kExtUBytes, (p.k2_half + h) * 64, 0);
    };
    int issued = 0, ext_issued = 0;
    const int early = min(k2, kExtSlots);
    auto issue_early = [&]() {
      if (early == 0) return;
      asm volatile("griddepcontrol.wait;" ::: "memory");  // sU written and visible
      for (; ext_issued < early; ++ext_issued) issue_ext(ext_issued);
    };
    bool ok = true;
    if (kn == 0) issue_early();
    for (int i = 0; i < kn; ++i) {
      const int s = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* xs = smem + s * kStageBytes;
      const int kg = kt0 + i;
      ptx::mbar_arrive_expect_tx(&full[s], kStageBytes);
      ptx::tma_load_2d(&tmX, &full[s], xs, kg * 64, 0);
      ptx::tma_load_2d(&tmC, &full[s], xs + kXBytes, kg * 32, n0);
      ++issued;
      if (i == kn / 2) issue_early();
    }
    if (ext_issued < early && ok) issue_early();
    for (int h = ext_issued; h < k2 && ok; ++h) {
      const int e = h % kExtSlots;
      if (!ptx::mbar_wait(&ext_empty[e], ((h / kExtSlots) & 1) ^ 1, kTimeoutCycles, abort_flag)) break;
      issue_ext(h);
      ++ext_issued;
    }
    // never leave with copies in flight into this CTA's shared memory
    for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
      ptx::mbar_wait(&full[i % kStages], (i / kStages) & 1, kTimeoutCycles, nullptr);
    for (int h = (ext_issued > kExtSlots ? ext_issued - kExtSlots : 0); h < ext_issued; ++h)
      ptx::mbar_wait(&ext_full[h % kExtSlots], (h / kExtSlots) & 1, kTimeoutCycles, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------ MMA issuer
    const uint32_t idesc = ptx::idesc_bf16(128, 16, 0, 0);
    bool ok = true;
    for (int i = 0; i < kn && ok; ++i) {
      const int s = i % kStages, a = i % kSlots;
      const uint32_t ph = (i / kStages) & 1, pa = (i / kSlots) & 1;
      if (!ptx::mbar_wait(&full[s], ph, kTimeoutCycles, abort_flag) ||
          !ptx::mbar_wait(&afull[a], pa, kTimeoutCycles, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t x_addr = ptx::smem_u32(smem + s * kStageBytes);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t bd = ptx::sw128_desc(x_addr + ks * 32, 16, 1024);
        umma_bf16_ts(tmem, tmem + 32 + 32 * a + 8 * ks, bd, idesc, (i | ks) != 0 ? 1u : 0u);
      }
      ptx::umma_commit(&empty[s]);   // the stage may be refilled
      ptx::umma_commit(&aempty[a]);  // the slot may be rewritten
    }
    for (int h = 0; h < k2 && ok; ++h) {
      const int e = h % kExtSlots;
      if (!ptx::mbar_wait(&ext_full[e], (h / kExtSlots) & 1, kTimeoutCycles, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(ext + e * kExtSlotBytes);
      const int steps = (h == p.k2_half - 1) ? p.k2_last_steps : 4;
      for (int part = 0; part < 2; ++part) {  // sU hi, then sU lo, against the same B tile
        const uint32_t b_addr = a_addr + kExtABytes + part * kExtUBytes;
        for (int ks = 0; ks < steps; ++ks)
          ptx::umma_bf16(tmem, ptx::sw128_desc(a_addr + ks * 32, 16, 1024),
                         ptx::sw128_desc(b_addr + ks * 32, 16, 1024), idesc,
                         (kn > 0 || h > 0 || part > 0 || ks > 0) ? 1u : 0u);
      }
      ptx::umma_commit(&ext_empty[e]);
    }
    ptx::umma_commit(accum);
    ptx::mbar_wait(accum, 0, kTimeoutCycles, nullptr);  // MMAs done before TMEM is freed
  } else if (warp >= 2) {
    const int grp = (warp - 2) >> 2;
    const int quarter = warp & 3;                 // TMEM lanes this warp may write / read
    const int row = 32 * quarter + lane;          // W row n0 + row = TMEM lane
    float lv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];
    const float mu = (p.w.dq_shift >= 0) ? __ldg(p.w.mean) : 0.0f;
    const int64_t wrow = static_cast<int64_t>(n0) + row;
    struct RawScale {
      float q, f;
      bool in;
    };
    auto load_scale = [&](int i) -> RawScale {
      if (i >= kn || wrow >= p.w.rows) return RawScale{0.0f, 0.0f, false};
      const int64_t b = wrow * (p.kblocks >> p.w.bs_shift) + ((kt0 + i) >> p.w.bs_shift);
      if (b >= p.nblocks) {
        report(p.st, QLORA_ERR_SHAPE, 221u);
        return RawScale{0.0f, 0.0f, false};
      }
      if (p.w.dq_shift < 0) return RawScale{1.0f, __ldg(p.w.factors + b), true};
      return RawScale{static_cast<float>(__ldg(p.w.scale_codes + b)),
                      __ldg(p.w.factors + (b >> p.w.dq_shift)), true};
    };
    RawScale r0 = load_scale(grp), r1 = load_scale(grp + 2), r2 = load_scale(grp + 4);
    for (int i = grp; i < kn; i += 2) {
      const int s = i % kStages, a = i % kSlots;
      const uint32_t ph = (i / kStages) & 1, pa = (i / kSlots) & 1;
      const float sc = !r0.in ? 0.0f
                       : (p.w.dq_shift < 0 ? r0.f : __fadd_rn(__fmul_rn(r0.q, r0.f), mu));
      r0 = r1;
      r1 = r2;
      r2 = load_scale(i + 6);
      // the stage's codes have landed; warp-uniform: the TMEM store below is a
      // warp-wide instruction
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&full[s], ph, kTimeoutCycles, abort_flag))) break;
      const uint8_t* codes = smem + s * kStageBytes + kXBytes + row * 32;
      const uint4 c0 = *reinterpret_cast<const uint4*>(codes);
      const uint4 c1 = *reinterpret_cast<const uint4*>(codes + 16);
      // these generic reads come before the next TMA into the slot (async proxy)
      ptx::fence_proxy_async_smem();
      uint32_t L[4], H[4];
      block_tables(lv, sc, L, H);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 e = expand8(words[j], L, H);  // k = 8j .. 8j + 7, two per column
        v[4 * j] = e.x;
        v[4 * j + 1] = e.y;
        v[4 * j + 2] = e.z;
        v[4 * j + 3] = e.w;
      }
      // the slot is free once the MMAs of its previous k-tile have completed
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&aempty[a], pa ^ 1, kTimeoutCycles, abort_flag)))
        break;
      ptx::tc_fence_after();
      tmem_st_x32(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 32 + 32 * a, v);
      tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&afull[a]);
    }
    if (grp == 0) {
      // ---------------------------------------------------------- epilogue
      bool ok = ptx::mbar_wait(accum, 0, kTimeoutCycles, abort_flag);
      ok = __all_sync(0xffffffffu, ok && !*abort_flag);
      if (p.cluster > 1) {
        // this split's tile into shared memory, summed over the cluster below
        uint32_t r[16];
        if (ok) {
          ptx::tc_fence_after();
          ptx::tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16), r);
          ptx::tmem_ld_wait();
        }
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < p.m) red[m * 128 + row] = ok ? __uint_as_float(r[m]) : 0.0f;
      } else if (ok) {
        ptx::tc_fence_after();
        uint32_t r[16];
        ptx::tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16), r);
        ptx::tmem_ld_wait();
        const int64_t n = wrow;
        if (n < p.n) {
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            if (m >= p.m) break;
            const int64_t idx = static_cast<int64_t>(m) * p.n + n;
            if (idx >= p.out_elems) {
              report(p.st, QLORA_ERR_SHAPE, 222u);
              break;
            }
            p.out[idx] = __float2bfloat16_rn(__uint_as_float(r[m]));
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (p.cluster > 1) {
    // the splits of this row tile summed in split order; CTA q of the cluster
    // writes the tokens m with m % cluster == q
    ptx::cluster_sync();
    if (warp >= 2 && warp < 6) {
      const int row = 32 * (warp & 3) + lane;
      const int64_t n = static_cast<int64_t>(n0) + row;
      const int q0 = static_cast<int>(ptx::cluster_ctarank());
      if (n < p.n) {
        for (int m = q0; m < p.m; m += p.cluster) {
          float x[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            x[q] = (q < p.cluster)
                       ? ptx::ld_cluster_f32(ptx::cluster_addr(&red[m * 128 + row], static_cast<uint32_t>(q)))
                       : 0.0f;
          float v = 0.0f;
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < p.cluster) v += x[q];
          const int64_t idx = static_cast<int64_t>(m) * p.n + n;
          if (idx < p.out_elems) p.out[idx] = __float2bfloat16_rn(v);
        }
      }
    }
    ptx::cluster_sync();  // every CTA keeps its tile until the others have read it
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.st, QLORA_ERR_DEVICE_TIMEOUT, 120u);
}

}  // namespace

int tc_decode_splits(int64_t M, int64_t N, int64_t K) {
  (void)M;
  const int64_t row_tiles = ceil_div(N, 128);
  const int64_t kt = K / 64;
  // two CTAs per SM (TMEM), one wave, at least 8 k-tiles per split
  int64_t s = (2 * 148) / row_tiles;
  const int64_t max_s = kt / 8 > 0 ? (kt / 8 < 8 ? kt / 8 : 8) : 1;  // a cluster holds the splits
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  const int64_t per = ceil_div(kt, s);
  return static_cast<int>(ceil_div(kt, per));
}

qlora_status tc_decode_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                               const void* sU, const void* B, int32_t r, void* out, int splits,
                               DeviceStatus* st, cudaStream_t s) {
  const int64_t N = w.rows, K = w.cols;
  if (M < 1 || M > 16) return QLORA_ERR_UNSUPPORTED;
  CUtensorMap mx, mc, mb2, mu2;
  if (!make_map(&mx, X, true, K, M, K, 64, 16, true) ||
      !make_map(&mc, w.codes, false, K / 2, N, K / 2, 32, 128, false) ||
      !make_map(&mb2, B, true, r, N, r, 64, 128, true) ||
      !make_map(&mu2, sU, true, 2 * lora_span(r), M, 2 * lora_span(r), 64, 16, true))
    return QLORA_ERR_CUDA;
  DecArgs p{};
  p.m = static_cast<int32_t>(M);
  p.n = static_cast<int32_t>(N);
  p.kt_total = static_cast<int32_t>(K / 64);
  p.k_tiles = static_cast<int32_t>(ceil_div(p.kt_total, splits));
  p.k2_half = (r + 63) / 64;
  p.k2_last_steps = ((r - 64 * (p.k2_half - 1)) + 15) / 16;
  p.w = w;
  p.kblocks = static_cast<int32_t>(K / 64);
  p.nblocks = (N * K / 64) >> w.bs_shift;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.out_elems = M * N;
  p.cluster = splits;
  p.st = st;
  const qlora_status cs =
      ensure_smem(reinterpret_cast<const void*>(tc_decode_fwd_kernel), kSmemBytes);
  if (cs != QLORA_OK) return cs;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ceil_div(N, 128)), static_cast<unsigned>(splits), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the U launch
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = static_cast<unsigned>(splits);
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = splits > 1 ? 2 : 1;
  count_launch();
  timing_mark(QLORA_KERNEL_FUSED_FWD, s, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, tc_decode_fwd_kernel, mx, mc, mb2, mu2, p, t);
  timing_mark(QLORA_KERNEL_FUSED_FWD, s, false);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  return after_launch("tc_decode(fwd)", s);
}

}  // namespace qlora

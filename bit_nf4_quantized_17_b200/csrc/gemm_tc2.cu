// Fused dequant GEMMs on CTA pairs, for large token counts.
//
// Same product as the single-CTA kernel of gemm_tc.cu: Y = X W^T + sU B^T
// (forward) or dX = dY W + sV A (backward), the 4-bit W dequantised on load
// to bf16 ("QLoRA技术从入门到精通", 3(2): restore a block to BF16, multiply,
// discard), the LoRA term added as extra K stages of the same accumulators.
// Here two CTAs of a cluster compute a 512 x tn output tile with pair MMAs
// (tcgen05.mma.cta_group::2, M = 256, N = tn, issued by the even CTA; tn =
// 256 for the backward, 192..256 for the forward, chosen per launch so that
// the tiles fill the last round of pair slots):
//
//   * each CTA holds its own 256 activation rows (two 128-row sub-tiles) and
//     HALF of the B tile: tn / 2 of the W rows (forward) or 128 of the 256
//     output columns (backward) - the MMA reads the other half from the peer;
//   * so each SM dequantises half of the W tile per k-tile and its shared
//     memory carries half of the B traffic, for the same MMA work per SM as
//     the single-CTA kernel with two accumulators;
//   * TMA loads of both CTAs count on the even CTA's barriers (no multicast:
//     every tile lands in the CTA that loads it); the odd CTA's dequant warps
//     arrive on the even CTA's barrier through the cluster; MMA completion is
//     committed to the barriers of both CTAs.
//
// Roles per CTA (640 threads): warp 0 TMA producer; warp 1 TMEM (both CTAs)
// and, in the even CTA, the MMA issuer; warps 4-19 dequantise in four groups
// of 128 threads (group g takes k-tiles kt % 4 == g), then drain the
// accumulators.  Every wait is bounded; a wait that gives up raises the
// CTA's abort flag and QLORA_ERR_DEVICE_TIMEOUT is reported.
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

using tc::block_tables;
using tc::expand8;
using tc::pack_bf16x2;

constexpr int kThreads = 640;
constexpr int kStages = 4;
constexpr int kGroupThreads = 128;      // dequant threads per group; 4 groups
constexpr int kABytes = 32768;          // 256 rows x 64 bf16 (two 128-row sub-tiles)
constexpr int kBBytes = 16384;          // this CTA's half of B: 128 x 64 bf16
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kCodeSlot = 4096;         // one k-tile of this CTA's codes
constexpr int kCodeSlots = 4;
constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kCodeSlots * kCodeSlot + 256;
constexpr long long kTimeoutCycles = 4000000000ll;  // ~2 s at 1.9 GHz

struct Tc2Args {
  int32_t m, n;              // output rows (tokens) and columns
  int32_t kt_total;          // main k-tiles
  int32_t k2_tiles, k2_half, k2_last_steps;
  int32_t b2_mn;             // extension B operand MN-major (backward)
  int32_t a_bytes;           // bytes of one CTA's activation tile per stage
  int32_t tn;                // output columns of a pair tile (a multiple of 16, <= 256);
                             // each CTA holds tn / 2 rows of the B tile
  QView w;
  int32_t kblocks;           // W.cols / 64
  int64_t nblocks;           // entries of w.scale_codes
  __nv_bfloat16* out;        // m x n, row stride ldo
  int64_t ldo;
  int64_t out_elems;
  DeviceStatus* st;
};

__device__ __forceinline__ void store16_bf16(const Tc2Args& p, int64_t row, int64_t col,
                                             const uint32_t (&r)[16]) {
  if (row >= p.m || col >= p.n) return;
  const int64_t base = row * p.ldo + col;
  const int64_t span = (p.n - col < 16) ? (p.n - col) : 16;
  if (base < 0 || base + span > p.out_elems) {
    report(p.st, QLORA_ERR_SHAPE, 210u);
    return;
  }
  __nv_bfloat16* o = p.out + base;
  if (col + 16 <= p.n) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
    reinterpret_cast<uint4*>(o)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(o)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    for (int j = 0; j < 16 && col + j < p.n; ++j) o[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
  }
}

template <int BMODE>
__global__ void __launch_bounds__(kThreads, 1)
tc2_fused_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                 const Tc2Args p, const LevelTable tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // [kStages x (A | B half)] [kCodeSlots x codes] [barriers]
  uint8_t* codes_ring = smem + kStages * kStageBytes;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(codes_ring + kCodeSlots * kCodeSlot);
  uint64_t* full_b = full_a + kStages;       // even CTA: both dequant halves written
  uint64_t* empty = full_b + kStages;        // both CTAs: the pair MMAs of the stage are done
  uint64_t* codes_full = empty + kStages;
  uint64_t* codes_empty = codes_full + kCodeSlots;
  uint64_t* accum = codes_empty + kCodeSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int m0 = static_cast<int>(blockIdx.x >> 1) * 512 + static_cast<int>(rank) * 256;
  const int hn = p.tn >> 1;                                 // B rows this CTA holds
  const int n0 = blockIdx.y * p.tn;                         // output columns of the pair tile
  const int nh = n0 + static_cast<int>(rank) * hn;          // this CTA's half of B
  const uint32_t code_bytes = (BMODE == B_DQ_K) ? static_cast<uint32_t>(hn) * 32u : kCodeSlot;
  const uint32_t b_bytes = static_cast<uint32_t>(hn) * 128u;
  const int total = p.kt_total + p.k2_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full_a[s], 1);
      ptx::mbar_init(&full_b[s], 2 * (kGroupThreads / 32));  // one arrival per dequant warp, both CTAs
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kCodeSlots; ++s) {
      ptx::mbar_init(&codes_full[s], 1);
      ptx::mbar_init(&codes_empty[s], kGroupThreads);
    }
    ptx::mbar_init(accum, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmA2);
    ptx::prefetch_tmap(&tmB2);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, 512);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  // both CTAs' barriers exist before either CTA signals the other's
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int kc = 0;  // next k-tile whose codes are loaded
    bool ok = true;
    auto issue_codes = [&](int upto) {
      while (ok && kc < p.kt_total && kc < upto) {
        const int cs = kc % kCodeSlots;
        if (!ptx::mbar_wait(&codes_empty[cs], ((kc / kCodeSlots) & 1) ^ 1, kTimeoutCycles,
                            abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* dst = codes_ring + cs * kCodeSlot;
        ptx::mbar_arrive_expect_tx(&codes_full[cs], code_bytes);
        if (BMODE == B_DQ_K)
          ptx::tma_load_2d(&tmB, &codes_full[cs], dst, kc * 32, nh);  // 128 W rows x 32 bytes
        else
          ptx::tma_load_2d(&tmB, &codes_full[cs], dst, nh / 2, kc * 64);  // 64 W rows x 64 bytes
        ++kc;
      }
    };
    issue_codes(kCodeSlots);
    int issued = 0;
    for (int kt = 0; kt < total && ok; ++kt) {
      const int s = kt % kStages;
      const uint32_t ph = (kt / kStages) & 1;
      if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) break;
      uint8_t* sa = smem + s * kStageBytes;
      uint8_t* sb = sa + kABytes;
      const uint32_t bar = ptx::cluster_addr(&full_a[s], 0);
      if (kt < p.kt_total) {
        if (rank == 0) ptx::mbar_arrive_expect_tx(&full_a[s], 2 * p.a_bytes);
        ptx::tma_load_2d_pair(&tmA, bar, sa, kt * 64, m0);
      } else {
        // extension stage tt: A2 columns [64 tt, 64 tt + 64) of [hi | lo];
        // this CTA's half of B2 at LoRA ranks [64 (tt mod half), ...)
        const int tt = kt - p.kt_total;
        // A2 (sU or sV) is the output of the launch before this one, which
        // lets this grid start early (programmatic dependent launch): the
        // main loop reads only the activations and W
        if (tt == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        const int k2a = tt * 64;
        const int k2b = (tt % p.k2_half) * 64;
        if (rank == 0) ptx::mbar_arrive_expect_tx(&full_a[s], 2 * (p.a_bytes + b_bytes));
        ptx::tma_load_2d_pair(&tmA2, bar, sa, k2a, m0);
        if (p.b2_mn) {
          ptx::tma_load_2d_pair(&tmB2, bar, sb, nh, k2b);
          ptx::tma_load_2d_pair(&tmB2, bar, sb + 8192, nh + 64, k2b);
        } else {
          ptx::tma_load_2d_pair(&tmB2, bar, sb, k2b, nh);
        }
      }
      ++issued;
      issue_codes(kt + 1 + kCodeSlots);
    }
    // this CTA's codes copies land before it exits; activation copies are
    // counted on the even CTA's barriers, which its MMA issuer waits for
    for (int c = (kc > kCodeSlots ? kc - kCodeSlots : 0); c < kc; ++c)
      ptx::mbar_wait(&codes_full[c % kCodeSlots], (c / kCodeSlots) & 1, kTimeoutCycles, nullptr);
    if (rank == 0)
      for (int kt = (issued > kStages ? issued - kStages : 0); kt < issued; ++kt)
        ptx::mbar_wait_cluster(&full_a[kt % kStages], (kt / kStages) & 1, kTimeoutCycles, nullptr);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------------ MMA issuer (even CTA)
    const uint32_t idesc = ptx::idesc_bf16(256, p.tn, 0, BMODE == B_DQ_MN ? 1 : 0);
    const uint32_t idesc2 = ptx::idesc_bf16(256, p.tn, 0, p.b2_mn);
    int done = 0;
    for (int kt = 0; kt < total; ++kt) {
      const int s = kt % kStages;
      const uint32_t ph = (kt / kStages) & 1;
      if (!ptx::mbar_wait_cluster(&full_a[s], ph, kTimeoutCycles, abort_flag)) break;
      const bool ext = kt >= p.kt_total;
      // full_b completes a phase per main k-tile only; the extension stages come last
      if (!ext && !ptx::mbar_wait_cluster(&full_b[s], ph, kTimeoutCycles, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(smem + s * kStageBytes);
      const uint32_t b_addr = a_addr + kABytes;
      const bool b_mn = ext ? (p.b2_mn != 0) : (BMODE == B_DQ_MN);
      const int steps =
          (ext && ((kt - p.kt_total) % p.k2_half) == p.k2_half - 1) ? p.k2_last_steps : 4;
      // One thread issues every MMA of the pair: keep its work per MMA to a
      // 64-bit add.  A shared-memory descriptor holds the start address in
      // 16-byte units in its low 14 bits, so the descriptor of an operand
      // advanced by `off` bytes inside the stage is the stage's descriptor plus
      // off / 16 (no carry: shared addresses stay below 256 KB).  Main k-tiles
      // are fully unrolled: 4 K steps x 2 accumulators.  (Building every
      // descriptor afresh in a runtime loop made this thread the limit of the
      // kernel: 10-17% slower.)
      const uint64_t a0 = ptx::sw128_desc(a_addr, 16, 1024);
      const uint64_t b0 = b_mn ? ptx::sw128_desc(b_addr, 8192, 1024)
                               : ptx::sw128_desc(b_addr, 16, 1024);
      const uint64_t b_step = b_mn ? (2048 >> 4) : (32 >> 4);
      const uint32_t acc0 = kt != 0 ? 1u : 0u;
      if (!ext) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bd = b0 + b_step * ks;
          ptx::umma_bf16_pair(tmem, a0 + ((ks * 32) >> 4), bd, idesc, ks ? 1u : acc0);
          ptx::umma_bf16_pair(tmem + 256, a0 + ((16384 + ks * 32) >> 4), bd, idesc,
                              ks ? 1u : acc0);
        }
      } else {
        for (int ks = 0; ks < steps; ++ks) {
          const uint64_t bd = b0 + b_step * ks;
          const uint32_t acc = (kt | ks) != 0 ? 1u : 0u;
          ptx::umma_bf16_pair(tmem, a0 + ((ks * 32) >> 4), bd, idesc2, acc);
          ptx::umma_bf16_pair(tmem + 256, a0 + ((16384 + ks * 32) >> 4), bd, idesc2, acc);
        }
      }
      ptx::umma_commit_pair(&empty[s]);
      ++done;
    }
    ptx::umma_commit_pair(accum);
    (void)done;
  } else if (warp >= 4) {
    const int grp = (threadIdx.x - 128) / kGroupThreads;  // k-tiles kt % 4 == grp
    const int td = (threadIdx.x - 128) % kGroupThreads;
    // ---------------------------------------------------- dequantisation
    // forward: thread td expands W row nh + td (one 64-weight block per k-tile);
    // backward: thread td expands block (nh / 64 + q) of W row 64 kt + row.
    float lv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];
    const float mu = (p.w.dq_shift >= 0) ? __ldg(p.w.mean) : 0.0f;
    const int row = (BMODE == B_DQ_K) ? td : (td & 63);
    const int q = (BMODE == B_DQ_K) ? 0 : (td >> 6);
    // forward: the threads past this CTA's hn W rows expand nothing but keep
    // their barrier arrivals
    const bool active = (BMODE == B_DQ_K) ? (td < hn) : true;
    const uint32_t leader_full_b0 = ptx::cluster_addr(&full_b[0], 0);
    struct RawScale {
      float q, f;
      bool in;
    };
    auto load_scale = [&](int kt) -> RawScale {
      if (kt >= p.kt_total || !active) return RawScale{0.0f, 0.0f, false};
      const int64_t wrow = (BMODE == B_DQ_K) ? static_cast<int64_t>(nh) + row
                                             : static_cast<int64_t>(kt) * 64 + row;
      const int64_t kb = (BMODE == B_DQ_K) ? kt : (nh / 64 + q);
      if (wrow >= p.w.rows || kb >= p.kblocks) return RawScale{0.0f, 0.0f, false};
      const int64_t b = wrow * (p.kblocks >> p.w.bs_shift) + (kb >> p.w.bs_shift);
      if (b >= p.nblocks) {
        report(p.st, QLORA_ERR_SHAPE, 211u);
        return RawScale{0.0f, 0.0f, false};
      }
      if (p.w.dq_shift < 0) return RawScale{1.0f, __ldg(p.w.factors + b), true};
      return RawScale{static_cast<float>(__ldg(p.w.scale_codes + b)),
                      __ldg(p.w.factors + (b >> p.w.dq_shift)), true};
    };
    RawScale r0 = load_scale(grp), r1 = load_scale(grp + 4);
    for (int kt = grp; kt < p.kt_total; kt += 4) {
      const int s = kt % kStages;  // == grp: each group owns one stage slot and one codes slot
      const uint32_t ph = (kt / kStages) & 1;
      const float sc = !r0.in ? 0.0f
                       : (p.w.dq_shift < 0 ? r0.f : __fadd_rn(__fmul_rn(r0.q, r0.f), mu));
      r0 = r1;
      r1 = load_scale(kt + 8);
      if (!ptx::mbar_wait(&codes_full[s], ph, kTimeoutCycles, abort_flag)) break;
      const uint8_t* slot = codes_ring + s * kCodeSlot;
      uint4 c0 = make_uint4(0u, 0u, 0u, 0u), c1 = c0;
      if (BMODE == B_DQ_K) {
        if (active) {
          c0 = *reinterpret_cast<const uint4*>(slot + row * 32);
          c1 = *reinterpret_cast<const uint4*>(slot + row * 32 + 16);
        }
      } else {
        c0 = *reinterpret_cast<const uint4*>(slot + row * 64 + q * 32);
        c1 = *reinterpret_cast<const uint4*>(slot + row * 64 + q * 32 + 16);
      }
      // the next TMA into the slot writes through the async proxy: order these
      // reads before it, then release the slot
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(&codes_empty[s]);
      uint32_t L[4], H[4];
      block_tables(lv, sc, L, H);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      // the B half of slot s is free once the pair MMAs of its previous use are done
      if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) break;
      uint8_t* sb = smem + s * kStageBytes + kABytes;
      uint8_t* dst_row = (BMODE == B_DQ_K) ? sb + row * 128 : sb + q * 8192 + row * 128;
      if (active) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(dst_row + 16 * (j ^ (row & 7))) = expand8(words[j], L, H);
      }
      // make the writes visible to the MMA (async proxy, possibly issued by
      // the peer CTA), then one arrival per warp on the even CTA's barrier
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(leader_full_b0 + 8u * s);
    }
    // ---------------------------------------------------------- epilogue
    bool ok = ptx::mbar_wait_cluster(accum, 0, kTimeoutCycles, abort_flag);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (ok) {
      ptx::tc_fence_after();
      const int quarter = warp & 3;
      const int cg = (warp - 4) >> 2;  // 0..3: accumulator cg & 1, column half cg >> 1
      const int t = cg & 1;
      const int64_t grow = static_cast<int64_t>(m0) + 128 * t + 32 * quarter + lane;
      const int chunks = p.tn >> 4;                 // 16-column chunks of the tile
      const int c_half = (chunks + 1) >> 1;
      const int c_begin = (cg >> 1) ? c_half : 0, c_end = (cg >> 1) ? chunks : c_half;
      for (int c = c_begin; c < c_end; ++c) {
        uint32_t r[16];
        ptx::tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + t * 256 + c * 16, r);
        ptx::tmem_ld_wait();
        store16_bf16(p, grow, static_cast<int64_t>(n0) + c * 16, r);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees TMEM) while the pair may still touch it
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.st, QLORA_ERR_DEVICE_TIMEOUT, 110u + BMODE);
}

template <int BMODE>
qlora_status launch_tc2(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& ma2,
                        const CUtensorMap& mb2, const Tc2Args& p, const LevelTable& t,
                        int64_t m_pairs, int64_t n_tiles, cudaStream_t s) {
  const qlora_status cs = ensure_smem(reinterpret_cast<const void*>(tc2_fused_kernel<BMODE>),
                                      kSmemBytes);
  if (cs != QLORA_OK) return cs;
  if (m_pairs < 1 || 2 * m_pairs > 0x7fffffff || n_tiles < 1 || n_tiles > 65535)
    return QLORA_ERR_SHAPE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * m_pairs), static_cast<unsigned>(n_tiles), 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // may overlap the U / V launch
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const int kind = BMODE == B_DQ_K ? QLORA_KERNEL_FUSED_FWD : QLORA_KERNEL_FUSED_DGRAD;
  count_launch();
  timing_mark(kind, s, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, tc2_fused_kernel<BMODE>, ma, mb, ma2, mb2, p, t);
  timing_mark(kind, s, false);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  return after_launch(BMODE == B_DQ_K ? "tc2_fused(fwd)" : "tc2_fused(dgrad)", s);
}

Tc2Args args_of(const QView& w, int64_t M, int64_t n_out, int32_t r, void* out, DeviceStatus* st) {
  Tc2Args p{};
  p.m = static_cast<int32_t>(M);
  p.n = static_cast<int32_t>(n_out);
  p.k2_half = (r + 63) / 64;
  p.k2_tiles = 2 * p.k2_half;
  p.k2_last_steps = ((r - 64 * (p.k2_half - 1)) + 15) / 16;
  p.a_bytes = kABytes;
  p.tn = 256;
  p.w = w;
  p.kblocks = static_cast<int32_t>(w.cols / 64);
  p.nblocks = (w.rows * w.cols / 64) >> w.bs_shift;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.ldo = n_out;
  p.out_elems = M * n_out;
  p.st = st;
  return p;
}

}  // namespace

bool tc2_eligible(int64_t M, const FusedShape& f) { return f.mt == 2 && f.splits == 1 && M > 256; }

// Output columns of a forward pair tile: 256 unless a narrower tile (down to
// 192, in steps of 16) ends the launch sooner.  An output 8192 wide at 2048
// tokens is 128 tiles of 256 on 74 pair slots (1.73 waves, two rounds); at
// 224 it is 148 tiles, two full rounds of narrower tiles.
static int tc2_pair_tile_width(int64_t M, int64_t n_out) {
  // pair slots of the device: one CTA per SM (shared memory), two per pair
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t slots = sms >= 2 ? sms / 2 : 1;
  const int64_t m_pairs = ceil_div(M, 512);
  // a pair tile's time grows with its width; pick the width that ends the
  // launch soonest (waves x width), the widest among equals
  int best = 256;
  int64_t best_cost = -1;
  for (int tn = 256; tn >= 192; tn -= 16) {
    const int64_t tiles = m_pairs * ceil_div(n_out, tn);
    const int64_t cost = ceil_div(tiles, slots) * tn;
    if (best_cost < 0 || cost < best_cost) {
      best = tn;
      best_cost = cost;
    }
  }
  return best;
}

qlora_status tc2_fused_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                               const void* sU, const void* B, int32_t r, void* Y,
                               DeviceStatus* st, cudaStream_t s) {
  const int64_t N = w.rows, K = w.cols;
  const int tn = tc2_pair_tile_width(M, N);
  const uint32_t hn = static_cast<uint32_t>(tn / 2);
  CUtensorMap ma, mb, ma2, mb2;
  if (!make_map(&ma, X, true, K, M, K, 64, 256, true) ||
      !make_map(&mb, w.codes, false, K / 2, N, K / 2, 32, hn, false) ||
      !make_map(&ma2, sU, true, 2 * lora_span(r), M, 2 * lora_span(r), 64, 256, true) ||
      !make_map(&mb2, B, true, r, N, r, 64, hn, true))
    return QLORA_ERR_CUDA;
  Tc2Args p = args_of(w, M, N, r, Y, st);
  p.kt_total = static_cast<int32_t>(K / 64);
  p.b2_mn = 0;
  p.tn = tn;
  return launch_tc2<B_DQ_K>(ma, mb, ma2, mb2, p, t, ceil_div(M, 512), ceil_div(N, tn), s);
}

qlora_status tc2_fused_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                             const void* sV, const void* A, int32_t r, void* dX,
                             DeviceStatus* st, cudaStream_t s) {
  const int64_t N = w.rows, K = w.cols;
  CUtensorMap ma, mb, ma2, mb2;
  if (!make_map(&ma, dY, true, N, M, N, 64, 256, true) ||
      !make_map(&mb, w.codes, false, K / 2, N, K / 2, 64, 64, false) ||
      !make_map(&ma2, sV, true, 2 * lora_span(r), M, 2 * lora_span(r), 64, 256, true) ||
      !make_map(&mb2, A, true, K, r, K, 64, 64, true))
    return QLORA_ERR_CUDA;
  Tc2Args p = args_of(w, M, K, r, dX, st);
  p.kt_total = static_cast<int32_t>(ceil_div(N, 64));
  p.b2_mn = 1;
  return launch_tc2<B_DQ_MN>(ma, mb, ma2, mb2, p, t, ceil_div(M, 512), ceil_div(K, 256), s);
}

}  // namespace qlora

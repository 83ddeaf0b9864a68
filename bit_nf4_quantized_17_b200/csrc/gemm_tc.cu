// Tensor-core (tcgen05 / TMEM / TMA) contractions of the QLoRA linear layer.
//
// One warp-specialised kernel computes a 128-row tile D[m0:m0+128, n0:n0+bn]
// of D = A . B^T with fp32 accumulation in TMEM:
//
//   warp 0      TMA producer: A tiles (bf16, K- or MN-major, 128B swizzle),
//               and either B tiles (bf16) or the packed 4-bit codes of W
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=bn,
//               K=16) and commits each stage back to the producer
//   warps 4-11  dequantise W on load (modes B_DQ_*): per 64-weight block
//               they build the 16 bf16 values fp32(level[k] * s_hat) of the
//               block's own table and expand every nibble with byte permutes
//               straight into the 128B-swizzled bf16 B tile; then they drain
//               the accumulator from TMEM and store the tile
//
// After the main loop optional "extension" stages append a second pair of
// bf16 operands along K (A2, B2): this is how the rank-r LoRA term
// s (X A^T) B^T (forward) or s (dY B) A (backward dX) is added into the same
// accumulator as the dequantised-weight product, so Y and dX leave the kernel
// once, in bf16, and the full-precision W never exists outside shared memory
// ("QLoRA技术从入门到精通", 3(2): dequantise one layer at a time and discard).
//
// Every mbarrier wait is bounded; a wait that gives up raises a CTA-wide
// abort, the kernel drains its own copies and MMAs, frees TMEM and reports
// QLORA_ERR_DEVICE_TIMEOUT in the workspace status word.
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

using tc::block_tables;
using tc::expand8;
using tc::pack_bf16x2;

// warps 0-3: TMA producer, MMA issuer (and TMEM owner), two idle;
// warps 4-19: dequantisation in two groups of 256 threads that take alternate
// stages (more warps in flight to hide the dependent byte-permute chains),
// then the epilogue
constexpr int kThreads = 640;
constexpr int kDqThreads = 256;  // per group
constexpr int kABytes = 16384;   // 128 rows x 64 bf16
constexpr int kCodeBytes = 8192;  // codes of one k-tile: 256 W rows x 32 B (fwd) or 64 x 128 B (bwd)

// The codes ring: kCG k-tiles per slot, kCSlots slots.  A slot of the
// decode-sized forward holds 64 contiguous bytes of each of 256 W rows
// (2 k-tiles), so that every row is read from DRAM in 64-byte pieces.
template <int BMODE, int MT>
struct CodesRing {
  static constexpr bool kWide = (BMODE == B_DQ_K && MT == 1);
  static constexpr int kCG = kWide ? 2 : 1;
  static constexpr int kSlots = kWide ? 2 : 4;
  static constexpr int kSlotBytes = kCG * kCodeBytes;
  static constexpr int kBytes = (BMODE == B_TMA_K) ? 0 : kSlots * kSlotBytes;
};
constexpr long long kTimeoutCycles = 4000000000ll;  // ~2 s at 1.9 GHz

struct TcArgs {
  int32_t m, n, bn;
  int32_t k_tiles;        // main-loop stages per CTA (per split)
  int32_t kt_total;       // main-loop stages of the whole contraction
  int32_t k2_tiles;       // extension stages: two halves of k2_half stages each
  int32_t k2_half;        // stages per half (64 LoRA ranks each)
  int32_t k2_last_steps;  // K=16 steps in the last stage of each half
  int32_t a_mn, b2_mn;
  int32_t b_bytes, stage_bytes, tmem_cols;
  int32_t a_bytes;        // bytes of A actually loaded per stage (rows beyond M are not fetched)
  QView w;
  int32_t kblocks;        // W.cols / 64
  float alpha;
  void* out;
  int64_t ldo;
  int32_t out_bf16;
  int64_t split_stride;
  int64_t out_elems;      // elements of `out` (stores beyond it are reported, not made)
  int64_t nblocks;        // entries of w.scale_codes (loads beyond it are reported)
  DeviceStatus* st;
};

__device__ __forceinline__ void store16(const TcArgs& p, int64_t row, int64_t col,
                                        const uint32_t (&r)[16]) {
  if (row >= p.m) return;
  const int64_t base = static_cast<int64_t>(blockIdx.z) * p.split_stride + row * p.ldo + col;
  const int64_t span = (p.n - col < 16) ? (p.n - col) : 16;
  if (base < 0 || base + span > p.out_elems) {
    report(p.st, QLORA_ERR_SHAPE, 200u);
    return;
  }
  if (p.out_bf16) {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + base;
    if (col + 16 <= p.n) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        w[j] = pack_bf16x2(p.alpha * __uint_as_float(r[2 * j]), p.alpha * __uint_as_float(r[2 * j + 1]));
      reinterpret_cast<uint4*>(o)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(o)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
      for (int j = 0; j < 16 && col + j < p.n; ++j)
        o[j] = __float2bfloat16_rn(p.alpha * __uint_as_float(r[j]));
    }
  } else {
    float* o = static_cast<float*>(p.out) + base;
    if (col + 16 <= p.n) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        reinterpret_cast<float4*>(o)[j] =
            make_float4(p.alpha * __uint_as_float(r[4 * j]), p.alpha * __uint_as_float(r[4 * j + 1]),
                        p.alpha * __uint_as_float(r[4 * j + 2]), p.alpha * __uint_as_float(r[4 * j + 3]));
    } else {
      for (int j = 0; j < 16 && col + j < p.n; ++j) o[j] = p.alpha * __uint_as_float(r[j]);
    }
  }
}

template <int BMODE, int STAGES, int MT>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
               const TcArgs p, const LevelTable tab) {
  // MT accumulators of 128 rows share every B tile: a CTA covers 128*MT rows.
  constexpr int kA = kABytes * MT;
  constexpr bool kDq = BMODE != B_TMA_K;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  using Ring = CodesRing<BMODE, MT>;
  constexpr int kCG = Ring::kCG, kCSlots = Ring::kSlots;
  // [STAGES x (A | B)] [kCSlots x codes] [barriers]
  uint8_t* codes_ring = smem + STAGES * p.stage_bytes;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(codes_ring + Ring::kBytes);
  uint64_t* full_b = full_a + STAGES;
  uint64_t* empty = full_b + STAGES;
  uint64_t* codes_full = empty + STAGES;
  uint64_t* codes_empty = codes_full + kCSlots;
  uint64_t* accum = codes_empty + kCSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * 128 * MT;
  const int n0 = blockIdx.x * p.bn;
  const int kt0 = blockIdx.z * p.k_tiles;
  const int k_tiles = min(p.k_tiles, p.kt_total - kt0);
  // with split-K the LoRA extension stages belong to split 0 only
  const int k2_tiles = blockIdx.z == 0 ? p.k2_tiles : 0;
  const int total = k_tiles + k2_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full_a[s], 1);
      ptx::mbar_init(&full_b[s], kDqThreads);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kCSlots; ++s) {
      ptx::mbar_init(&codes_full[s], 1);
      // a slot holding several k-tiles is read by both dequant groups
      ptx::mbar_init(&codes_empty[s], kCG > 1 ? 2 * kDqThreads : kDqThreads);
    }
    ptx::mbar_init(accum, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    if (k2_tiles) {
      ptx::prefetch_tmap(&tmA2);
      ptx::prefetch_tmap(&tmB2);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, p.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    // A (and B when it is bf16) go into stage kt % STAGES once the MMAs of
    // its previous use are done; the 4-bit codes run ahead in their own ring
    // (groups of kCG k-tiles), freed as soon as the dequant warps read them.
    int issued = 0, kc = 0;
    const int n_groups = (k_tiles + kCG - 1) / kCG;
    bool ok = true;
    auto issue_codes = [&](int upto) {
      while (ok && kc < n_groups && kc < upto) {
        const int cs = kc % kCSlots;
        if (!ptx::mbar_wait(&codes_empty[cs], ((kc / kCSlots) & 1) ^ 1, kTimeoutCycles,
                            abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* dst = codes_ring + cs * Ring::kSlotBytes;
        const int kg = kt0 + kc * kCG;
        ptx::mbar_arrive_expect_tx(&codes_full[cs], Ring::kSlotBytes);
        if (BMODE == B_DQ_K)
          ptx::tma_load_2d(&tmB, &codes_full[cs], dst, kg * 32, n0);
        else
          ptx::tma_load_2d(&tmB, &codes_full[cs], dst, n0 / 2, kg * 64);
        ++kc;
      }
    };
    if (kDq) issue_codes(kCSlots);
    for (int kt = 0; kt < total && ok; ++kt) {
      const int s = kt % STAGES;
      const uint32_t ph = (kt / STAGES) & 1;
      if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) break;
      uint8_t* sa = smem + s * p.stage_bytes;
      uint8_t* sb = sa + kA;
      if (kt < k_tiles) {
        const int kg = kt0 + kt;
        ptx::mbar_arrive_expect_tx(&full_a[s], p.a_bytes + (kDq ? 0 : p.bn * 128));
        if (p.a_mn) {
          // MN-major A (only with MT == 1): two 64-row halves
          ptx::tma_load_2d(&tmA, &full_a[s], sa, m0, kg * 64);
          ptx::tma_load_2d(&tmA, &full_a[s], sa + 8192, m0 + 64, kg * 64);
        } else {
          ptx::tma_load_2d(&tmA, &full_a[s], sa, kg * 64, m0);
        }
        if (!kDq) ptx::tma_load_2d(&tmB, &full_a[s], sb, kg * 64, n0);
      } else {
        // extension stage tt: A2 columns [64 tt, 64 tt + 64) of [hi | lo], B2 ranks
        // [64 (tt mod half), ...): both halves multiply the same B2 tiles
        const int tt = kt - k_tiles;
        const int k2a = tt * 64;
        const int k2b = (tt % p.k2_half) * 64;
        // A2 (sU or sV) is the output of the launch before this one, which
        // lets the fused kernels start early (programmatic dependent launch):
        // the main loop reads only the activations and W
        if (tt == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
        ptx::mbar_arrive_expect_tx(&full_a[s], p.a_bytes + 32768);
        ptx::tma_load_2d(&tmA2, &full_a[s], sa, k2a, m0);
        if (p.b2_mn) {
#pragma unroll
          for (int h = 0; h < 4; ++h)
            ptx::tma_load_2d(&tmB2, &full_a[s], sb + h * 8192, n0 + 64 * h, k2b);
        } else {
          ptx::tma_load_2d(&tmB2, &full_a[s], sb, k2b, n0);
        }
      }
      ++issued;
      if (kDq) issue_codes(kt / kCG + kCSlots);
    }
    // never leave with copies in flight into this CTA's shared memory
    for (int kt = max(0, issued - STAGES); kt < issued; ++kt)
      ptx::mbar_wait(&full_a[kt % STAGES], (kt / STAGES) & 1, kTimeoutCycles, nullptr);
    for (int c = max(0, kc - kCSlots); c < kc; ++c)
      ptx::mbar_wait(&codes_full[c % kCSlots], (c / kCSlots) & 1, kTimeoutCycles, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------ MMA issuer
    const uint32_t idesc = ptx::idesc_bf16(128, p.bn, p.a_mn, BMODE == B_DQ_MN ? 1 : 0);
    const uint32_t idesc2 = ptx::idesc_bf16(128, p.bn, 0, p.b2_mn);
    for (int kt = 0; kt < total; ++kt) {
      const int s = kt % STAGES;
      const uint32_t ph = (kt / STAGES) & 1;
      if (!ptx::mbar_wait(&full_a[s], ph, kTimeoutCycles, abort_flag)) break;
      const bool ext = kt >= k_tiles;
      if (kDq && !ext && !ptx::mbar_wait(&full_b[s], ph, kTimeoutCycles, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(smem + s * p.stage_bytes);
      const uint32_t b_addr = a_addr + kA;
      const bool a_mn = !ext && p.a_mn;
      const bool b_mn = ext ? (p.b2_mn != 0) : (BMODE == B_DQ_MN);
      const int steps = (ext && ((kt - k_tiles) % p.k2_half) == p.k2_half - 1) ? p.k2_last_steps : 4;
      // descriptors stepped by their 16-byte address field from one per
      // operand and stage (see gemm_tc2.cu: building each afresh made the
      // issuing thread the limit); main k-tiles unrolled
      const uint64_t a0 = a_mn ? ptx::sw128_desc(a_addr, 8192, 1024) : ptx::sw128_desc(a_addr, 16, 1024);
      const uint64_t b0 = b_mn ? ptx::sw128_desc(b_addr, 8192, 1024) : ptx::sw128_desc(b_addr, 16, 1024);
      const uint64_t a_step = a_mn ? (2048 >> 4) : (32 >> 4);
      const uint64_t b_step = b_mn ? (2048 >> 4) : (32 >> 4);
      if (steps == 4) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (int t = 0; t < MT; ++t)
            ptx::umma_bf16(tmem + t * p.bn, a0 + a_step * ks + t * (kABytes >> 4), b0 + b_step * ks,
                           ext ? idesc2 : idesc, (kt | ks) != 0 ? 1u : 0u);
        }
      } else {
        for (int ks = 0; ks < steps; ++ks) {
#pragma unroll
          for (int t = 0; t < MT; ++t)
            ptx::umma_bf16(tmem + t * p.bn, a0 + a_step * ks + t * (kABytes >> 4), b0 + b_step * ks,
                           ext ? idesc2 : idesc, (kt | ks) != 0 ? 1u : 0u);
        }
      }
      ptx::umma_commit(&empty[s]);
    }
    ptx::umma_commit(accum);
    ptx::mbar_wait(accum, 0, kTimeoutCycles, nullptr);  // MMAs done before TMEM is freed
  } else if (warp >= 4) {
    const int grp = (threadIdx.x - 128) / kDqThreads;  // dequant group: stages kt % 2 == grp
    const int td = (threadIdx.x - 128) % kDqThreads;
    if (kDq) {
      // ---------------------------------------------------- dequantisation
      // forward: thread td expands W row n0 + td (one 64-weight block per stage);
      // backward: thread td expands block q = td / 64 of W row (stage rows) + td % 64.
      float lv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];
      const float mu = (p.w.dq_shift >= 0) ? __ldg(p.w.mean) : 0.0f;
      const int row = (BMODE == B_DQ_K) ? td : (td & 63);
      const int q = (BMODE == B_DQ_K) ? 0 : (td >> 6);
      // Raw inputs of the scale of the block this thread expands at stage kt:
      // the int8 code and the group factor (or the fp32 absmax without double
      // quantisation); `in` is false outside W.  They are loaded four of this
      // group's stages ahead and combined only when used, so the loads stay in
      // flight meanwhile (at small M every scale is a first touch from DRAM).
      struct RawScale {
        float q, f;
        bool in;
      };
      auto load_scale = [&](int kt) -> RawScale {
        if (kt >= k_tiles) return RawScale{0.0f, 0.0f, false};
        const int kg = kt0 + kt;
        const int64_t wrow = (BMODE == B_DQ_K) ? static_cast<int64_t>(n0) + row
                                               : static_cast<int64_t>(kg) * 64 + row;
        const int64_t kb = (BMODE == B_DQ_K) ? kg : (n0 / 64 + q);
        if (wrow >= p.w.rows || kb >= p.kblocks) return RawScale{0.0f, 0.0f, false};
        const int64_t b = wrow * (p.kblocks >> p.w.bs_shift) + (kb >> p.w.bs_shift);
        if (b >= p.nblocks) {
          report(p.st, QLORA_ERR_SHAPE, 201u);
          return RawScale{0.0f, 0.0f, false};
        }
        if (p.w.dq_shift < 0) return RawScale{1.0f, __ldg(p.w.factors + b), true};
        return RawScale{static_cast<float>(__ldg(p.w.scale_codes + b)),
                        __ldg(p.w.factors + (b >> p.w.dq_shift)), true};
      };
      const float mu_eff = (p.w.dq_shift >= 0) ? mu : 0.0f;
      RawScale r0 = load_scale(grp), r1 = load_scale(grp + 2), r2 = load_scale(grp + 4),
               r3 = load_scale(grp + 6);
      for (int kt = grp; kt < k_tiles; kt += 2) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        const int g = kt / kCG, sub = kt % kCG;
        const int cs = g % kCSlots;
        // s_hat = fp32(fp32(q * f) + mean) (absmax without double quantisation);
        // 0 outside W, which makes the whole table 0
        const float sc = !r0.in ? 0.0f
                         : (p.w.dq_shift < 0 ? r0.f : __fadd_rn(__fmul_rn(r0.q, r0.f), mu_eff));
        r0 = r1;
        r1 = r2;
        r2 = r3;
        r3 = load_scale(kt + 8);
        if (!ptx::mbar_wait(&codes_full[cs], (g / kCSlots) & 1, kTimeoutCycles, abort_flag))
          break;
        // this thread's 32 code bytes: fwd decode slots are 64-byte rows, the
        // backward slot 128-byte rows with the 128B swizzle (16-byte chunk c of
        // row r at c ^ (r & 7)), the large-M forward slot 32-byte rows
        const uint8_t* slot = codes_ring + cs * Ring::kSlotBytes;
        uint4 c0, c1;
        if (BMODE == B_DQ_K && !Ring::kWide) {
          c0 = *reinterpret_cast<const uint4*>(slot + row * 32);
          c1 = *reinterpret_cast<const uint4*>(slot + row * 32 + 16);
        } else if (BMODE == B_DQ_K) {
          c0 = *reinterpret_cast<const uint4*>(slot + row * 64 + 32 * sub);
          c1 = *reinterpret_cast<const uint4*>(slot + row * 64 + 32 * sub + 16);
        } else {
          const int chunk = (BMODE == B_DQ_K) ? 2 * sub : 2 * q;
          c0 = *reinterpret_cast<const uint4*>(slot + row * 128 + 16 * (chunk ^ (row & 7)));
          c1 = *reinterpret_cast<const uint4*>(slot + row * 128 + 16 * ((chunk + 1) ^ (row & 7)));
        }
        // this group's last read of the slot (it reads every other k-tile of it)
        if (sub + 2 >= kCG || kt + 2 >= k_tiles) {
          // The next TMA into this slot writes through the async proxy: order
          // these generic-proxy reads before it, then release the slot.
          // (Without the proxy fence the barrier alone let the TMA overwrite
          // codes that single threads had not yet read.)
          ptx::fence_proxy_async_smem();
          ptx::mbar_arrive(&codes_empty[cs]);
        }
        uint32_t L[4], H[4];
        block_tables(lv, sc, L, H);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        // B slot s is free once the MMAs of its previous use have completed
        if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) break;
        uint8_t* sb = smem + s * p.stage_bytes + kA;
        uint8_t* dst_row = (BMODE == B_DQ_K) ? sb + row * 128 : sb + q * 8192 + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(dst_row + 16 * (j ^ (row & 7))) = expand8(words[j], L, H);
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(&full_b[s]);
      }
    }
    // ---------------------------------------------------------- epilogue
    bool ok = ptx::mbar_wait(accum, 0, kTimeoutCycles, abort_flag);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (ok) {
      ptx::tc_fence_after();
      const int quarter = warp & 3;
      const int cg = (warp - 4) >> 2;  // 0..3: four warps per TMEM lane quarter
      const int nchunks = p.bn / 16;
      // MT == 2: warps cg drain accumulator cg & 1, column half cg >> 1;
      // MT == 1: the four column groups interleave over 16-column chunks
      const int t = (MT == 2) ? (cg & 1) : 0;
      const int c_first = (MT == 2) ? (cg >> 1) * ((nchunks + 1) / 2) : cg;
      const int c_end = (MT == 2) ? min(nchunks, c_first + (nchunks + 1) / 2) : nchunks;
      const int c_step = (MT == 2) ? 1 : 4;
      const int64_t row = static_cast<int64_t>(m0) + 128 * t + 32 * quarter + lane;
      for (int c = c_first; c < c_end; c += c_step) {
        uint32_t r[16];
        ptx::tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + t * p.bn + c * 16, r);
        ptx::tmem_ld_wait();
        store16(p, row, static_cast<int64_t>(n0) + c * 16, r);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, p.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.st, QLORA_ERR_DEVICE_TIMEOUT, 100u + BMODE);
}

// Deterministic split-K reduction.  v = sum_z part[z][i][j] (+ part[z][i][j + lo]
// when lo > 0), summed in a fixed order; then the outputs of tc::reduce_store.
// With o2_pad the padding columns of o2 ([cols, o2_lo) and [o2_lo + cols,
// 2 o2_lo) of every row) are written as zeros too, so o2 needs no memset.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t rows,
                                     int cols, int pcols, int lo, float* o1, int64_t ld1,
                                     int trans1, float a1, int acc1, __nv_bfloat16* o2, int64_t ld2,
                                     float a2, int o2_lo, __nv_bfloat16* o3, int64_t ld3, float a3,
                                     int o3_lo, int o2_pad, const int32_t* __restrict__ seg,
                                     int seg_cols) {
  const int64_t total = rows * cols;
  const int pad = (o2 && o2_pad) ? o2_lo - cols : 0;
  const int64_t total_pad = rows * 2 * pad;
  const int64_t split_stride = rows * pcols;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       e < total + total_pad; e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e >= total) {
      const int64_t p = e - total;
      const int64_t i = p / (2 * pad);
      const int c = static_cast<int>(p - i * 2 * pad);
      o2[i * ld2 + ((c < pad) ? cols + c : o2_lo + cols + (c - pad))] = __float2bfloat16_rn(0.0f);
      continue;
    }
    const int64_t i = e / cols;
    const int j = static_cast<int>(e - i * cols);
    const float* src = part + i * pcols + j;
    // up to 8 splits are loaded together, then added in split order
    float v = 0.0f;
    for (int z0 = 0; z0 < splits; z0 += 8) {
      float h[8], l[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        h[u] = (z0 + u < splits) ? src[(z0 + u) * split_stride] : 0.0f;
        l[u] = (lo && z0 + u < splits) ? src[(z0 + u) * split_stride + lo] : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (z0 + u < splits) {
          v += h[u];
          if (lo) v += l[u];
        }
      }
    }
    if (seg && __ldg(seg + i) != j / seg_cols) v = 0.0f;
    tc::reduce_store(v, i, j, o1, ld1, trans1, a1, acc1, o2, ld2, a2, o2_lo, o3, ld3, a3, o3_lo);
  }
}

// Same reduction with one warp per output: lane l sums splits l, l + 32, ...,
// then the lanes are combined by a butterfly (a fixed order: deterministic).
// Used when there are few outputs and many splits.
__global__ void splitk_reduce_warp_kernel(const float* __restrict__ part, int splits, int64_t rows,
                                          int cols, int pcols, int lo, float* o1, int64_t ld1,
                                          int trans1, float a1, int acc1, __nv_bfloat16* o2,
                                          int64_t ld2, float a2, int o2_lo, __nv_bfloat16* o3,
                                          int64_t ld3, float a3, int o3_lo, int o2_pad,
                                          const int32_t* __restrict__ seg, int seg_cols) {
  const int64_t total = rows * cols;
  const int64_t split_stride = rows * pcols;
  const int lane = threadIdx.x & 31;
  if (o2 && o2_pad) {
    // the padding columns of o2, one thread each
    const int pad = o2_lo - cols;
    for (int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         p < rows * 2 * pad; p += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t i = p / (2 * pad);
      const int c = static_cast<int>(p - i * 2 * pad);
      o2[i * ld2 + ((c < pad) ? cols + c : o2_lo + cols + (c - pad))] = __float2bfloat16_rn(0.0f);
    }
  }
  for (int64_t e = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; e < total;
       e += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t i = e / cols;
    const int j = static_cast<int>(e - i * cols);
    const float* src = part + i * pcols + j;
    float v = 0.0f;
    for (int z = lane; z < splits; z += 32) {
      v += src[z * split_stride];
      if (lo) v += src[z * split_stride + lo];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (seg && __ldg(seg + i) != j / seg_cols) v = 0.0f;
    if (lane == 0)
      tc::reduce_store(v, i, j, o1, ld1, trans1, a1, acc1, o2, ld2, a2, o2_lo, o3, ld3, a3, o3_lo);
  }
}

// out[j][i] = hi = bf16(in[i][j]) and, if lo_rows > 0, out[j + lo_rows][i] =
// bf16(in[i][j] - hi), for a rows x cols fp32 or bf16 matrix.
template <typename T>
__global__ void transpose_bf16_kernel(const T* __restrict__ in, int64_t rows, int cols,
                                      int64_t ld_in, __nv_bfloat16* __restrict__ out,
                                      int64_t ld_out, int lo_rows) {
  const int64_t total = rows * cols;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / cols;
    const int j = static_cast<int>(e - i * cols);
    float v;
    if constexpr (sizeof(T) == 4)
      v = in[i * ld_in + j];
    else
      v = __bfloat162float(in[i * ld_in + j]);
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    out[j * ld_out + i] = h;
    if (lo_rows) out[(j + lo_rows) * ld_out + i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// ----------------------------------------------------------------- host

}  // namespace

using EncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeFn encode_fn() {
  static EncodeFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeFn>(nullptr);
    return reinterpret_cast<EncodeFn>(f);
  }();
  return fn;
}

// 2-D map over a row-major matrix: `inner` contiguous elements per row, `outer`
// rows `ld` elements apart; box = box_inner x box_outer elements.
bool make_map(CUtensorMap* map, const void* base, bool bf16, uint64_t inner, uint64_t outer,
              uint64_t ld, uint32_t box_inner, uint32_t box_outer, bool swizzle) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const int es = bf16 ? 2 : 1;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld * es};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

int pow2_cols(int bn) {
  int c = 32;
  while (c < bn) c <<= 1;
  return c;
}

template <int BMODE, int STAGES, int MT>
qlora_status launch_tc(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& a2,
                       const CUtensorMap& b2, TcArgs p, const LevelTable& t, dim3 grid,
                       cudaStream_t s) {
  const size_t smem = 1024 + static_cast<size_t>(STAGES) * p.stage_bytes +
                      CodesRing<BMODE, MT>::kBytes + 256;
  const qlora_status cs =
      ensure_smem(reinterpret_cast<const void*>(tc_gemm_kernel<BMODE, STAGES, MT>), 232448);
  if (cs != QLORA_OK) return cs;
  count_launch();
  constexpr int kind = BMODE == B_TMA_K   ? QLORA_KERNEL_LORA_GEMM
                       : BMODE == B_DQ_K ? QLORA_KERNEL_FUSED_FWD
                                         : QLORA_KERNEL_FUSED_DGRAD;
  timing_mark(kind, s, true);
  if constexpr (BMODE == B_TMA_K) {
    tc_gemm_kernel<BMODE, STAGES, MT><<<grid, kThreads, smem, s>>>(a, b, a2, b2, p, t);
  } else {
    // the fused kernels read the previous launch's output only in their LoRA
    // stages: they may start while it runs
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, tc_gemm_kernel<BMODE, STAGES, MT>, a, b, a2, b2, p, t) !=
        cudaSuccess) {
      timing_mark(kind, s, false);
      return QLORA_ERR_CUDA;
    }
  }
  timing_mark(kind, s, false);
  return after_launch(BMODE == B_TMA_K ? "tc_gemm(lora)" : BMODE == B_DQ_K ? "tc_gemm(fwd)" : "tc_gemm(dgrad)", s);
}

TcArgs base_args(int m, int n, int bn, DeviceStatus* st) {
  TcArgs p{};
  p.m = m;
  p.n = n;
  p.bn = bn;
  p.k2_last_steps = 4;
  p.k2_half = 1;
  p.tmem_cols = pow2_cols(bn);
  p.alpha = 1.0f;
  p.st = st;
  return p;
}

}  // namespace

// Rows of the activation tile actually fetched: the MMA always runs 128 rows
// per accumulator, but rows at or beyond M only feed accumulator rows that are
// never stored, so they need not be loaded.
uint32_t a_rows(int64_t M, int mt) {
  const int64_t full = 128 * mt;
  const int64_t r16 = (M + 15) / 16 * 16;
  return static_cast<uint32_t>(r16 < full ? r16 : full);
}

// Splits of a rank-r GEMM: as many as keep the grid within one wave (two
// CTAs per SM), and at least four k-tiles per split.
int tc_split_count(int64_t m_tiles, int64_t k_tiles) {
  int64_t s = (2 * 148) / m_tiles;
  const int64_t max_s = k_tiles / 4 > 0 ? k_tiles / 4 : 1;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  const int64_t per = (k_tiles + s - 1) / s;
  return static_cast<int>((k_tiles + per - 1) / per);
}

// Tile shape of the fused kernels: MT 128-row accumulators per CTA and a
// split of the contraction when the output alone gives too few CTAs.
FusedShape fused_shape(int64_t M, int64_t n_out, int64_t kt_total) {
  FusedShape f;
  const int64_t n_tiles = ceil_div(n_out, 256);
  f.mt = (M > 128) ? 2 : 1;
  const int64_t m_tiles = ceil_div(M, 128 * f.mt);
  f.splits = 1;
  if (m_tiles * n_tiles < 148) {
    // one CTA per SM fits (shared memory): stay within a single wave
    int64_t s = 148 / (m_tiles * n_tiles);
    const int64_t max_s = kt_total / 2 > 0 ? kt_total / 2 : 1;
    if (s > max_s) s = max_s;
    const int64_t per = ceil_div(kt_total, s);
    f.splits = static_cast<int>(ceil_div(kt_total, per));
  }
  return f;
}

namespace {

template <int BMODE>
qlora_status launch_fused(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& ma2,
                          const CUtensorMap& mb2, TcArgs p, const LevelTable& t, int64_t M,
                          int64_t n_out, const FusedShape& f, cudaStream_t s) {
  p.k_tiles = static_cast<int>(ceil_div(p.kt_total, f.splits));
  p.a_bytes = static_cast<int32_t>(a_rows(M, f.mt)) * 128;
  p.b_bytes = 32768;
  p.stage_bytes = f.mt * kABytes + 32768;
  p.tmem_cols = f.mt == 2 ? 512 : 256;
  dim3 grid(static_cast<unsigned>(ceil_div(n_out, 256)),
            static_cast<unsigned>(ceil_div(M, 128 * f.mt)), static_cast<unsigned>(f.splits));
  if (f.mt == 2) return launch_tc<BMODE, 3, 2>(ma, mb, ma2, mb2, p, t, grid, s);
  return launch_tc<BMODE, 4, 1>(ma, mb, ma2, mb2, p, t, grid, s);
}

}  // namespace

qlora_status tc_fused_forward(const QView& w, const LevelTable& t, const void* X, int64_t M,
                              const void* sU, const void* B, int32_t r, void* out,
                              const FusedShape& f, DeviceStatus* st, cudaStream_t s) {
  if (tc2_eligible(M, f)) return tc2_fused_forward(w, t, X, M, sU, B, r, out, st, s);
  const int64_t N = w.rows, K = w.cols;
  const uint32_t rows = a_rows(M, f.mt);
  CUtensorMap ma, mb, ma2, mb2;
  if (!make_map(&ma, X, true, K, M, K, 64, rows, true) ||
      !(f.mt == 1 ? make_map(&mb, w.codes, false, K / 2, N, K / 2, 64, 256, false)
                  : make_map(&mb, w.codes, false, K / 2, N, K / 2, 32, 256, false)) ||
      !make_map(&ma2, sU, true, 2 * lora_span(r), M, 2 * lora_span(r), 64, rows, true) ||
      !make_map(&mb2, B, true, r, N, r, 64, 256, true))
    return QLORA_ERR_CUDA;
  TcArgs p = base_args(static_cast<int>(M), static_cast<int>(N), 256, st);
  p.kt_total = static_cast<int>(K / 64);
  p.k2_half = (r + 63) / 64;
  p.k2_tiles = 2 * p.k2_half;
  p.k2_last_steps = ((r - 64 * (p.k2_half - 1)) + 15) / 16;
  p.w = w;
  p.kblocks = static_cast<int>(K / 64);
  p.nblocks = (N * K / 64) >> w.bs_shift;
  p.out = out;
  p.ldo = N;
  p.out_bf16 = f.splits == 1 ? 1 : 0;
  p.split_stride = M * N;
  p.out_elems = static_cast<int64_t>(f.splits) * M * N;
  return launch_fused<B_DQ_K>(ma, mb, ma2, mb2, p, t, M, N, f, s);
}

qlora_status tc_fused_dgrad(const QView& w, const LevelTable& t, const void* dY, int64_t M,
                            const void* sV, const void* A, int32_t r, void* out,
                            const FusedShape& f, DeviceStatus* st, cudaStream_t s) {
  if (tc2_eligible(M, f)) return tc2_fused_dgrad(w, t, dY, M, sV, A, r, out, st, s);
  const int64_t N = w.rows, K = w.cols;
  const uint32_t rows = a_rows(M, f.mt);
  CUtensorMap ma, mb, ma2, mb2;
  if (!make_map(&ma, dY, true, N, M, N, 64, rows, true) ||
      !make_map(&mb, w.codes, false, K / 2, N, K / 2, 128, 64, true) ||
      !make_map(&ma2, sV, true, 2 * lora_span(r), M, 2 * lora_span(r), 64, rows, true) ||
      !make_map(&mb2, A, true, K, r, K, 64, 64, true))
    return QLORA_ERR_CUDA;
  TcArgs p = base_args(static_cast<int>(M), static_cast<int>(K), 256, st);
  p.kt_total = static_cast<int>(ceil_div(N, 64));
  p.k2_half = (r + 63) / 64;
  p.k2_tiles = 2 * p.k2_half;
  p.k2_last_steps = ((r - 64 * (p.k2_half - 1)) + 15) / 16;
  p.b2_mn = 1;
  p.w = w;
  p.kblocks = static_cast<int>(K / 64);
  p.nblocks = (N * K / 64) >> w.bs_shift;
  p.out = out;
  p.ldo = K;
  p.out_bf16 = f.splits == 1 ? 1 : 0;
  p.split_stride = M * K;
  p.out_elems = static_cast<int64_t>(f.splits) * M * K;
  return launch_fused<B_DQ_MN>(ma, mb, ma2, mb2, p, t, M, K, f, s);
}

// part[z] (m_rows x n_cols fp32) = A . B^T over split z of the contraction; A is
// m_rows x kdim (K-major, or MN-major: stored kdim x m_rows), B is b_rows x kdim
// K-major (ld_b), read as n_cols rows (a multiple of 16; rows past b_rows are zero).
qlora_status tc_lora_gemm(const void* A, bool a_mn, int64_t m_rows, int64_t kdim, int64_t ld_a,
                          const void* B, int64_t ld_b, int32_t b_rows, int32_t n_cols,
                          float* part, int splits, DeviceStatus* st, cudaStream_t s) {
  const int bn = n_cols < 256 ? n_cols : 256;
  CUtensorMap ma, mb;
  bool ok = a_mn ? make_map(&ma, A, true, m_rows, kdim, ld_a, 64, 64, true)
                 : make_map(&ma, A, true, kdim, m_rows, ld_a, 64, 128, true);
  ok = ok && make_map(&mb, B, true, kdim, b_rows, ld_b, 64, bn, true);
  if (!ok) return QLORA_ERR_CUDA;
  TcArgs p = base_args(static_cast<int>(m_rows), n_cols, bn, st);
  p.kt_total = static_cast<int>(ceil_div(kdim, 64));
  p.k_tiles = static_cast<int>(ceil_div(p.kt_total, splits));
  p.a_mn = a_mn ? 1 : 0;
  p.b_bytes = (bn * 128 + 1023) / 1024 * 1024;
  p.stage_bytes = kABytes + p.b_bytes;
  p.a_bytes = kABytes;
  p.out = part;
  p.ldo = n_cols;
  p.out_bf16 = 0;
  p.split_stride = m_rows * n_cols;
  p.out_elems = static_cast<int64_t>(splits) * m_rows * n_cols;
  dim3 grid(static_cast<unsigned>(ceil_div(n_cols, bn)), static_cast<unsigned>(ceil_div(m_rows, 128)),
            static_cast<unsigned>(splits));
  LevelTable unused{};
  return launch_tc<B_TMA_K, 4, 1>(ma, mb, ma, mb, p, unused, grid, s);
}

qlora_status splitk_reduce(const ReduceArgs& a, cudaStream_t s) {
  const int64_t total = a.rows * a.cols;
  count_launch();
  if (a.splits >= 16 && total < 32768) {
    const int grid = static_cast<int>(std::min<int64_t>(ceil_div(total * 32, 256), 148 * 8));
    splitk_reduce_warp_kernel<<<grid, 256, 0, s>>>(
        a.part, a.splits, a.rows, a.cols, a.pcols, a.lo, a.o1, a.ld1, a.trans1 ? 1 : 0, a.a1,
        a.acc1 ? 1 : 0, static_cast<__nv_bfloat16*>(a.o2), a.ld2, a.a2, a.o2_lo,
        static_cast<__nv_bfloat16*>(a.o3), a.ld3, a.a3, a.o3_lo, a.o2_pad, a.seg,
        a.seg ? a.seg_cols : 1);
  } else {
    const int64_t pad_items = (a.o2 && a.o2_pad) ? a.rows * 2 * (a.o2_lo - a.cols) : 0;
    const int grid =
        static_cast<int>(std::min<int64_t>(ceil_div(total + pad_items, 256), 148 * 8));
    splitk_reduce_kernel<<<grid, 256, 0, s>>>(
        a.part, a.splits, a.rows, a.cols, a.pcols, a.lo, a.o1, a.ld1, a.trans1 ? 1 : 0, a.a1,
        a.acc1 ? 1 : 0, static_cast<__nv_bfloat16*>(a.o2), a.ld2, a.a2, a.o2_lo,
        static_cast<__nv_bfloat16*>(a.o3), a.ld3, a.a3, a.o3_lo, a.o2_pad, a.seg,
        a.seg ? a.seg_cols : 1);
  }
  return after_launch("splitk_reduce", s);
}

qlora_status transpose_to_bf16(const void* in, bool in_f32, int64_t rows, int cols, int64_t ld_in,
                               void* out, int64_t ld_out, int lo_rows, cudaStream_t s) {
  const int64_t total = rows * cols;
  const int grid = static_cast<int>(std::min<int64_t>(ceil_div(total, 256), 148 * 8));
  count_launch();
  if (in_f32)
    transpose_bf16_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float*>(in), rows, cols,
                                                      ld_in, static_cast<__nv_bfloat16*>(out),
                                                      ld_out, lo_rows);
  else
    transpose_bf16_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(in), rows, cols, ld_in,
        static_cast<__nv_bfloat16*>(out), ld_out, lo_rows);
  return after_launch("transpose_to_bf16", s);
}

}  // namespace qlora

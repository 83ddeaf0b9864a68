// Merging a trained adapter into a restored 16-bit weight on the tensor cores.
//
//   W_merged[n][k] = bf16( fp32(level[idx] * s_hat) + s * sum_j B[n][j] A[j][k] )
//
// ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section 3: B A has the shape
// of W and is added to the restored weight.)  The dense form takes a bf16 base
// W_in instead of the NF4 decode.
//
// One CTA per 128 x 128 tile of W.  The rank-r product B A is one tcgen05.mma
// chain (M = 128 rows of B, N = 128 columns of A, K = the ranks in steps of 16)
// into 128 TMEM columns: B's rows arrive K-major and A's columns MN-major, by
// TMA in 128B-swizzled boxes, 64 ranks per stage.  The epilogue gives each TMEM
// lane (one W row) to one thread: the row's codes and block scales are
// requested before the wait for the MMAs; then per 16-column chunk it reads the
// fp32 products, restores the chunk's 16 base weights, adds s times the
// product with the same two roundings as the CUDA-core form, rounds once to
// bf16 and writes 32 bytes.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-5 the epilogue.  The epilogue waits on memory, not on issue, so the
// tile is narrow and the registers few enough for four CTAs per SM: at r <= 64
// the CTA takes one pipeline stage (34 KB of shared memory), and the launch
// asks for at least 47 KB so that no fifth CTA fits and the four CTAs' TMEM
// columns (4 x 128) stay within the SM's 512.  Every wait is bounded; the merge
// calls take no status word, so a wait that gives up (it does not in correct
// operation) leaves NaN in its CTA's tile.
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 192;
constexpr int kTileRows = 128, kTileCols = 128;
constexpr int kStages = 2;
constexpr int kABytes = 16384;                   // 128 rows of B x 64 ranks
constexpr int kBBytes = 16384;                   // 64 ranks x 128 columns of A (two boxes)
constexpr int kStageBytes = kABytes + kBBytes;
// [alignment slack][barriers, TMEM address, abort flag, levels: 1024][stages]
constexpr int kHeadBytes = 1024;
constexpr int smem_bytes(int stages) { return 1024 + kHeadBytes + stages * kStageBytes; }
constexpr int kMinSmemBytes = 47 * 1024;  // 5 x (47 KB + 1 KB reserved) > 228 KB per SM
constexpr uint32_t kTmemCols = 128;
constexpr long long kTimeoutCycles = 4000000000ll;

struct MergeTcArgs {
  QView w;                    // NF4 base (DENSE = false)
  const __nv_bfloat16* win;   // bf16 base (DENSE = true); may be `out`
  __nv_bfloat16* out;
  int64_t rows, cols;
  int32_t kt_total;           // 64-rank stages
  int32_t last_steps;         // 16-rank MMA steps of the last stage
  float s;                    // alpha / r
};

template <bool DENSE>
__global__ void __launch_bounds__(kThreads, 4)
merge_tc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmA,
                const MergeTcArgs p, const LevelTable tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kStages;
  uint64_t* accum = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* lv = reinterpret_cast<float*>(smem + 128);  // 16 levels
  uint8_t* stages = smem + kHeadBytes;  // min(kStages, stages the ranks need) of them

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kTileRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kTileCols;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accum, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmB);
    ptx::prefetch_tmap(&tmA);
  }
  if (!DENSE && threadIdx.x == 64) {  // warp 2: no warp-wide TMEM instruction before the barrier
#pragma unroll
    for (int j = 0; j < 16; ++j) lv[j] = tab.level[j];  // constant indices: no local copy
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
    int issued = 0;
    for (int i = 0; i < p.kt_total; ++i) {
      const int s = i % kStages;
      if (!ptx::mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, kTimeoutCycles, abort_flag)) break;
      uint8_t* sa = stages + s * kStageBytes;
      ptx::mbar_arrive_expect_tx(&full[s], kStageBytes);
      ptx::tma_load_2d(&tmB, &full[s], sa, i * 64, static_cast<int>(n0));  // 128 rows x 64 ranks
      for (int h = 0; h < kTileCols / 64; ++h)                              // 64 ranks x 64 columns
        ptx::tma_load_2d(&tmA, &full[s], sa + kABytes + h * 8192, static_cast<int>(k0) + 64 * h,
                         i * 64);
      ++issued;
    }
    // never leave with copies in flight into this CTA's shared memory
    for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
      ptx::mbar_wait(&full[i % kStages], (i / kStages) & 1, kTimeoutCycles, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------ MMA issuer
    const uint32_t idesc = ptx::idesc_bf16(kTileRows, kTileCols, 0, 1);
    for (int i = 0; i < p.kt_total; ++i) {
      const int s = i % kStages;
      if (!ptx::mbar_wait(&full[s], (i / kStages) & 1, kTimeoutCycles, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(stages + s * kStageBytes);
      const uint64_t a0 = ptx::sw128_desc(a_addr, 16, 1024);               // K-major rows of B
      const uint64_t b0 = ptx::sw128_desc(a_addr + kABytes, 8192, 1024);   // MN-major columns of A
      const int steps = (i == p.kt_total - 1) ? p.last_steps : 4;
      for (int ks = 0; ks < steps; ++ks)
        ptx::umma_bf16(tmem, a0 + ((32 * ks) >> 4), b0 + ((2048 * ks) >> 4), idesc,
                       (i | ks) != 0 ? 1u : 0u);
      ptx::umma_commit(&empty[s]);
    }
    ptx::umma_commit(accum);
    ptx::mbar_wait(accum, 0, kTimeoutCycles, nullptr);  // MMAs done before TMEM is freed
  } else if (warp >= 2) {
    // ------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31
    const int row = 32 * quarter + lane;
    const int64_t n = n0 + row;
    const bool row_in = n < p.rows;
    // this row's codes and block scales for the whole tile, requested before
    // the wait for the MMAs so that their latency overlaps it
    uint4 cw[kTileCols / 32];
    float scv[kTileCols / 64];
    if constexpr (!DENSE) {
      const float mu = (p.w.dq_shift >= 0) ? __ldg(p.w.mean) : 0.0f;
      const int64_t nb_row = p.cols >> (6 + p.w.bs_shift);
#pragma unroll
      for (int c = 0; c < kTileCols / 32; ++c) {
        const int64_t k = k0 + 32 * c;
        cw[c] = make_uint4(0u, 0u, 0u, 0u);
        if (row_in && k < p.cols)
          cw[c] = __ldg(reinterpret_cast<const uint4*>(p.w.codes + (n * p.cols + k) / 2));
      }
#pragma unroll
      for (int c = 0; c < kTileCols / 64; ++c) {
        const int64_t k = k0 + 64 * c;
        scv[c] = 0.0f;
        if (row_in && k < p.cols) scv[c] = block_scale(p.w, n * nb_row + (k >> (6 + p.w.bs_shift)), mu);
      }
    }
    bool ok = ptx::mbar_wait(accum, 0, kTimeoutCycles, abort_flag);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    ptx::tc_fence_after();
    // the TMEM loads are warp-wide: every lane takes part in each chunk, and
    // the rows past the end skip only the loads and stores of W
#pragma unroll
    for (int c = 0; c < kTileCols / 16; ++c) {
      const int64_t k = k0 + 16 * c;
      if (k >= p.cols) break;  // uniform: cols is a multiple of 64, a chunk is all in or all out
      __syncwarp();
      uint32_t acc[16];
      if (ok) {
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 16 * c;
        ptx::tmem_ld_x16(taddr, acc);
        ptx::tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0u;
      }
      if (row_in) {
        float base[16];
        if constexpr (DENSE) {
          const uint4* src = reinterpret_cast<const uint4*>(p.win + n * p.cols + k);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint4 v = src[q];
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              base[8 * q + 2 * u] = __uint_as_float(vw[u] << 16);
              base[8 * q + 2 * u + 1] = __uint_as_float(vw[u] & 0xffff0000u);
            }
          }
        } else {
          // 16 codes (8 bytes) of one block, and its restored scale s_hat
          const float sc = scv[c >> 2];
          const uint4 c4 = cw[c >> 1];
          const uint32_t words[2] = {(c & 1) ? c4.z : c4.x, (c & 1) ? c4.w : c4.y};
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int u = 0; u < 8; ++u)
              base[8 * q + u] = __fmul_rn(lv[(words[q] >> (4 * u)) & 15u], sc);
        }
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float v0 = ok ? __fadd_rn(base[j], __fmul_rn(p.s, __uint_as_float(acc[j])))
                              : __uint_as_float(0x7fc00000u);
          const float v1 = ok ? __fadd_rn(base[j + 1], __fmul_rn(p.s, __uint_as_float(acc[j + 1])))
                              : __uint_as_float(0x7fc00000u);
          o[j / 2] = tc::pack_bf16x2(v0, v1);
        }
        uint4* dst = reinterpret_cast<uint4*>(p.out + n * p.cols + k);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool DENSE>
qlora_status launch(const QView& w, const LevelTable& t, const void* W_in, int64_t rows,
                    int64_t cols, const void* A, const void* B, int32_t r, float alpha, void* out,
                    cudaStream_t s) {
  CUtensorMap mb, ma;
  // B: rows x r (ranks contiguous), 64-rank x 128-row boxes; A: r x cols
  // (columns contiguous), 64-column x 64-rank boxes.  Ranks past r read as 0.
  if (!make_map(&mb, B, true, r, rows, r, 64, kTileRows, true) ||
      !make_map(&ma, A, true, cols, r, cols, 64, 64, true))
    return QLORA_ERR_CUDA;
  MergeTcArgs p{};
  p.w = w;
  p.win = static_cast<const __nv_bfloat16*>(W_in);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.rows = rows;
  p.cols = cols;
  p.kt_total = static_cast<int32_t>(ceil_div(r, 64));
  p.last_steps = static_cast<int32_t>(ceil_div(r - 64 * (p.kt_total - 1), 16));
  p.s = alpha / static_cast<float>(r);
  const qlora_status cs =
      ensure_smem(reinterpret_cast<const void*>(merge_tc_kernel<DENSE>), smem_bytes(kStages));
  // one stage when the ranks fit in one (r <= 64), so that four CTAs share an
  // SM; never less than a fifth of an SM's shared memory, so that no fifth CTA
  // fits and the CTAs' TMEM columns (4 x 128) stay within the SM's 512
  int smem = smem_bytes(p.kt_total < kStages ? p.kt_total : kStages);
  if (smem < kMinSmemBytes) smem = kMinSmemBytes;
  if (cs != QLORA_OK) return cs;
  const int64_t gx = ceil_div(cols, kTileCols), gy = ceil_div(rows, kTileRows);
  if (gx > 0x7fffffff || gy > 65535) return QLORA_ERR_SHAPE;
  count_launch();
  timing_mark(QLORA_KERNEL_MERGE, s, true);
  merge_tc_kernel<DENSE><<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kThreads,
                           smem, s>>>(mb, ma, p, t);
  timing_mark(QLORA_KERNEL_MERGE, s, false);
  return after_launch(DENSE ? "merge_tc(dense)" : "merge_tc", s);
}

}  // namespace

bool merge_tc_eligible(int64_t cols, int32_t r) {
  // TMA rows of B are r bf16: a multiple of 16 bytes; column chunks of 32
  return r >= 1 && r <= 256 && r % 8 == 0 && cols % 64 == 0;
}

qlora_status launch_merge_tc(const QView& w, const LevelTable& t, const void* A, const void* B,
                             int32_t r, float alpha, void* out, cudaStream_t s) {
  return launch<false>(w, t, nullptr, w.rows, w.cols, A, B, r, alpha, out, s);
}

qlora_status launch_merge_dense_tc(const void* W_in, int64_t rows, int64_t cols, const void* A,
                                   const void* B, int32_t r, float alpha, void* out,
                                   cudaStream_t s) {
  QView w{};
  w.rows = rows;
  w.cols = cols;
  return launch<true>(w, LevelTable{}, W_in, rows, cols, A, B, r, alpha, out, s);
}

}  // namespace qlora

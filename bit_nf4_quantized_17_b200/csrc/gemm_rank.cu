// Rank-r contractions of the QLoRA linear layer for large token counts,
// reduced inside a thread-block cluster.
//
// The four rank-r products of a training step ("LoRA 与 QLoRA：把大模型微调拆成
// 可负担的工程", 2 and 6; "QLoRA技术从入门到精通", 3(2) 双轨计算 and 3(3)):
//   U = X A^T (M x r, over d_in),      V = dY B (M x r, over d_out),
//   dB = s dY^T U (d_out x r, over M),  dA = s V^T X (r x d_in, over M),
// are thin: r <= 256 output columns against a contraction of thousands.  They
// move X or dY once and are bound by that read.  One launch computes
// D = A . B^T for 128-row tiles of A: the contraction is split over the S CTAs
// of a cluster (S = 1 .. 8) so that the grid covers the SMs, each CTA
// accumulates its share in TMEM (tcgen05.mma kind::f16, M = 128, N = bn,
// operands by TMA in 128B-swizzled tiles), and the S fp32 partial tiles are
// summed in distributed shared memory, in split order (deterministic), by the
// CTA that owns each slice of ceil(128 / S) rows.  The sums go straight to the outputs the
// callers need (fp32, bf16 [hi | lo] pairs, transposed copies), so no partial
// reaches global memory and no separate reduce launch follows.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer,
// warps 2-5 drain the accumulator into shared memory and reduce.  Every wait
// on an mbarrier is bounded; a wait that gives up raises the CTA's abort flag,
// the CTA still takes part in both cluster barriers (writing zeros), and
// QLORA_ERR_DEVICE_TIMEOUT is reported.
#include <cudaTypedefs.h>

#include "internal.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 192;
constexpr int kABytes = 16384;               // 128 rows x 64 bf16
// stages of A and B tiles (the reduce buffer reuses them): small enough for
// two CTAs per SM where the partial tile allows, for bytes in flight
constexpr int kSmemBudget = 100 * 1024;
constexpr long long kTimeoutCycles = 4000000000ll;

// fp32 load from another CTA's shared memory (a shared::cluster address);
// volatile so that it stays between the two cluster barriers around it.
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

struct RankArgs {
  int32_t m_rows;        // rows of A (and of the result)
  int32_t kt_total;      // 64-wide k-tiles of the whole contraction
  int32_t k_tiles;       // k-tiles per split
  int32_t a_mn;          // A stored MN-major (its rows contiguous)
  int32_t b_mn;          // B stored MN-major (its n_cols columns contiguous): bn / 64 boxes
  int32_t bn;            // MMA N: columns of the partial tile (multiple of 16, <= 256)
  int32_t b_bytes, stage_bytes, stages, tmem_cols;
  int32_t red_ld;        // fp32 row stride of the shared-memory partial tile
  ReduceArgs o;          // outputs; o.part and o.splits are not used
  DeviceStatus* st;
};

__global__ void __launch_bounds__(kThreads, 1)
rank_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const RankArgs p) {
  // the fused GEMM that follows may start now: it reads this launch's output
  // only after its own grid-dependency wait
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const size_t red_bytes = static_cast<size_t>(128) * p.red_ld * sizeof(float);
  const size_t stage_area = static_cast<size_t>(p.stages) * p.stage_bytes;
  const size_t data_bytes = stage_area > red_bytes ? stage_area : red_bytes;
  // [stages x (A | B)], reused as the fp32 partial tile once the MMAs are done
  float* red = reinterpret_cast<float*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + data_bytes);
  uint64_t* empty = full + 8;
  uint64_t* accum = empty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t S = gridDim.z;                       // splits = CTAs of the cluster
  const uint32_t z = ptx::cluster_ctarank();          // == blockIdx.z (cluster spans z)
  const int m0 = blockIdx.y * 128;
  const int n0 = blockIdx.x * p.bn;
  const int kt0 = static_cast<int>(z) * p.k_tiles;
  const int kn = max(0, min(p.k_tiles, p.kt_total - kt0));

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accum, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
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
    int issued = 0;
    for (int i = 0; i < kn; ++i) {
      const int s = i % p.stages;
      const uint32_t ph = (i / p.stages) & 1;
      if (!ptx::mbar_wait(&empty[s], ph ^ 1, kTimeoutCycles, abort_flag)) break;
      uint8_t* sa = smem + s * p.stage_bytes;
      const int kg = kt0 + i;
      ptx::mbar_arrive_expect_tx(&full[s], kABytes + p.b_bytes);
      if (p.a_mn) {
        // A^T tiles: 64 contraction rows x 64 output rows, two halves
        ptx::tma_load_2d(&tmA, &full[s], sa, m0, kg * 64);
        ptx::tma_load_2d(&tmA, &full[s], sa + 8192, m0 + 64, kg * 64);
      } else {
        ptx::tma_load_2d(&tmA, &full[s], sa, kg * 64, m0);
      }
      if (p.b_mn) {
        // B^T tiles: 64 contraction rows x 64 columns, one per 64 columns
        for (int h = 0; h < p.bn / 64; ++h)
          ptx::tma_load_2d(&tmB, &full[s], sa + kABytes + h * 8192, n0 + 64 * h, kg * 64);
      } else {
        ptx::tma_load_2d(&tmB, &full[s], sa + kABytes, kg * 64, n0);
      }
      ++issued;
    }
    // never leave with copies in flight into this CTA's shared memory
    for (int i = (issued > p.stages ? issued - p.stages : 0); i < issued; ++i)
      ptx::mbar_wait(&full[i % p.stages], (i / p.stages) & 1, kTimeoutCycles, nullptr);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------ MMA issuer
    const uint32_t idesc = ptx::idesc_bf16(128, p.bn, p.a_mn, p.b_mn);
    for (int i = 0; i < kn; ++i) {
      const int s = i % p.stages;
      const uint32_t ph = (i / p.stages) & 1;
      if (!ptx::mbar_wait(&full[s], ph, kTimeoutCycles, abort_flag)) break;
      ptx::tc_fence_after();
      const uint32_t a_addr = ptx::smem_u32(smem + s * p.stage_bytes);
      const uint32_t b_addr = a_addr + kABytes;
      // descriptors stepped by their 16-byte address field (see gemm_tc2.cu)
      const uint64_t a0 = p.a_mn ? ptx::sw128_desc(a_addr, 8192, 1024)
                                 : ptx::sw128_desc(a_addr, 16, 1024);
      const uint64_t b0 = p.b_mn ? ptx::sw128_desc(b_addr, 8192, 1024)
                                 : ptx::sw128_desc(b_addr, 16, 1024);
      const uint64_t a_step = p.a_mn ? (2048 >> 4) : (32 >> 4);
      const uint64_t b_step = p.b_mn ? (2048 >> 4) : (32 >> 4);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        ptx::umma_bf16(tmem, a0 + a_step * ks, b0 + b_step * ks, idesc, (i | ks) != 0 ? 1u : 0u);
      ptx::umma_commit(&empty[s]);
    }
    ptx::umma_commit(accum);
    ptx::mbar_wait(accum, 0, kTimeoutCycles, nullptr);  // MMAs done before TMEM is freed
  }

  // -------------------------------------------- partial tile -> shared memory
  if (warp >= 2) {
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31 (warps 2..5 -> 2, 3, 0, 1)
    const int row = 32 * quarter + lane;
    bool ok = kn > 0 && ptx::mbar_wait(accum, 0, kTimeoutCycles, abort_flag);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (ok) ptx::tc_fence_after();
    for (int c = 0; c < p.bn / 16; ++c) {
      uint32_t r[16];
      if (ok) {
        ptx::tmem_ld_x16(tmem + (static_cast<uint32_t>(32 * quarter) << 16) + 16 * c, r);
        ptx::tmem_ld_wait();
      }
      float* dst = red + static_cast<size_t>(row) * p.red_ld + 16 * c;
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(dst + j) =
            ok ? make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                             __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]))
               : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
  }
  ptx::tc_fence_before();
  // the role branches above leave warps 0 and 1 diverged: reconverge every
  // warp before the aligned cluster barrier; then every partial tile of the
  // cluster is in shared memory
  __syncthreads();
  ptx::cluster_sync();

  // --------------------------- sum over the splits, in order, and store
  if (warp >= 2) {
    const ReduceArgs& o = p.o;
    // this CTA's slice of the 128 rows: ceil(128 / S) rows, the last slice shorter
    const int slice = (128 + static_cast<int>(S) - 1) / static_cast<int>(S);
    const int i0 = static_cast<int>(z) * slice;
    const int rows_per = max(0, min(slice, 128 - i0));
    const int cols = o.cols;
    const int tid = threadIdx.x - 64;
    uint32_t peer[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      peer[q] = (q < static_cast<int>(S)) ? ptx::cluster_addr(red, static_cast<uint32_t>(q)) : 0u;
    // four consecutive columns per thread and step (cols, lo and the row
    // stride are multiples of 4 floats: 16-byte loads)
    const int cols4 = cols >> 2;
    for (int e = tid; e < rows_per * cols4; e += 128) {
      const int il = i0 + e / cols4;
      const int j = 4 * (e - (e / cols4) * cols4);
      const int64_t gi = static_cast<int64_t>(m0) + il;
      if (gi >= p.m_rows) continue;
      const uint32_t off = static_cast<uint32_t>((il * p.red_ld + (j - n0)) * 4);
      float4 h[8], l[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        h[q] = (q < static_cast<int>(S)) ? ld_dsmem_f32x4(peer[q] + off)
                                         : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        l[q] = (o.lo && q < static_cast<int>(S)) ? ld_dsmem_f32x4(peer[q] + off + 4u * o.lo)
                                                 : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      }
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q < static_cast<int>(S)) {
          v[0] += h[q].x;
          v[1] += h[q].y;
          v[2] += h[q].z;
          v[3] += h[q].w;
          if (o.lo) {
            v[0] += l[q].x;
            v[1] += l[q].y;
            v[2] += l[q].z;
            v[3] += l[q].w;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float x = v[u];
        if (o.seg && __ldg(o.seg + gi) != (j + u) / o.seg_cols) x = 0.0f;
        tc::reduce_store(x, gi, j + u, o.o1, o.ld1, o.trans1 ? 1 : 0, o.a1, o.acc1 ? 1 : 0,
                         static_cast<__nv_bfloat16*>(o.o2), o.ld2, o.a2, o.o2_lo,
                         static_cast<__nv_bfloat16*>(o.o3), o.ld3, o.a3, o.o3_lo);
      }
    }
    if (o.o2 && o.o2_pad && (cols % 8) == 0 && (o.o2_lo % 8) == 0 && (o.ld2 % 8) == 0 &&
        (reinterpret_cast<uintptr_t>(o.o2) & 15) == 0) {
      // the padding columns of o2 of this CTA's rows, [cols, o2_lo) and
      // [o2_lo + cols, 2 o2_lo), in 16-byte stores: both runs start and end
      // on 8-column boundaries
      const int chunks = (o.o2_lo - cols) / 8;  // per run
      uint4* o2 = static_cast<uint4*>(o.o2);
      const int64_t ld16 = o.ld2 / 8;
      for (int e = tid; e < rows_per * 2 * chunks; e += 128) {
        const int il = i0 + e / (2 * chunks);
        const int c = e - (e / (2 * chunks)) * 2 * chunks;
        const int64_t gi = static_cast<int64_t>(m0) + il;
        if (gi >= p.m_rows) continue;
        o2[gi * ld16 + ((c < chunks) ? cols / 8 + c : (o.o2_lo + cols) / 8 + (c - chunks))] =
            make_uint4(0u, 0u, 0u, 0u);
      }
    } else if (o.o2 && o.o2_pad) {
      // the same, one column at a time
      const int pad = o.o2_lo - cols;
      __nv_bfloat16* o2 = static_cast<__nv_bfloat16*>(o.o2);
      for (int e = tid; e < rows_per * 2 * pad; e += 128) {
        const int il = i0 + e / (2 * pad);
        const int c = e - (e / (2 * pad)) * 2 * pad;
        const int64_t gi = static_cast<int64_t>(m0) + il;
        if (gi >= p.m_rows) continue;
        o2[gi * o.ld2 + ((c < pad) ? cols + c : o.o2_lo + cols + (c - pad))] =
            __float2bfloat16_rn(0.0f);
      }
    }
  }
  // no CTA leaves (or frees TMEM) while the others may still read its tile
  __syncthreads();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, p.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort_flag) report(p.st, QLORA_ERR_DEVICE_TIMEOUT, 130u);
}

int pow2_at_least(int v) {
  int c = 32;
  while (c < v) c <<= 1;
  return c;
}

}  // namespace

bool tc_rank_eligible(int32_t n_cols, int32_t cols, int32_t lo) {
  return n_cols >= 16 && n_cols <= 256 && n_cols % 16 == 0 && cols % 4 == 0 && lo % 4 == 0 &&
         cols + lo <= n_cols;
}

int tc_rank_splits(int64_t m_tiles, int64_t k_tiles) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // up to two CTAs per SM in one wave, at least 8 k-tiles per split, at most
  // 8 (a cluster holds the splits); the launch steps down from there while
  // the clusters would not all be resident (large clusters run about one CTA
  // per SM, small ones two)
  int64_t s = m_tiles > 0 ? (2 * static_cast<int64_t>(sms)) / m_tiles : 1;
  if (s > 8) s = 8;
  if (s > k_tiles / 8) s = k_tiles / 8;
  if (s < 1) s = 1;
  return static_cast<int>(s);
}

qlora_status tc_rank_gemm(const void* A, bool a_mn, int64_t m_rows, int64_t kdim, int64_t ld_a,
                          const void* B, bool b_mn, int64_t ld_b, int32_t b_rows, int32_t n_cols,
                          const ReduceArgs& out, DeviceStatus* st, cudaStream_t s) {
  if (!tc_rank_eligible(n_cols, out.cols, out.lo) || m_rows < 1 || kdim < 1)
    return QLORA_ERR_UNSUPPORTED;
  // an MN-major B is read in 64-column boxes: n_cols a multiple of 64
  if (b_mn && n_cols % 64 != 0) return QLORA_ERR_UNSUPPORTED;
  CUtensorMap ma, mb;
  bool ok = a_mn ? make_map(&ma, A, true, m_rows, kdim, ld_a, 64, 64, true)
                 : make_map(&ma, A, true, kdim, m_rows, ld_a, 64, 128, true);
  ok = ok && (b_mn ? make_map(&mb, B, true, b_rows, kdim, ld_b, 64, 64, true)
                   : make_map(&mb, B, true, kdim, b_rows, ld_b, 64, n_cols, true));
  if (!ok) return QLORA_ERR_CUDA;
  RankArgs p{};
  p.m_rows = static_cast<int32_t>(m_rows);
  p.kt_total = static_cast<int32_t>(ceil_div(kdim, 64));
  const int64_t m_tiles = ceil_div(m_rows, 128);
  int splits = tc_rank_splits(m_tiles, p.kt_total);
  p.k_tiles = static_cast<int32_t>(ceil_div(p.kt_total, splits));
  p.a_mn = a_mn ? 1 : 0;
  p.b_mn = b_mn ? 1 : 0;
  p.bn = n_cols;
  p.b_bytes = n_cols * 128;
  p.stage_bytes = kABytes + p.b_bytes;
  p.stages = kSmemBudget / p.stage_bytes;
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 3) p.stages = 3;  // wide partial tiles: one CTA per SM
  p.tmem_cols = pow2_at_least(n_cols);
  p.red_ld = n_cols + 4;
  p.o = out;
  p.st = st;
  const size_t red_bytes = static_cast<size_t>(128) * p.red_ld * sizeof(float);
  const size_t stage_area = static_cast<size_t>(p.stages) * p.stage_bytes;
  const size_t smem = 1024 + (stage_area > red_bytes ? stage_area : red_bytes) + 256;
  if (smem > 200 * 1024) return QLORA_ERR_UNSUPPORTED;
  // the limit is raised once to what any launch of this kernel may use, so
  // that the occupancy query below prices this launch's own size
  const qlora_status cs = ensure_smem(reinterpret_cast<const void*>(rank_gemm_kernel), 200 * 1024);
  if (cs != QLORA_OK) return cs;
  // the largest shared-memory carveout, so that two CTAs fit on an SM (the
  // driver would otherwise size the carveout for one) - once per device
  constexpr int kCarveoutTag = 2;
  int carve = 0;
  if (!cached_value(reinterpret_cast<const void*>(rank_gemm_kernel), kCarveoutTag, &carve)) {
    if (cudaFuncSetAttribute(reinterpret_cast<const void*>(rank_gemm_kernel),
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess) {
      (void)cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    store_value(reinterpret_cast<const void*>(rank_gemm_kernel), kCarveoutTag, 1);
  }
  if (m_tiles > 65535) return QLORA_ERR_SHAPE;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // fewer splits while the clusters would not all be resident at once
  while (splits > 1) {
    attr[0].val.clusterDim.z = static_cast<unsigned>(splits);
    cfg.gridDim = dim3(1u, static_cast<unsigned>(m_tiles), static_cast<unsigned>(splits));
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, rank_gemm_kernel, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      break;
    }
    if (static_cast<int64_t>(resident) >= m_tiles) break;
    splits -= 1;
  }
  p.k_tiles = static_cast<int32_t>(ceil_div(p.kt_total, splits));
  cfg.gridDim = dim3(1u, static_cast<unsigned>(m_tiles), static_cast<unsigned>(splits));
  attr[0].val.clusterDim.z = static_cast<unsigned>(splits);
  count_launch();
  timing_mark(QLORA_KERNEL_LORA_GEMM, s, true);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, rank_gemm_kernel, ma, mb, p);
  timing_mark(QLORA_KERNEL_LORA_GEMM, s, false);
  if (e != cudaSuccess) return QLORA_ERR_CUDA;
  return after_launch("rank_gemm", s);
}

}  // namespace qlora

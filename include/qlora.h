/*
 * qlora.h - C ABI of libqlora.so: a QLoRA linear layer on one B200 (sm_100a).
 *
 * The frozen base weight W (d_out x d_in) is stored block-wise in 4 bits:
 * absmax per block of `blocksize` consecutive weights, the nearest of 16
 * levels (NF4 or the uniform grid), two indices per byte, and the fp32 block
 * scales quantised again to int8 ("double quantisation").  The layer adds a
 * trainable bf16 LoRA branch:
 *
 *     forward   Y  = X W^T + s (X A^T) B^T,            s = alpha / r
 *     backward  dX = dY W + s (dY B) A,  dB = s dY^T (X A^T),  dA = s (dY B)^T X
 *
 * with no gradient for W.  Sources (page title, section):
 *   - quantise / store:  "QLoRA技术从入门到精通", 3(1) 基座模型初始化量化;
 *                         "LoRA 与 QLoRA：用一块 GPU 微调大模型", 量化 (分块缩放, NF4, 存储和计算)
 *   - dequantise:         "QLoRA技术从入门到精通", 3(2) 前向传播 (X_deq = grid[idx] * scale)
 *   - forward:            "LoRA 与 QLoRA：把大模型微调拆成可负担的工程", 2 (h = W x + (α/r) B A x)
 *   - backward:           "QLoRA技术从入门到精通", 3(3) 反向传播; same page as forward, 6
 *
 * Conventions for every call:
 *   - All matrices are dense row-major.  X: M x d_in, Y and dY: M x d_out,
 *     A: r x d_in, B: d_out x r, dX: M x d_in (all bf16); U: M x r,
 *     dA: r x d_in, dB: d_out x r (all fp32).
 *   - Pointers named "device" are CUDA device pointers, 16-byte aligned.  The
 *     caller owns and allocates every buffer (sizes from the *_sizes and
 *     *_workspace queries); the library never allocates, frees or keeps a
 *     pointer after a call returns - except qlora_paged_alloc and
 *     qlora_paged_free, whose whole job is that.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous: they return after enqueueing work.
 *     The backward pass of larger batches forks its dA/dB work onto a second,
 *     library-owned stream (one per host thread and device, created on first
 *     use and kept until the process exits) and joins it back before it
 *     returns, so the call stays ordered on `stream` and can be captured in a
 *     CUDA graph.
 *   - Argument errors are found on the host and returned before any launch.
 *     Errors found on the device (a non-finite weight, a bounded wait that
 *     gave up) are written to a status word at the start of the workspace;
 *     qlora_check() synchronises the stream and returns it.  A workspace must
 *     be zero-filled before its first use; the library leaves its status word
 *     zero unless it reports an error (qlora_check clears it again).
 *   - No call exits, aborts or traps.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = 1,           /* a required pointer is NULL */
  QLORA_ERR_ALIGN = 2,          /* a device pointer is not 16-byte aligned */
  QLORA_ERR_SHAPE = 3,          /* a size is out of range or sizes disagree */
  QLORA_ERR_UNSUPPORTED = 4,    /* valid request this build does not implement */
  QLORA_ERR_NONFINITE = 5,      /* quantise met a NaN or an infinity (device status) */
  QLORA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait gave up (device status) */
  QLORA_ERR_CUDA = 7,           /* a CUDA runtime call or launch failed */
  QLORA_ERR_WORKSPACE = 8       /* workspace missing or smaller than the query said */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* Level tables.  NF4: medians of equal-probability intervals of N(0,1),
 * 7 below zero, an exact 0, 8 above, each half scaled so the ends are -1 and
 * +1 ("QLoRA技术从入门到精通", 2(3)2) NF4非均匀格点).  UNIFORM: -1 + k*2/15
 * ("QLoRA 量化微调", 7.1). */
typedef enum { QLORA_TABLE_NF4 = 0, QLORA_TABLE_UNIFORM = 1 } qlora_table;

/* A quantised weight.  Block b covers flattened row-major elements
 * [b*blocksize, (b+1)*blocksize); group g covers blocks [g*dq_blocksize,
 * (g+1)*dq_blocksize).  n = rows*cols, nb = ceil(n/blocksize),
 * ng = ceil(nb/dq_blocksize).
 *   codes        device, ceil(n/2) bytes: element 2j in the low nibble of
 *                byte j, element 2j+1 in the high nibble
 *   scale_codes  device, nb int8 (dq_blocksize > 0), else unused (may be NULL)
 *   factors      device fp32: ng group factors absmax_g/127 (dq_blocksize > 0),
 *                or the nb block absmax values themselves (dq_blocksize = 0)
 *   mean         device, 1 fp32: mean of the block scales (dq_blocksize > 0),
 *                else unused (may be NULL)
 * Block b dequantises with s_b = fp32(fp32(scale_codes[b] * factors[b/dq]) + mean)
 * (or factors[b] without double quantisation) and w = fp32(level[idx] * s_b). */
typedef struct {
  int64_t rows;          /* d_out */
  int64_t cols;          /* d_in */
  int32_t blocksize;     /* 64, 128, 256, 512 or 1024 */
  int32_t dq_blocksize;  /* 0 (no double quantisation), 64, 128, 256, 512 or 1024 */
  int32_t table;         /* qlora_table */
  int32_t reserved;      /* set to 0 */
  uint8_t* codes;
  int8_t* scale_codes;
  float* factors;
  float* mean;
} qlora_nf4;

/* Human-readable name of a status code (static storage). */
const char* qlora_status_string(qlora_status s);

/* The library's own 16 fp32 levels of `table` (host memory, ascending). */
qlora_status qlora_levels(int32_t table, float levels_out[16]);

/* Byte sizes of the arrays of a quantised rows x cols weight and of the
 * workspace qlora_quantize needs.  Any output pointer may be NULL.
 * QLORA_ERR_SHAPE for rows, cols < 1 or more than 2^36 elements;
 * QLORA_ERR_UNSUPPORTED for a blocksize or dq_blocksize not listed above. */
qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int32_t blocksize,
                             int32_t dq_blocksize, size_t* codes_bytes,
                             size_t* scale_codes_bytes, size_t* factors_bytes,
                             size_t* mean_bytes, size_t* workspace_bytes);

/* Quantise W (device, rows*cols values of w_dtype, row-major) into the arrays
 * of *q (host struct holding device pointers; rows, cols, blocksize,
 * dq_blocksize and table describe the request).  Steps: block absmax, divide
 * (IEEE fp32), nearest level (exact; a value halfway between two levels takes
 * the lower index), pack; then, with double quantisation, the mean of the
 * block scales on a fixed-point grid of 2^(E-32) (E = binary exponent of the
 * largest scale; order-independent), int8 codes of scale - mean per group
 * with factor absmax/127, round half to even.  A non-finite weight sets
 * QLORA_ERR_NONFINITE in the workspace status (outputs then undefined).
 * workspace: device, >= workspace_bytes from qlora_nf4_sizes. */
qlora_status qlora_quantize(const void* W, int32_t w_dtype, const qlora_nf4* q,
                            void* workspace, size_t workspace_bytes, void* stream);

/* qlora_quantize without a workspace argument, for callers that cannot
 * allocate one: code whose device memory belongs to a pool that has already
 * reserved the GPU, and loops that cannot pay the device-wide synchronisation
 * of cudaMalloc/cudaFree.  The pages have no counterpart to this call; it is a
 * library convenience.  Same inputs, outputs and results as qlora_quantize.
 * The reduction workspace is a fixed array in the library's own device memory
 * (one copy per GPU that loads the library, 4 MiB + 512 B, kept until exit).
 * With double quantisation it holds one fp32 per block: at most 2^20 blocks
 * (64 Mi weights at blocksize 64), larger tensors return QLORA_ERR_WORKSPACE
 * before any work is enqueued.  Without double quantisation (dq_blocksize 0)
 * only its 512-byte header is used and there is no such limit.  Argument
 * checks and their errors are those of qlora_quantize.  All calls on a
 * device share the array: calls whose work overlaps on the GPU race; calls on
 * one stream are safe.  Each call clears the words that must start at zero
 * (status, maximum, sum) and rewrites the per-block values before reading
 * them, so nothing carries over from an earlier call.  status_out
 * (device, 4 bytes, may be NULL) receives the device status when the work
 * completes: 0, or QLORA_ERR_NONFINITE for a NaN or infinite weight.  The
 * first call on a device looks up the array (cudaGetSymbolAddress on the
 * current device); make that first call before any stream capture. */
qlora_status qlora_quantize_noalloc(const void* W, int32_t w_dtype, const qlora_nf4* q,
                                    uint32_t* status_out, void* stream);

/* Dequantise *q into W_out (device, rows*cols values of out_dtype):
 * fp32 out is w = fp32(level[idx] * s_b) bit for bit; bf16 out is that value
 * rounded to nearest even.  Needs no workspace. */
qlora_status qlora_dequantize(const qlora_nf4* q, void* W_out, int32_t out_dtype,
                              void* stream);

/* Workspace bytes for qlora_linear_fwd / qlora_linear_bwd at these sizes
 * (N = d_out, K = d_in).  Either output may be NULL. */
qlora_status qlora_linear_workspace(int64_t M, int64_t N, int64_t K, int32_t r,
                                    size_t* fwd_bytes, size_t* bwd_bytes);

/* Forward pass Y = X W^T + s (X A^T) B^T with W dequantised on the fly (a
 * full-precision W is never written to memory).  Requirements: W->cols a
 * multiple of W->blocksize, so that no block straddles two rows (else
 * QLORA_ERR_UNSUPPORTED; every blocksize, double-quantisation setting and
 * table of qlora_quantize is accepted), 1 <= r <= 256,
 * M >= 0 (M = 0 is a no-op).  Device buffers: A (r x K bf16), B (N x r bf16),
 * X (M x K bf16), Y (M x N bf16, written), U_save (M x r fp32, written with
 * X A^T; may be NULL), workspace (>= fwd_bytes). */
qlora_status qlora_linear_fwd(const qlora_nf4* W, const void* A, const void* B,
                              int32_t r, float alpha, const void* X, int64_t M,
                              void* Y, float* U_save, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Backward pass: dX = dY W + s V A, dB = s dY^T U, dA = s V^T X, V = dY B.
 * W receives no gradient.  U (M x r fp32, from the forward) may be NULL: it is
 * then recomputed as X A^T.  dX (M x K bf16) may be NULL to skip it.  dA
 * (r x K fp32) and dB (N x r fp32) are overwritten, or added to when
 * accumulate != 0.  Same requirements as the forward; workspace >= bwd_bytes. */
qlora_status qlora_linear_bwd(const qlora_nf4* W, const void* A, const void* B,
                              int32_t r, float alpha, const void* X, const float* U,
                              const void* dY, int64_t M, void* dX, float* dA,
                              float* dB, int32_t accumulate, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Several adapters over one quantised base ("LoRA 与 QLoRA：把大模型微调拆成
 * 可负担的工程", section 3: one base, one small adapter per task, switched per
 * request).  n_adapters adapters of rank r share W; token m uses adapter
 * adapter[m] (device int32; an id outside [0, n_adapters), e.g. -1, selects
 * none: that token gets the base output only).  With a = adapter[m]:
 *     Y[m]  = X[m] W^T + s (X[m] A_a^T) B_a^T,           s = alpha / r
 *     dX[m] = dY[m] W + s (dY[m] B_a) A_a
 *     dA_a  = s sum_{m: a} (dY[m] B_a)^T X[m],  dB_a = s sum_{m: a} dY[m]^T (X[m] A_a^T)
 * The adapters are stacked along the rank: A is (n_adapters r) x K bf16 with
 * A_a in rows [a r, (a+1) r); B is N x (n_adapters r) bf16 with B_a in
 * columns [a r, (a+1) r); dA and dB (fp32) have the same layouts and U_save /
 * U are M x (n_adapters r) fp32 holding X[m] A_a^T in the token's own
 * columns and zeros elsewhere.  Workspace sizes: qlora_linear_workspace with
 * rank n_adapters * r.  Requirements as qlora_linear_fwd / _bwd, plus
 * n_adapters >= 1, n_adapters * r <= 256, and N and n_adapters * r multiples
 * of 8 (else QLORA_ERR_UNSUPPORTED); `adapter` 4-byte aligned, NULL only
 * when M = 0. */
qlora_status qlora_linear_fwd_multi(const qlora_nf4* W, const void* A, const void* B,
                                    int32_t n_adapters, int32_t r, float alpha,
                                    const int32_t* adapter, const void* X, int64_t M, void* Y,
                                    float* U_save, void* workspace, size_t workspace_bytes,
                                    void* stream);
qlora_status qlora_linear_bwd_multi(const qlora_nf4* W, const void* A, const void* B,
                                    int32_t n_adapters, int32_t r, float alpha,
                                    const int32_t* adapter, const void* X, const float* U,
                                    const void* dY, int64_t M, void* dX, float* dA, float* dB,
                                    int32_t accumulate, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Merge a trained adapter into a restored 16-bit weight ("LoRA 与 QLoRA：把
 * 大模型微调拆成可负担的工程", section 3: after training B A has the shape of
 * W and is added to it; 4-bit storage cannot take the update):
 *   W_out[n][k] = bf16( fp32(level[idx] * s_hat) + (alpha / r) sum_j B[n][j] A[j][k] )
 * with the rank-r sum accumulated in fp32 and one final rounding to bf16.
 * Device buffers: A (r x K bf16), B (N x r bf16), W_out (N x K bf16,
 * written; 16-byte aligned).  Requirements as for qlora_linear_fwd (W->cols a
 * multiple of W->blocksize, 1 <= r <= 256); errors QLORA_ERR_NULL, _ALIGN,
 * _SHAPE, _UNSUPPORTED, _CUDA.  Stream-ordered; allocates nothing.  The
 * result can be quantised again with qlora_quantize.  For r a multiple of 8 the
 * rank-r product runs on the tensor cores; its device-side waits are bounded,
 * and as the call takes no status word, a wait that gives up (it does not in
 * correct operation) leaves NaN in its 128 x 128 tile of W_out. */
qlora_status qlora_merge(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                         float alpha, void* W_out, void* stream);

/* The same update on a dense bf16 weight: W_out = bf16(W_in + (alpha / r) B A),
 * accumulated in fp32 and rounded once.  With -alpha it takes a merged
 * adapter out again (unmerge), or, applied twice, moves a merged weight from
 * one adapter to another.  Device buffers: W_in and W_out (rows x cols bf16,
 * row-major; W_out may be W_in: in place), A (r x cols bf16), B (rows x r
 * bf16), all 16-byte aligned.  Errors: QLORA_ERR_NULL, _ALIGN, _SHAPE (rows or
 * cols < 1, cols % 8 != 0, r outside [1, 256], rows > 2^22), _CUDA.  With r a
 * multiple of 8 and cols a multiple of 64 it takes the tensor-core form, with
 * the same NaN-tile behaviour as qlora_merge on a wait that gives up. */
qlora_status qlora_merge_dense(const void* W_in, int64_t rows, int64_t cols, const void* A,
                               const void* B, int32_t r, float alpha, void* W_out, void* stream);

/* One AdamW step (Adam with decoupled weight decay) over n adapter
 * parameters - the optimiser that updates only A and B ("QLoRA技术从入门到精
 * 通", section 3(3)).  For step >= 1, per element, g' = grad_scale * grad:
 *   m = beta1 m + (1 - beta1) g',  v = beta2 v + (1 - beta2) g'^2,
 *   param -= lr (m / (1 - beta1^step) / (sqrt(v / (1 - beta2^step)) + eps)
 *                + weight_decay param),
 * then param_bf16 = bf16(param) when param_bf16 is not NULL.  Device buffers
 * (any device-accessible memory, managed memory included): param, grad, m, v
 * (n fp32 each; param, m, v updated in place), param_bf16 (n bf16, written).
 * All 16-byte aligned.  The flat dA/dB buffer of a data-parallel step can be
 * passed whole.  Errors: QLORA_ERR_NULL, _ALIGN, _SHAPE (n < 0, step < 1),
 * _UNSUPPORTED (beta outside [0, 1), eps <= 0, lr < 0), _CUDA. */
qlora_status qlora_adamw(float* param, void* param_bf16, const float* grad, float* m, float* v,
                         int64_t n, int32_t step, float lr, float beta1, float beta2, float eps,
                         float weight_decay, float grad_scale, void* stream);

/* The general form of the two calls above, with LoRA dropout on the adapter
 * input ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section 4.3,
 * lora_dropout; "QLoRA 量化微调", training recipe).  The adapter branch reads
 * X~ = D (.) X / (1 - p) for a keep mask D that the caller draws, the base
 * branch reads X:
 *     Y  = X W^T + s U B^T,               U = X~ A^T   (U_save / U hold this U)
 *     dX = dY W + s D (.) (V A) / (1 - p),  dA = s V^T X~,  dB = s dY^T U
 * Fields of qlora_adapter_opts:
 *   n_adapters, adapter  as for the *_multi calls (n_adapters = 1 and
 *                        adapter = NULL: one adapter for every token);
 *   dropout_p            p in [0, 1); keep_mask = NULL turns dropout off;
 *   keep_mask            device, M x K/8 bytes: bit (k % 8) of byte
 *                        m K/8 + k/8 set = keep X[m][k];
 *   x_drop               device, M x K bf16, 16-byte aligned: written by the
 *                        forward with D (.) X (kept values, unscaled), read
 *                        by the backward (pass the same buffer and mask).
 * Dropout needs the same conditions as several adapters (N and the stacked
 * rank multiples of 8, else QLORA_ERR_UNSUPPORTED).  Errors as the *_multi
 * calls, plus QLORA_ERR_UNSUPPORTED for p outside [0, 1) and QLORA_ERR_NULL
 * for a mask without x_drop. */
typedef struct {
  int32_t n_adapters;
  int32_t reserved;
  const int32_t* adapter;
  float dropout_p;
  int32_t reserved2;
  const uint8_t* keep_mask;
  void* x_drop;
} qlora_adapter_opts;
qlora_status qlora_linear_fwd_ex(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                                 float alpha, const qlora_adapter_opts* opts, const void* X,
                                 int64_t M, void* Y, float* U_save, void* workspace,
                                 size_t workspace_bytes, void* stream);
qlora_status qlora_linear_bwd_ex(const qlora_nf4* W, const void* A, const void* B, int32_t r,
                                 float alpha, const qlora_adapter_opts* opts, const void* X,
                                 const float* U, const void* dY, int64_t M, void* dX, float* dA,
                                 float* dB, int32_t accumulate, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Paged optimiser states.  The optimiser moments can live in CUDA managed
 * (unified) memory, which the driver migrates between host and device pages
 * on demand, so that they need not stay in HBM ("LoRA 与 QLoRA：把大模型微调
 * 拆成可负担的工程", section 6.3; "QLoRA 量化微调", paged optimisers).
 *   qlora_paged_alloc:    `bytes` of managed memory (global attachment,
 *                         256-byte aligned, zero-filled) into *ptr.
 *   qlora_paged_prefetch: enqueue on `stream` a migration of [ptr, ptr+bytes)
 *                         to the current device (to_device != 0) or to host
 *                         memory (to_device == 0).  Optional: pages that are
 *                         not resident move on first touch anyway.
 *   qlora_paged_free:     release a pointer from qlora_paged_alloc (waits for
 *                         the device, as cudaFree does).  NULL is a no-op.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_SHAPE (bytes == 0), QLORA_ERR_CUDA
 * (allocation failed or the device cannot prefetch managed memory). */
qlora_status qlora_paged_alloc(size_t bytes, void** ptr);
qlora_status qlora_paged_prefetch(void* ptr, size_t bytes, int32_t to_device, void* stream);
qlora_status qlora_paged_free(void* ptr);

/* Diagnostic of the failure path: one CTA waits, with the library's bounded
 * wait, on an mbarrier that nothing completes, gives up after `limit_cycles`
 * clock cycles (1 .. 2^32) and writes QLORA_ERR_DEVICE_TIMEOUT to the status
 * word of `workspace` (at least 256 bytes), as the library's kernels do when
 * one of their waits runs out.  qlora_check then returns that code and clears
 * it; the context stays usable.  Errors: QLORA_ERR_NULL, _SHAPE, _ALIGN, _CUDA. */
qlora_status qlora_selftest_timeout(int64_t limit_cycles, void* workspace, void* stream);

/* Synchronise `stream`, then return and clear the device status word that
 * calls given this workspace wrote (QLORA_OK if none). */
qlora_status qlora_check(void* workspace, void* stream);

/* Number of kernels this library has enqueued since it was loaded (all
 * threads, all calls; memsets not counted).  Host only, never fails. */
uint64_t qlora_launch_count(void);

/* Kernel timing (measurement aid).  Between qlora_timing_begin and
 * qlora_timing_end the library records a pair of CUDA events on the launching
 * stream around every launch of the kernel kinds in `kind_mask` (bit k set =
 * kind k), for at most `max_launches` launches in all (later ones are not
 * timed).  qlora_timing_end waits for the recorded events, writes the summed
 * device time in milliseconds and the launch count of each kind to
 * ms[QLORA_KERNEL_KINDS] and launches[QLORA_KERNEL_KINDS] (either may be
 * NULL), and releases the events.  The events are library-owned host
 * objects; no device memory is allocated.  Calls captured into a CUDA graph
 * while timing is on record their events as graph nodes: qlora_timing_end,
 * after the graph has run, reads the times of that run.  Launches from several host
 * threads at once are not supported while timing is on.
 * Errors: QLORA_ERR_SHAPE for max_launches outside [1, 65536],
 * QLORA_ERR_UNSUPPORTED for begin while timing is already on or end while it
 * is off, QLORA_ERR_CUDA if an event cannot be created or read. */
typedef enum {
  QLORA_KERNEL_QUANTIZE = 0,     /* block absmax, nearest level, nibble packing */
  QLORA_KERNEL_FUSED_FWD = 1,    /* fused dequant GEMM of the forward pass */
  QLORA_KERNEL_FUSED_DGRAD = 2,  /* fused dequant GEMM of dX */
  QLORA_KERNEL_LORA_GEMM = 3,    /* tensor-core rank-r GEMMs (U, V, dA, dB) */
  QLORA_KERNEL_MERGE = 4,        /* qlora_merge */
  QLORA_KERNEL_KINDS = 5
} qlora_kernel_kind;
qlora_status qlora_timing_begin(uint32_t kind_mask, int32_t max_launches);
qlora_status qlora_timing_end(float* ms, int32_t* launches);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H */

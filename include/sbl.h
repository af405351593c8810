/*
 * sbl.h -- C ABI of the Sparse-BitLinear operator for NVIDIA B200 (sm_100a).
 *
 * Sparse-BitLinear is the layer of Sparse-BitNet: per step it recomputes an
 * N:M magnitude mask on the bf16 master weight W, quantises W to ternary
 * with an absmean scale, masks the ternary weight, quantises activations
 * per token to int8, multiplies on int8 tensor cores, and back-propagates
 * with a "Dual" straight-through estimator that gives masked weights their
 * full gradient.
 *
 * Pages cited below (by title and section):
 *   [summary]   "Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏", the
 *               structured summary of arXiv 2603.05168: 前置知识 (1.58-bit
 *               BitNet 量化; 半结构化 N:M 稀疏; STE), 核心方法,
 *               方法步骤详情 (Algorithm 1), 实验结果 (Table 3).
 *   [explainer] "什麼是 Sparse-BitNet？核心概念一次搞懂": 1.58 位元量化的技術原理;
 *               N:M 半結構化稀疏性的運作機制.
 *   [article]   "突破性发现：极低位量化与稀疏化的完美协同": 7.1 推理优化技巧.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (CUDA global memory) owned by
 *     the caller; the library never frees or retains them.  The library
 *     allocates no device memory except fixed-size static state created on
 *     first use (tensor-map encoder entry point, attribute settings).
 *   - Matrices are row-major with the last index contiguous.  "bf16" means
 *     IEEE bfloat16 bit patterns (uint16 per element).
 *   - Every pointer must be 16-byte aligned.  d_in must be a multiple of 16
 *     and of M; d_out must be a multiple of 8.  T (tokens) may be any value
 *     >= 0; with T = 0 no token row is written (sbl_backward's dW, a sum
 *     over tokens, is then zero-filled, or left as it is when accumulating).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on `stream` and returns; it
 *     never synchronises.
 *   - Return value: SBL_OK, or an error code.  Argument errors are detected on
 *     the host before anything is launched and leave all outputs untouched.
 *     Launch failures return SBL_ERR_CUDA.  Errors found by a kernel while it
 *     runs (a bounded wait that expired, a pack input with more than N
 *     nonzeros in a group) are latched in a device word and returned by the
 *     next sbl_check() on that device.
 *   - No call throws or aborts across the ABI.
 *   - The library caches per-device state the first time a device is used
 *     (the address of its device error word, of sbl_mask_quant_noalloc's
 *     scratch array, kernel attributes).  cudaDeviceReset() destroys the
 *     context that state points into: after resetting a device, do not call
 *     this library on that device again in the same process.
 */
#ifndef SBL_H_
#define SBL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SBL_OK = 0,
  SBL_ERR_INVALID_ARG = 1, /* null pointer, N/M out of range, bad flag       */
  SBL_ERR_SHAPE = 2,       /* d_in % 16, d_in % M, d_out % 8, negative sizes */
  SBL_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                */
  SBL_ERR_UNSUPPORTED = 4, /* device is not sm_100, or an unsupported N:M     */
  SBL_ERR_WORKSPACE = 5,   /* workspace (or packed buffer) too small          */
  SBL_ERR_TIMEOUT = 6,     /* a kernel's bounded wait expired (latched)       */
  SBL_ERR_CUDA = 7,        /* a CUDA runtime call failed                      */
  SBL_ERR_DEVICE_CHECK = 8 /* a kernel rejected its input data (latched)      */
} sbl_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* sbl_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int sbl_version(void);

/* Select the tensor-core kernel used by sbl_forward and sbl_backward for
 * all later calls in this process: 0 = pairs of CTAs computing 256 x 256
 * tiles with tcgen05 cta_group::2 (the default), 1 = one CTA per 128 x 256
 * tile.  Results are identical (integer forward) or differ only in fp32
 * summation order (backward).  A process-wide setting, not a per-stream
 * one: safe to call from any thread (an atomic store); calls enqueued after
 * it returns use the new kernel. */
sbl_status sbl_set_gemm_variant(int variant);

/* Select the decode GEMV kernel used by sbl_gemv_packed(_group) and
 * sbl_gemv_dense2_group for all later calls in this process: 0 = the
 * default: the dense 2-bit layout (and the 8:8 format) through small blocks
 * whose warps fill TMA rings before waiting for the previous kernel, so
 * consecutive launches overlap; the N:M formats through kernel 2; 1 = one
 * block-wide TMA tile ring with producer and epilogue warps, 2 = persistent
 * blocks in which each warp streams its own 16-row slices through its own
 * TMA ring, for every format.  Results
 * are identical (exact int32 sums, the same scaling).  Process-wide and
 * thread-safe like sbl_set_gemm_variant. */
sbl_status sbl_set_gemv_variant(int variant);

/* Failure-detection self-test.  Every spin-wait of this library gives up
 * after a time limit, latches SBL_ERR_TIMEOUT in the device's error word and
 * returns, so a lost signal ends as an error status instead of a hung
 * device.  This call launches one kernel that takes that path on purpose: it
 * waits on a barrier phase that nothing completes for limit_us microseconds
 * (1..1000000), then latches the timeout and exits.  The next sbl_check on
 * this device returns SBL_ERR_TIMEOUT and clears it; the CUDA context stays
 * usable.  The pages have no counterpart: it checks the library's own error
 * path. */
sbl_status sbl_selftest_wait_timeout(unsigned limit_us, void* stream);

/* Synchronise `stream`, then return (and clear) the first error latched by a
 * kernel of this library on the current device since the previous check;
 * SBL_OK if none.  Also reports a pending CUDA error as SBL_ERR_CUDA. */
sbl_status sbl_check(void* stream);

/* ------------------------------------------------------------------------
 * Weight side: mask, absmean scale, ternary quantiser, quant-then-mask.
 * [summary] 前置知识 / 1.58-bit BitNet 量化: gamma = ||W||_1/(d_out*d_in),
 *   W_q = RoundClip(W/(gamma+eps), -1, +1), eps = 1e-5, round half to even;
 * [summary] 半结构化 N:M 稀疏 and 核心方法 (i)-(iii), Algorithm 1 steps
 *   (2), (4), (5): keep the top-N of |W| among each M consecutive weights
 *   along d_in (ties -> lowest index), W_eff = W_q (.) mask.
 *
 *   W          [d_out, d_in] bf16, read only.
 *   N, M       M in {4, 8}, 1 <= N <= M.
 *   W_eff      [d_out, d_in] int8 out, values in {-1, 0, +1}.
 *   W_eff_bf16 optional (NULL): [d_out, d_in] bf16 out, the same values as
 *              exact bf16 (the operand of the backward dX product).
 *   mask_bits  optional (NULL): [d_out, d_in/8] uint8 out; bit p of byte b of
 *              a row is the keep flag of weight 8*b + p of that row.
 *   gamma      1 float out (device): the absmean scale.  It is the exact
 *              sum of |W| rounded once to fp64, divided by d_out*d_in in
 *              fp64, rounded to fp32.
 *   workspace  device scratch of at least sbl_mask_quant_workspace_bytes()
 *              bytes, 256-byte aligned; contents on entry are ignored.
 *              Calls that share a workspace must be ordered on one stream.
 * ---------------------------------------------------------------------- */
size_t sbl_mask_quant_workspace_bytes(int d_out, int d_in);
sbl_status sbl_mask_quant(const void* W, int d_out, int d_in, int N, int M,
                          int8_t* W_eff, void* W_eff_bf16, uint8_t* mask_bits,
                          float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream);

/* The weight step with the pages' mask-source ablation ([gist] 2.2 compares
 * the mask taken from the master weight with one taken from the ternary
 * weight).  flags = 0 is exactly sbl_mask_quant; SBL_MASK_FROM_QUANTISED
 * takes the mask as the top-N of |W_q| per group (ties to the lowest
 * index: the nonzero ternary codes first, then the lowest zero positions).
 * Other arguments as sbl_mask_quant; unknown flag bits give
 * SBL_ERR_INVALID_ARG. */
#define SBL_MASK_FROM_QUANTISED 1u
sbl_status sbl_mask_quant_ex(const void* W, int d_out, int d_in, int N, int M, unsigned flags,
                             int8_t* W_eff, void* W_eff_bf16, uint8_t* mask_bits,
                             float* gamma, void* workspace, size_t workspace_bytes,
                             void* stream);

/* The ablation without the Dual-STE: dW (.) M in place, so masked weights
 * receive no gradient.  [summary] 核心方法 (the Dual-STE keeps their
 * gradient; the ablation removes it).
 *   dW         [d_out, d_in] float, in place (e.g. after sbl_backward).
 *   mask_bits  [d_out, d_in/8] uint8 from sbl_mask_quant(_ex). */
sbl_status sbl_mask_grad(float* dW, const uint8_t* mask_bits, int d_out, int d_in,
                         void* stream);

/* ------------------------------------------------------------------------
 * The optimizer step, fused with the first pass of the next weight step.
 * [summary] Algorithm 1 step (8): AdamW updates the master weight (the
 * pages: beta = (0.9, 0.95), eps = 1e-5, weight decay 0.1, grad clip 1.0,
 * BF16 master weight); step (2) recomputes the mask from the new W on the
 * next step; 独立分析的弱点 names the mask flip rate (Fig. 3b).
 *
 * sbl_grad_sqnorm: *sumsq += sum_i dW_i^2, each square exact in fp64 and
 *   the sum in fp64 (deterministic for a given n: fixed per-block shares,
 *   partials added in block order).  Call once per gradient tensor on one
 *   stream, after zeroing *sumsq, to get the global squared norm that
 *   sbl_adamw_step clips by.
 *   dW       [n] float (any n >= 0; n = 0 adds nothing).
 *   sumsq    1 double (device, 8-byte aligned), read and written.
 *   workspace as sbl_mask_quant (sbl_mask_quant_workspace_bytes, 256-byte
 *            aligned); calls sharing one workspace must be ordered.
 * ---------------------------------------------------------------------- */
sbl_status sbl_grad_sqnorm(const float* dW, size_t n, double* sumsq, void* workspace,
                           size_t workspace_bytes, void* stream);

/* sbl_adamw_step: one AdamW update of W, then the weight step of the new W
 * (exactly what sbl_mask_quant would give for it), in two launches; the
 * update shares its read of W with the exact gamma pass.
 *   Per element, IEEE fp32 operations in this order (no contraction):
 *     g  = dW * c
 *     m' = beta1 * m + (1 - beta1) * g
 *     v' = beta2 * v + ((1 - beta2) * g) * g
 *     w' = w * (1 - lr * wd) - alpha * (m' / (sqrt(v') / b2s + eps))
 *   with alpha = lr / (1 - beta1^t), b2s = sqrt(1 - beta2^t), and every
 *   scalar (beta1, beta2, eps, 1 - beta1, 1 - beta2, alpha, b2s,
 *   1 - lr * wd) computed in fp64 and rounded once to fp32.
 *   c = 1 when grad_sqnorm is NULL, else fl32(min(1, max_norm /
 *   (sqrt(S) + 1e-6))) in fp64 with S = *grad_sqnorm (device, read).
 *   W          [d_out, d_in] bf16, in place: the new W is bf16_rn(w').
 *   W32        optional [d_out, d_in] float master copy, in place.  NULL:
 *              W itself is the master (w = W); else w = W32, W32 := w'.
 *   dW         [d_out, d_in] float in.   m, v  [d_out, d_in] float, in place.
 *   step       t >= 1 (the update's index, for the bias corrections).
 *   lr >= 0, 0 <= beta1, beta2 < 1, eps > 0, weight_decay >= 0,
 *   max_norm > 0 when grad_sqnorm is given.
 *   W_eff, W_eff_bf16, mask_bits, gamma, workspace: outputs and scratch as
 *              sbl_mask_quant, for the new W.
 *   flips      optional 1 unsigned long long (device, 8-byte aligned): adds
 *              the number of positions whose keep flag differs between the
 *              mask in mask_bits on entry (the mask of the old W, from the
 *              previous sbl_mask_quant or sbl_adamw_step) and the mask of
 *              the new W.  Needs mask_bits; NULL skips the count. */
sbl_status sbl_adamw_step(void* W, float* W32, const float* dW, float* m, float* v, int d_out,
                          int d_in, int N, int M, double lr, double beta1, double beta2,
                          double eps, double weight_decay, long long step,
                          const double* grad_sqnorm, double max_norm, int8_t* W_eff,
                          void* W_eff_bf16, uint8_t* mask_bits, float* gamma,
                          unsigned long long* flips, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ------------------------------------------------------------------------
 * sbl_mask_quant without a caller-supplied workspace.  The paper has no
 * counterpart for this call: it exists for callers that cannot allocate
 * device memory when the weight step runs, such as processes that reserve
 * their whole device-memory budget at start-up and forbid any later
 * cudaMalloc, or host frameworks whose plugin interface passes only the
 * input and output buffers.  It computes exactly what sbl_mask_quant
 * computes (same arguments, minus the workspace) and allocates nothing: the
 * scratch is a fixed array of sbl_mask_quant_noalloc_scratch_bytes() bytes
 * (7040) in the library's static device memory, which every device that
 * loads the library holds until the process exits.
 *   - Size limit: W may have at most 2^32 - 1 elements (d_out * d_in);
 *     larger W returns SBL_ERR_SHAPE without launching anything.
 *   - The first call on a device looks up the scratch array's device address
 *     (once per device, with that device current) and caches it; make that
 *     first call before any stream capture.  A cudaDeviceReset() leaves the
 *     cached address stale (see the conventions above).
 *   - All calls on a device share the one scratch array.  Each call clears
 *     the part that must start at zero, but calls that overlap on the GPU
 *     (different streams, or different host threads without ordering) race
 *     on it and give wrong results: order them on one stream.
 * ---------------------------------------------------------------------- */
size_t sbl_mask_quant_noalloc_scratch_bytes(void);
sbl_status sbl_mask_quant_noalloc(const void* W, int d_out, int d_in, int N, int M,
                                  int8_t* W_eff, void* W_eff_bf16, uint8_t* mask_bits,
                                  float* gamma, void* stream);

/* ------------------------------------------------------------------------
 * Per-token absmax int8 activation quantiser.
 * [summary] 前置知识 (activations absmax-quantised to 8-bit integers) and
 * Algorithm 1 step (3).
 *   X     [T, d_in] bf16 in.
 *   Xq    [T, d_in] int8 out: clip(rint(fp32(x * fp32(127 / amax_t))), -128, 127).
 *   amax  [T] float out: amax_t = max(max_j |x_tj|, 1e-5).
 * ---------------------------------------------------------------------- */
sbl_status sbl_act_quant(const void* X, int T, int d_in, int8_t* Xq, float* amax,
                         void* stream);

/* Norm fused with the activation quantiser: x~ = Q_a(Norm(x)).
 * [summary] Algorithm 1 step (3).  Norm is RMSNorm with a per-channel gain
 * (the pages do not name the norm), computed so that no summation order
 * shows in the result:
 *   ss = sum_j x_tj^2 in fp64, v = fl32(ss / d_in + eps),
 *   r = fl32(1 / fl32(sqrt(v))), xn_tj = bf16_rn(fl32(fl32(x_tj * r) * g_j)),
 * then Xq and amax of the bf16 row xn exactly as sbl_act_quant.  One pass
 * over X instead of a norm pass plus sbl_act_quant.
 *   X    [T, d_in] bf16 in (the un-normalised activation).
 *   g    [d_in] bf16 in (the norm's gain).   eps > 0 (fp32).
 *   Xn   optional (NULL): [T, d_in] bf16 out, the normalised row (the X
 *        operand of sbl_backward's dW).
 *   Xq   [T, d_in] int8 out;  amax [T] float out. */
sbl_status sbl_rmsnorm_act_quant(const void* X, const void* g, float eps, int T, int d_in,
                                 void* Xn, int8_t* Xq, float* amax, void* stream);

/* ------------------------------------------------------------------------
 * Forward product on int8 tensor cores (tcgen05, int32 accumulation).
 * [summary] Algorithm 1 step (6): y = s * W_eff x~, with s absorbing the
 * quantisation scales: y[t,o] = fp32(fp32(acc) * fp32(gamma * fp32(amax_t/127))),
 * acc[t,o] = sum_j Xq[t,j] * W_eff[o,j] (exact int32).
 *   Xq     [T, d_in] int8, amax [T] float (from sbl_act_quant).
 *   W_eff  [d_out, d_in] int8 (from sbl_mask_quant), gamma 1 float (device).
 *   Y      [T, d_out] float out.
 *   acc    optional (NULL): [T, d_out] int32 out, the raw accumulators.
 * ---------------------------------------------------------------------- */
sbl_status sbl_forward(const int8_t* Xq, const float* amax, const int8_t* W_eff,
                       const float* gamma, int T, int d_in, int d_out, float* Y,
                       int32_t* acc, void* stream);

/* Several forward products (e.g. the seven projections of a layer):
 * problem i is exactly sbl_forward on its own buffers.  While the products
 * together have at most four 256 x 256 output tiles per pair of SMs (short
 * token batches, such as a prefill of a few hundred tokens) they run in one
 * launch, which pays the fixed start-up cost once; inside it a product whose
 * K is at least twice the group's shortest is split in K (exact integer
 * partial sums added into Y, then scaled in place by a second pass, so Y is
 * written twice).  Larger groups run one launch per product (as do all
 * products under sbl_set_gemm_variant(1)).  Same citation as sbl_forward.
 *   problems  HOST array of `count` descriptors (read before the call
 *             returns; the pointers inside are device pointers); each is
 *             validated as sbl_forward validates its arguments. */
typedef struct {
  const int8_t* Xq;     /* [T, d_in] int8                          */
  const float* amax;    /* [T] float                               */
  const int8_t* W_eff;  /* [d_out, d_in] int8                      */
  const float* gamma;   /* 1 float (device)                        */
  int T, d_in, d_out;
  float* Y;             /* [T, d_out] float out                    */
  int32_t* acc;         /* optional [T, d_out] int32 out (NULL)    */
} sbl_forward_problem;
sbl_status sbl_forward_group(const sbl_forward_problem* problems, int count, void* stream);

/* Forward product with the weight read from the packed format (prefill on a
 * deployed model): the same result as sbl_forward on the unpacked W_eff, bit
 * for bit.  [summary] Algorithm 1 step (6); [article] 7.1 (cached sparse
 * format); the packed weight is expanded tile by tile into shared memory
 * right before the int8 tensor-core MMA, so HBM only carries 2.5 bit/weight
 * at 6:8.
 *   packed  sbl_pack output of the [d_out, d_in] weight, N:M as packed.
 *   other arguments as sbl_forward. */
sbl_status sbl_forward_packed(const int8_t* Xq, const float* amax, const uint8_t* packed,
                              const float* gamma, int T, int d_in, int d_out, int N, int M,
                              float* Y, int32_t* acc, void* stream);

/* ------------------------------------------------------------------------
 * 2:4 weights on the sparse tensor core (tcgen05.mma.sp, kind::i8).
 * [summary] 前置知识 / 半结构化 N:M 稀疏 (2:4 is the pattern sparse tensor
 * cores accelerate) and 核心方法 (the mask is applied after quantisation,
 * so a 2:4 W_eff is already in the structure the hardware takes).
 *
 * sbl_compress24 turns a 2:4 W_eff ([d_out, d_in] int8, at most two
 * nonzeros in every group of four) into the compressed buffer the sparse
 * forward reads:
 *   values plane    d_out rows of ceil16(d_in / 2) bytes: the int8 values
 *                   of each group's two slots, ascending position order;
 *   selector plane  from the first 1024-byte boundary after the values: the
 *                   4-bit selector i0 | i1 << 2 of every group, in blocks of
 *                   128 rows x 256 weights (4096 bytes; block (mb, kb) at
 *                   (mb * ceil(d_in/256) + kb) * 4096), each block two
 *                   halves of 128 rows x 16 bytes, row r at 16 r, two groups
 *                   per byte (low nibble = even group).  Rows are padded to a
 *                   multiple of 256 and weights to a multiple of 256 with
 *                   selector 0x4 (slots 0, 1) and zero values.
 * Slots are the group's nonzero positions plus its lowest zero positions.
 * A group with more than two nonzeros latches SBL_ERR_DEVICE_CHECK (its
 * first two nonzeros are kept).
 *   out        device buffer of at least sbl_compress24_bytes() bytes.
 *
 * sbl_forward_sparse24 computes exactly sbl_forward on the W_eff that was
 * compressed, bit for bit (same int32 accumulators, same fp32 epilogue),
 * with the multiply skipped for the two dropped weights of every group.
 *   w24        sbl_compress24 output for this [d_out, d_in].
 *   other arguments as sbl_forward.
 * ---------------------------------------------------------------------- */
size_t sbl_compress24_bytes(int d_out, int d_in);
sbl_status sbl_compress24(const int8_t* W_eff, int d_out, int d_in, uint8_t* out,
                          size_t out_bytes, void* stream);
sbl_status sbl_forward_sparse24(const int8_t* Xq, const float* amax, const uint8_t* w24,
                                const float* gamma, int T, int d_in, int d_out, float* Y,
                                int32_t* acc, void* stream);

/* ------------------------------------------------------------------------
 * Dual-STE backward on bf16 tensor cores (tcgen05, fp32 accumulation).
 * [summary] 前置知识 / STE and 核心方法 (masked weights receive the full
 * gradient), Algorithm 1 step (7):
 *   dX = gamma * (dY . W_eff)          [T, d_in]
 *   dW = dY^T . X  (dense, unmasked)   [d_out, d_in]
 *   dY          [T, d_out] bf16;  X [T, d_in] bf16 (the layer input);
 *   W_eff_bf16  [d_out, d_in] bf16 (from sbl_mask_quant); gamma 1 float.
 *   dX          optional (NULL skips it): [T, d_in] float out.
 *   dW          optional (NULL skips it): [d_out, d_in] float out;
 *               accumulate_dW != 0 adds into the existing contents (gradient
 *               accumulation), 0 overwrites.
 *   workspace   device scratch of sbl_backward_workspace_bytes() bytes (may
 *               be NULL when that is 0).
 * ---------------------------------------------------------------------- */
size_t sbl_backward_workspace_bytes(int T, int d_in, int d_out);
sbl_status sbl_backward(const void* dY, const void* X, const void* W_eff_bf16,
                        const float* gamma, int T, int d_in, int d_out, float* dX,
                        float* dW, int accumulate_dW, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Packed inference format: 2-bit ternary codes + N:M slot index.
 * [article] 7.1 (pre-compute and cache the sparse format for inference);
 * [summary] 核心方法 (masking after quantisation makes the deployed ternary
 * weights N:M-structured).
 * Layout, per weight row, two planes each padded with zero bytes to a
 * multiple of 16 bytes.  A chunk is 8 consecutive positions; it holds
 * K = 8N/M slots s_0 < ... < s_(K-1) (its groups' slots in position order),
 * and H = ceil(K/2).
 *   codes plane: one 2K-bit field per chunk, little-endian, chunk c at bit
 *     2K*c.  Inside a field the code of s_q (q < H) sits at bits 4q..4q+1
 *     and the code of s_(H+q) at bits 4q+2..4q+3; codes +1 = 00, -1 = 01,
 *     0 = 10.
 *   index plane: the M-bit slot mask of every group (bit p = position p is a
 *     slot), little-endian bit stream (group g at bit g*M); for M = 8 one
 *     mask byte per chunk.
 * Slots are the group's nonzero positions plus, if fewer than N, its lowest
 * zero positions.  Buffer = d_out code rows, then d_out index rows; sbl_pack
 * writes the padding as zero bytes.
 * A group with more than N nonzeros latches SBL_ERR_DEVICE_CHECK.
 * ---------------------------------------------------------------------- */
size_t sbl_packed_bytes(int d_out, int d_in, int N, int M);
sbl_status sbl_pack(const int8_t* W_eff, int d_out, int d_in, int N, int M,
                    uint8_t* packed, size_t packed_bytes, void* stream);

/* Unpack: the packed format back to int8 W_eff [d_out, d_in] (bit for bit
 * the W_eff that was packed).  [article] 7.1 (the cached format is decoded
 * where it is used).  For prefill over many tokens, unpacking once and
 * calling sbl_forward is faster than sbl_forward_packed, which decodes the
 * weight again for every 256-token tile.
 *   packed  sbl_pack output of the [d_out, d_in] weight, N:M as packed.
 *   W_eff   [d_out, d_in] int8 out. */
sbl_status sbl_unpack(const uint8_t* packed, int d_out, int d_in, int N, int M,
                      int8_t* W_eff, void* stream);

/* Decode GEMV on the packed format, batch 1..16 tokens.
 * [summary] 实验结果 / Table 3 (decode on the 6:8 ternary model).
 * The kernel is launched with programmatic dependent launch: it may start
 * while the previous kernel of `stream` is finishing, build its tables and
 * begin streaming `packed`; it reads Xq, amax and gamma and writes Y only
 * after that kernel has completed.  No kernel of this library that lets its
 * successor start early writes a packed buffer, so plain stream order is
 * enough for every sequence of library calls.
 *   Xq [batch, d_in] int8, amax [batch] float, gamma 1 float (device),
 *   Y  [batch, d_out] float out, same formula as sbl_forward. */
sbl_status sbl_gemv_packed(const int8_t* Xq, const float* amax, int batch,
                           const uint8_t* packed, const float* gamma, int d_in,
                           int d_out, int N, int M, float* Y, void* stream);

/* Several decode GEMVs in one launch (e.g. the projections of a layer, or of
 * several layers): problem i is exactly sbl_gemv_packed on its own buffers.
 * Same citation as sbl_gemv_packed.
 *   problems  HOST array of `count` descriptors (read before the call
 *             returns; the pointers inside are device pointers).
 *   batch     tokens (1..16), N:M shared by all problems. */
typedef struct {
  const uint8_t* packed; /* sbl_pack output of a [d_out, d_in] weight */
  const int8_t* Xq;      /* [batch, d_in] int8 activations            */
  const float* amax;     /* [batch] per-token absmax (sbl_act_quant)  */
  const float* gamma;    /* 1 float, the weight's absmean scale       */
  float* Y;              /* [batch, d_out] float out                  */
  int d_in, d_out;
} sbl_gemv_problem;
sbl_status sbl_gemv_packed_group(const sbl_gemv_problem* problems, int count, int batch,
                                 int N, int M, void* stream);

/* ------------------------------------------------------------------------
 * Dense 2-bit ternary layout, a denser decode format: every position keeps
 * its 2-bit code and there is no index plane (for an N:M weight the dropped
 * positions hold the code of 0).  [article] 7.1 (cached low-bit format for
 * inference).  For ternary weights it is smaller than the packed format
 * (2.0 vs 2.5 bit/weight at 6:8: a 6:8 index costs 8 bits per chunk and
 * saves 4 bits of codes) and decodes without a table or a scatter.
 * Layout per row, padded to 16 bytes: d_in/8 little-endian 16-bit fields;
 * in a field the code of position q (q < 4) sits at bits 4q..4q+1 and the
 * code of position q+4 at bits 4q+2..4q+3 (+1 = 00, -1 = 01, 0 = 10) -- the
 * codes plane of the 8:8 packed format.
 *   sbl_pack_dense2:       W_eff [d_out, d_in] int8 -> out (>= sbl_dense2_bytes).
 *   sbl_gemv_dense2_group: decode GEMV on dense buffers, as
 *                          sbl_gemv_packed_group (problems[i].packed points at
 *                          the dense buffer of problem i; same dependent-launch
 *                          behaviour).
 * ---------------------------------------------------------------------- */
size_t sbl_dense2_bytes(int d_out, int d_in);
sbl_status sbl_pack_dense2(const int8_t* W_eff, int d_out, int d_in, uint8_t* out,
                           size_t out_bytes, void* stream);
sbl_status sbl_gemv_dense2_group(const sbl_gemv_problem* problems, int count, int batch,
                                 void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SBL_H_ */

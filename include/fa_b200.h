/*
 * fa_b200.h - C ABI of the B200 (sm_100a) BF16 FlashAttention library.
 *
 * What the calls compute (the statement of attention on the pages):
 *   S = scale * Q K^T, P = softmax(S) row by row, O = P V
 *   ("Is Flash Attention Stable?", chibakuma.com: the standard/baseline
 *   attention that FlashAttention reorders with tiling and kernel fusion),
 * evaluated the FlashAttention way: K/V tiles streamed through shared memory,
 * an online safe softmax with a running row maximum m and row sum l, the
 * unnormalised output P_bar V accumulated in FP32 and divided by l at the end,
 * and the log-sum-exp kept for a backward pass that recomputes P
 * (yicaiai article, abstract and sections 1.1, 3.4, 4.3).
 *
 * The repeated-max fix ("Why Low-Precision Transformer Training Fails: An
 * Analysis on Flash Attention", admirer.cn summary, "mechanism 2"): per row,
 * detect whether the maximum of S occurs more than once; if it does, raise
 * the safe-softmax shift m so that every exponent, the ones at the maximum
 * included, is strictly below 1.  This library raises m by
 * delta = -log2(1 - 2^-8) in the base-2 exponent domain, which maps each
 * maximum to exactly 1 - 2^-8 = 0.99609375, the largest bf16 value below 1.
 * P_bar is rounded to bf16 (round to nearest even) before the P_bar V
 * product; l sums the unrounded FP32 P.
 *
 * Conventions shared by every call
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are bf16, contiguous [B, H, N, d]
 *     (row-major, d fastest).  LSE is float32 [B, H, N] in natural-log units.
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or keeps a pointer after a call returns.
 *     Base addresses must be 16-byte aligned (TMA requirement).
 *   - d is 64 or 128.  N >= 1, any value (ragged tails are masked).  B, H >= 1.
 *     B*H*N*d must be below 2^31.  scale must be finite and > 0.
 *   - causal: 0 = every key visible; 1 = key j visible to query i iff j <= i.
 *   - stream is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on it; the return value reports argument and launch
 *     errors only.  Kernel-side watchdog timeouts are reported by
 *     fa_check_device_error().
 *   - On any error nothing is launched and outputs are left untouched.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = -1,      /* a required pointer is NULL                       */
  FA_ERR_SHAPE = -2,     /* B, H or N < 1, or B*H*N*d too large               */
  FA_ERR_HEADDIM = -3,   /* d not in {64, 128}                                */
  FA_ERR_ALIGN = -4,     /* a tensor base is not 16-byte aligned              */
  FA_ERR_FIXMODE = -5,   /* fix_mode not in {0, 1, 2, 3, 4, 5}                */
  FA_ERR_WORKSPACE = -6, /* workspace NULL, misaligned or too small           */
  FA_ERR_LAUNCH = -7,    /* the CUDA runtime refused a launch                 */
  FA_ERR_TIMEOUT = -8,   /* a kernel's bounded wait expired (device flag)     */
  FA_ERR_ARG = -9,       /* causal not in {0,1}, scale not finite and > 0, or
                            elem not an fa_elem value                         */
  FA_ERR_DEVICE = -10,   /* no sm_100 device, or the driver entry point for
                            tensor maps is unavailable                        */
  FA_ERR_SCRATCH_LIMIT = -11, /* fa_bwd_noalloc: the problem needs more scratch
                            than FA_BWD_NOALLOC_SCRATCH_BYTES                 */
  FA_ERR_BUILD = -12     /* the kernels were compiled with a register count
                            per thread that their register split does not
                            expect; nothing is launched                       */
} fa_status;

/*
 * fa_fwd - attention forward pass with the optional repeated-max fix.
 *   q, k, v  in : bf16 [B,H,N,d], device.
 *   o        out: bf16 [B,H,N,d], device.  O = (P_bar V) / l, rounded to bf16.
 *   lse      out: float32 [B,H,N], device.  LSE_i = log sum_j exp(S_ij).
 *   fix_mode    : 0 = plain safe softmax (shift = row max);
 *                 1 = repeated-max fix as described above (maxima -> 1 - 2^-8);
 *                 the variants below measure which choices remove the bias
 *                 (the pages leave the amount of the shift open):
 *                 2 = the fix with the shift raised by 1 (base 2): maxima ->
 *                     0.5, on the bf16 grid;
 *                 3 = the fix with the shift raised by 1/16 (natural log):
 *                     maxima -> exp(-1/16) = 0.93941, off the grid (P_bar
 *                     0.9375 there);
 *                 4 = plain shift, but O = (P_bar V) / sum_j P_bar_ij, the
 *                     sum of the rounded P_bar (self-normalised);
 *                 5 = fix_mode 1 triggered by near ties: two or more entries
 *                     whose P (plain shift) rounds to bf16 1.0, i.e.
 *                     P >= 1 - 2^-9, over the whole row (the two largest
 *                     scores are carried across key tiles).
 *                 LSE is the unrounded log-sum-exp in every mode.
 * Returns FA_OK or a negative fa_status.
 */
FA_API int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, int causal, float scale, int fix_mode,
           void* stream);

/* Element formats of fa_fwd_ex / fa_bwd_ex / fa_fwd_debug. */
typedef enum { FA_ELEM_BF16 = 0, FA_ELEM_F16 = 1 } fa_elem;

/*
 * fa_fwd_ex / fa_bwd_ex - fa_fwd / fa_bwd for every combination of:
 *   - elem: the element format (FA_ELEM_BF16 or FA_ELEM_F16) of every
 *     [.,.,N,d] tensor and of P_bar.  The pages treat FP16 and BF16 together
 *     as the low-precision formats of the instability (yicaiai article,
 *     abstract).  With FP16 the fix modes carry over on the fp16 grid: 1 and 5
 *     map repeated maxima to 1 - 2^-11, the largest fp16 value below 1;
 *     2, 3 and 4 are as in fa_fwd; 5 counts entries whose P rounds to fp16
 *     1.0, i.e. P >= 1 - 2^-12.
 *   - H query heads over Hkv key/value heads (grouped-query attention, the
 *     head layout of the larger Llama 2 models that "Is Flash Attention
 *     Stable?" names; MQA when Hkv == 1; ordinary attention when Hkv == H):
 *     query head h reads key/value head h / (H / Hkv).
 *       q, o, dout, dq : [B,H,N,d];  k, v, dk, dv : [B,Hkv,N,d];
 *       lse            : float32 [B,H,N].
 *     dK and dV of a shared head are the sums over the query heads of its
 *     group.  Hkv must divide H (FA_ERR_SHAPE otherwise).  The workspace is
 *     fa_bwd_workspace_size(B, H, N, d) (query heads).
 *   - any fix_mode 0-5.
 * fa_fwd and fa_bwd are these calls with elem = FA_ELEM_BF16 and Hkv = H.
 * Layouts, ownership, the workspace and the error codes are theirs;
 * FA_ERR_ARG also reports an unknown elem.
 */
FA_API int fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int Hkv, int N, int d, int causal, float scale,
                     int fix_mode, int elem, void* stream);
FA_API int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv,
                     void* workspace, size_t workspace_bytes, int B, int H, int Hkv,
                     int N, int d, int causal, float scale, int elem, void* stream);

/*
 * fa_fwd_debug - fa_fwd_ex plus per-row records that show the fix at work
 * inside the kernel ("Why Low-Precision Transformer Training Fails",
 * admirer.cn summary, mechanism 2: detect a repeated row maximum of S and
 * raise the shift so that every exponent, the maxima included, is strictly
 * below 1; the same section places the bias in the forward's unnormalised
 * output).  Same kernel and arithmetic as fa_fwd_ex; O and LSE are
 * bit-identical to its outputs.  Any of the three records may be NULL, not
 * all (FA_ERR_NULL).
 *   tie_count_out out: int32 [B,H,N], device.
 *       Bits 0-28: the number of visible keys whose FP32 score equals the row
 *       maximum of S (at most N < 2^25).
 *       Bit 29: the row's final shift is the raised one, i.e. the fix applies
 *       to its output (fix_mode 1, 2, 3 with a repeated maximum; fix_mode 5
 *       with two or more entries that round to 1).
 *       Bit 30: the detector fired at some key tile: the running maximum was
 *       repeated (fix_mode 0-4), or two or more entries rounded to 1
 *       (fix_mode 5).
 *   one_hit_out   out: int32 [B,H,N], device.  The number of entries of the
 *       row whose P_bar, as the kernel rounded it for the P_bar V product,
 *       is exactly 1.0, counted among the entries produced under the row's
 *       final shift (a move of the shift rescales O and l exactly, so
 *       entries rounded earlier no longer enter O with weight P_bar).  A row
 *       whose final shift is raised (bit 29 above) has 0: no exponent reaches
 *       1.  A row with the plain shift has at least 1 (its maximum).
 *   o_f32_out     out: float32 [B,H,N,d], device, 16-byte aligned.  O before
 *       its rounding to the element format: the FP32 values (P_bar V) / l
 *       whose round-to-nearest-even is the returned O.  It shows the error
 *       of the P_bar V path without the error of the output's own rounding.
 */
FA_API int fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse,
                        int32_t* tie_count_out, int32_t* one_hit_out, float* o_f32_out,
                        int B, int H, int Hkv, int N, int d, int causal, float scale,
                        int fix_mode, int elem, void* stream);

/*
 * fa_bwd_workspace_size - bytes of device scratch fa_bwd needs:
 *   an FP32 dQ accumulator [B,H,N,d] and FP32 D_i = sum_k dO_ik O_ik [B,H,N].
 * Returns 0 for invalid shapes.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * fa_bwd - attention backward pass that recomputes P from the LSE.
 *   q, k, v, o, dout in : bf16 [B,H,N,d], device (o and lse from fa_fwd).
 *   lse              in : float32 [B,H,N], device.
 *   dq, dk, dv       out: bf16 [B,H,N,d], device.
 *   workspace        tmp: device, >= fa_bwd_workspace_size() bytes, 16-byte
 *                         aligned; contents on entry are ignored.
 * Gradients of sum(dO * O): dV = P^T dO, dS = P * (dO V^T - D),
 * dQ = scale dS K, dK = scale dS^T Q.  No fix_mode argument: LSE does not
 * depend on the shift, so the recomputed P is the same either way.
 */
FA_API int fa_bwd(const void* q, const void* k, const void* v, const void* o,
           const float* lse, const void* dout, void* dq, void* dk, void* dv,
           void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
           int causal, float scale, void* stream);

/*
 * The three launches fa_bwd makes, callable one by one (same arguments and
 * checks as fa_bwd; all three must see the same workspace, in this order):
 *   fa_bwd_preprocess  D_i = sum_k dO_ik O_ik into the workspace, and a zeroed
 *                      FP32 dQ accumulator (reads O and dO once).
 *   fa_bwd_main        recompute P per (key tile, query tile), write dK and dV,
 *                      and add the unscaled dQ contributions into the
 *                      accumulator.
 *   fa_bwd_finish      dQ = scale * accumulator, rounded to bf16.
 */
FA_API int fa_bwd_preprocess(const void* o, const void* dout, void* workspace,
                             size_t workspace_bytes, int B, int H, int N, int d,
                             void* stream);
FA_API int fa_bwd_main(const void* q, const void* k, const void* v,
                       const float* lse, const void* dout, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes, int B, int H,
                       int N, int d, int causal, float scale, void* stream);
FA_API int fa_bwd_finish(void* dq, const void* workspace, size_t workspace_bytes,
                         int B, int H, int N, int d, float scale, void* stream);

/*
 * fa_bwd_noalloc - fa_bwd for callers that must not allocate device memory.
 * The paper has no counterpart: this is an interface convenience.
 *
 * Who needs it: code that runs where cudaMalloc is off limits - a plugin
 * inside a host that owns all device memory through its own pool, a process
 * whose allocator is reserved up front to a fixed budget, or a real-time loop
 * that must not take the driver's allocation locks.  fa_bwd asks such a
 * caller for a workspace it has no way to get; this call needs none.
 *
 * Arguments and results are those of fa_bwd without workspace/workspace_bytes.
 * The scratch (FP32 dQ accumulator and D) lives instead in one fixed array of
 * FA_BWD_NOALLOC_SCRATCH_BYTES (32 MiB) compiled into the library as a
 * device global: every GPU that loads the library holds those 32 MiB until
 * the process exits, whether or not this call is used.
 *   - Limit: fa_bwd_workspace_size(B,H,N,d) <= FA_BWD_NOALLOC_SCRATCH_BYTES,
 *     which allows B*H*N <= 129055 rows at d = 64 (8 x 12 x 1024 = 98304
 *     fits) and <= 65027 rows at d = 128.  Larger problems return
 *     FA_ERR_SCRATCH_LIMIT and launch nothing.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device (the current device) looks up the array's
 *     device address once; make that first call before any stream capture
 *     begins on that device.
 *   - The array is shared by every call on a device and keeps the last call's
 *     contents; each call clears the accumulator before use.  Calls whose
 *     kernels overlap on the GPU (concurrent streams, or host threads without
 *     stream ordering between them) race on the array and give wrong
 *     gradients: order them on one stream, or serialise them.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
FA_API int fa_bwd_noalloc(const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dout,
                          void* dq, void* dk, void* dv, int B, int H, int N,
                          int d, int causal, float scale, void* stream);

/* fa_status_string - static, NUL-terminated description of a status code. */
FA_API const char* fa_status_string(int status);

/*
 * fa_watchdog_selftest - test hook for the kernels' failure handling; the
 * paper has no counterpart.  Launches one small kernel on `stream` whose
 * bounded mbarrier wait (the same code every attention kernel uses) is made to
 * expire after `timeout_us` microseconds (1 .. 1000000), while a second warp
 * waits with the kernels' own limit and must leave on the CTA's abort mark.
 * Nothing faults or hangs; the kernel returns, and the next
 * fa_check_device_error() on that stream reports FA_ERR_TIMEOUT.
 * Returns FA_OK, FA_ERR_ARG (timeout out of range), FA_ERR_DEVICE or
 * FA_ERR_LAUNCH.
 */
FA_API int fa_watchdog_selftest(unsigned timeout_us, void* stream);

/*
 * fa_check_device_error - synchronises `stream`, then reads and clears the
 * library's device error flag on the current device.  Returns FA_OK,
 * FA_ERR_TIMEOUT if a kernel gave up on a bounded wait since the last check,
 * FA_ERR_DEVICE if a kernel found its shared memory misaligned and did no
 * work, or FA_ERR_LAUNCH if the stream reports a CUDA error.
 */
FA_API int fa_check_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */

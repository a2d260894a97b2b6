/*
 * fa_b200.h -- C ABI of libfa_b200.so: BF16 FlashAttention forward and
 * backward for NVIDIA B200 (sm_100a) with the stabilised safe softmax of
 * Qiu & Yao, "Why Low-Precision Transformer Training Fails: An Analysis on
 * Flash Attention" (arXiv 2510.04212).
 *
 * What the operations compute (sources: the web page
 * itsolotime.com/archives/23922, sections "mechanism two" (safe softmax) and
 * "minimal fix" (the shift rule, with its pseudocode); the web page
 * 91haoming.cn/news/show-608006, section 3 (the delta step of the backward)):
 *
 *   S     = Q K^T * scale,  scale = 1/sqrt(d)     (fp32 accumulation)
 *   rm    = rowmax(S),  rs = number of j with S[i,j] == rm[i]
 *   m     = rm                                     (FA_SOFTMAX_STANDARD)
 *   m     = beta*rm  if rs > 1 and rm > 0          (FA_SOFTMAX_STABILIZED)
 *           0        if rs > 1 and rm < 0
 *           beta-1   if rs > 1 and rm == 0   <- reading: the pages' "else"
 *                                               would leave exact ones in
 *                                               P_bar; the rm > 0 rule with
 *                                               |rm| replaced by 1 is used
 *           rm       otherwise
 *   m2    = m + margin rule                        (FA_SOFTMAX_STABILIZED_MARGIN)
 *           on rows with rs > 1 where m - rm < 2^-8 (fp32 subtraction),
 *           m2 = rm + 2^-8 (fp32 add); otherwise m2 = m.  The rule above keeps
 *           the fp32 max(P_bar) below 1, but bf16(P_bar) still rounds to 1
 *           when m - rm < 2^-9; with the margin, exp(rm - m2) <= exp(-2^-8)
 *           and its bf16 value is below 1 too.  (The pages give the fp32
 *           rule; the margin carries their goal, max(P_bar) < 1, to the bf16
 *           operand of the P V product.)
 *   P_bar = exp(S - m),  l = rowsum(P_bar),  P = P_bar / l,  O = P V
 *   lse   = m + ln(l)                          (natural logarithm)
 *
 *   backward: delta = rowsum(dO o O), dV = P^T dO, dP = dO V^T,
 *             dS = P o (dP - delta), dQ = dS K * scale, dK = dS^T Q * scale,
 *   with P recomputed as exp(S - lse) (standard) or as
 *   exp(S - m) * (1/l), l = exp(lse - m) (both stabilised modes, m from the
 *   forward).
 *
 * Layout: Q, K, V, O, dO, dQ, dK, dV are bf16 arrays [B, H, N, d], contiguous
 * (d fastest), base addresses 16-byte aligned.  lse, delta and the row
 * statistics are fp32 (rs: int32) arrays [B, H, N].  Query and key lengths
 * are equal (N).  Causal masking hides key j from query i when j > i.
 *
 * Ownership: every pointer is caller-owned device memory (global memory of
 * the current device).  The library allocates and frees nothing; it keeps
 * no state between calls except the per-kernel timing records of
 * fa_timing_* and the device error word of fa_device_error.
 *
 * Execution: calls are asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = the legacy default stream).  Argument errors are returned
 * synchronously before anything is launched.  A failed launch returns
 * FA_ERR_CUDA.  Every wait inside the kernels is bounded (2 s); a kernel
 * whose wait runs out records a code in a device error word, frees its
 * tensor memory and returns: fa_device_error reports it as FA_ERR_TIMEOUT.
 *
 * Domain: d in {64, 128}; any N >= 0 (a ragged last tile of fewer than 128
 * rows is masked); B, H >= 0, and a problem with B*H*N == 0 is a valid
 * no-op; B*H*N*d < 2^40 and B*H*ceil(N/128) < 2^31.  beta must be finite
 * and > 1 in the stabilised modes (ignored in standard mode).
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, bad size or mode, beta <= 1 */
  FA_ERR_UNSUPPORTED = 2,  /* valid request outside the implemented domain (d, N) */
  FA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  FA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or kernel launch failed */
  FA_ERR_TIMEOUT = 5       /* a kernel gave up on a bounded wait (see fa_device_error) */
} fa_status;

typedef enum {
  FA_SOFTMAX_STANDARD = 0,
  FA_SOFTMAX_STABILIZED = 1,
  FA_SOFTMAX_STABILIZED_MARGIN = 2
} fa_softmax_mode;

/* Optional per-row outputs of the forward, each [B, H, N]; any may be NULL.
 * rm: row max of S; rs: its tie count; m: the shift used (this is what
 * fa_bwd consumes as row_m in stabilised mode); pbar_max: exp(rm - m), the
 * largest P_bar of the row (1 when m == rm, < 1 when the shift moved). */
typedef struct {
  float* rm;
  int32_t* rs;
  float* m;
  float* pbar_max;
} fa_row_stats;

/* Forward.  Inputs q, k, v; outputs o (bf16) and lse (fp32); stats optional
 * (the struct pointer itself may be NULL).  One kernel launch. */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const fa_row_stats* stats,
                 int B, int H, int N, int d, int causal, int softmax_mode, float beta, void* stream);

/* Bytes of device workspace fa_bwd needs: delta (fp32 [B,H,N]), the fp32 dQ
 * accumulator [B,H,N,d] and a 256-byte block that holds the work-item counter
 * of the d = 128 kernel, each part 256-byte aligned.  0 on bad sizes. */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/* Byte offset of delta and of the fp32 dQ accumulator inside the workspace
 * (the work-item counter follows the accumulator). */
size_t fa_bwd_workspace_delta_offset(int B, int H, int N, int d);
size_t fa_bwd_workspace_dq_offset(int B, int H, int N, int d);

/* Backward.  Inputs q, k, v, o, dO (bf16), lse (fp32, from fa_fwd), row_m
 * (fp32 shift m from fa_fwd's stats; required in the stabilised modes,
 * ignored otherwise); outputs dq, dk, dv (bf16).  workspace: caller-owned device
 * memory of at least fa_bwd_workspace_bytes, 256-byte aligned; its contents
 * on entry do not matter and on exit hold delta and the fp32 dQ.  Launches
 * three kernels on `stream`: delta (which also clears the accumulator and the
 * work-item counter), main (dK, dV, partial dQ), dQ convert.  softmax_mode
 * must match the one the forward used. */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 const float* row_m, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                 int H, int N, int d, int causal, int softmax_mode, float beta, void* stream);

/* High-precision O (the pages' O_hp; reading of their localisation remedy:
 * keep the rounded O_lp out of the delta term of the backward).
 *
 * fa_fwd_o_hp: as fa_fwd (the bf16 o and every other output are the same,
 * bit for bit), and also writes o_hp, fp32 [B, H, N, d] (16-byte aligned,
 * caller-owned): O with P_bar carried to about 16 bits -- P_bar is split into
 * P_hi = bf16(P_bar) and P_lo = bf16(P_bar - P_hi), the two parts are
 * multiplied by V into separate fp32 accumulators and o_hp = (O_hi + O_lo)/l.
 * The bf16 o is O_hi / l rounded, as in fa_fwd.  Costs a second P V product
 * and a 512-column TMEM allocation (one CTA per SM).
 *
 * fa_bwd_o_hp: as fa_bwd, with delta = rowsum(dO o O_hp) taken from the fp32
 * O instead of the bf16 one; every other step is fa_bwd's.  Same workspace,
 * same errors (o_hp NULL or misaligned: FA_ERR_INVALID_ARG). */
fa_status fa_fwd_o_hp(const void* q, const void* k, const void* v, void* o, float* o_hp, float* lse,
                      const fa_row_stats* stats, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                      void* stream);
fa_status fa_bwd_o_hp(const void* q, const void* k, const void* v, const float* o_hp, const void* dO,
                      const float* lse, const float* row_m, void* dq, void* dk, void* dv, void* workspace,
                      size_t workspace_bytes, int B, int H, int N, int d, int causal, int softmax_mode, float beta,
                      void* stream);

/* Static description of a status code. */
const char* fa_status_string(fa_status s);

/* The CUDA failure behind the last FA_ERR_CUDA returned to the calling
 * thread: the failing step and CUDA's error name (thread-local storage owned
 * by the library; "" if none yet). */
const char* fa_last_error_string(void);

/* Synchronises the current device, then reads and clears the device error
 * word that kernels set when a bounded wait ran out.  *code (may be NULL)
 * receives the raw word (kernel id << 24 | wait site << 16 | block), the
 * kernel id being one of FA_ERRWORD_*.  Returns FA_OK if it was clear,
 * FA_ERR_TIMEOUT if set, FA_ERR_CUDA if the synchronisation failed. */
enum { FA_ERRWORD_FWD = 1, FA_ERRWORD_BWD_D64 = 3, FA_ERRWORD_BWD_D128 = 4 };
fa_status fa_device_error(unsigned int* code);

/* Test hooks for the bounded-wait exit path (the pages have no counterpart;
 * they exist so that the error exit can be exercised on a GPU without a
 * fault).  Both write a device variable of the current device with a
 * synchronous copy; call them between launches, never while a kernel of this
 * library runs.
 *
 * fa_debug_set_wait_limit_ns: time limit of every bounded wait of every
 * kernel launched afterwards (0 restores the default, 2 s).  A short limit
 * (milliseconds) makes a withheld arrive end quickly; it must stay well above
 * the longest legitimate wait of the problem being run.
 *
 * fa_debug_inject_stall: kernel_id = FA_ERRWORD_FWD, _BWD_D64 or _BWD_D128
 * makes CTA 0 of every later launch of that kernel withhold its elementwise
 * warps' first arrive on the barrier that hands P_bar (forward) or P^T
 * (backward) to the MMA warp.  No bulk copy is outstanding on that barrier:
 * the MMA warp's wait runs out, the kernel records the error word, drains its
 * copies and products, frees its tensor memory and returns; fa_device_error
 * then reports FA_ERR_TIMEOUT, and the outputs of that launch are undefined.
 * 0 switches the injection off.  Any other id: FA_ERR_INVALID_ARG. */
fa_status fa_debug_set_wait_limit_ns(unsigned long long ns);
fa_status fa_debug_inject_stall(unsigned int kernel_id);

/* Per-kernel timing.  While enabled, every launch made by fa_fwd / fa_bwd is
 * bracketed by two CUDA events recorded on the launching stream.
 * fa_timing_read synchronises on the recorded events, adds the elapsed times
 * per kernel id (FA_KERNEL_*), writes launch counts and total milliseconds
 * into the caller's arrays (length FA_NUM_KERNELS) and clears the records.
 * Not thread-safe. */
enum { FA_KERNEL_FWD = 0, FA_KERNEL_BWD_DELTA = 1, FA_KERNEL_BWD_MAIN = 2, FA_KERNEL_BWD_DQ = 3, FA_NUM_KERNELS = 4 };
fa_status fa_timing_enable(int enable);
fa_status fa_timing_read(int* launches, double* total_ms);

/* Allocation-free backward.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory themselves --
 * runtimes that fix every device buffer at start-up under a static memory
 * plan and forbid allocation afterwards, and plug-ins that are handed tensors
 * by a host framework but own no allocator.  Such callers cannot provide the
 * workspace fa_bwd asks for.
 *
 * Same arguments and results as fa_bwd without the workspace.  The scratch
 * (delta and the fp32 dQ accumulator) lives in one static device array of
 * FA_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads the
 * library holds that array until the process exits.  A problem whose
 * fa_bwd_workspace_bytes exceeds it is rejected with FA_ERR_WORKSPACE before
 * anything is launched.  The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress, with the device current); make that first
 * call before any stream capture.  All calls share the one array and it keeps
 * the last call's contents (the dQ accumulator is cleared by the call itself
 * before use), so calls that overlap on the GPU -- on different streams, or
 * from different host threads -- race on it and must be serialised by the
 * caller.  The looked-up address is kept for the life of the process: a
 * device reset (cudaDeviceReset) or any other teardown of the device's
 * primary context invalidates it, and calling fa_bwd_noalloc after one is not
 * supported.  Returns FA_ERR_CUDA if the address lookup fails. */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                         const float* lse, const float* row_m, void* dq, void* dk, void* dv, int B, int H, int N,
                         int d, int causal, int softmax_mode, float beta, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H_ */

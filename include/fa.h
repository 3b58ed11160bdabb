/*
 * fa.h -- C ABI of libfa.so: exact scaled-dot-product attention, forward and
 * backward, as fused tiled kernels for NVIDIA B200 (sm_100a).
 *
 * What is computed (per head (b, h); heads are independent):
 *
 *   O = softmax(scale * Q K^T [+ causal mask]) V
 *
 * -- the "Vanilla Attention" definition of the FlashAttention review
 * (mrodiduger, "Vanilla Attention", with the scale the review leaves out),
 * computed the IO-aware way the same review ("Tiling", "Recomputation") and the
 * FlashAttention summary ("Architecture, step by step") describe: tiles of
 * Q, K and V are staged on chip, a running max m and normaliser l combine the
 * blocks (online softmax), and only O and the per-row statistics reach HBM.
 * The N x N score matrix is never written to memory.  The statistics are
 * stored folded into one log-sum-exp, LSE_i = m_i + ln(l_i) (natural log).
 * The backward pass recomputes S and P from Q, K and LSE
 * ("Recomputation") and returns dQ, dK, dV for an upstream gradient dO.
 *
 * Causal mask: key j is masked (-inf) for query i when j > i (the diagonal is
 * kept; queries and keys share positions 0..N-1).
 *
 * Layout and types (all tensors caller-owned, device memory, contiguous):
 *   q, k, v, o, dO, dq, dk, dv : [B, H, N, d] bf16 (passed as raw 16-bit words)
 *   lse                        : [B, H, N] fp32, natural-log LSE
 *   workspace (fa_bwd only)    : fa_bwd_workspace_bytes(B, H, N, d) bytes
 * Every pointer must be 16-byte aligned (a TMA requirement).  Outputs must not
 * overlap inputs.  Inputs are never written.
 *
 * Supported: d in {64, 128}; B, H, N >= 1; B*H*N*d < 2^31 elements per tensor;
 * scale finite and > 0; causal in {0, 1}; an sm_100 device.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 * default stream).  The return value reports argument and launch errors only;
 * on an argument error nothing is launched and no output is touched.  A
 * device-side failure (a pipeline wait that exceeded its time limit) is
 * recorded in a library-owned device status word and returned by
 * fa_device_status().  No exception crosses this interface.  The library
 * allocates only that status word (32 bytes per device, once, on the first
 * call that reaches the device) and host-side state; all tensors and the
 * workspace come from the caller.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,   /* null pointer, N/B/H < 1, bad scale or causal flag */
    FA_ERR_UNSUPPORTED = 2,   /* d not in {64,128}, tensor too large, device not sm_100 */
    FA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    FA_ERR_WORKSPACE = 4,     /* workspace null or smaller than fa_bwd_workspace_bytes() */
    FA_ERR_NO_DEVICE = 5,     /* no CUDA device could be used */
    FA_ERR_CUDA = 6,          /* a CUDA runtime/driver call or a launch failed */
    FA_ERR_DEVICE_TIMEOUT = 7, /* a kernel gave up on a pipeline wait (fa_device_status) */
    FA_ERR_DEVICE_INTERNAL = 8 /* a kernel found its launch environment unusable
                                  (e.g. a misaligned shared-memory window) */
} fa_status;

/*
 * Forward pass.  Writes o [B,H,N,d] bf16 and lse [B,H,N] fp32.
 * Source: FlashAttention summary "Architecture, step by step" (tile inputs,
 * compute locally, online normalisation, write compact output) and the review's
 * "Tiling" section (online softmax instead of the three-loop safe softmax).
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N, int d, float scale, int causal, void *stream);

/*
 * Bytes of scratch fa_bwd needs: an fp32 dQ accumulator [B,H,N,d], plus two
 * fp32 vectors [B,H,Np] with Np = N rounded up to a multiple of 128 -- the
 * per-row D_i = rowsum(dO * O) and LSE_i * log2(e) -- so
 * 4*B*H*(N*d + 2*Np) bytes, rounded up to a multiple of 256; then 256 bytes
 * more, whose first word counts the work units the backward kernel's CTAs
 * have taken (one CTA per SM, each taking (head, key tile) units in turn).
 * Returns 0 for unsupported or invalid shapes.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass.  Given the forward inputs, its outputs o and lse, and the
 * upstream gradient dO, writes dq, dk, dv [B,H,N,d] bf16.  Source: the review's
 * "Recomputation" section (keep the softmax statistics, recompute S and P in the
 * backward pass); the gradient formulas are the chain rule through softmax.
 * `workspace` (device, 16-byte aligned, caller-owned, contents ignored on entry)
 * must hold fa_bwd_workspace_bytes(B,H,N,d) bytes; it is overwritten.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o,
           const void *dO, const float *lse, void *dq, void *dk, void *dv,
           int B, int H, int N, int d, float scale, int causal,
           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward pass that also writes the rounding residual of O:
 *   o_lo [B,H,N,d] bf16 = bf16(O_fp32 - o),
 * i.e. what rounding the fp32 result to the bf16 output o dropped, so that
 * o + o_lo carries about 16 significant bits of O.  The backward's
 * D_i = rowsum(dO_i o O_i) is a difference-sensitive quantity: in rows where
 * softmax is nearly one-hot, dS = P (dP - D) cancels almost exactly and an
 * 8-bit O would dominate the gradient error.  Passing o_lo to fa_bwd_ex
 * removes that error.  o_lo must not overlap any other tensor; NULL makes
 * this call identical to fa_fwd.  This is not a step of the pages' method but
 * a precision choice of this implementation (the pages leave the backward's
 * arithmetic open).
 */
int fa_fwd_residual(const void *q, const void *k, const void *v, void *o,
                    void *o_lo, float *lse, int B, int H, int N, int d,
                    float scale, int causal, void *stream);

/*
 * FP8 forward pass (the FlashAttention topic page names FP8 as a
 * FlashAttention-3 feature, "FlashAttention-3 (2024)", without a scheme).
 * Inputs are e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * the "fn" variant without infinities) with one fp32 descale factor per head:
 *   q8, k8, v8           [B, H, N, d] uint8 e4m3 codes (device, 16-byte aligned)
 *   descale_q/_k/_v      [B, H] fp32 (device, 4-byte aligned); the inputs are the
 *                        reals code_value * descale
 *   o                    [B, H, N, d] bf16 output, lse [B, H, N] fp32 (natural log)
 * It computes O = softmax(scale * Q K^T [+ causal mask]) V of those reals, as
 * fa_fwd does, with two differences of precision: S = Q K^T accumulates the
 * exact e4m3 products in fp32, and the probabilities P are rounded to e4m3
 * (relative error <= 2^-4, absolute <= 2^-10 below 2^-6) before the PV
 * product; O is divided by the fp32 row sum of the unrounded P, and lse is
 * that of the unrounded P.  Supported: d = 128 only (FA_ERR_UNSUPPORTED
 * otherwise); other arguments, errors and ownership as fa_fwd.
 */
int fa_fwd_fp8(const void *q8, const void *k8, const void *v8,
               const float *descale_q, const float *descale_k,
               const float *descale_v, void *o, float *lse, int B, int H,
               int N, int d, float scale, int causal, void *stream);

/*
 * Forward pass with dropout on the attention probabilities (the fused dropout
 * the FlashAttention pages count among the method's largest speed-ups): the
 * same arguments as fa_fwd_residual (o_lo may be NULL), plus
 *   rate    dropout probability, 0 <= rate < 1 (FA_ERR_INVALID_ARG otherwise);
 *   seed    64-bit key of the Philox4x32-10 generator (Salmon et al., SC 2011);
 *   offset  counter word 3 (e.g. the training step): a new mask per value.
 * Mask: for head bh = b*H + h, query row i and key j, the generator's counter is
 * (i, j >> 4, bh, offset) and its key (seed & 0xffffffff, seed >> 32); the
 * 8-bit draw of key j is byte (j & 3) of output word ((j & 15) >> 2); key j is
 * kept for row i iff the draw is >= T = floor(rate * 256) (the rate takes steps
 * of 1/256: a rate below 1/256 drops nothing, 0.1 drops with probability
 * 25/256).  Then
 *   O_i = sum_j P_ij * keep_ij * 256/(256 - T) * V_j
 * with P = softmax(scale * Q K^T [+ causal mask]); lse is that of P, without
 * dropout.  The mask is never stored: fa_bwd_dropout regenerates it.
 */
int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o,
                   void *o_lo, float *lse, int B, int H, int N, int d,
                   float scale, int causal, float rate, unsigned long long seed,
                   unsigned int offset, void *stream);

/*
 * Backward pass of fa_fwd_dropout, given the same rate, seed and offset (and
 * that call's o, o_lo, lse): dV = (P o Z)^T dO, dP = Z o (dO V^T),
 * dS = P o (dP - D) with D_i = rowsum(dO_i o O_i), dQ = scale dS K,
 * dK = scale dS^T Q, where Z = keep * 256/(256 - T).  Workspace, layout and
 * errors as fa_bwd_ex (without events).
 */
int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o,
                   const void *o_lo, const void *dO, const float *lse, void *dq,
                   void *dk, void *dv, int B, int H, int N, int d, float scale,
                   int causal, float rate, unsigned long long seed,
                   unsigned int offset, void *workspace, size_t workspace_bytes,
                   void *stream);

/*
 * The dropout mask itself, for inspection and tests: mask [B,H,N,N] uint8
 * (device, caller-owned, row-major over keys) receives keep_ij in {0, 1} as
 * defined for fa_fwd_dropout.  This writes N*N bytes per head, the O(N^2)
 * object the fused kernels never materialise.
 */
int fa_dropout_mask(int B, int H, int N, float rate, unsigned long long seed,
                    unsigned int offset, void *mask, void *stream);

/*
 * Backward pass with the optional extras:
 *   o_lo    NULL, or the residual written by fa_fwd_residual (then
 *           D_i = rowsum(dO o (o + o_lo)) instead of rowsum(dO o o));
 *   events  NULL, or a host array of four cudaEvent_t handles owned by the
 *           caller, recorded on `stream` before the preprocess kernel, after
 *           it, after the main dK/dV/dQ kernel and after the dQ conversion, so
 *           each kernel can be timed with cudaEventElapsedTime.
 * Otherwise the same arguments, layout and errors as fa_bwd (FA_ERR_INVALID_ARG
 * if an event handle is NULL, FA_ERR_CUDA if recording one fails).
 */
int fa_bwd_ex(const void *q, const void *k, const void *v, const void *o,
              const void *o_lo, const void *dO, const float *lse, void *dq,
              void *dk, void *dv, int B, int H, int N, int d, float scale,
              int causal, void *workspace, size_t workspace_bytes,
              void *stream, void *const *events);

/*
 * Deterministic backward pass: the same results as fa_bwd_ex (without events)
 * within the same tolerances, and the same bits on every call with the same
 * inputs on the same GPU model.
 *
 * In fa_bwd, each 128-row key tile adds its contribution dS_ij K_j to dQ_i into
 * an fp32 accumulator as it finishes, so the order of the fp32 additions, and
 * with it the last bits of dQ, can change from run to run.  Here dQ is
 * computed by a separate kernel, one CTA per (head, 128-row query tile), which
 * recomputes S_ij = Q_i K_j^T, P_ij (from LSE, as in the review's
 * "Recomputation" section), dP_ij = dO_i V_j^T and dS_ij (the chain rule
 * through softmax) and sums dQ_i over the key tiles in ascending j in tensor
 * memory.  dK and dV come from the fused kernel run without its dQ product, bit
 * for bit as in fa_bwd (the same products in the same order).  Costs 7 tile
 * products per (query tile, key tile) pair against fa_bwd's 5: 1.4x the
 * tensor-core work.
 *
 * Arguments, layout, ownership and errors: as fa_bwd_ex with events = NULL
 * (o_lo may be NULL); the workspace size is fa_bwd_workspace_bytes(B, H, N, d).
 */
int fa_bwd_deterministic(const void *q, const void *k, const void *v,
                         const void *o, const void *o_lo, const void *dO,
                         const float *lse, void *dq, void *dk, void *dv,
                         int B, int H, int N, int d, float scale, int causal,
                         void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * Backward pass for callers that cannot allocate device memory.
 *
 * Some callers may not call cudaMalloc at all: code that runs where an
 * allocation could block, fail or be forbidden (for example inside a memory
 * pool or allocator of its own, in a real-time path with a fixed memory
 * budget, or where device memory is handed out by a host framework that owns
 * it).  This entry point computes exactly what fa_bwd computes, with the same
 * arguments except the workspace: its scratch -- the fp32 dQ accumulator and
 * the per-row D and LSE*log2(e) vectors -- lives in one static array of
 * FA_NOALLOC_SCRATCH_BYTES bytes inside this library's device image.  Every
 * GPU on which the library is loaded holds that array until the process exits.
 * No counterpart exists in the pages; this is a deployment variant only.
 *
 * Limit: shapes whose scratch, fa_bwd_workspace_bytes(B, H, N, d), exceeds
 * FA_NOALLOC_SCRATCH_BYTES are rejected with FA_ERR_WORKSPACE before anything
 * is launched (e.g. at d = 128 about B*H*N <= 64 000 rows).
 *
 * The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine.  Its first call on a device does a one-time set-up on that
 * device (it looks up the array's device address with cudaGetSymbolAddress and
 * sets kernel attributes); make that first call before any stream capture.
 * Every call shares the one array and each call re-initialises the part it
 * uses (the dQ accumulator is zeroed by the first kernel of the call), so calls
 * whose kernels overlap on the GPU -- on different streams, or from different
 * host threads -- race on the array and must be serialised by the caller.
 * A device-side wait timeout in these kernels is recorded in a status word that
 * also lives in the static image (dq/dk/dv are then undefined).
 * fa_device_status() does not see that word (it owns a separately allocated
 * one): read it with fa_noalloc_device_status() after the call.
 */
#define FA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                   const void *dO, const float *lse, void *dq, void *dk,
                   void *dv, int B, int H, int N, int d, float scale,
                   int causal, void *stream);

/*
 * The failure record of fa_bwd_noalloc: synchronises `stream`, then returns and
 * clears the status word in the static image that fa_bwd_noalloc's kernels
 * write -- FA_OK, or FA_ERR_DEVICE_TIMEOUT if one of them gave up on a wait
 * since the last read (its dq/dk/dv are then undefined) -- and copies the
 * record into info[0..3] as fa_device_status_info() does (info may be NULL).
 * Allocates nothing; the first no-alloc call on a device does the same
 * one-time set-up as fa_bwd_noalloc.  FA_ERR_CUDA if a CUDA call fails.
 */
int fa_noalloc_device_status(void *stream, int *info);

/*
 * fa_selftest_timeout() aimed at fa_bwd_noalloc's status word: one thread
 * waits on a barrier nothing completes, gives up after 1 s and records
 * FA_ERR_DEVICE_TIMEOUT (kernel id 5, wait tag 1) there, so that
 * fa_noalloc_device_status() can be checked without a fault.  Allocates
 * nothing.
 */
int fa_noalloc_selftest_timeout(void *stream);

/* Static, human-readable name of a status code (never NULL). */
const char *fa_status_string(int status);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: FA_OK, or FA_ERR_DEVICE_TIMEOUT if a kernel launched since
 * the last call gave up on a wait (its outputs are then undefined).
 * Returns FA_ERR_CUDA if the synchronisation itself fails.
 */
int fa_device_status(void *stream);

/*
 * Like fa_device_status(), and also copies the failure record into info[0..3]:
 * {kernel id (1 fwd, 2 bwd, 4 deterministic dQ, 5 fa_selftest_timeout), wait tag, block
 * index, launch sequence number}; zeros when there was no failure.  `info` is a
 * host pointer to 4 ints (may be NULL).
 */
int fa_device_status_info(void *stream, int *info);

/*
 * Diagnostic of the device-side failure path.  Launches one thread on `stream`
 * that waits on a pipeline barrier nothing will complete.  Like every wait in
 * the kernels, that wait is bounded: after its time limit (1 s) the kernel
 * records FA_ERR_DEVICE_TIMEOUT in the status word (kernel id 5, wait tag 1)
 * and returns, so the context stays usable.  The next fa_device_status() then
 * returns FA_ERR_DEVICE_TIMEOUT and clears the word.  Returns FA_OK once the
 * kernel is launched, or FA_ERR_NO_DEVICE / FA_ERR_UNSUPPORTED / FA_ERR_CUDA.
 */
int fa_selftest_timeout(void *stream);

/* Library version, MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */

/*
 * fa_vanilla.h -- standard (materialising) attention on B200: the baseline the
 * IO-aware kernels in fa.h are measured against.
 *
 * Source: the FlashAttention review (mrodiduger.github.io, "Flash Attention"
 * post), section "Vanilla Attention": S0 = Q K^T and S1 = softmax(S0) are each
 * written to HBM and read back, then O = S1 V.  Here S0 carries the scale
 * (S0 = scale * Q K^T), the causal mask is applied to S0 before the softmax, and
 * the backward pass keeps S1 (= P) from the forward as its activation, the way
 * standard attention stores the softmax output for the gradient.
 *
 * Memory: the workspace holds, per head, S0 (later dP) as fp32 and P (later
 * dS) as bf16: 6*N*N bytes -- the O(N^2) footprint the IO-aware method avoids.
 * The three GEMMs of each pass are cuBLAS strided-batched GEMMs (bf16 inputs,
 * fp32 accumulation); the row softmax and its backward are kernels of this
 * library.
 *
 * Layout and conventions follow fa.h: q, k, v, o, dO, dq, dk, dv are device
 * pointers to [B,H,N,d] contiguous bf16 (16-bit words); lse is [B,H,N] fp32
 * (natural log); d in {64, 128}; N >= 1; 16-byte aligned pointers; finite
 * scale > 0; causal in {0, 1}.  Calls are asynchronous on `stream` (a
 * cudaStream_t, NULL for the default stream).  Return values are fa_status
 * codes from fa.h: argument errors return before any launch and touch nothing;
 * FA_ERR_CUDA reports a failed launch or cuBLAS call.  cuBLAS keeps one handle
 * per device (created on first use) and may allocate its own scratch.
 */
#ifndef FA_VANILLA_H
#define FA_VANILLA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Workspace bytes for fa_vanilla_fwd / fa_vanilla_bwd: 6*B*H*N*N (fp32 S0 or
 * dP, then bf16 P or dS, per head), rounded up to 256.  0 for invalid shapes
 * or when the size does not fit a size_t.
 */
size_t fa_vanilla_workspace_bytes(int B, int H, int N, int d);

/*
 * Forward: S0 = scale*Q K^T (fp32, into the workspace), masked (j > i) when
 * causal; P = softmax(S0) row by row (bf16, into the workspace) with
 * LSE_i = max_j S0_ij + ln sum_j exp(S0_ij - max); O = P V (bf16).
 * The workspace keeps P for fa_vanilla_bwd.
 */
int fa_vanilla_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int N, int d, float scale, int causal,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward, given the workspace exactly as fa_vanilla_fwd left it for the
 * same q, k, v (its P): dP = dO V^T (fp32, over S0); dV = P^T dO;
 * dS = P o (dP - D) with D_i = sum_j P_ij dP_ij (bf16, over P);
 * dQ = scale*dS K; dK = scale*dS^T Q.  o and lse are not read (they are
 * accepted for symmetry with fa_bwd).
 */
int fa_vanilla_bwd(const void *q, const void *k, const void *v, const void *o,
                   const void *dO, const float *lse, void *dq, void *dk, void *dv,
                   int B, int H, int N, int d, float scale, int causal,
                   void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_VANILLA_H */

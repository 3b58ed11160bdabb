// vanilla.cu -- standard (materialising) attention, the baseline of the IO-aware
// kernels: the "Vanilla Attention" section of the FlashAttention review
// (S0 = Q K^T and S1 = softmax(S0) written to and read back from HBM, then
// O = S1 V), with the scale and causal mask applied to S0 and the softmax
// output kept for the backward pass.  C ABI in include/fa_vanilla.h.
//
// GEMMs: cuBLAS strided-batched, bf16 operands, fp32 accumulation.  cuBLAS is
// column-major; a row-major [R x C] matrix is read by it as the column-major
// [C x R] transpose, so every product below is written for the transposes
// (row-major X = A B  <=>  column-major X^T = B^T A^T).
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_vanilla.h"

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
cublasHandle_t g_handle[kMaxDevices] = {};

cublasHandle_t handle_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_handle[dev] && cublasCreate(&g_handle[dev]) != CUBLAS_STATUS_SUCCESS) g_handle[dev] = nullptr;
  return g_handle[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape and argument checks shared by both entry points (the same support as fa.h).
int check_args(int B, int H, int N, int d, float scale, int causal) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  const long long elems = static_cast<long long>(B) * H * N * d;
  if (elems >= (1ll << 31)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t workspace_bytes(int B, int H, int N) {
  const unsigned long long nn = static_cast<unsigned long long>(N) * static_cast<unsigned long long>(N);
  const unsigned long long heads = static_cast<unsigned long long>(B) * static_cast<unsigned long long>(H);
  if (nn != 0 && heads > ~0ull / nn / 8) return 0;
  const unsigned long long total = heads * nn * 6ull;
  return static_cast<size_t>((total + 255ull) / 256ull * 256ull);
}

// ------------------------------------------------------------------ kernels
constexpr int kRowThreads = 256;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float *red) {
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red[] may still be read from the previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[lane < kRowThreads / 32 ? lane : 0];
  if (lane >= kRowThreads / 32) v = is_max ? -INFINITY : 0.f;
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  return v;
}

// One CTA per row of S0: P = exp(S0 - max) / sum (bf16), masked entries 0;
// LSE = max + ln(sum).  Reads the fp32 row twice (the second pass from cache).
__global__ void __launch_bounds__(kRowThreads) softmax_rows(const float *__restrict__ S, __nv_bfloat16 *__restrict__ P,
                                                            float *__restrict__ lse, int N, int causal) {
  __shared__ float red[kRowThreads / 32];
  const size_t row = blockIdx.x;
  const int i = static_cast<int>(row % static_cast<size_t>(N));
  const int valid = causal ? i + 1 : N;  // keys j < valid take part
  const float *s = S + row * static_cast<size_t>(N);
  __nv_bfloat16 *p = P + row * static_cast<size_t>(N);
  float m = -INFINITY;
  for (int j = threadIdx.x; j < valid; j += kRowThreads) m = fmaxf(m, s[j]);
  m = block_reduce(m, true, red);
  float l = 0.f;
  for (int j = threadIdx.x; j < valid; j += kRowThreads) l += expf(s[j] - m);
  l = block_reduce(l, false, red);
  const float inv = 1.f / l;
  for (int j = threadIdx.x; j < N; j += kRowThreads)
    p[j] = __float2bfloat16_rn(j < valid ? expf(s[j] - m) * inv : 0.f);
  if (threadIdx.x == 0) lse[row] = m + logf(l);
}

// One CTA per row: D = sum_j P_ij dP_ij; dS_ij = P_ij (dP_ij - D), bf16, written
// over P (masked entries have P = 0 and stay 0).
__global__ void __launch_bounds__(kRowThreads) softmax_bwd_rows(const float *__restrict__ dP,
                                                                __nv_bfloat16 *__restrict__ P, int N) {
  __shared__ float red[kRowThreads / 32];
  const size_t row = blockIdx.x;
  const float *dp = dP + row * static_cast<size_t>(N);
  __nv_bfloat16 *p = P + row * static_cast<size_t>(N);
  float acc = 0.f;
  for (int j = threadIdx.x; j < N; j += kRowThreads) acc += __bfloat162float(p[j]) * dp[j];
  const float D = block_reduce(acc, false, red);
  for (int j = threadIdx.x; j < N; j += kRowThreads) {
    const float pj = __bfloat162float(p[j]);
    p[j] = __float2bfloat16_rn(pj * (dp[j] - D));
  }
}

// C = alpha * op(A) op(B), column-major, bf16 operands, fp32 accumulation.
cublasStatus_t gemm(cublasHandle_t h, cublasOperation_t ta, cublasOperation_t tb, int m, int n, int k, float alpha,
                    const void *A, int lda, long long sA, const void *B, int ldb, long long sB, void *C,
                    cudaDataType ctype, int ldc, long long sC, int batch) {
  const float beta = 0.f;
  return cublasGemmStridedBatchedEx(h, ta, tb, m, n, k, &alpha, A, CUDA_R_16BF, lda, sA, B, CUDA_R_16BF, ldb, sB,
                                    &beta, C, ctype, ldc, sC, batch, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
}

}  // namespace

extern "C" size_t fa_vanilla_workspace_bytes(int B, int H, int N, int d) {
  if (check_args(B, H, N, d, 1.f, 0) != FA_OK) return 0;
  return workspace_bytes(B, H, N);
}

extern "C" int fa_vanilla_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N,
                              int d, float scale, int causal, void *workspace, size_t ws_bytes, void *stream) {
  int st = check_args(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(workspace))
    return FA_ERR_MISALIGNED;
  const size_t need = workspace_bytes(B, H, N);
  if (need == 0 || ws_bytes < need) return FA_ERR_WORKSPACE;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return FA_ERR_NO_DEVICE;
  cublasHandle_t h = handle_for_current_device();
  if (!h) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) return FA_ERR_CUDA;
  const int BH = B * H;
  const long long nd = static_cast<long long>(N) * d, nn = static_cast<long long>(N) * N;
  float *S = static_cast<float *>(workspace);
  __nv_bfloat16 *P = reinterpret_cast<__nv_bfloat16 *>(S + static_cast<size_t>(BH) * nn);
  // S0 (row-major N x N) = scale Q K^T  <=>  column-major S0^T = scale K Q^T, with
  // K and Q read as the column-major [d x N] matrices K^T and Q^T.
  if (gemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, N, d, scale, k, d, nd, q, d, nd, S, CUDA_R_32F, N, nn, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  softmax_rows<<<static_cast<unsigned>(static_cast<long long>(BH) * N), kRowThreads, 0, s>>>(S, P, lse, N, causal);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  // O (row-major N x d) = P V  <=>  column-major O^T = V^T P^T.
  if (gemm(h, CUBLAS_OP_N, CUBLAS_OP_N, d, N, N, 1.f, v, d, nd, P, N, nn, o, CUDA_R_16BF, d, nd, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  return FA_OK;
}

extern "C" int fa_vanilla_bwd(const void *q, const void *k, const void *v, const void *o, const void *dO,
                              const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                              int causal, void *workspace, size_t ws_bytes, void *stream) {
  (void)o;
  (void)lse;
  int st = check_args(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (!q || !k || !v || !dO || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(workspace))
    return FA_ERR_MISALIGNED;
  const size_t need = workspace_bytes(B, H, N);
  if (need == 0 || ws_bytes < need) return FA_ERR_WORKSPACE;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) return FA_ERR_NO_DEVICE;
  cublasHandle_t h = handle_for_current_device();
  if (!h) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) return FA_ERR_CUDA;
  const int BH = B * H;
  const long long nd = static_cast<long long>(N) * d, nn = static_cast<long long>(N) * N;
  float *dPm = static_cast<float *>(workspace);  // over S0
  __nv_bfloat16 *P = reinterpret_cast<__nv_bfloat16 *>(dPm + static_cast<size_t>(BH) * nn);
  // dP = dO V^T  <=>  column-major dP^T = V dO^T.
  if (gemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, N, d, 1.f, v, d, nd, dO, d, nd, dPm, CUDA_R_32F, N, nn, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  // dV = P^T dO  <=>  column-major dV^T = dO^T P (P read as column-major P^T, transposed).
  if (gemm(h, CUBLAS_OP_N, CUBLAS_OP_T, d, N, N, 1.f, dO, d, nd, P, N, nn, dv, CUDA_R_16BF, d, nd, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  softmax_bwd_rows<<<static_cast<unsigned>(static_cast<long long>(BH) * N), kRowThreads, 0, s>>>(dPm, P, N);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  // dQ = scale dS K  <=>  column-major dQ^T = scale K^T dS^T.
  if (gemm(h, CUBLAS_OP_N, CUBLAS_OP_N, d, N, N, scale, k, d, nd, P, N, nn, dq, CUDA_R_16BF, d, nd, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  // dK = scale dS^T Q  <=>  column-major dK^T = scale Q^T dS.
  if (gemm(h, CUBLAS_OP_N, CUBLAS_OP_T, d, N, N, scale, q, d, nd, P, N, nn, dk, CUDA_R_16BF, d, nd, BH) !=
      CUBLAS_STATUS_SUCCESS)
    return FA_ERR_CUDA;
  return FA_OK;
}

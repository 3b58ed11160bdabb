// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument
// validation, TMA descriptor encoding, the per-device status block, and the
// launches of the forward, backward and deterministic-dQ kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_dq.cuh"
#include "fa_fwd.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kStatusInts = 8;
// The forward's unit counters: a launch uses slot seq % kFwdCounterSlots, zeroed on
// its stream just before it, so launches in flight at the same time use distinct
// slots unless kFwdCounterSlots of them are.
constexpr int kFwdCounterSlots = 4096;

struct DeviceState {
  bool ready = false;
  int *status = nullptr;        // kStatusInts ints, device memory
  int *fwd_counters = nullptr;  // kFwdCounterSlots ints, after the status block
  int num_sms = 0;
  bool attrs_set = false;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::atomic<int> g_seq{1};

int next_seq() {
  int s = g_seq.fetch_add(1);
  if (s <= 0) {  // wrapped: sequence numbers stay positive (0 marks "none")
    g_seq.store(2);
    s = 1;
  }
  return s;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor maps are pure functions of (address, type, dims, box), so encoded maps
// are kept in a small least-recently-used cache: a call on tensors seen before
// copies its maps instead of encoding them again.
struct MapKey {
  int dev;
  const void *ptr;
  int dt, D, N, BH, box_x;
  bool operator==(const MapKey &o) const {
    return dev == o.dev && ptr == o.ptr && dt == o.dt && D == o.D && N == o.N && BH == o.BH && box_x == o.box_x;
  }
};
struct MapSlot {
  MapKey key;
  CUtensorMap map;
  uint64_t used = 0;  // 0: empty
};
constexpr int kMapSlots = 64;
std::mutex g_map_mu;
MapSlot g_maps[kMapSlots];
uint64_t g_map_tick = 0;

int encode_3d_uncached(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem_bytes, int D, int N,
                       int BH, int box_x);

// [BH, N, D] tensor viewed as 3-D (x = feature, y = row, z = head); box of
// 64 (or 32 for fp32, 128 for bytes) features x 128 rows x 1 head, 128-byte
// swizzle, zero fill.
int encode_3d(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem_bytes, int D, int N, int BH,
              int box_x) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  const MapKey key{dev, ptr, static_cast<int>(dt), D, N, BH, box_x};
  {
    std::lock_guard<std::mutex> lock(g_map_mu);
    for (MapSlot &sl : g_maps)
      if (sl.used != 0 && sl.key == key) {
        sl.used = ++g_map_tick;
        *m = sl.map;
        return FA_OK;
      }
  }
  const int st = encode_3d_uncached(m, ptr, dt, elem_bytes, D, N, BH, box_x);
  if (st != FA_OK) return st;
  std::lock_guard<std::mutex> lock(g_map_mu);
  MapSlot *victim = &g_maps[0];
  for (MapSlot &sl : g_maps)
    if (sl.used < victim->used) victim = &sl;
  victim->key = key;
  victim->map = *m;
  victim->used = ++g_map_tick;
  return FA_OK;
}

int encode_3d_uncached(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem_bytes, int D, int N,
                       int BH, int box_x) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * elem_bytes,
                           static_cast<cuuint64_t>(N) * D * elem_bytes};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int encode_bf16(CUtensorMap *m, const void *ptr, int D, int N, int BH) {
  return encode_3d(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, N, BH, 64);
}

// e4m3 codes as bytes: 128-element (128-byte) box rows.
int encode_u8(CUtensorMap *m, const void *ptr, int D, int N, int BH) {
  return encode_3d(m, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, N, BH, 128);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by both passes (no CUDA calls).
int check_shape(int B, int H, int N, int d, float scale, int causal) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long double elems = static_cast<long double>(B) * H * N * d;
  if (elems >= 2147483648.0L) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

template <int D, bool CAUSAL, bool DROPOUT, bool FP8 = false>
cudaError_t fwd_set_attribute() {
  return cudaFuncSetAttribute(fa::fa_fwd_kernel<D, CAUSAL, DROPOUT, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              fa::FwdCfg<D, FP8>::kSmemBytes);
}

// Dropout rate -> the generator's threshold and the kept entries' scale.
// Returns false for a rate outside [0, 1).
bool dropout_params(float rate, unsigned long long seed, unsigned int offset, fa::DropoutParams *dp) {
  if (!std::isfinite(rate) || rate < 0.f || rate >= 1.f) return false;
  const double t = std::floor(static_cast<double>(rate) * 256.0);
  if (t >= 256.0) return false;
  dp->T = static_cast<uint32_t>(t);
  dp->seed_lo = static_cast<uint32_t>(seed & 0xffffffffull);
  dp->seed_hi = static_cast<uint32_t>(seed >> 32);
  dp->offset = offset;
  dp->inv_keep = static_cast<float>(256.0 / (256.0 - t));
  return true;
}

// Lazily set up the current device: compute capability check, SM count and
// the status block.  Returns a status code.
int device_state(DeviceState **out, int *dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  if (dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState &s = g_dev[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
    int *st = nullptr;
    const size_t bytes = (kStatusInts + kFwdCounterSlots) * sizeof(int);
    if (cudaMalloc(&st, bytes) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    if (cudaMemset(st, 0, bytes) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(st);
      return FA_ERR_CUDA;
    }
    s.status = st;
    s.fwd_counters = st + kStatusInts;
    s.num_sms = sms;
    s.ready = true;
  }
  if (!s.attrs_set) {
    cudaError_t e = cudaSuccess;
    e = (e == cudaSuccess) ? fwd_set_attribute<64, false, false>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<64, true, false>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, false, false>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, true, false>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<64, false, true>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<64, true, true>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, false, true>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, true, true>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, false, false, true>() : e;
    e = (e == cudaSuccess) ? fwd_set_attribute<128, true, false, true>() : e;
    e = (e == cudaSuccess) ? fa::bwd_set_attributes() : e;
    e = (e == cudaSuccess) ? fa::dq_set_attributes() : e;
    if (e != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    s.attrs_set = true;
  }
  *out = &s;
  if (dev_out) *dev_out = dev;
  return FA_OK;
}

// Persistent grid: one CTA per SM (one resident CTA fits), or one per unit if fewer.
template <int D, bool CAUSAL, bool DROPOUT, bool FP8 = false>
cudaError_t launch_fwd(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v, const fa::FwdParams &p,
                       int num_sms, cudaStream_t stream) {
  const long units = static_cast<long>(p.BH) * p.n_qpairs;
  const dim3 grid(static_cast<unsigned>(units < num_sms ? units : num_sms));
  fa::fa_fwd_kernel<D, CAUSAL, DROPOUT, FP8>
      <<<grid, fa::FwdCfg<D, FP8>::kThreads, fa::FwdCfg<D, FP8>::kSmemBytes, stream>>>(q, k, v, p);
  return cudaGetLastError();
}

template <bool DROPOUT>
cudaError_t launch_fwd_any(int d, int causal, const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                           const fa::FwdParams &p, int n, cudaStream_t s) {
  if (d == 64)
    return causal ? launch_fwd<64, true, DROPOUT>(q, k, v, p, n, s) : launch_fwd<64, false, DROPOUT>(q, k, v, p, n, s);
  return causal ? launch_fwd<128, true, DROPOUT>(q, k, v, p, n, s) : launch_fwd<128, false, DROPOUT>(q, k, v, p, n, s);
}

// Zero the launch's unit-counter slot on its stream.
int fwd_counter(DeviceState *ds, int seq, cudaStream_t s, int **out) {
  int *c = ds->fwd_counters + (seq & (kFwdCounterSlots - 1));
  if (cudaMemsetAsync(c, 0, sizeof(int), s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  *out = c;
  return FA_OK;
}

// Dropout mask writer: one thread per (head, query row, 16-key block).
__global__ void fa_dropout_mask_kernel(uint8_t *mask, long BH, int N, fa::DropoutParams dp) {
  const long nblk = (N + 15) / 16;
  const long total = BH * N * nblk;
  for (long t = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<long>(gridDim.x) * blockDim.x) {
    const long jb = t % nblk, row = t / nblk;
    const long i = row % N, bh = row / N;
    const uint32_t bits = fa::dropout_keep16(dp, static_cast<uint32_t>(i), static_cast<uint32_t>(jb),
                                             static_cast<uint32_t>(bh));
    uint8_t *out = mask + row * N + jb * 16;
    for (int u = 0; u < 16 && jb * 16 + u < N; ++u) out[u] = static_cast<uint8_t>((bits >> u) & 1u);
  }
}

// Self-test of the device-side failure path: one thread waits on an mbarrier
// that nothing arrives on.  The bounded wait gives up after its time limit,
// records the failure in the status block (kernel kKernelSelftest, wait tag
// kSelftestTag) and the kernel returns normally, leaving the context usable.
constexpr int kKernelSelftest = 5;
constexpr int kSelftestTag = 1;

__global__ void fa_selftest_timeout_kernel(int *status, int seq) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    fa::mbar_init(&bar, 1);
    fa::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const fa::WaitCtx ctx{status, reinterpret_cast<volatile int *>(&abort_flag), kKernelSelftest, seq};
    fa::mbar_wait(ctx, &bar, 0, kSelftestTag);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// The shared bodies of the entry points: argument checks, tensor maps, launch.

static int fwd_common(const void *q, const void *k, const void *v, void *o, void *o_lo, float *lse, int B, int H,
                      int N, int d, float scale, int causal, const fa::DropoutParams *drop, void *stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (o_lo && !aligned16(o_lo)))
    return FA_ERR_MISALIGNED;
  DeviceState *ds = nullptr;
  st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;

  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (encode_bf16(&tq, q, d, N, BH) || encode_bf16(&tk, k, d, N, BH) || encode_bf16(&tv, v, d, N, BH))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.o_lo = static_cast<uint16_t *>(o_lo);
  p.status = ds->status;
  p.seq = next_seq();
  p.N = N;
  p.BH = BH;
  p.n_qpairs = (N + 255) / 256;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.drop = drop ? *drop : fa::DropoutParams{0u, 0u, 0u, 0u, 1.f};
  p.descale_q = p.descale_k = p.descale_v = nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fwd_counter(ds, p.seq, s, &p.unit_counter);
  if (st != FA_OK) return st;
  const int n = ds->num_sms;
  const cudaError_t e = drop ? launch_fwd_any<true>(d, causal, tq, tk, tv, p, n, s)
                             : launch_fwd_any<false>(d, causal, tq, tk, tv, p, n, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// e4m3 forward: Q, K, V as byte codes with per-head descale factors; O bf16.
static int fwd_fp8_common(const void *q8, const void *k8, const void *v8, const float *dq, const float *dk,
                          const float *dv, void *o, float *lse, int B, int H, int N, int d, float scale, int causal,
                          void *stream) {
  if (!q8 || !k8 || !v8 || !dq || !dk || !dv || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(dq) & 3u) || (reinterpret_cast<uintptr_t>(dk) & 3u) ||
      (reinterpret_cast<uintptr_t>(dv) & 3u))
    return FA_ERR_MISALIGNED;
  DeviceState *ds = nullptr;
  st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (encode_u8(&tq, q8, d, N, BH) || encode_u8(&tk, k8, d, N, BH) || encode_u8(&tv, v8, d, N, BH))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = static_cast<uint16_t *>(o);
  p.lse = lse;
  p.o_lo = nullptr;
  p.status = ds->status;
  p.seq = next_seq();
  p.N = N;
  p.BH = BH;
  p.n_qpairs = (N + 255) / 256;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.drop = fa::DropoutParams{0u, 0u, 0u, 0u, 1.f};
  p.descale_q = dq;
  p.descale_k = dk;
  p.descale_v = dv;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = fwd_counter(ds, p.seq, s, &p.unit_counter);
  if (st != FA_OK) return st;
  const cudaError_t e = causal ? launch_fwd<128, true, false, true>(tq, tk, tv, p, ds->num_sms, s)
                               : launch_fwd<128, false, false, true>(tq, tk, tv, p, ds->num_sms, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// deterministic: dQ from fa_dq_kernel (a fixed summation order over key tiles)
// instead of the fp32 accumulator that key tiles add into as they finish.
static int bwd_common(const void *q, const void *k, const void *v, const void *o, const void *o_lo, const void *dO,
                      const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                      int causal, void *workspace, size_t workspace_bytes, void *stream, void *const *events,
                      const fa::DropoutParams *drop, bool deterministic) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (o_lo && !aligned16(o_lo)))
    return FA_ERR_MISALIGNED;
  const int BH = B * H;
  if (!workspace || workspace_bytes < fa::bwd_workspace_bytes(BH, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  if (events && (!events[0] || !events[1] || !events[2] || !events[3])) return FA_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;

  fa::BwdLaunch L;
  L.q = q; L.k = k; L.v = v; L.o = o; L.o_lo = o_lo; L.dO = dO; L.lse = lse;
  L.dq = dq; L.dk = dk; L.dv = dv;
  L.BH = BH; L.N = N; L.d = d; L.scale = scale; L.causal = causal;
  L.workspace = workspace;
  L.status = ds->status;
  L.seq = next_seq();
  L.num_sms = ds->num_sms;
  L.events = reinterpret_cast<cudaEvent_t const *>(events);
  L.drop = drop;
  CUtensorMap maps[7], tdq;
  if (encode_bf16(&maps[0], q, d, N, BH) || encode_bf16(&maps[1], k, d, N, BH) ||
      encode_bf16(&maps[2], v, d, N, BH) || encode_bf16(&maps[3], dO, d, N, BH) ||
      encode_3d(&maps[6], L.workspace, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, BH, 32) ||
      (deterministic && encode_bf16(&tdq, dq, d, N, BH)))
    return FA_ERR_CUDA;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = deterministic ? fa::bwd_launch_deterministic(L, maps, tdq, s) : fa::bwd_launch(L, maps, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" {

int fa_version(void) { return 300; }  // 0.3.0: fa_fwd_fp8, the no-alloc status reader

const char *fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported shape or device";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
    case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE: no usable CUDA device";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call or launch failed";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT: a kernel gave up on a pipeline wait";
    case FA_ERR_DEVICE_INTERNAL: return "FA_ERR_DEVICE_INTERNAL: kernel launch environment unusable";
    default: return "unknown fa_status";
  }
}

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
           float scale, int causal, void *stream) {
  return fwd_common(q, k, v, o, nullptr, lse, B, H, N, d, scale, causal, nullptr, stream);
}

int fa_fwd_residual(const void *q, const void *k, const void *v, void *o, void *o_lo, float *lse, int B, int H,
                    int N, int d, float scale, int causal, void *stream) {
  return fwd_common(q, k, v, o, o_lo, lse, B, H, N, d, scale, causal, nullptr, stream);
}

int fa_fwd_fp8(const void *q8, const void *k8, const void *v8, const float *descale_q, const float *descale_k,
               const float *descale_v, void *o, float *lse, int B, int H, int N, int d, float scale, int causal,
               void *stream) {
  return fwd_fp8_common(q8, k8, v8, descale_q, descale_k, descale_v, o, lse, B, H, N, d, scale, causal, stream);
}

int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, void *o_lo, float *lse, int B, int H, int N,
                   int d, float scale, int causal, float rate, unsigned long long seed, unsigned int offset,
                   void *stream) {
  fa::DropoutParams dp;
  if (!dropout_params(rate, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
  return fwd_common(q, k, v, o, o_lo, lse, B, H, N, d, scale, causal, &dp, stream);
}

int fa_dropout_mask(int B, int H, int N, float rate, unsigned long long seed, unsigned int offset, void *mask,
                    void *stream) {
  if (!mask) return FA_ERR_INVALID_ARG;
  int st = check_shape(B, H, N, 64, 1.f, 0);
  if (st != FA_OK) return st;
  fa::DropoutParams dp;
  if (!dropout_params(rate, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
  DeviceState *ds = nullptr;
  st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;
  const long BH = static_cast<long>(B) * H;
  fa_dropout_mask_kernel<<<ds->num_sms * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint8_t *>(mask), BH, N, dp);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 1.f, 0) != FA_OK) return 0;
  return fa::bwd_workspace_bytes(B * H, N, d);
}

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dO, const float *lse, void *dq,
           void *dk, void *dv, int B, int H, int N, int d, float scale, int causal, void *workspace,
           size_t workspace_bytes, void *stream) {
  return bwd_common(q, k, v, o, nullptr, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                    workspace_bytes, stream, nullptr, nullptr, false);
}

int fa_bwd_ex(const void *q, const void *k, const void *v, const void *o, const void *o_lo, const void *dO,
              const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale, int causal,
              void *workspace, size_t workspace_bytes, void *stream, void *const *events) {
  return bwd_common(q, k, v, o, o_lo, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes,
                    stream, events, nullptr, false);
}

int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o, const void *o_lo, const void *dO,
                   const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                   int causal, float rate, unsigned long long seed, unsigned int offset, void *workspace,
                   size_t workspace_bytes, void *stream) {
  fa::DropoutParams dp;
  if (!dropout_params(rate, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
  return bwd_common(q, k, v, o, o_lo, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes,
                    stream, nullptr, &dp, false);
}

int fa_bwd_deterministic(const void *q, const void *k, const void *v, const void *o, const void *o_lo,
                         const void *dO, const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                         float scale, int causal, void *workspace, size_t workspace_bytes, void *stream) {
  return bwd_common(q, k, v, o, o_lo, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes,
                    stream, nullptr, nullptr, true);
}

int fa_device_status_info(void *stream, int *info) {
  if (info) std::memset(info, 0, 4 * sizeof(int));
  DeviceState *ds = nullptr;
  int st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  int h[kStatusInts];
  if (cudaMemcpy(h, ds->status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (h[0] == 0) return FA_OK;
  if (info) {
    info[0] = h[1];
    info[1] = h[2];
    info[2] = h[3];
    info[3] = h[4];
  }
  if (cudaMemset(ds->status, 0, kStatusInts * sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return h[0] == fa::kStatusInternal ? FA_ERR_DEVICE_INTERNAL : FA_ERR_DEVICE_TIMEOUT;
}

int fa_device_status(void *stream) { return fa_device_status_info(stream, nullptr); }

int fa_selftest_timeout(void *stream) {
  DeviceState *ds = nullptr;
  const int st = device_state(&ds, nullptr);
  if (st != FA_OK) return st;
  fa_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ds->status, next_seq());
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_bwd_noalloc: fa_bwd for callers that cannot allocate device memory.  The
// scratch it needs is this file-scope array in the library's device image.  In
// host code the array's name is only a host-side stand-in, so its device
// address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and passed to the kernels.
static __device__ __align__(256) unsigned char fa_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];
static __device__ __align__(256) int fa_noalloc_status[kStatusInts];

namespace {

struct NoAllocState {
  bool ready = false;
  void *scratch = nullptr;  // device address of fa_noalloc_scratch on this device
  int *status = nullptr;    // device address of fa_noalloc_status on this device
  int num_sms = 0;
};

NoAllocState g_noalloc[kMaxDevices];

// One-time set-up on the current device; performs no allocation.
int noalloc_state(NoAllocState **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return FA_ERR_NO_DEVICE;
  }
  if (dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocState &s = g_noalloc[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_NO_DEVICE;
    }
    if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;
    void *scratch = nullptr, *status = nullptr;
    if (cudaGetSymbolAddress(&scratch, fa_noalloc_scratch) != cudaSuccess ||
        cudaGetSymbolAddress(&status, fa_noalloc_status) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    if (fa::bwd_set_attributes() != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    s.scratch = scratch;
    s.status = static_cast<int *>(status);
    s.num_sms = sms;
    s.ready = true;
  }
  *out = &s;
  return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const void *dO,
                              const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                              float scale, int causal, void *stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  const int BH = B * H;
  if (fa::bwd_workspace_bytes(BH, N, d) > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES)) return FA_ERR_WORKSPACE;
  NoAllocState *ns = nullptr;
  st = noalloc_state(&ns);
  if (st != FA_OK) return st;

  fa::BwdLaunch L;
  L.q = q; L.k = k; L.v = v; L.o = o; L.o_lo = nullptr; L.dO = dO; L.lse = lse;
  L.dq = dq; L.dk = dk; L.dv = dv;
  L.BH = BH; L.N = N; L.d = d; L.scale = scale; L.causal = causal;
  L.workspace = ns->scratch;
  L.status = ns->status;
  L.seq = next_seq();
  L.num_sms = ns->num_sms;
  CUtensorMap maps[7];
  if (encode_bf16(&maps[0], q, d, N, BH) || encode_bf16(&maps[1], k, d, N, BH) ||
      encode_bf16(&maps[2], v, d, N, BH) || encode_bf16(&maps[3], dO, d, N, BH) ||
      encode_3d(&maps[6], L.workspace, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, BH, 32))
    return FA_ERR_CUDA;
  cudaError_t e = fa::bwd_launch(L, maps, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The no-alloc path's failure record: its kernels write device-side wait
// timeouts into fa_noalloc_status (in the static image), which the separately
// allocated word read by fa_device_status() never sees.  These two calls read
// and clear that word, and exercise it with the bounded-wait self-test.  Like
// fa_bwd_noalloc, neither allocates device memory.
extern "C" int fa_noalloc_device_status(void *stream, int *info) {
  if (info) std::memset(info, 0, 4 * sizeof(int));
  NoAllocState *ns = nullptr;
  int st = noalloc_state(&ns);
  if (st != FA_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h[kStatusInts];
  if (cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemcpyAsync(h, ns->status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (h[0] == 0) return FA_OK;
  if (info) {
    info[0] = h[1];
    info[1] = h[2];
    info[2] = h[3];
    info[3] = h[4];
  }
  if (cudaMemsetAsync(ns->status, 0, kStatusInts * sizeof(int), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  return h[0] == fa::kStatusInternal ? FA_ERR_DEVICE_INTERNAL : FA_ERR_DEVICE_TIMEOUT;
}

extern "C" int fa_noalloc_selftest_timeout(void *stream) {
  NoAllocState *ns = nullptr;
  const int st = noalloc_state(&ns);
  if (st != FA_OK) return st;
  fa_selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ns->status, next_seq());
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

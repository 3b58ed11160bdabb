// fa_dq.cuh -- deterministic dQ for the exact-attention backward pass (sm_100a).
//
// The fused backward (fa_bwd.cuh) adds each key tile's dQ contribution into an
// fp32 accumulator in L2, in whatever order the CTAs get there: exact up to the
// order of fp32 additions, so the last bits of dQ can change from run to run.
// This kernel computes dQ query-tile-major instead, the way the forward walks
// the key tiles: one CTA per (head, 128-row query tile i) keeps dQ_i in tensor
// memory and accumulates over j = 0, 1, ... in that fixed order, so the result
// is the same bits on every run, with no atomics.  It recomputes, per key tile,
//   S    = Q_i K_j^T                       (smem x smem)  -> TMEM
//   P    = 2^(c*S - LSE_i*log2(e))         (the stored log-sum-exp)
//   dP   = dO_i V_j^T                      (smem x smem)  -> TMEM
//   dS   = P o (dP - D_i),  D_i = rowsum(dO_i o O_i)  (from the preprocess)
//   dQ_i += dS K_j                         (TMEM x smem)
// and writes dQ_i = scale * dQ_i as bf16 at the end: the chain rule through
// softmax, with the recomputation of the review's "Recomputation" section.
//
// Roles (320 threads):
//   warps 0-7  compute.  Warp w owns query rows 32*(w%4)..+31 (its TMEM lane
//              quarter) and key columns 64h..64h+63, h = w/4, of every tile.
//              A thread holds its row's LSE and D in registers.
//   warp  8    TMA producer: Q_i and dO_i once, then K_0, V_0, K_1, V_1, ...
//              through a ring of single-tile slots.
//   warp  9    MMA issuer (one elected lane) and TMEM owner.  Per key tile it issues
//              S(j+1) before dQ(j), so the compute warps start on tile j+1's
//              exponentials while dQ(j) and dP(j+1) run.
// A slot is released by the MMA that reads its tile last: V_j by dP(j), K_j by
// dQ(j).
//
// TMEM columns (512 allocated): S/dS double buffer [0,128) and [128,256), dP
// [256,384), dQ [384,384+D).  The bf16 dS of column half h (two per column) is
// written over S columns [64h, 64h+32), inside the half its warp has read, and
// is the A operand of the dQ MMA straight from TMEM.  S(j+2) reuses the buffer
// of dS(j): its MMA comes from the same thread as dQ(j), and the tensor pipe
// runs them in issue order.
#pragma once

#include "fa_bwd.cuh"
#include "ptx.cuh"

namespace fa {

struct DqParams {
  const float *ws_lse2;  // [BH, Npad]  LSE * log2(e), +inf on padded rows
  const float *ws_D;     // [BH, Npad]  rowsum(dO o O), 0 on padded rows
  int *status;
  int seq;
  int N;
  int Npad;
  int BH;
  float scale_log2;
  float scale;
};

template <int D>
struct DqCfg {
  static constexpr int kTile = 128 * D * 2;          // one 128 x D bf16 tile
  static constexpr int kBoxes = D / 64;              // 64-feature TMA boxes per tile
  static constexpr int kSlots = (D == 128) ? 5 : 8;  // K/V ring slots (one tile each)
  static constexpr int kOffQ = 0;
  static constexpr int kOffdO = kTile;
  static constexpr int kOffKV = 2 * kTile;
  static constexpr int kOffBar = kOffKV + kSlots * kTile;
  // mbarriers: qdo, kv_full[kSlots], kv_empty[kSlots], s_full[2], dp_full,
  // ds_full, dq_done, epi, drain; then the TMEM address slot and the abort flag.
  static constexpr int kNumBars = 8 + 2 * kSlots;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr int kThreads = 320;
  static constexpr int kComputeThreads = 256;
  static constexpr int kProducerWarp = 8;
  static constexpr int kIssuerWarp = 9;
  static constexpr uint32_t kColS = 0, kColdP = 256, kColdQ = 384;
};

enum DqTag : int {
  kQTagQdo = 31, kQTagKvFull = 32, kQTagKvEmpty = 33, kQTagSFull = 34, kQTagDpFull = 35, kQTagDsFull = 36,
  kQTagDqDone = 37, kQTagEpi = 38
};

// CTA -> (head, query tile): chunks of kHeadChunk heads (their K and V stay in
// L2 while the chunk runs); inside a chunk the last query tile first (the
// heaviest when causal).
__device__ __forceinline__ void dq_unit(int block, int BH, int nq, int &bh, int &i) {
  const int per_chunk = kHeadChunk * nq;
  const int c = block / per_chunk, rem = block % per_chunk;
  const int g = min(kHeadChunk, BH - c * kHeadChunk);
  i = nq - 1 - rem / g;
  bh = c * kHeadChunk + rem % g;
}

// Ring position of the key tile (load 2j) and value tile (load 2j+1) of step j.
__device__ __forceinline__ int dq_slot(int idx, int slots) { return idx % slots; }
__device__ __forceinline__ uint32_t dq_phase(int idx, int slots) { return static_cast<uint32_t>(idx / slots) & 1u; }

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    fa_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const __grid_constant__ CUtensorMap tmdQ, const DqParams p) {
  using C = DqCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *bar_qdo = bars + 0;
  uint64_t *bar_kv_full = bars + 1;               // [kSlots]
  uint64_t *bar_kv_empty = bars + 1 + C::kSlots;  // [kSlots]
  uint64_t *bar_s_full = bars + 1 + 2 * C::kSlots;  // [2]
  uint64_t *bar_dp_full = bar_s_full + 2;
  uint64_t *bar_ds_full = bar_dp_full + 1;
  uint64_t *bar_dq_done = bar_ds_full + 1;
  uint64_t *bar_epi = bar_dq_done + 1;
  uint64_t *bar_drain = bar_epi + 1;
  static_assert(8 + 2 * C::kSlots == C::kNumBars, "barrier count");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  uint8_t *sQ = smem + C::kOffQ;
  uint8_t *sdO = smem + C::kOffdO;
  uint8_t *sKV = smem + C::kOffKV;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nq = p.Npad / 128;
  int bh, i;  // head and query tile of this CTA
  dq_unit(blockIdx.x, p.BH, nq, bh, i);
  const int n_kv = CAUSAL ? i + 1 : nq;  // key tiles 0 .. n_kv-1

  const WaitCtx ctx{p.status, abort_flag, kKernelDq, p.seq};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) record_failure(ctx, kStatusInternal, 0);
    mbar_init(bar_qdo, 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    mbar_init(&bar_s_full[0], 1);
    mbar_init(&bar_s_full[1], 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_full, C::kComputeThreads);
    mbar_init(bar_dq_done, 1);
    mbar_init(bar_epi, C::kComputeThreads);
    mbar_init(bar_drain, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == C::kIssuerWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(bar_qdo, 2 * C::kTile);
      for (int b = 0; b < C::kBoxes; ++b) {
        tma_load_3d(&tmQ, bar_qdo, sQ + b * 16384, b * 64, i * 128, bh);
        tma_load_3d(&tmdO, bar_qdo, sdO + b * 16384, b * 64, i * 128, bh);
      }
      bool ok = true;
      int idx = 0;
      for (; idx < 2 * n_kv; ++idx) {
        const int s = dq_slot(idx, C::kSlots), n = idx / C::kSlots;
        if (n > 0 && !mbar_wait(ctx, &bar_kv_empty[s], (n - 1) & 1, kQTagKvEmpty)) {
          ok = false;
          break;
        }
        const int j = idx >> 1;
        uint8_t *dst = sKV + s * C::kTile;
        mbar_arrive_expect_tx(&bar_kv_full[s], C::kTile);
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d((idx & 1) ? &tmV : &tmK, &bar_kv_full[s], dst + b * 16384, b * 64, j * 128, bh);
      }
      if (!ok) {
        // Drain the copies still in flight before the CTA can exit.
        mbar_drain(bar_qdo, 0);
        for (int s = 0; s < C::kSlots && s < idx; ++s) {
          const int last = s + ((idx - 1 - s) / C::kSlots) * C::kSlots;
          mbar_drain(&bar_kv_full[s], dq_phase(last, C::kSlots));
        }
      }
    }
    __syncwarp();
  } else if (warp == C::kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (warp-uniform descriptors and TMEM
    // addresses); one elected lane issues each MMA and commit.
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    if (__all_sync(0xffffffffu, *abort_flag == 0)) {
      auto wait = [&](uint64_t *bar, int parity, int tag) {
        return __all_sync(0xffffffffu, mbar_wait(ctx, bar, static_cast<uint32_t>(parity), tag));
      };
      constexpr uint32_t id_ss = make_idesc_bf16(128, 128, 0, 0);  // S, dP (both operands K-major)
      constexpr uint32_t id_dq = make_idesc_bf16(128, D, 0, 1);    // dQ: A = dS (TMEM), B = K_j MN-major
      const uint64_t dQk = make_sdesc(smem_u32(sQ), 16, 1024);
      const uint64_t dOk = make_sdesc(smem_u32(sdO), 16, 1024);
      const uint64_t kvk0 = make_sdesc(smem_u32(sKV), 16, 1024);     // slot 0, K-major view
      const uint64_t kvm0 = make_sdesc(smem_u32(sKV), 16384, 1024);  // slot 0, MN-major view
      const uint32_t tdP = tm + C::kColdP, tdQ = tm + C::kColdQ;
      auto issue_S = [&](int j) {  // S(j) = Q_i K_j^T -> S buffer j & 1
        const uint64_t kd = sdesc_add(kvk0, dq_slot(2 * j, C::kSlots) * C::kTile);
        const uint32_t tS = tm + C::kColS + 128 * (j & 1);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_w(tS, sdesc_add(dQk, off), sdesc_add(kd, off), id_ss, ks > 0);
        }
        mma_commit_w(&bar_s_full[j & 1]);
      };
      auto issue_dP = [&](int j) {  // dP(j) = dO_i V_j^T; V_j's slot is free once it completes
        const int sv = dq_slot(2 * j + 1, C::kSlots);
        const uint64_t vd = sdesc_add(kvk0, sv * C::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_w(tdP, sdesc_add(dOk, off), sdesc_add(vd, off), id_ss, ks > 0);
        }
        mma_commit_w(bar_dp_full);
        mma_commit_w(&bar_kv_empty[sv]);
      };
      auto issue_dQ = [&](int j) {  // dQ += dS(j) K_j; K_j's slot is free once it completes
        const int sk = dq_slot(2 * j, C::kSlots);
        const uint64_t km = sdesc_add(kvm0, sk * C::kTile);
        const uint32_t tS = tm + C::kColS + 128 * (j & 1);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_w(tdQ, tS + ks * 8 + (ks >= 4 ? 32 : 0), sdesc_add(km, ks * 2048), id_dq,
                 (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit_w(&bar_kv_empty[sk]);
      };
      auto wait_kv = [&](int idx) {
        return wait(&bar_kv_full[dq_slot(idx, C::kSlots)], static_cast<int>(dq_phase(idx, C::kSlots)), kQTagKvFull);
      };
      bool ok = wait(bar_qdo, 0, kQTagQdo) && wait_kv(0) && wait_kv(1);
      if (ok) {
        tc_fence_after();
        issue_S(0);
        issue_dP(0);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 1 < n_kv) {
          ok = wait_kv(2 * j + 2);
          if (!ok) break;
          tc_fence_after();
          issue_S(j + 1);
        }
        ok = wait(bar_ds_full, j & 1, kQTagDsFull);
        if (!ok) break;
        tc_fence_after();
        issue_dQ(j);
        if (j + 1 < n_kv) {
          ok = wait_kv(2 * j + 3);
          if (!ok) break;
          tc_fence_after();
          issue_dP(j + 1);
        }
      }
      if (ok) {
        mma_commit_w(bar_dq_done);
      } else {
        // Let every MMA this warp issued finish before TMEM is released.
        mma_commit_w(bar_drain);
        mbar_drain(bar_drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute
    const int h = warp >> 2;                 // key-column half of every tile
    const int rq = warp & 3;                 // TMEM lane quarter
    const int r = rq * 32 + lane;            // query row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(rq * 32) << 16;
    const size_t srow = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * 128 + r;
    const float lse2 = p.ws_lse2[srow];  // +inf on padded rows: P = 0 there
    const float Dr = p.ws_D[srow];
    const float c = p.scale_log2;
    bool ok = !*abort_flag;
    for (int j = 0; j < n_kv && ok; ++j) {
      const uint32_t tS = tmem + lane_off + C::kColS + 128 * (j & 1) + 64 * h;
      ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_s_full[j & 1], (j >> 1) & 1, kQTagSFull));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(tS, sv);
      tmem_ld32(tS + 32, sv + 32);
      tmem_wait_ld();
      // Keys j*128 + 64h + cc are valid when cc < nv (tail of N, causal diagonal).
      int nvalid = min(128, p.N - j * 128);
      if (CAUSAL && j == i) nvalid = min(nvalid, r + 1);
      const int nv = nvalid - 64 * h;
      float pf[64];
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) pf[cc] = cc < nv ? ex2(fmaf(__uint_as_float(sv[cc]), c, -lse2)) : 0.f;
      ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dp_full, j & 1, kQTagDpFull));
      if (!ok) break;
      tc_fence_after();
      uint32_t dsk[32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dp[32];
        tmem_ld32(tmem + lane_off + C::kColdP + 64 * h + 32 * ch, dp);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int c0 = 32 * ch + 2 * t;
          dsk[16 * ch + t] = pack_bf16(pf[c0] * (__uint_as_float(dp[2 * t]) - Dr),
                                       pf[c0 + 1] * (__uint_as_float(dp[2 * t + 1]) - Dr));
        }
      }
      tmem_st32(tS, dsk);  // inside the columns this warp has read
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_ds_full);
    }
    // ---------------------------------------------------------- epilogue
    // Once the last dQ MMA has completed no MMA or load is in flight, so the Q
    // buffer is free: dQ_i * scale is staged there (swizzled) and written by TMA.
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dq_done, 0, kQTagDqDone));
    if (ok) {
      tc_fence_after();
      const uint32_t st = smem_u32(sQ);
      const uint32_t tdQ = tmem + lane_off + C::kColdQ;
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) {
        const int col0 = h * (D / 2) + 32 * ch;  // first feature of this 32-column chunk
        uint32_t a[32], w[16];
        tmem_ld32(tdQ + col0, a);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 16; ++t)
          w[t] = pack_bf16(__uint_as_float(a[2 * t]) * p.scale, __uint_as_float(a[2 * t + 1]) * p.scale);
        const int box = col0 >> 6, chunk0 = (col0 & 63) >> 3;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          st_shared_v4(st + box * 16384 + bsw128(r, chunk0 + t), w[4 * t], w[4 * t + 1], w[4 * t + 2],
                       w[4 * t + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_epi);
      if (threadIdx.x == 0 && mbar_wait(ctx, bar_epi, 0, kQTagEpi)) {
        for (int b = 0; b < C::kBoxes; ++b) tma_store_3d(&tmdQ, sQ + b * 16384, b * 64, i * 128, bh);
        bulk_commit();
        bulk_wait_read<0>();
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::kIssuerWarp) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ host side
template <int D, bool CAUSAL>
inline cudaError_t dq_set_attribute() {
  return cudaFuncSetAttribute(fa_dq_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              DqCfg<D>::kSmemBytes);
}

inline cudaError_t dq_set_attributes() {
  const cudaError_t es[4] = {dq_set_attribute<64, false>(), dq_set_attribute<64, true>(),
                             dq_set_attribute<128, false>(), dq_set_attribute<128, true>()};
  for (cudaError_t e : es)
    if (e != cudaSuccess) return e;
  return cudaSuccess;
}

template <int D, bool CAUSAL>
inline void dq_launch(const CUtensorMap *m, const CUtensorMap &tmdQ, const DqParams &p, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.Npad / 128));
  fa_dq_kernel<D, CAUSAL><<<grid, DqCfg<D>::kThreads, DqCfg<D>::kSmemBytes, s>>>(m[0], m[1], m[2], m[3], tmdQ, p);
}

// The deterministic backward: the preprocess (D, LSE * log2(e)), the fused
// kernel for dK and dV (its dQ additions land in the workspace accumulator and
// are not used), then fa_dq_kernel for dQ.  dK and dV are the fused kernel's,
// bit for bit; dQ no longer depends on the order in which CTAs finish.
// maps: as for bwd_launch; tmdQ: the bf16 dQ output (3-D, 64-feature boxes).
inline cudaError_t bwd_launch_deterministic(const BwdLaunch &L, const CUtensorMap *maps, const CUtensorMap &tmdQ,
                                            cudaStream_t s) {
  const int Npad = pad128(L.N);
  float *ws_dq = static_cast<float *>(L.workspace);
  float *ws_lse2 = ws_dq + static_cast<size_t>(L.BH) * L.N * L.d;
  float *ws_D = ws_lse2 + static_cast<size_t>(L.BH) * Npad;
  int *counter = reinterpret_cast<int *>(static_cast<uint8_t *>(L.workspace) +
                                         bwd_workspace_main_bytes(L.BH, L.N, L.d));
  const int pre_grid = L.num_sms * 8;
  // No dQ accumulator here (dQ comes from fa_dq_kernel): nullptr skips its zeroing.
  if (L.d == 64)
    fa_bwd_pre_kernel<64><<<pre_grid, 256, 0, s>>>(static_cast<const uint16_t *>(L.o),
                                                   static_cast<const uint16_t *>(L.o_lo),
                                                   static_cast<const uint16_t *>(L.dO), L.lse, ws_D, ws_lse2, nullptr, counter,
                                                   L.N, Npad, L.BH);
  else
    fa_bwd_pre_kernel<128><<<pre_grid, 256, 0, s>>>(static_cast<const uint16_t *>(L.o),
                                                    static_cast<const uint16_t *>(L.o_lo),
                                                    static_cast<const uint16_t *>(L.dO), L.lse, ws_D, ws_lse2, nullptr, counter,
                                                    L.N, Npad, L.BH);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BwdParams p;
  p.drop = DropoutParams{0u, 0u, 0u, 0u, 1.f};
  p.ws_lse2 = ws_lse2;
  p.ws_D = ws_D;
  p.ws_dq = ws_dq;
  p.unit_counter = counter;
  p.dk = static_cast<uint16_t *>(L.dk);
  p.dv = static_cast<uint16_t *>(L.dv);
  p.status = L.status;
  p.seq = L.seq;
  p.N = L.N;
  p.Npad = Npad;
  p.BH = L.BH;
  p.scale_log2 = L.scale * 1.4426950408889634f;
  p.scale = L.scale;
  const int nkv = Npad / 128;
  // dK, dV from the fused kernel without its dQ product (NO_DQ).
  if (L.d == 64)
    L.causal ? bwd_main_launch<64, true, false, true>(maps, p, nkv, L.num_sms, s)
             : bwd_main_launch<64, false, false, true>(maps, p, nkv, L.num_sms, s);
  else
    L.causal ? bwd_main_launch<128, true, false, true>(maps, p, nkv, L.num_sms, s)
             : bwd_main_launch<128, false, false, true>(maps, p, nkv, L.num_sms, s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DqParams q;
  q.ws_lse2 = ws_lse2;
  q.ws_D = ws_D;
  q.status = L.status;
  q.seq = L.seq;
  q.N = L.N;
  q.Npad = Npad;
  q.BH = L.BH;
  q.scale_log2 = p.scale_log2;
  q.scale = L.scale;
  if (L.d == 64)
    L.causal ? dq_launch<64, true>(maps, tmdQ, q, s) : dq_launch<64, false>(maps, tmdQ, q, s);
  else
    L.causal ? dq_launch<128, true>(maps, tmdQ, q, s) : dq_launch<128, false>(maps, tmdQ, q, s);
  return cudaGetLastError();
}

}  // namespace fa

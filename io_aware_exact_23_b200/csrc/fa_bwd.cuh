// fa_bwd.cuh -- exact-attention backward pass for sm_100a.
//
// The backward pass keeps no N x N matrix either: following the review's
// "Recomputation" section, it rebuilds S and P tile by tile from Q, K and the
// stored log-sum-exp, P_ij = 2^(c*S_ij - LSE_i*log2(e)).  The gradients are the
// chain rule through softmax:
//   dV = P^T dO,  dP = dO V^T,  dS = P o (dP - D),  D_i = sum_k dO_ik O_ik,
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three kernels on one stream:
//   1. fa_bwd_pre_kernel   D_i = rowsum(dO o O) (O = o + o_lo when the forward
//                          wrote its rounding residual) and LSE_i*log2(e) into the
//                          workspace (padded to whole 128-row tiles), and zero
//                          the fp32 dQ accumulator.
//   2. fa_bwd_kernel       one CTA per (head, 128-row key tile j): K_j, V_j stay
//                          in smem, dK_j and dV_j accumulate in TMEM while the
//                          CTA walks the query tiles; each query tile's dQ
//                          contribution is added into the fp32 accumulator.
//   3. fa_dq_convert_kernel  dQ (bf16) = accumulator.
//
// fa_bwd_kernel roles (448 threads at d = 64; 320 at d = 128 and without dQ):
//   warps 0-3   compute, query columns 0..63 of each tile (thread = key row)
//   warps 4-7   compute, query columns 64..127
//   dQ drain    TMEM dQ rows -> registers (TMEM released at once) -> scale ->
//               the Q_i / dO_i stage buffers of the finished tile (together
//               exactly one fp32 dQ tile) -> TMA bulk reduce-add into the fp32
//               accumulator in L2, then the stage goes back to the producer.
//               At d = 64 four warps (8-11) do it, their leader issuing the
//               reduce-add; at d = 128 the compute warps stage dQ themselves
//               after each tile's dS and the producer issues the reduce-add.
//   producer    (warp 12 / 8) TMA: K_j, V_j once; Q_i, dO_i, LSE_i, D_i per
//               tile (2 stages)
//   issuer      (warp 13 / 9) MMAs (one elected lane), five per query tile:
//                 S^T  = K_j Q_i^T      (smem x smem)      -> TMEM
//                 dP^T = V_j dO_i^T     (smem x smem)      -> TMEM
//                 dV  += P^T dO_i       (TMEM x smem)
//                 dK  += dS^T Q_i       (smem x smem)
//                 dQ_i = dS K_j         (smem x smem, dS read transposed)
//
// TMEM columns (512): S^T [0,128) with P^T (bf16) of query columns 64w..64w+63
// over S^T columns [64w, 64w+32) (w = 0, 1: the half each compute warp reads);
// dP^T [128,256); dK [256,256+D); dV [256+D,256+2D); dQ reuses dP^T's columns
// when D = 128 (dP^T is dead once dS is formed) and [384,448) when D = 64.
// dS^T (bf16) is written to smem in the 128-byte-swizzled K-major layout,
// which is at the same time the MN-major layout of dS for the dQ MMA.
// CTAs are ordered in chunks of kHeadChunk heads, heaviest key tiles first
// within a chunk: the fp32 dQ rows of a chunk stay resident in L2 while its
// key tiles add into them.
#pragma once

#include "dropout.cuh"
#include "ptx.cuh"

namespace fa {

struct BwdParams {
  const float *ws_lse2;  // [BH, Npad]  LSE * log2(e), +inf on padded rows
  const float *ws_D;     // [BH, Npad]  rowsum(dO o O), 0 on padded rows
  float *ws_dq;          // [BH, N, D]  fp32 dQ accumulator (zeroed by the preprocess)
  int *unit_counter;     // units handed out past the first wave (zeroed by the preprocess)
  uint16_t *dk, *dv;     // [BH, N, D]  bf16 outputs
  int *status;
  int seq;
  int N;
  int Npad;
  int BH;
  float scale_log2;
  float scale;
  DropoutParams drop;  // read only by the DROPOUT instantiations
};

constexpr int kHeadChunk = 8;  // heads whose CTAs are scheduled together

// CTA -> (head, key tile): chunks of kHeadChunk heads; inside a chunk all heads'
// key tile 0 first, then tile 1, ... (tile 0 is the heaviest when causal).
__device__ __forceinline__ void bwd_unit(int block, int BH, int nkv, int &bh, int &j) {
  const int per_chunk = kHeadChunk * nkv;
  const int c = block / per_chunk, rem = block % per_chunk;
  const int g = min(kHeadChunk, BH - c * kHeadChunk);
  j = rem / g;
  bh = c * kHeadChunk + rem % g;
}

template <int D>
struct BwdCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  // Q_i / dO_i stages: three at d = 64, where shared memory has room, so that a
  // stage's reload (behind the drain of the tile two back) has a tile of slack;
  // two at d = 128, where shared memory is full.
  static constexpr int kQStages = (D == 64) ? 3 : 2;
  static constexpr int kOffQ = 2 * kTile;                 // [kQStages]
  static constexpr int kOffdO = (2 + kQStages) * kTile;   // [kQStages]
  static constexpr int kOffdS = (2 + 2 * kQStages) * kTile;  // 128 x 128 bf16
  static constexpr int kOffL = kOffdS + 32768;                // [kQStages][128] fp32
  static constexpr int kOffDv = kOffL + 512 * kQStages;       // [kQStages][128] fp32
  static constexpr int kOffBar = kOffDv + 512 * kQStages;
  // then the TMEM address slot, the abort flag and the two-slot unit ring
  static constexpr int kNumBars = 3 * kQStages + 14;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr uint32_t kColS = 0, kColdP = 128, kColdK = 256, kColdV = 256 + D;
  static constexpr uint32_t kColdQ = (D == 128) ? 128 : 384;
};

// Warp roles.  With the dQ product at d = 64 there are four drain warps (8-11)
// that stage each tile's dQ for the reduce-add.  At d = 128 the compute warps
// drain dQ themselves, in the time they would otherwise spend waiting for dK,
// dQ and the next S^T, and the producer reduce-adds the staged tile just before
// it reloads that stage; without the dQ product (the deterministic mode) there
// is nothing to drain.  Either way ten warps, and up to 168 registers a thread.
template <int D, bool NO_DQ>
struct BwdRoles {
  static constexpr bool kComputeDrain = (D == 128) || NO_DQ;
  static constexpr int kThreads = kComputeDrain ? 320 : 448;
  static constexpr int kProducerWarp = kComputeDrain ? 8 : 12;
  static constexpr int kIssuerWarp = kComputeDrain ? 9 : 13;
};

enum BwdTag : int {
  kBTagKV = 11, kBTagQdoFull = 12, kBTagQdoEmpty = 13, kBTagSFull = 14, kBTagDpFull = 15, kBTagPFull = 16,
  kBTagDsFull = 17, kBTagDvDone = 18, kBTagDkqDone = 19, kBTagDqEmpty = 20, kBTagEpi = 21, kBTagDrained = 22,
  kBTagStage = 23, kBTagUnit = 24
};

__device__ __forceinline__ uint32_t bsw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ----------------------------------------------------------- preprocess
// Lanes-per-row = D / 8 (each lane handles 8 features = 16 bytes).
template <int D>
__global__ void __launch_bounds__(256, 4) fa_bwd_pre_kernel(const uint16_t *__restrict__ o,
                                                         const uint16_t *__restrict__ o_lo,
                                                         const uint16_t *__restrict__ dO,
                                                         const float *__restrict__ lse, float *__restrict__ ws_D,
                                                         float *__restrict__ ws_lse2, float *__restrict__ ws_dq,
                                                         int *__restrict__ unit_counter, int N, int Npad, int BH) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *unit_counter = 0;
  constexpr int LPR = D / 8;     // lanes per row, 16 bytes each
  constexpr int RPW = 32 / LPR;  // rows per warp pass
  constexpr int U = 4;           // passes whose loads are in flight together
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, part = lane % LPR;
  const long warps = static_cast<long>(gridDim.x) * (blockDim.x / 32);
  const long gw = static_cast<long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const long rows = static_cast<long>(BH) * Npad;
  const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
  for (long base = gw * RPW * U; base < rows; base += warps * RPW * U) {
    uint4 a[U], b[U], c[U];
    bool valid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long row = base + u * RPW + sub;
      const int bh = row < rows ? static_cast<int>(row / Npad) : 0;
      const int i = row < rows ? static_cast<int>(row % Npad) : 0;
      valid[u] = row < rows && i < N;
      a[u] = b[u] = c[u] = zero4;
      if (valid[u]) {
        const size_t off = (static_cast<size_t>(bh) * N + i) * D + part * 8;
        a[u] = *reinterpret_cast<const uint4 *>(o + off);
        b[u] = *reinterpret_cast<const uint4 *>(dO + off);
        if (o_lo != nullptr) c[u] = *reinterpret_cast<const uint4 *>(o_lo + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t av[4] = {a[u].x, a[u].y, a[u].z, a[u].w}, bv[4] = {b[u].x, b[u].y, b[u].z, b[u].w};
      const uint32_t cv[4] = {c[u].x, c[u].y, c[u].z, c[u].w};
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        // O = o + o_lo when the forward wrote its rounding residual.
        const float b_lo = __uint_as_float(bv[t] << 16), b_hi = __uint_as_float(bv[t] & 0xFFFF0000u);
        acc = fmaf(__uint_as_float(av[t] << 16), b_lo, acc);
        acc = fmaf(__uint_as_float(av[t] & 0xFFFF0000u), b_hi, acc);
        if (o_lo != nullptr) {
          acc = fmaf(__uint_as_float(cv[t] << 16), b_lo, acc);
          acc = fmaf(__uint_as_float(cv[t] & 0xFFFF0000u), b_hi, acc);
        }
      }
#pragma unroll
      for (int w = LPR / 2; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
      const long row = base + u * RPW + sub;
      if (row < rows && part == 0) {
        const int bh = static_cast<int>(row / Npad), i = static_cast<int>(row % Npad);
        ws_D[row] = valid[u] ? acc : 0.f;
        ws_lse2[row] = valid[u] ? lse[static_cast<size_t>(bh) * N + i] * 1.4426950408889634f : INFINITY;
      }
    }
  }
  if (ws_dq == nullptr) return;  // no dQ accumulator to zero (the deterministic mode)
  const long n4 = static_cast<long>(BH) * N * D / 4;
  const long tid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long nthreads = static_cast<long>(gridDim.x) * blockDim.x;
  float4 *z = reinterpret_cast<float4 *>(ws_dq);
  for (long t = tid; t < n4; t += nthreads) z[t] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// --------------------------------------------------------- dQ conversion
__global__ void __launch_bounds__(256) fa_dq_convert_kernel(const float *__restrict__ ws_dq,
                                                            uint16_t *__restrict__ dq, long n4) {
  constexpr int U = 4;  // loads in flight per thread
  const long tid = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long nthreads = static_cast<long>(gridDim.x) * blockDim.x;
  const float4 *src = reinterpret_cast<const float4 *>(ws_dq);
  uint2 *dst = reinterpret_cast<uint2 *>(dq);
  for (long t0 = tid; t0 < n4; t0 += nthreads * U) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long t = t0 + u * nthreads;
      v[u] = t < n4 ? __ldcs(src + t) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long t = t0 + u * nthreads;
      if (t < n4) dst[t] = make_uint2(pack_bf16(v[u].x, v[u].y), pack_bf16(v[u].z, v[u].w));
    }
  }
}

// ------------------------------------------------------------ main kernel
// NO_DQ: the instantiation of the deterministic mode, whose dQ comes from
// fa_dq_kernel.  It skips the dQ product and its drain; dK(i) then closes each
// query tile (its commit takes the place of dQ(i)'s), the issue order is
// S^T(0) dP^T(0) | dV(i) S^T(i+1) dK(i) dP^T(i+1) | ... at both head dims, and
// the producer reloads each Q_i / dO_i stage once dK(i) has completed.
//
// Persistent CTAs: the grid holds one CTA per SM (or one per unit, if fewer);
// CTA c starts on unit c and then takes units from a counter in the workspace,
// in the same heaviest-first order, each when its current unit is nearly done.  Every per-tile barrier phase and stage
// runs on t, the CTA's count of query tiles over all its units.  The producer
// hands each unit to the other roles through a two-slot ring in shared memory,
// loads the next unit's K_j and V_j once the previous unit's last dK / dQ have
// completed (after its first query tile), and its stage reloads carry on across
// units; the next unit's first MMAs overlap the previous unit's last dQ
// reduce-adds and its epilogue.  A unit's first dV and dK overwrite the
// accumulators, but they follow P and dS of its first tile, which the compute
// warps produce only after the previous epilogue has read them.
template <int D, bool CAUSAL, bool DROPOUT = false, bool NO_DQ = false>
__global__ void __launch_bounds__(BwdRoles<D, NO_DQ>::kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
  using C = BwdCfg<D>;
  using R = BwdRoles<D, NO_DQ>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (threadIdx.x == 0) FA_TRACE(1);

  constexpr int S = C::kQStages;  // query tile t sits in stage t % S
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *bar_kv = bars + 0;
  // At d = 64 a stage's loads land on two barriers: Q_i and LSE_i on q_full, dO_i
  // and D_i on do_full, so that S^T(i) (and P) need not wait for the dO half
  // (1.03-1.07x there).  At d = 128 the split measured slower (0.97-0.99x: S^T(i)
  // waits for the issuer's turn behind tile i-1, not for the load) and all four
  // loads land on q_full.
  constexpr bool kSplitStage = (D == 64);
  uint64_t *bar_q_full = bars + 1;             // [S]
  uint64_t *bar_do_full = bars + 1 + S;        // [S], d = 64
  uint64_t *bar_qdo_empty = bars + 1 + 2 * S;  // [S] drain-warp layout: the stage is free again
  // [S] compute-drain layout: every compute thread staged its dQ part; without
  // dQ, the issuer's commit after dK(t).  (A per-stage barrier: a wait on it
  // cannot fall two phases behind, which one on dkq_done could across units.)
  uint64_t *bar_staged = bar_qdo_empty;
  uint64_t *bar_s_full = bars + 1 + 3 * S;
  uint64_t *bar_dp_full = bar_s_full + 1;
  uint64_t *bar_p_full = bar_s_full + 2;
  uint64_t *bar_ds_full = bar_s_full + 3;
  uint64_t *bar_dkq_done = bar_s_full + 4;
  uint64_t *bar_dq_empty = bar_s_full + 5;
  uint64_t *bar_drain = bar_s_full + 6;
  uint64_t *bar_stage = bar_s_full + 7;       // dQ drain warps: all 128 rows staged
  uint64_t *bar_unit_full = bar_s_full + 8;   // [2] unit ring: the producer wrote the slot
  uint64_t *bar_unit_empty = bar_s_full + 10; // [2] unit ring: every consumer warp read it
  uint64_t *bar_kv_free = bar_s_full + 12;    // a unit's last MMA completed: K_j, V_j are dead
  static_assert(1 + 3 * S + 13 == C::kNumBars, "barrier count");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + C::kNumBars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *unit_ring = reinterpret_cast<volatile int *>(tmem_slot + 2);  // [2]

  uint8_t *sK = smem + C::kOffK;
  uint8_t *sV = smem + C::kOffV;
  uint8_t *sQ = smem + C::kOffQ;
  uint8_t *sdO = smem + C::kOffdO;
  uint8_t *sdS = smem + C::kOffdS;
  float *sL = reinterpret_cast<float *>(smem + C::kOffL);
  float *sDv = reinterpret_cast<float *>(smem + C::kOffDv);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nq = (p.N + 127) / 128;
  const int n_units = p.BH * nq;
  constexpr int kConsumerWarps = 1 + 8 + (R::kComputeDrain ? 0 : 4);  // issuer, compute, drain

  const WaitCtx ctx{p.status, abort_flag, kKernelBwd, p.seq};

  // Query tile i of head bh into stage t % S: Q and LSE*log2(e) on q_full; dO and
  // D on do_full (d = 64) or on q_full as well (d = 128).
  auto load_tile = [&](int t, int bh, int i) {
    const int s = t % S;
    uint64_t *bq = &bar_q_full[s];
    uint64_t *bd = kSplitStage ? &bar_do_full[s] : bq;
    if constexpr (kSplitStage) {
      mbar_arrive_expect_tx(bq, C::kTile + 512);
      mbar_arrive_expect_tx(bd, C::kTile + 512);
    } else {
      mbar_arrive_expect_tx(bq, 2 * C::kTile + 1024);
    }
    for (int b = 0; b < C::kBoxes; ++b) {
      tma_load_3d(&tmQ, bq, sQ + s * C::kTile + b * 16384, b * 64, i * 128, bh);
      tma_load_3d(&tmdO, bd, sdO + s * C::kTile + b * 16384, b * 64, i * 128, bh);
    }
    const size_t soff = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * 128;
    bulk_load_1d(sL + s * 128, p.ws_lse2 + soff, 512, bq);
    bulk_load_1d(sDv + s * 128, p.ws_D + soff, 512, bd);
  };
  // Key tile j of head bh: K_j, V_j.
  auto load_kv = [&](int bh, int j) {
    mbar_arrive_expect_tx(bar_kv, 2 * C::kTile);
    for (int b = 0; b < C::kBoxes; ++b) {
      tma_load_3d(&tmK, bar_kv, sK + b * 16384, b * 64, j * 128, bh);
      tma_load_3d(&tmV, bar_kv, sV + b * 16384, b * 64, j * 128, bh);
    }
  };

  // The producer thread sets up the barriers and starts the first unit's loads
  // (its first query tile, K_j, V_j) before the block-wide barrier, so that they
  // overlap the TMEM allocation and the other warps' start.
  if (warp == R::kProducerWarp && lane == 0) {
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) record_failure(ctx, kStatusInternal, 0);
    mbar_init(bar_kv, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar_q_full[s], 1);
      mbar_init(&bar_do_full[s], 1);
      // bar_staged in the compute-drain layout: 256 stagers, or the issuer's commit
      mbar_init(&bar_qdo_empty[s], R::kComputeDrain ? (NO_DQ ? 1 : 256) : 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_unit_full[s], 1);
      mbar_init(&bar_unit_empty[s], kConsumerWarps);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_full, 256);
    mbar_init(bar_ds_full, 256);
    mbar_init(bar_dkq_done, 1);
    mbar_init(bar_dq_empty, R::kComputeDrain ? 256 : 128);
    mbar_init(bar_drain, 1);
    mbar_init(bar_stage, 128);
    mbar_init(bar_kv_free, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmdO);
    if (static_cast<int>(blockIdx.x) < n_units) {
      int bh, j;
      bwd_unit(blockIdx.x, p.BH, nq, bh, j);
      load_tile(0, bh, CAUSAL ? j : 0);
      load_kv(bh, j);
    }
  }
  if (warp == R::kIssuerWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) FA_TRACE(0);

  // A consumer warp (all lanes) takes unit u from the ring: its index, or -1 (no
  // more units), broadcast from lane 0 so that the compiler knows it is
  // warp-uniform.
  auto take_unit = [&](int u, int &unit) -> bool {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_unit_full[u & 1], (u >> 1) & 1, kBTagUnit));
    if (!ok) return false;
    unit = __shfl_sync(0xffffffffu, unit_ring[u & 1], 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_unit_empty[u & 1]);
    return true;
  };

  if (warp == R::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort_flag) {
      bool ok = true;
      int t = 0;            // query tiles handled so far, over all units
      int n_loaded = 0;     // query tiles whose loads were issued
      int n_kv = 0;         // K/V loads issued
      int stage_row[S] = {}, stage_bh[S] = {};  // the tile each stage holds
      // Compute-drain layout: query tile tt's stage is reloaded (for tile tt + S)
      // once the tile is done with -- after the issuer's commit behind dK(tt)
      // without the dQ product; else once every compute thread has staged its
      // part of dQ(tt) there and this thread has reduce-added the staged tile into
      // the accumulator and TMA has read it.  (Reloading Q as soon as the Q
      // buffer's half had been read measured no faster: at d = 128, S^T(tt + S)
      // waits for the issuer's turn behind tile tt + S - 1, not for the stage.)
      // reload = false: the last S tiles, with no load behind them.
      auto free_stage = [&](int tt, bool reload, int bh, int i) -> bool {
        const int st = tt % S;
        if (tt < 256) FA_TRACE(3000 + tt * 3 + 0);
        if (!mbar_wait(ctx, &bar_staged[st], (tt / S) & 1, kBTagStage)) return false;
        if (tt < 256) FA_TRACE(3000 + tt * 3 + 1);
        if constexpr (!NO_DQ) {
          for (int half = 0; half < 2; ++half)
            for (int b = 0; b < D / 64; ++b)
              tma_reduce_add_3d(&tmdQacc, (half == 0 ? sQ : sdO) + st * C::kTile + b * 16384,
                                half * (D / 2) + 32 * b, stage_row[st], stage_bh[st]);
          bulk_commit();
          bulk_wait_read<0>();
          if (tt < 256) FA_TRACE(3000 + tt * 3 + 2);
        }
        if (reload) load_tile(tt + S, bh, i);
        return true;
      };
      int unit = static_cast<int>(blockIdx.x) < n_units ? static_cast<int>(blockIdx.x) : -1;
      for (int u = 0; ok; ++u) {
        // Hand unit u (or the end, -1) to the other roles.
        if (u >= 2 && !(ok = mbar_wait(ctx, &bar_unit_empty[u & 1], ((u >> 1) - 1) & 1, kBTagUnit))) break;
        unit_ring[u & 1] = unit;
        mbar_arrive(&bar_unit_full[u & 1]);
        if (unit < 0) break;
        int bh, j;
        bwd_unit(unit, p.BH, nq, bh, j);
        const int i0 = CAUSAL ? j : 0, n_it = nq - i0;
        for (int it = 0; it < n_it; ++it) {
          const int s = t % S, n = t / S;
          if (u == 0 && it == 0) {  // loaded before the block-wide barrier
            n_loaded = n_kv = 1;
          } else {
            if constexpr (R::kComputeDrain) {
              if (t >= S) {
                if (!(ok = free_stage(t - S, true, bh, i0 + it))) break;
              } else {
                load_tile(t, bh, i0 + it);
              }
            } else {
              if (n > 0 && !(ok = mbar_wait(ctx, &bar_qdo_empty[s], (n - 1) & 1, kBTagQdoEmpty))) break;
              load_tile(t, bh, i0 + it);
            }
            ++n_loaded;
            if (it == 0) {
              // K_j, V_j of this unit, once every MMA of the previous one has
              // completed (the issuer's per-unit commit; a wait on dkq_done could
              // miss its phase, with three stages this thread runs far enough
              // ahead).  The wait cannot alias: the next commit needs this load.
              if (!(ok = mbar_wait(ctx, bar_kv_free, (u - 1) & 1, kBTagKV))) break;
              load_kv(bh, j);
              ++n_kv;
            }
          }
          stage_row[s] = (i0 + it) * 128;
          stage_bh[s] = bh;
          ++t;
        }
        if (!ok) break;
        // The next unit is claimed once this one's last tile is loaded, a tile or
        // two before it ends: claimed earlier, it would wait behind this unit while
        // other CTAs run dry (heaviest-first order needs claims at finish time), and
        // the atomic's latency still hides behind the remaining tiles.
        unit = static_cast<int>(gridDim.x) + atomicAdd(p.unit_counter, 1);
        if (unit >= n_units) unit = -1;
      }
      if constexpr (R::kComputeDrain && !NO_DQ) {
        // The last S tiles have no load behind them: reduce-add their staged dQ
        // here.  (Without the dQ product there is nothing to wait for.)
        for (int tt = t >= S ? t - S : 0; tt < t && ok; ++tt) ok = free_stage(tt, false, 0, 0);
        bulk_wait<0>();  // every reduction has landed before the CTA exits
      }
      // The last loads have landed before the CTA can exit (immediate unless a
      // consumer gave up before taking them).
      if (n_kv > 0) mbar_drain(bar_kv, (n_kv - 1) & 1);
      for (int s = 0; s < S && s < n_loaded; ++s) {
        const int last = s + ((n_loaded - 1 - s) / S) * S;
        mbar_drain(&bar_q_full[s], (last / S) & 1);
        if (kSplitStage) mbar_drain(&bar_do_full[s], (last / S) & 1);
      }
    }
    __syncwarp();
  } else if (warp == R::kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop, so that its descriptors and TMEM
    // addresses are warp-uniform values; one elected lane issues each MMA and
    // commit (the warp-wide forms in ptx.cuh).
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    if (__all_sync(0xffffffffu, *abort_flag == 0)) {
      auto wait = [&](uint64_t *bar, int parity, int tag) {
        return __all_sync(0xffffffffu, mbar_wait(ctx, bar, static_cast<uint32_t>(parity), tag));
      };
      constexpr uint32_t id_ss = make_idesc_bf16(128, 128, 0, 0);     // S^T, dP^T
      constexpr uint32_t id_kxmn = make_idesc_bf16(128, D, 0, 1);     // dV (A in TMEM), dK
      constexpr uint32_t id_mnmn = make_idesc_bf16(128, D, 1, 1);     // dQ
      // Base descriptors (K-major "k" and MN-major "m" views), advanced per k-step.
      const uint64_t dKk = make_sdesc(smem_u32(sK), 16, 1024), dKm = make_sdesc(smem_u32(sK), 16384, 1024);
      const uint64_t dVk = make_sdesc(smem_u32(sV), 16, 1024);
      const uint64_t dSk = make_sdesc(smem_u32(sdS), 16, 1024), dSm = make_sdesc(smem_u32(sdS), 16384, 1024);
      const uint64_t dQk0 = make_sdesc(smem_u32(sQ), 16, 1024), dQm0 = make_sdesc(smem_u32(sQ), 16384, 1024);
      const uint64_t dOk0 = make_sdesc(smem_u32(sdO), 16, 1024), dOm0 = make_sdesc(smem_u32(sdO), 16384, 1024);
      const uint32_t tS = tm + C::kColS, tdP = tm + C::kColdP, tdK = tm + C::kColdK;
      const uint32_t tdV = tm + C::kColdV, tdQ = tm + C::kColdQ;
      // t: the tile's index over all units (its stage is t % 2); acc: accumulate
      // into dK / dV (false for a unit's first query tile).
      auto issue_sT = [&](int t) {  // S^T = K_j Q_i^T
        const uint64_t dQk = sdesc_add(dQk0, (t % S) * C::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_w(tS, sdesc_add(dKk, off), sdesc_add(dQk, off), id_ss, ks > 0);
        }
        mma_commit_w(bar_s_full);
        if (lane == 0) FA_TRACE(16 + t * 8 + 0);
      };
      auto issue_dPT = [&](int t) {  // dP^T = V_j dO_i^T
        const uint64_t dOk = sdesc_add(dOk0, (t % S) * C::kTile);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_w(tdP, sdesc_add(dVk, off), sdesc_add(dOk, off), id_ss, ks > 0);
        }
        mma_commit_w(bar_dp_full);
        if (lane == 0) FA_TRACE(16 + t * 8 + 1);
      };
      auto issue_dV = [&](int t, bool acc) {  // dV += P^T dO_i; P^T of query columns 64w.. at S^T columns 64w..64w+31
        const uint64_t dOm = sdesc_add(dOm0, (t % S) * C::kTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ts_w(tdV, tS + ks * 8 + (ks >= 4 ? 32 : 0), sdesc_add(dOm, ks * 2048), id_kxmn,
                 (acc || ks > 0) ? 1u : 0u);
        if (lane == 0) FA_TRACE(16 + t * 8 + 2);
      };
      auto issue_dK = [&](int t, bool acc) {  // dK += dS^T Q_i
        const uint64_t dQm = sdesc_add(dQm0, (t % S) * C::kTile);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_ss_w(tdK, sdesc_add(dSk, off), sdesc_add(dQm, ks * 2048), id_kxmn, (acc || ks > 0) ? 1u : 0u);
        }
      };
      auto issue_dQ = [&](int t) {  // dQ_i = dS K_j; the dQ drain releases the Q/dO stage after staging through it
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss_w(tdQ, sdesc_add(dSm, ks * 2048), sdesc_add(dKm, ks * 2048), id_mnmn, ks > 0);
        mma_commit_w(bar_dkq_done);
        if (lane == 0) FA_TRACE(16 + t * 8 + 3);
      };
      // Tile t's Q and LSE (for S^T, dK) and its dO and D (for dP^T, dV).
      auto wait_q = [&](int t) { return wait(&bar_q_full[t % S], (t / S) & 1, kBTagQdoFull); };
      auto wait_do = [&](int t) { return !kSplitStage || wait(&bar_do_full[t % S], (t / S) & 1, kBTagQdoFull); };
      // S^T(i+1) overwrites P^T(i), which dV(i) reads, and dP^T(i+1) the dP^T(i)
      // the compute warps have turned into dS(i): neither waits for an MMA to
      // complete, since one lane issues them all and the pipe runs them in order.
      bool ok = true;
      int t = 0;  // query tiles issued so far, over all units
      for (int u = 0; ok; ++u) {
        int unit;
        if (!(ok = take_unit(u, unit))) break;
        if (unit < 0) break;
        int bh, j;
        bwd_unit(unit, p.BH, nq, bh, j);
        const int n_it = nq - (CAUSAL ? j : 0), t0 = t;
        if (!(ok = wait(bar_kv, u & 1, kBTagKV))) break;
        if (NO_DQ || D == 64) {
          // Order S^T(0) dP^T(0) | dV(i) S^T(i+1) dK(i) [dQ(i)] dP^T(i+1) | ...: the
          // next tile's S^T goes in ahead of dK(i) (and dQ(i), which has columns of
          // its own at d = 64), so the compute warps start tile i+1 while those run.
          // Without dQ, dK(i)'s commit closes the tile and frees its stage.
          if (!(ok = wait_q(t0))) break;
          tc_fence_after();
          issue_sT(t0);
          if (!(ok = wait_do(t0))) break;
          tc_fence_after();
          issue_dPT(t0);
          for (int it = 0; it < n_it && ok; ++it) {
            t = t0 + it;
            if (!(ok = wait(bar_p_full, t & 1, kBTagPFull))) break;
            tc_fence_after();
            issue_dV(t, it > 0);
            if (it + 1 < n_it) {
              if (!(ok = wait_q(t + 1))) break;
              tc_fence_after();
              issue_sT(t + 1);
            }
            if (!(ok = wait(bar_ds_full, t & 1, kBTagDsFull))) break;
            tc_fence_after();
            issue_dK(t, it > 0);
            if constexpr (NO_DQ) {
              mma_commit_w(bar_dkq_done);
              mma_commit_w(&bar_staged[t % S]);
            } else {
              if (t > 0) {  // dQ of the previous tile has left its columns
                if (!(ok = wait(bar_dq_empty, (t - 1) & 1, kBTagDqEmpty))) break;
                tc_fence_after();
              }
              issue_dQ(t);
            }
            if (it + 1 < n_it) {
              if (!(ok = wait_do(t + 1))) break;
              tc_fence_after();
              issue_dPT(t + 1);
            }
          }
        } else {
          // Order S^T(i) dP^T(i) dV(i) dK(i) dQ(i).  dQ(i) accumulates in dP^T's
          // columns, so dP^T(i+1) also waits for the drain to have read dQ(i).
          for (int it = 0; it < n_it && ok; ++it) {
            t = t0 + it;
            if (!(ok = wait_q(t))) break;
            tc_fence_after();
            issue_sT(t);
            if (t > 0 && !(ok = wait(bar_dq_empty, (t - 1) & 1, kBTagDqEmpty))) break;
            if (!(ok = wait_do(t))) break;
            tc_fence_after();
            issue_dPT(t);
            if (!(ok = wait(bar_p_full, t & 1, kBTagPFull))) break;
            tc_fence_after();
            issue_dV(t, it > 0);
            if (!(ok = wait(bar_ds_full, t & 1, kBTagDsFull))) break;
            tc_fence_after();
            issue_dK(t, it > 0);
            issue_dQ(t);
          }
        }
        if (!ok) break;
        mma_commit_w(bar_kv_free);  // every MMA of this unit: K_j, V_j may be reloaded
        t = t0 + n_it;
      }
      if (!ok) {
        mma_commit_w(bar_drain);
        mbar_drain(bar_drain, 0);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ compute
    const int w = warp >> 2;                 // query-column half
    const int r = (warp & 3) * 32 + lane;    // key row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS;
    const uint32_t tdP = tmem + lane_off + C::kColdP;
    const uint32_t dS_addr = smem_u32(sdS) + w * 16384;
    // This warp's 4 KB of the dS tile (the rows it writes there): the epilogue's
    // staging for its 32 rows x D/2 columns of dV, then of dK.
    const uint32_t my_dS = smem_u32(sdS) + w * 16384 + (warp & 3) * 4096;
    const float c = p.scale_log2;
    bool ok = !*abort_flag;
    int t0 = 0;  // this unit's first tile, counted over all units
    for (int u = 0; ok; ++u) {
      int unit;
      if (!(ok = take_unit(u, unit))) break;
      if (unit < 0) break;
      // Only the tile count lives through the tile loop (registers are tight): the
      // head and key tile are derived again where they are needed.
      int n_it;
      {
        int bh_u, j_u;
        bwd_unit(unit, p.BH, nq, bh_u, j_u);
        n_it = nq - (CAUSAL ? j_u : 0);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        const int t = t0 + it;
        const int s = t % S, n = t / S;
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_s_full, t & 1, kBTagSFull) &&
                                         mbar_wait(ctx, &bar_q_full[s], n & 1, kBTagQdoFull));
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == 0) FA_TRACE(16 + t * 8 + 4);
        // Dropout: keep bit cc for query i*128 + 64w + cc and this thread's key.
        // The generator's counter blocks run along keys, so the warp draws the
        // 64 x 32 block together (four calls per lane, 16 keys each) and transposes
        // it through its own rows of the dS tile, free once the previous tile's
        // dK / dQ are done.
        uint64_t keep = ~0ull;
        if constexpr (DROPOUT) {
          if (t > 0) ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dkq_done, (t - 1) & 1, kBTagDkqDone));
          if (!ok) break;
          int bh, j;
          bwd_unit(unit, p.BH, nq, bh, j);
          const int i = (CAUSAL ? j : 0) + it;
          const uint32_t slot = smem_u32(sdS) + w * 16384 + (warp & 3) * 4096;  // [64 queries][32 keys] u8
          const int b = lane & 1;
          const uint32_t jblk = static_cast<uint32_t>(j * 128 + (warp & 3) * 32) / 16 + b;
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            const int ii = (lane >> 1) + 16 * q4;
            const uint4 wv = dropout_words(p.drop, i * 128 + 64 * w + ii, jblk, bh);
            st_shared_v4(slot + ii * 32 + 16 * b, wv.x, wv.y, wv.z, wv.w);
          }
          __syncwarp();
          const uint8_t *draws = reinterpret_cast<const uint8_t *>(sdS + w * 16384 + (warp & 3) * 4096);
          keep = 0;
  #pragma unroll
          for (int ii = 0; ii < 64; ++ii) keep |= static_cast<uint64_t>(draws[ii * 32 + lane] >= p.drop.T) << ii;
          __syncwarp();
        }
        uint32_t sv[64];
        tmem_ld32(tS + 64 * w, sv);
        tmem_ld32(tS + 64 * w + 32, sv + 32);
        tmem_wait_ld();
        const float *lse2 = sL + s * 128 + 64 * w;
        float pf[64];
  #pragma unroll
        for (int cc = 0; cc < 64; ++cc) pf[cc] = ex2(fmaf(__uint_as_float(sv[cc]), c, -lse2[cc]));
        if (CAUSAL && it == 0) {  // the diagonal tile (i = j)
          // Diagonal tile: key row r is masked for query columns before it.
  #pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (64 * w + cc < r) pf[cc] = 0.f;
        }
        // Z = keep / (keep probability): dV takes (P o Z)^T, dS the dP o Z.
        auto zval = [&](int cc) { return DROPOUT ? (((keep >> cc) & 1ull) ? p.drop.inv_keep : 0.f) : 1.f; };
        uint32_t pk[32];
  #pragma unroll
        for (int t = 0; t < 32; ++t) pk[t] = pack_bf16(pf[2 * t] * zval(2 * t), pf[2 * t + 1] * zval(2 * t + 1));
        tmem_st32(tS + 64 * w, pk);  // inside the columns this warp has read
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_full);
        if (threadIdx.x == 0) FA_TRACE(16 + t * 8 + 5);

        // dP^T, and D (it came with dO: the issuer waited for both before dP^T, but
        // the data's visibility to these threads comes with their own wait).
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dp_full, t & 1, kBTagDpFull) &&
                                         (!kSplitStage || mbar_wait(ctx, &bar_do_full[s], n & 1, kBTagQdoFull)));
        // The previous tile's dK / dQ MMAs read dS from smem: wait until they are done.
        if (ok && t > 0) ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dkq_done, (t - 1) & 1, kBTagDkqDone));
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == 0) FA_TRACE(16 + t * 8 + 6);
        const float *Dv = sDv + s * 128 + 64 * w;
  #pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t dp[32];
          tmem_ld32(tdP + 64 * w + 32 * ch, dp);
          tmem_wait_ld();
          uint32_t dsk[16];
  #pragma unroll
          for (int t = 0; t < 16; ++t) {
            const int c0 = 32 * ch + 2 * t;
            float z0 = 1.f, z1 = 1.f;
            if constexpr (DROPOUT) {
              z0 = keep_bit_fresh(keep, c0) ? p.drop.inv_keep : 0.f;
              z1 = keep_bit_fresh(keep, c0 + 1) ? p.drop.inv_keep : 0.f;
            }
            const float d0 = pf[c0] * (__uint_as_float(dp[2 * t]) * z0 - Dv[c0]);
            const float d1 = pf[c0 + 1] * (__uint_as_float(dp[2 * t + 1]) * z1 - Dv[c0 + 1]);
            dsk[t] = pack_bf16(d0, d1);
          }
  #pragma unroll
          for (int t = 0; t < 4; ++t)
            st_shared_v4(dS_addr + bsw128(r, 4 * ch + t), dsk[4 * t], dsk[4 * t + 1], dsk[4 * t + 2], dsk[4 * t + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_ds_full);
        if (threadIdx.x == 0) FA_TRACE(16 + t * 8 + 7);
        if constexpr (R::kComputeDrain && !NO_DQ) {
          // dQ drain: once dK(i) and dQ(i) have completed, read this warp's part of
          // dQ (its lane quarter's rows, columns 64w..) out of TMEM -- which frees
          // the columns for dP^T(i+1) -- and stage it, scaled, as fp32 in tile i's
          // Q (w = 0) or dO (w = 1) stage buffer for the producer's reduce-add.
          ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dkq_done, t & 1, kBTagDkqDone));
          if (!ok) break;
          tc_fence_after();
          if (threadIdx.x == 0) FA_TRACE(1024 + t * 2 + 0);
          uint32_t v[64];
          const uint32_t tdQ = tmem + lane_off + C::kColdQ + 64 * w;
          tmem_ld32(tdQ, v);
          tmem_ld32(tdQ + 32, v + 32);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar_dq_empty);
          const uint32_t buf = smem_u32((w == 0 ? sQ : sdO) + s * C::kTile);
  #pragma unroll
          for (int b = 0; b < 2; ++b)
  #pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int c0 = 32 * b + 4 * t;
              st_shared_v4(buf + b * 16384 + bsw128(r, t), __float_as_uint(__uint_as_float(v[c0]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 1]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 2]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 3]) * p.scale));
            }
          fence_proxy_async_smem();
          mbar_arrive(&bar_staged[s]);
          if (threadIdx.x == 0) FA_TRACE(1024 + t * 2 + 1);
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      // After the unit's last dK / dQ (this warp's own drain already waited at
      // d = 128 with dQ), dV and dK are final: read this warp's rows out of TMEM
      // -- which also frees the accumulators for the next unit's first dV, dK
      // (they follow that unit's first P and dS, which this warp forms later) --
      // and write them out through the warp's own part of the dS tile (free: the
      // MMAs that read it completed).  Stores of whole 128-byte row segments, and
      // nothing waits for them.
      const int t_last = t0 + n_it - 1;
      int bh, j;
      bwd_unit(unit, p.BH, nq, bh, j);
      if constexpr (!R::kComputeDrain || NO_DQ)
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dkq_done, t_last & 1, kBTagDkqDone));
      if (!ok) break;
      tc_fence_after();
      if (threadIdx.x == 0) FA_TRACE(2);
      constexpr int kChunks = D / 16;        // 16-byte chunks in a row's D/2 bf16 columns
      constexpr int kRowsPerPass = 512 / D;  // rows one warp-wide 16-byte access covers
      const int row0 = j * 128 + (warp & 3) * 32;  // this warp's first key row
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {  // dV, then dK (times the softmax scale)
        const uint32_t tacc = tmem + lane_off + (pass == 0 ? C::kColdV : C::kColdK) + w * (D / 2);
        const float f = pass == 0 ? 1.f : p.scale;
        uint16_t *out = pass == 0 ? p.dv : p.dk;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {  // 32 columns at a time (registers are tight)
          uint32_t a[32];
          tmem_ld32(tacc + 32 * ch, a);
          tmem_wait_ld();
#pragma unroll
          for (int cq = 0; cq < 4; ++cq) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              wv[e] = pack_bf16(__uint_as_float(a[8 * cq + 2 * e]) * f, __uint_as_float(a[8 * cq + 2 * e + 1]) * f);
            st_shared_v4(my_dS + epi_offset<D>(lane, 4 * ch + cq), wv[0], wv[1], wv[2], wv[3]);
          }
        }
        if (pass == 1) tc_fence_before();  // both accumulators read: the next unit may overwrite them
        __syncwarp();
        const int cq = lane % kChunks;
#pragma unroll
        for (int ps = 0; ps < 32 / kRowsPerPass; ++ps) {
          const int row = ps * kRowsPerPass + lane / kChunks;
          if (row0 + row < p.N) {
            const size_t e = (static_cast<size_t>(bh) * p.N + row0 + row) * D + w * (D / 2) + cq * 8;
            *reinterpret_cast<uint4 *>(out + e) = ld_shared_u4(my_dS + epi_offset<D>(row, cq));
          }
        }
        __syncwarp();  // the staging is rewritten by dK, then by the next unit's dS
      }
      if (threadIdx.x == 0) FA_TRACE(3);
      t0 += n_it;
    }
    __syncwarp();
  } else if constexpr (!R::kComputeDrain) {
    // ------------------------------------------------------------ dQ drain
    // Staging: the fp32 dQ tile is 128 rows x D columns = 4 * D * 128 bytes, split
    // into 32-column boxes (128-byte swizzle); boxes 0..D/64-1 go to Q_i's stage
    // buffer and the rest to dO_i's (each buffer holds D/64 boxes of 16 KB).
    const int r = (warp & 3) * 32 + lane;  // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tdQ = tmem + lane_off + C::kColdQ;
    const bool leader = (warp == 8 && lane == 0);
    constexpr int kBoxesPerBuf = D / 64;  // 16 KB boxes per stage buffer
    bool ok = !*abort_flag;
    int t0 = 0;  // this unit's first tile, counted over all units
    for (int u = 0; ok; ++u) {
      int unit;
      if (!(ok = take_unit(u, unit))) break;
      if (unit < 0) break;
      int bh, j;
      bwd_unit(unit, p.BH, nq, bh, j);
      const int i0 = CAUSAL ? j : 0, n_it = nq - i0;
      for (int it = 0; it < n_it && ok; ++it) {
        const int t = t0 + it, s = t % S;
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, bar_dkq_done, t & 1, kBTagDkqDone));
        if (!ok) break;
        tc_fence_after();
        if (r == 0) FA_TRACE(1024 + t * 2 + 0);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // Columns [half*D/2, (half+1)*D/2) -> the Q (half 0) or dO (half 1) stage buffer.
          uint32_t v[D / 2];
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) tmem_ld32(tdQ + half * (D / 2) + 32 * ch, v + 32 * ch);
          tmem_wait_ld();
          if (half == 1) {
            tc_fence_before();
            mbar_arrive(bar_dq_empty);  // dQ is out of TMEM
          }
          const uint32_t buf = smem_u32((half == 0 ? sQ : sdO) + s * C::kTile);
#pragma unroll
          for (int b = 0; b < kBoxesPerBuf; ++b)
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int c0 = 32 * b + 4 * q;
              st_shared_v4(buf + b * 16384 + bsw128(r, q), __float_as_uint(__uint_as_float(v[c0]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 1]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 2]) * p.scale),
                           __float_as_uint(__uint_as_float(v[c0 + 3]) * p.scale));
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_stage);
        if (leader) {
          ok = mbar_wait(ctx, bar_stage, t & 1, kBTagStage);
          if (ok) {
            for (int half = 0; half < 2; ++half)
              for (int b = 0; b < kBoxesPerBuf; ++b)
                tma_reduce_add_3d(&tmdQacc, (half == 0 ? sQ : sdO) + s * C::kTile + b * 16384,
                                  half * (D / 2) + 32 * b, (i0 + it) * 128, bh);
            bulk_commit();
            bulk_wait_read<0>();
          }
          // The stage (Q_i, dO_i) is free for the producer: the MMAs that read it
          // completed (bar_dkq_done) and TMA has read the staged dQ.
          mbar_arrive(&bar_qdo_empty[s]);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (r == 0) FA_TRACE(1024 + t * 2 + 1);
      }
      t0 += n_it;
    }
    if (leader) bulk_wait<0>();  // every reduction has landed before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) FA_TRACE(7);
  if (warp == R::kIssuerWarp) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ host side
inline int pad128(int n) { return (n + 127) / 128 * 128; }

// Workspace: the fp32 dQ accumulator, the LSE*log2(e) and D vectors, then 256
// bytes whose first word counts the units fa_bwd_kernel's CTAs have taken.
inline size_t bwd_workspace_main_bytes(int BH, int N, int d) {
  const size_t dq = static_cast<size_t>(BH) * N * d * 4;
  const size_t vec = static_cast<size_t>(BH) * pad128(N) * 4;
  return (dq + 2 * vec + 255) / 256 * 256;
}
inline size_t bwd_workspace_bytes(int BH, int N, int d) { return bwd_workspace_main_bytes(BH, N, d) + 256; }

struct BwdLaunch {
  const void *q, *k, *v, *o, *o_lo, *dO;
  const float *lse;
  void *dq, *dk, *dv;
  int BH, N, d, causal;
  float scale;
  void *workspace;
  int *status;
  int seq;
  int num_sms;
  cudaEvent_t const *events = nullptr;  // optional: 4 events recorded around the stages
  const DropoutParams *drop = nullptr;  // dropout on the probabilities, or none
};

template <int D, bool CAUSAL, bool DROPOUT, bool NO_DQ = false>
inline cudaError_t bwd_set_attribute() {
  return cudaFuncSetAttribute(fa_bwd_kernel<D, CAUSAL, DROPOUT, NO_DQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              BwdCfg<D>::kSmemBytes);
}

inline cudaError_t bwd_set_attributes() {
  const cudaError_t es[12] = {bwd_set_attribute<64, false, false>(), bwd_set_attribute<64, true, false>(),
                              bwd_set_attribute<128, false, false>(), bwd_set_attribute<128, true, false>(),
                              bwd_set_attribute<64, false, true>(), bwd_set_attribute<64, true, true>(),
                              bwd_set_attribute<128, false, true>(), bwd_set_attribute<128, true, true>(),
                              bwd_set_attribute<64, false, false, true>(), bwd_set_attribute<64, true, false, true>(),
                              bwd_set_attribute<128, false, false, true>(),
                              bwd_set_attribute<128, true, false, true>()};
  for (cudaError_t e : es)
    if (e != cudaSuccess) return e;
  return cudaSuccess;
}

// Persistent grid: one CTA per SM (one resident CTA fits), or one per unit if fewer.
template <int D, bool CAUSAL, bool DROPOUT, bool NO_DQ = false>
inline void bwd_main_launch(const CUtensorMap *m, const BwdParams &p, int nkv, int num_sms, cudaStream_t s) {
  const long units = static_cast<long>(p.BH) * nkv;
  const dim3 grid(static_cast<unsigned>(units < num_sms ? units : num_sms));
  fa_bwd_kernel<D, CAUSAL, DROPOUT, NO_DQ><<<grid, BwdRoles<D, NO_DQ>::kThreads, BwdCfg<D>::kSmemBytes, s>>>(
      m[0], m[1], m[2], m[3], m[6], p);
}

// maps: Q, K, V, dO, dK, dV (bf16, 3-D, 64-feature boxes), dQ accumulator
// (fp32, 3-D, 32-feature boxes).
inline cudaError_t bwd_launch(const BwdLaunch &L, const CUtensorMap *maps, cudaStream_t s) {
  const int Npad = pad128(L.N);
  float *ws_dq = static_cast<float *>(L.workspace);
  float *ws_lse2 = ws_dq + static_cast<size_t>(L.BH) * L.N * L.d;
  float *ws_D = ws_lse2 + static_cast<size_t>(L.BH) * Npad;
  int *counter = reinterpret_cast<int *>(static_cast<uint8_t *>(L.workspace) +
                                         bwd_workspace_main_bytes(L.BH, L.N, L.d));
  const int pre_grid = L.num_sms * 8;
  cudaError_t e = cudaSuccess;
  if (L.events && (e = cudaEventRecord(L.events[0], s)) != cudaSuccess) return e;
  if (L.d == 64)
    fa_bwd_pre_kernel<64><<<pre_grid, 256, 0, s>>>(static_cast<const uint16_t *>(L.o),
                                                   static_cast<const uint16_t *>(L.o_lo),
                                                   static_cast<const uint16_t *>(L.dO), L.lse, ws_D, ws_lse2, ws_dq, counter,
                                                   L.N, Npad, L.BH);
  else
    fa_bwd_pre_kernel<128><<<pre_grid, 256, 0, s>>>(static_cast<const uint16_t *>(L.o),
                                                    static_cast<const uint16_t *>(L.o_lo),
                                                    static_cast<const uint16_t *>(L.dO), L.lse, ws_D, ws_lse2, ws_dq, counter,
                                                    L.N, Npad, L.BH);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (L.events && (e = cudaEventRecord(L.events[1], s)) != cudaSuccess) return e;
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
  if (L.drop) p.drop = *L.drop;
  if (L.drop) {
    if (L.d == 64)
      L.causal ? bwd_main_launch<64, true, true>(maps, p, nkv, L.num_sms, s) : bwd_main_launch<64, false, true>(maps, p, nkv, L.num_sms, s);
    else
      L.causal ? bwd_main_launch<128, true, true>(maps, p, nkv, L.num_sms, s)
               : bwd_main_launch<128, false, true>(maps, p, nkv, L.num_sms, s);
  } else {
    if (L.d == 64)
      L.causal ? bwd_main_launch<64, true, false>(maps, p, nkv, L.num_sms, s)
               : bwd_main_launch<64, false, false>(maps, p, nkv, L.num_sms, s);
    else
      L.causal ? bwd_main_launch<128, true, false>(maps, p, nkv, L.num_sms, s)
               : bwd_main_launch<128, false, false>(maps, p, nkv, L.num_sms, s);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (L.events && (e = cudaEventRecord(L.events[2], s)) != cudaSuccess) return e;
  const long n4 = static_cast<long>(L.BH) * L.N * L.d / 4;
  fa_dq_convert_kernel<<<L.num_sms * 4, 256, 0, s>>>(ws_dq, static_cast<uint16_t *>(L.dq), n4);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (L.events) e = cudaEventRecord(L.events[3], s);
  return e;
}

}  // namespace fa

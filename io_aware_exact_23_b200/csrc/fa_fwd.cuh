// fa_fwd.cuh -- fused exact-attention forward kernel for sm_100a.
//
// One CTA computes O and LSE for a pair of 128-row query tiles of one head:
// the "tile inputs / compute locally / online normalisation / write compact
// output" steps of the FlashAttention summary ("Architecture, step by step"),
// with the online softmax of the review's "Tiling" section.  The N x N scores
// live only on chip, one 128 x 128 tile at a time: the fp32 S
// and the bf16 P in tensor memory (TMEM).
//
// Roles (352 threads):
//   warps 0-7  softmax.  Warp w owns rows 32*(w%4)..+31 (its TMEM lane
//              quarter) and the column half h = w/4 of every S tile.  All eight
//              warps work on tile 0 of KV step j, then on tile 1, then on tile 0
//              of step j+1 ...: while they run one tile's softmax, the tensor
//              pipe runs the other tile's PV and next S.  The two warps that
//              share rows exchange their half-row maxima through smem.
//   warp  8    TMA producer: Q0, Q1 once, then K / V tiles through a smem ring.
//   warp  9    MMA issuer for tile 0 (one elected lane); warp 10 for tile 1.  Two
//              independent issuers let the pipe take whichever tile is ready.
// A K/V ring stage is released when both issuers' MMAs that read it completed.
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D).  The bf16 P (two per column) of column half h is written
// over S columns [64h, 64h+32) -- inside the half its warp has already read --
// and is the A operand of the PV MMA straight from TMEM.  The next S of a tile
// overwrites those columns; its issuer puts it in the pipe right behind that
// tile's PV (one issuing lane: the MMAs execute in order), without waiting.
//
// Online softmax, in the log2 domain with c = scale*log2(e):
//   m' = max(m, c*rowmax(S));  P = 2^(c*S - m');  l = 2^(m-m') l + rowsum(P);
//   O = 2^(m-m') O + P V.
// O is divided by the row sum of P as rounded to bf16 (the weights the MMA
// actually applied), LSE uses the fp32 row sum.
// The running max is only moved when it grows by more than 8 (a factor 256):
// O and l are both kept relative to the same stale max, which is exact, and
// P <= 256 cannot overflow fp32 or bf16.  Most tiles then skip the O rescale.
// After the first KV step P is computed against the running max before the
// row max of the new tile is known (the half maxima travel through smem in the
// meantime); only a row whose max grew by more than 8 recomputes its P.
// Every exponential runs on the MUFU unit (one per 4d FLOPs; at d = 128 its
// rate equals the tensor rate).  Moving a share of them to the FMA pipe as a
// polynomial was measured slower: FP32-pipe pressure from the softmax warps
// delays the MMA issue more than the MUFU queue does.
#pragma once

#include "dropout.cuh"
#include "ptx.cuh"

namespace fa {

struct FwdParams {
  uint16_t *o;       // [BH, N, D] bf16
  int *unit_counter;  // units handed out past the first wave (zeroed on the stream before the launch)
  float *lse;        // [BH, N] fp32 (natural log)
  uint16_t *o_lo;    // optional [BH, N, D] bf16: bf16(O_fp32 - O), or nullptr
  int *status;       // device status block
  int seq;           // launch sequence number (for the status block)
  int N;
  int BH;
  int n_qpairs;      // ceil(N / 256)
  float scale_log2;  // scale * log2(e)
  DropoutParams drop;  // read only by the DROPOUT instantiations
  // FP8 instantiations only: per-head descale factors [BH] of the e4m3 Q, K, V
  // (the inputs are code * descale).
  const float *descale_q, *descale_k, *descale_v;
};

// FP8: Q, K, V as e4m3 (one byte per element); the output O stays bf16.
template <int D, bool FP8 = false>
struct FwdCfg {
  static_assert(!FP8 || D == 128, "the e4m3 forward takes d = 128 (one 128-byte swizzle row per tile row)");
  static constexpr int kElemBytes = FP8 ? 1 : 2;
  static constexpr int kTileBytes = 128 * D * kElemBytes;  // one 128 x D input tile
  static constexpr int kBoxCols = 128 / kElemBytes;        // input elements per 128-byte TMA box row
  static constexpr int kBoxes = kTileBytes / 16384;        // 128-row TMA boxes (16 KB) per input tile
  static constexpr int kStages = (FP8 || D == 64) ? 8 : 4;  // K/V ring depth
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kXOff = kKVOff + kStages * kTileBytes;  // half-row maxima [2 tiles][2 halves][128]
  static constexpr int kLOff = kXOff + 2048;                   // half-row sums [2 tiles][2 halves][2][128]
  // Epilogue staging, 2 KB per softmax warp: 32 rows x 32 bf16 columns at a time,
  // so that a unit's epilogue leaves the ring and Q buffers to the next unit.
  static constexpr int kEpiOff = kLOff + 4096;
  static constexpr int kBarOff = kEpiOff + 8 * 2048;
  // mbarriers: q[2], kv_full/kv_empty[kStages], s_full/p_full/pv_done/drain
  // [2] each (one per query tile), the max and sum exchanges [2][4] (one per
  // tile and warp pair), q_free[2] (a unit's last S_k completed) and the unit
  // ring's full / empty [2]; then the TMEM address slot, the abort flag and the
  // two-slot unit ring.
  static constexpr int kNumBars = 2 + 2 * kStages + 30;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = 352;
  static constexpr int kSoftmaxThreads = 256;
  static constexpr int kProducerWarp = 8;
  static constexpr int kIssuerWarp = 9;  // 9: tile 0 (and TMEM owner), 10: tile 1
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

enum FwdTag : int {
  kTagQ = 1, kTagKvFull = 2, kTagKvEmpty = 3, kTagSFull = 4, kTagPFull = 5, kTagPvDone = 6, kTagEpi = 7,
  kTagXmax = 8, kTagLsum = 9, kTagQfree = 10, kTagUnit = 24
};

// Load order of the K/V ring: K tiles run one KV step ahead of V tiles
// (K0, K1, V0, K2, V1, ..., K_{n-1}, V_{n-2}, V_{n-1}), because S of step j+1
// is issued while P of step j is still being computed.  Ring slot of each load:
__device__ __forceinline__ int kv_idx_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int kv_idx_v(int j, int n) { return (j + 1 < n) ? 2 * j + 2 : 2 * j + 1; }

// Position of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled
// tile: TMA's SWIZZLE_128B pattern XORs the chunk index with row % 8.
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}


// FP8: e4m3 Q, K, V with per-head descale factors (kind::f8f6f4 MMAs, K = 32
// per instruction); P is rounded to e4m3 for the PV product, four per TMEM
// column, and O is divided by the fp32 row sum of the unrounded P.
//
// Persistent CTAs: the grid holds one CTA per SM (or one per unit, if fewer).
// CTA c starts on unit c and then claims units from a counter, in the same
// order, each when its current unit's last K/V load has been issued.  Barrier
// phases run on counts over all the CTA's units (K/V loads, and each tile's KV
// steps); the producer hands units to the other roles through a two-slot ring
// in shared memory, reloads Q_k for the next unit once the previous unit's last
// S_k completed, and keeps the K/V ring going across units.  A unit's first
// PV_k overwrites O_k, but it follows P_k of that unit, which the softmax warps
// write only after their epilogue has read O_k.
template <int D, bool CAUSAL, bool DROPOUT = false, bool FP8 = false>
__global__ void __launch_bounds__(352, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!(FP8 && DROPOUT), "no dropout in the e4m3 forward");
  using C = FwdCfg<D, FP8>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (threadIdx.x == 0) FA_TRACE(1);

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *bar_q = bars + 0;                        // [2]
  uint64_t *bar_kv_full = bars + 2;                  // [kStages]
  uint64_t *bar_kv_empty = bars + 2 + C::kStages;    // [kStages]
  uint64_t *bar_s_full = bars + 2 + 2 * C::kStages;  // [2] S_k in TMEM
  uint64_t *bar_p_full = bar_s_full + 2;             // [2] P_k in TMEM (and O_k rescaled)
  uint64_t *bar_pv_done = bar_p_full + 2;            // [2] PV_k completed
  uint64_t *bar_drain = bar_pv_done + 2;             // [2] abort path: the issuer's MMAs completed
  uint64_t *bar_x = bar_drain + 2;                   // [2][4] half-row max exchange, per warp pair
  uint64_t *bar_l = bar_x + 8;                       // [2][4] half-row sum exchange, per warp pair
  uint64_t *bar_q_free = bar_l + 8;                  // [2] the unit's last S_k completed
  uint64_t *bar_unit_full = bar_q_free + 2;          // [2] unit ring: the producer wrote the slot
  uint64_t *bar_unit_empty = bar_unit_full + 2;      // [2] unit ring: every consumer warp read it
  static_assert(2 + 2 * C::kStages + 30 == C::kNumBars, "barrier count");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_unit_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *unit_ring = reinterpret_cast<volatile int *>(tmem_slot + 2);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_kv_all = (p.N + 127) / 128;
  const int n_units = p.BH * p.n_qpairs;
  constexpr int kConsumerWarps = 2 + 8;  // the two issuers, the eight softmax warps

  const WaitCtx ctx{p.status, abort_flag, kKernelFwd, p.seq};

  if (threadIdx.x == 0) {
    // The swizzle arithmetic and the UMMA descriptors assume a 1024-byte
    // aligned shared-memory window.
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) record_failure(ctx, kStatusInternal, 0);
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bar_q[k], 1);
      mbar_init(&bar_q_free[k], 1);
      mbar_init(&bar_unit_full[k], 1);
      mbar_init(&bar_unit_empty[k], kConsumerWarps);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 2);  // one arrival per MMA issuer
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bar_s_full[k], 1);
      mbar_init(&bar_p_full[k], C::kSoftmaxThreads);
      mbar_init(&bar_pv_done[k], 1);
      for (int q = 0; q < 4; ++q) {
        // Warps q and q+4 share rows 32q..32q+31 (and an SM sub-partition).
        mbar_init(&bar_x[k * 4 + q], 64);
        mbar_init(&bar_l[k * 4 + q], 64);
      }
      mbar_init(&bar_drain[k], 1);
    }
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
  if (threadIdx.x == 0) FA_TRACE(0);

  uint8_t *sQ = smem + C::kQOff;
  uint8_t *sKV = smem + C::kKVOff;

  // Work unit -> (head, query-tile pair): heads in chunks of 8 (their K/V stay
  // resident in L2 while the chunk runs); inside a chunk, longest pairs first.
  auto decode = [&](int unit, int &bh, int &u) {
    constexpr int kChunk = 8;
    const int per_chunk = kChunk * p.n_qpairs;
    const int ch = unit / per_chunk, rem = unit % per_chunk;
    const int g = min(kChunk, p.BH - ch * kChunk);
    u = p.n_qpairs - 1 - rem / g;
    bh = ch * kChunk + rem % g;
  };
  // KV steps of the pair's query tiles 0 and 1 (n1 >= n0).
  auto steps = [&](int u, int &n0, int &n1) {
    n0 = CAUSAL ? min(2 * u + 1, n_kv_all) : n_kv_all;
    n1 = CAUSAL ? min(2 * u + 2, n_kv_all) : n_kv_all;
  };
  // A consumer warp (all lanes) takes unit i from the ring (-1: no more units).
  // The value is broadcast from lane 0, so the compiler knows it is warp-uniform.
  auto take_unit = [&](int i, int &unit) -> bool {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_unit_full[i & 1], (i >> 1) & 1, kTagUnit));
    if (!ok) return false;
    unit = __shfl_sync(0xffffffffu, unit_ring[i & 1], 0);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_unit_empty[i & 1]);
    return true;
  };

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      bool ok = true;
      int g = 0;             // K/V loads issued so far, over all units (the ring index)
      int nq[2] = {0, 0};    // Q_k loads issued so far
      int unit = static_cast<int>(blockIdx.x) < n_units ? static_cast<int>(blockIdx.x) : -1;
      for (int ui = 0; ok; ++ui) {
        // Hand unit ui (or the end, -1) to the other roles.
        if (ui >= 2 && !(ok = mbar_wait(ctx, &bar_unit_empty[ui & 1], ((ui >> 1) - 1) & 1, kTagUnit))) break;
        unit_ring[ui & 1] = unit;
        mbar_arrive(&bar_unit_full[ui & 1]);
        if (unit < 0) break;
        int bh, u, n0, n_kv;
        decode(unit, bh, u);
        steps(u, n0, n_kv);
        // Q_k of this unit, once the previous unit's last S_k has completed.
        if (ui > 0 && !(ok = mbar_wait(ctx, &bar_q_free[0], (ui - 1) & 1, kTagQfree))) break;
        mbar_arrive_expect_tx(&bar_q[0], C::kTileBytes);
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(&tmQ, &bar_q[0], sQ + b * 16384, b * C::kBoxCols, (2 * u) * 128, bh);
        ++nq[0];
        for (int idx = 0; idx < 2 * n_kv && ok; ++idx, ++g) {
          // Which tile is load number idx in the K-ahead order.
          const bool is_k = (idx == 0) || ((idx & 1) && (idx + 1) / 2 < n_kv);
          const int j = (idx == 0) ? 0 : (is_k ? (idx + 1) / 2 : (idx == 2 * n_kv - 1 ? n_kv - 1 : idx / 2 - 1));
          const int s = g % C::kStages, r = g / C::kStages;
          if (r > 0 && !(ok = mbar_wait(ctx, &bar_kv_empty[s], (r - 1) & 1, kTagKvEmpty))) break;
          uint8_t *dst = sKV + s * C::kTileBytes;
          mbar_arrive_expect_tx(&bar_kv_full[s], C::kTileBytes);
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_3d(is_k ? &tmK : &tmV, &bar_kv_full[s], dst + b * 16384, b * C::kBoxCols, j * 128, bh);
          if (idx == 0) {
            if (ui > 0 && !(ok = mbar_wait(ctx, &bar_q_free[1], (ui - 1) & 1, kTagQfree))) {
              ++g;
              break;
            }
            mbar_arrive_expect_tx(&bar_q[1], C::kTileBytes);
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_3d(&tmQ, &bar_q[1], sQ + C::kTileBytes + b * 16384, b * C::kBoxCols, (2 * u + 1) * 128,
                          bh);
            ++nq[1];
          }
        }
        if (!ok) break;
        // The next unit, claimed once this one's loads are all issued (a KV step
        // or two before its end): claimed earlier, it would wait behind this unit
        // while other CTAs run dry; the atomic's latency hides behind those steps.
        unit = static_cast<int>(gridDim.x) + atomicAdd(p.unit_counter, 1);
        if (unit >= n_units) unit = -1;
      }
      // The last loads have landed before the CTA can exit (immediate unless a
      // consumer gave up before taking them).
      for (int k = 0; k < 2; ++k)
        if (nq[k] > 0) mbar_drain(&bar_q[k], (nq[k] - 1) & 1);
      for (int s = 0; s < C::kStages && s < g; ++s) {
        const int last = s + ((g - 1 - s) / C::kStages) * C::kStages;
        mbar_drain(&bar_kv_full[s], (last / C::kStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == C::kIssuerWarp || warp == C::kIssuerWarp + 1) {
    // ------------------------------------------------------------ MMA issuers
    // The whole warp runs the issue loop (waits, unit decode, descriptors), so
    // that every value it computes is warp-uniform; one elected lane issues each
    // MMA and commit.  (Run from a single lane, the loop took about 100 SM cycles
    // per MMA while the softmax warps kept the sub-partition busy; 60-70 this way.)
    const int k = __shfl_sync(0xffffffffu, warp, 0) - C::kIssuerWarp;  // query tile owned by this issuer
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    if (__all_sync(0xffffffffu, *abort_flag == 0)) {
      constexpr uint32_t idesc_qk = FP8 ? make_idesc_e4m3(128, 128, 0, 0) : make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = FP8 ? make_idesc_e4m3(128, D, 0, 1) : make_idesc_bf16(128, D, 0, 1);
      // Base descriptors: Q_k (K-major), ring stage 0 as K (K-major) and as V (MN-major).
      const uint64_t q_desc = make_sdesc(smem_u32(sQ + k * C::kTileBytes), 16, 1024);
      const uint64_t k_desc0 = make_sdesc(smem_u32(sKV), 16, 1024);
      const uint64_t v_desc0 = make_sdesc(smem_u32(sKV), 16384, 1024);
      const uint32_t tS = tm + 128 * k;
      const uint32_t tO = tm + 256 + k * D;
      bool ok = true;
      int gb = 0;  // K/V loads of the previous units
      int cs = 0;  // this tile's KV steps in the previous units
      auto wait = [&](uint64_t *bar, int parity, int tag) {
        return __all_sync(0xffffffffu, mbar_wait(ctx, bar, static_cast<uint32_t>(parity), tag));
      };
      for (int ui = 0; ok; ++ui) {
        int unit;
        if (!(ok = take_unit(ui, unit))) break;
        if (unit < 0) break;
        int bh, u, n0, n_kv;
        decode(unit, bh, u);
        steps(u, n0, n_kv);
        const int n_k = (k == 0) ? n0 : n_kv;
        if (!(ok = wait(&bar_q[k], ui & 1, kTagQ))) break;
        for (int j = 0; j < n_kv && ok; ++j) {
          const int iK = gb + kv_idx_k(j), sK = iK % C::kStages;
          const int iV = gb + kv_idx_v(j, n_kv), sV = iV % C::kStages;
          // Arrivals on kv_empty must follow the matching kv_full phase, so even
          // a tile that skips K_j / V_j (causal tile 0 past its diagonal) waits.
          ok = wait(&bar_kv_full[sK], (iK / C::kStages) & 1, kTagKvFull);
          if (!ok) break;
          if (j >= n_k) {
            if (lane == 0) mbar_arrive(&bar_kv_empty[sK]);
            ok = wait(&bar_kv_full[sV], (iV / C::kStages) & 1, kTagKvFull);
            if (ok && lane == 0) mbar_arrive(&bar_kv_empty[sV]);
            continue;
          }
          // S_k aliases P_k, which the previous PV_k reads.  Both MMAs come from
          // this warp's elected lane and the tensor pipe runs them in issue order,
          // so S_k is issued right behind PV_k without waiting for it to complete.
          const uint64_t k_desc = sdesc_add(k_desc0, sK * C::kTileBytes);
          // One MMA per 32-byte K slice of the 128-byte swizzled rows (16 bf16 or 32 e4m3).
#pragma unroll
          for (int ks = 0; ks < D * C::kElemBytes / 32; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            if constexpr (FP8)
              mma_ss_f8_w(tS, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, ks > 0);
            else
              mma_ss_w(tS, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, ks > 0);
          }
          mma_commit_w(&bar_s_full[k]);
          mma_commit_w(&bar_kv_empty[sK]);
          if (j == n_k - 1) mma_commit_w(&bar_q_free[k]);  // Q_k is not read again in this unit
          if (lane == 0) FA_TRACE(16 + k * 256 + 4 * j + 0);
          ok = wait(&bar_kv_full[sV], (iV / C::kStages) & 1, kTagKvFull);
          if (ok) ok = wait(&bar_p_full[k], (cs + j) & 1, kTagPFull);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) FA_TRACE(16 + k * 256 + 4 * j + 2);
          const uint64_t v_desc = sdesc_add(v_desc0, sV * C::kTileBytes);
          // K steps over the 128 keys: 16 (bf16) or 32 (e4m3) keys, 8 TMEM columns of P
          // and 16 or 32 rows of V each; P of keys 64h.. starts at column 64h.
          if constexpr (FP8) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_ts_f8_w(tO, tS + ks * 8 + (ks >= 2 ? 48 : 0), sdesc_add(v_desc, ks * 4096), idesc_pv,
                          (j > 0 || ks > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_ts_w(tO, tS + ks * 8 + (ks >= 4 ? 32 : 0), sdesc_add(v_desc, ks * 2048), idesc_pv,
                       (j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit_w(&bar_pv_done[k]);
          mma_commit_w(&bar_kv_empty[sV]);
          if (lane == 0) FA_TRACE(16 + k * 256 + 4 * j + 1);
        }
        gb += 2 * n_kv;
        cs += n_k;
      }
      if (!ok) {
        // Let every MMA this warp issued finish before TMEM is released.
        mma_commit_w(&bar_drain[k]);
        mbar_drain(&bar_drain[k], 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int h = warp >> 2;                 // column half of every S tile
    const int rq = warp & 3;                 // TMEM lane quarter
    const int r = rq * 32 + lane;            // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(rq * 32) << 16;
    float *xm = reinterpret_cast<float *>(smem + C::kXOff);  // [k][h][128]
    // This warp's 2 KB of the epilogue staging: 32 rows x 32 bf16 columns.
    const uint32_t stg = smem_u32(smem + C::kEpiOff) + warp * 2048;
    bool ok = !*abort_flag;
    int cs[2] = {0, 0};  // each tile's KV steps in the previous units
    for (int ui = 0; ok; ++ui) {
      int unit;
      if (!(ok = take_unit(ui, unit))) break;
      if (unit < 0) break;
      int bh, u, n_kv0, n_kv;
      decode(unit, bh, u);
      steps(u, n_kv0, n_kv);
      // c = scale * log2(e), times the descale factors of Q and K for e4m3 inputs.
      const float c = FP8 ? p.scale_log2 * p.descale_q[bh] * p.descale_k[bh] : p.scale_log2;
      const uint64_t c2 = f2pack(c, c);
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, lr[2] = {0.f, 0.f};
      const int n_k[2] = {n_kv0, n_kv};
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int k = 0; k < 2 && ok; ++k) {
          if (j >= n_k[k]) continue;
          const int qt = 2 * u + k;
          const uint32_t tS = tmem + lane_off + 128 * k + 64 * h;
          ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_s_full[k], (cs[k] + j) & 1, kTagSFull));
          if (!ok) break;
          tc_fence_after();
          if (r == 0 && h == 0) FA_TRACE(528 + k * 256 + 4 * j + 0);
          uint32_t s[64];
          tmem_ld32(tS, s);
          tmem_ld32(tS + 32, s + 32);
          tmem_wait_ld();
          // Keys j*128 + 64h + col are valid when col < nv (tail of N, causal diagonal).
          int nvalid = min(128, p.N - j * 128);
          if (CAUSAL && j == qt) nvalid = min(nvalid, r + 1);
          const int nv = nvalid - 64 * h;
          if (nv < 64) {
  #pragma unroll
            for (int cc = 0; cc < 64; ++cc)
              if (cc >= nv) s[cc] = __float_as_uint(-INFINITY);
          }
          // Dropout: keys j*128 + 64h + 16q .. +15 of query row qt*128 + r come from
          // generator call jb0 + q (the counter's key block), drawn in the
          // exponential loop below, one call per 16 keys.
          const uint32_t jb0 = static_cast<uint32_t>(j * 128 + 64 * h) >> 4;
          const uint32_t c256 = DROPOUT ? (256u - p.drop.T) * 0x00010001u : 0u;
          // Half-row max as a shallow tree (eight independent chains of four).
          float mq[8];
  #pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float *v = reinterpret_cast<const float *>(s + 8 * q);
            mq[q] = fmaxf(fmax3(fmax3(fmax3(v[0], v[1], v[2]), v[3], v[4]), v[5], v[6]), v[7]);
          }
          const float mh = fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
          xm[(k * 2 + h) * 128 + r] = mh;
          mbar_arrive(&bar_x[k * 4 + rq]);
          // P = 2^(c*S - m) for this half row, with the row sums of P in fp32
          // (for the LSE) and of P rounded to bf16 (the PV weights; O's normaliser).
          uint32_t pk[32];
          float psum = 0.f, prsum = 0.f;
          auto exps = [&](float mref) {
            const float neg = (mref == -INFINITY) ? 0.f : -mref;
            const uint64_t n2 = f2pack(neg, neg);
            if constexpr (FP8) {
              // P rounded to e4m3, four keys per word; O's normaliser is the fp32
              // sum of the unrounded P (the same sum as the LSE's).
              uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
  #pragma unroll
              for (int cq = 0; cq < 16; ++cq) {
                const uint64_t xa = ffma2(f2pack(__uint_as_float(s[4 * cq]), __uint_as_float(s[4 * cq + 1])), c2, n2);
                const uint64_t xb =
                    ffma2(f2pack(__uint_as_float(s[4 * cq + 2]), __uint_as_float(s[4 * cq + 3])), c2, n2);
                float x0, x1, x2, x3;
                f2unpack(xa, x0, x1);
                f2unpack(xb, x2, x3);
                const float a0 = ex2(x0), a1 = ex2(x1), a2 = ex2(x2), a3 = ex2(x3);
                acc[cq & 3] = fadd2(acc[cq & 3], fadd2(f2pack(a0, a1), f2pack(a2, a3)));
                pk[cq] = pack_e4m3x4(a0, a1, a2, a3);
              }
              float u0, u1, u2, u3, u4, u5, u6, u7;
              f2unpack(acc[0], u0, u1);
              f2unpack(acc[1], u2, u3);
              f2unpack(acc[2], u4, u5);
              f2unpack(acc[3], u6, u7);
              psum = ((u0 + u1) + (u2 + u3)) + ((u4 + u5) + (u6 + u7));
              prsum = psum;
              return;
            }
            uint64_t acc[2] = {0ull, 0ull}, racc[2] = {0ull, 0ull};
            uint4 wd = make_uint4(0u, 0u, 0u, 0u);
  #pragma unroll
            for (int cc = 0; cc < 32; ++cc) {
              if constexpr (DROPOUT) {
                if ((cc & 7) == 0) wd = dropout_words(p.drop, qt * 128 + r, jb0 + (cc >> 3), bh);
              }
              const uint64_t x2 = ffma2(f2pack(__uint_as_float(s[2 * cc]), __uint_as_float(s[2 * cc + 1])), c2, n2);
              float x0, x1;
              f2unpack(x2, x0, x1);
              const float a = ex2(x0), b = ex2(x1);
              acc[cc & 1] = fadd2(acc[cc & 1], f2pack(a, b));
              const uint32_t w = pack_bf16(a, b);
              // The sums are of P before dropout; the PV product takes the kept entries
              // (the 1/keep-probability scale is applied to O in the epilogue).
              pk[cc] = DROPOUT ? (w & dropout_pair_mask(wd, cc & 7, c256)) : w;
              racc[cc & 1] = fadd2(racc[cc & 1], f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
            }
            float u0, u1, u2, u3, v0, v1, v2, v3;
            f2unpack(acc[0], u0, u1);
            f2unpack(acc[1], u2, u3);
            f2unpack(racc[0], v0, v1);
            f2unpack(racc[1], v2, v3);
            psum = (u0 + u1) + (u2 + u3);
            prsum = (v0 + v1) + (v2 + v3);
          };
          const float m_old = m[k];
          if (m_old != -INFINITY) exps(m_old);  // optimistic: the running max usually holds
          ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_x[k * 4 + rq], (cs[k] + j) & 1, kTagXmax));
          if (!ok) break;
          const float m_cand = fmaxf(mh, xm[(k * 2 + (h ^ 1)) * 128 + r]) * c;
          float alpha = 1.f;
          bool rescale = false;
          if (m_cand > m_old + 8.f) {  // also taken on the first tile (m = -inf)
            alpha = ex2(m_old - m_cand);
            rescale = (m_old != -INFINITY);
            m[k] = m_cand;
            exps(m_cand);
          }
          l[k] = l[k] * alpha + psum;
          lr[k] = lr[k] * alpha + prsum;
          if (__any_sync(0xffffffffu, rescale)) {
            // O_k still holds the previous step's PV: wait for it, then rescale
            // this warp's column half of O.
            ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[k], (cs[k] + j - 1) & 1, kTagPvDone));
            if (!ok) break;
            tc_fence_after();
            const uint32_t tO = tmem + lane_off + 256 + k * D + h * (D / 2);
  #pragma unroll
            for (int ch = 0; ch < D / 64; ++ch) {
              uint32_t o[32];
              tmem_ld32(tO + ch * 32, o);
              tmem_wait_ld();
  #pragma unroll
              for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
              tmem_st32(tO + ch * 32, o);
            }
          }
          if constexpr (FP8)
            tmem_st16(tS, pk);  // 64 keys of e4m3 P in 16 columns
          else
            tmem_st32(tS, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bar_p_full[k]);
          if (r == 0 && h == 0) FA_TRACE(528 + k * 256 + 4 * j + 1);
          if (lane == 0 && j < 16) FA_TRACE(1024 + (k * 8 + warp) * 16 + j);
        }
      }
      if (!ok) break;
      // -------------------------------------------------------- epilogue
      // Once tile k's last PV of the unit has completed, O_k is final (tile 0's
      // epilogue runs while tile 1's last PV does).  Each warp turns its 32 rows
      // x D/2 columns of O_k (and of the rounding residual) into bf16 32 columns
      // at a time, stages them in its own 2 KB
      // (16-byte chunks XOR-swizzled by row pair, so that the row-wise writes and
      // the chunk-wise read-back are free of bank conflicts) and writes them out
      // with 16-byte stores covering whole 64-byte row segments.  The staging is
      // its own, so the next unit's loads and first S MMAs run meanwhile, and
      // nothing waits for the stores.
      for (int k = 0; k < 2 && ok; ++k) {
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[k], (cs[k] + n_k[k] - 1) & 1, kTagPvDone));
        if (!ok) break;
        tc_fence_after();
        const int qt = 2 * u + k;
        // Whole-row sums from the two column halves.
        float *ls = reinterpret_cast<float *>(smem + C::kLOff) + k * 512;  // [h][2][128]
        ls[(h * 2 + 0) * 128 + r] = l[k];
        ls[(h * 2 + 1) * 128 + r] = lr[k];
        mbar_arrive(&bar_l[k * 4 + rq]);
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_l[k * 4 + rq], ui & 1, kTagLsum));
        if (!ok) break;
        if (r == 0 && h == 0) FA_TRACE(4 + k);
        const float lt = l[k] + ls[((h ^ 1) * 2 + 0) * 128 + r];
        const float lrt = lr[k] + ls[((h ^ 1) * 2 + 1) * 128 + r];
        const float inv_l = (FP8 ? p.descale_v[bh] : (DROPOUT ? p.drop.inv_keep : 1.f)) / lrt;
        const uint32_t tO = tmem + lane_off + 256 + k * D + h * (D / 2);
        const int row0 = qt * 128 + rq * 32;  // this warp's first query row
#pragma unroll 1
        for (int rd = 0; rd < D / 64; ++rd) {  // 32 columns at a time
          uint32_t o[32];
          tmem_ld32(tO + 32 * rd, o);
          tmem_wait_ld();
          for (int part = 0; part < 2; ++part) {  // O, then its rounding residual
            if (part == 1 && p.o_lo == nullptr) break;
            uint16_t *out = part == 0 ? p.o : p.o_lo;
            uint32_t wv[16];
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const float a = __uint_as_float(o[2 * t]) * inv_l, b = __uint_as_float(o[2 * t + 1]) * inv_l;
              const uint32_t hi = pack_bf16(a, b);
              // The residual: what rounding O to bf16 dropped, itself rounded to
              // bf16 (O ~ o + o_lo to about 16 significant bits; the backward's
              // D = rowsum(dO o O) uses it).
              wv[t] = part == 0 ? hi : pack_bf16(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xFFFF0000u));
            }
#pragma unroll
            for (int cq = 0; cq < 4; ++cq)
              st_shared_v4(stg + epi_offset<64>(lane, cq), wv[4 * cq], wv[4 * cq + 1], wv[4 * cq + 2], wv[4 * cq + 3]);
            __syncwarp();
            const int cq = lane & 3;
#pragma unroll
            for (int ps = 0; ps < 4; ++ps) {
              const int row = ps * 8 + (lane >> 2);
              if (row0 + row < p.N) {
                const size_t e = (static_cast<size_t>(bh) * p.N + row0 + row) * D + h * (D / 2) + rd * 32 + cq * 8;
                *reinterpret_cast<uint4 *>(out + e) = ld_shared_u4(stg + epi_offset<64>(row, cq));
              }
            }
            __syncwarp();  // the staging is rewritten by the next round
          }
        }
        const int grow = qt * 128 + r;
        if (h == 0 && grow < p.N) p.lse[static_cast<size_t>(bh) * p.N + grow] = (m[k] + log2f(lt)) * 0.69314718055994531f;
      }
      if (ok && threadIdx.x == 0) FA_TRACE(6);
      cs[0] += n_k[0];
      cs[1] += n_k[1];
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) FA_TRACE(7);
  if (warp == C::kIssuerWarp) tmem_dealloc(tmem, 512);
}

}  // namespace fa

// Backward main pass on CTA pairs (head dim 128): the same products as
// attn_bwd_kernel, executed as cta_group::2 MMAs by clusters of two CTAs that
// own adjacent 128-key tiles of one (batch, kv head) and sweep the same 64-query
// blocks ("AI Infra series ch. 6, GPU performance engineering (II)", section 7,
// item 3: one UMMA spans a CTA pair, each CTA loads half of the operand data,
// and the dQ reductions are halved).
//
// Per query block i, for the pair's 256 keys (rank r owns keys [128 r, 128 r + 128)):
//   S^T  = K Q_i^T    M = 256, N = 64    A: own K tile      B: Q_i rows [32 r, 32 r + 32)
//   dP^T = V dO_i^T   M = 256, N = 64    A: own V tile      B: dO_i rows [32 r, 32 r + 32)
//   P^T, dS^T in each CTA's tensor memory (softmax warps, as in the one-CTA pass)
//   dV  += P^T dO_i   M = 256, N = 128   A: own P^T (TMEM)  B: dO_i columns [64 r, 64 r + 64)
//   dK  += dS^T Q_i   M = 256, N = 128   A: own dS^T (TMEM) B: Q_i columns [64 r, 64 r + 64)
//   dQ_i^T = K^T dS^T M = 128, N = 64, contraction over all 256 keys
//                     A: K^T rows [64 r, 64 r + 64) of both tiles   B: dS^T columns [32 r, 32 r + 32)
// so per CTA the B operands of S^T, dP^T, dV and dK are half as large as in the
// one-CTA pass, and each CTA adds a 64 x 64 dQ tile (its half of the head dim)
// instead of a 64 x 128 one.
//
// dS^T reaches the dQ^T operand of both CTAs without generic stores into the
// other CTA (the cluster-scope proxy fence they need costs ~2000 clk): every
// softmax thread writes its own CTA's shared memory -- the query half of its own
// rank straight into the operand, the other half into a staging tile -- and a
// copy warp moves the staging tile into the other CTA's operand with one bulk
// copy whose bytes complete on that CTA's barrier.  The exchange overlaps the
// next block's S^T and dP^T MMAs: only dQ^T waits for it.
//
// Rank 0 issues every MMA and commits each completion to the barrier of both
// CTAs (two commits: no multicast).  Every TMA copy completes on a barrier of the
// CTA it fills, so each producer drains exactly the copies it issued; rank 1
// relays "landed" to rank 0 with one arrival, and its softmax and dQ warps arrive
// on rank 0's barriers remotely.  Every wait is bounded; before leaving, the two
// CTAs exchange one arrival each, so neither exits or frees its tensor memory
// while the other can still touch it.
//
// Warps: 0-7 softmax / dS and the dK, dV epilogue, 8-11 dQ staging, 12 TMA,
// 13 TMEM + MMA issue (rank 0) / relay of the tile arrivals (rank 1), 14 dQ
// reduce-adds, 15 dS^T exchange.
#pragma once

#include "bwd_kernels.cuh"

namespace attn {

template <bool DET>
struct BwdPairLayout {
  static constexpr int D = 128;
  static constexpr int BN = 128;                 // keys per CTA
  static constexpr int BQ = 64;                  // queries per block
  static constexpr int BOX = 128 * 128;          // 128 rows x 128 B
  static constexpr int HBOX = 32 * 128;          // 32 rows x 128 B
  static constexpr int QBOX = 64 * 128;          // 64 rows x 128 B
  static constexpr int K_OFF = 0;                // own K tile (two boxes)
  static constexpr int V_OFF = K_OFF + 2 * BOX;  // own V tile
  static constexpr int KT_OFF = V_OFF + 2 * BOX; // [t] = K of the pair's tile t, columns [64 r, 64 r + 64)
  static constexpr int STAGE_OFF = KT_OFF + 2 * BOX;
  // one stage: Q / dO rows [32 r, 32 r + 32) (two 4 KB boxes each), Q / dO columns [64 r, 64 r + 64)
  static constexpr int ST_QH = 0, ST_DOH = 2 * HBOX, ST_QB = 4 * HBOX, ST_DOB = ST_QB + QBOX;
  static constexpr int STAGE_BYTES = ST_DOB + QBOX;  // 32 KB
  static constexpr int NST = 2;                      // Q/dO ring depth
  static constexpr int NDS = DET ? 1 : 2;            // dS^T operand buffers
  static constexpr int NDQ = DET ? 2 : 1;            // dQ staging tiles
  // dS^T operand: [256 keys][32 queries] bf16, 64-byte rows, 64-byte swizzle (16-byte
  // chunk c of row R at chunk c ^ ((R / 2) % 4)); rows [128 t, 128 t + 128) come from rank t
  static constexpr int DS_OFF = STAGE_OFF + NST * STAGE_BYTES;
  static constexpr int DS_BYTES = 256 * 64;
  static constexpr int HALF_DS = 128 * 64;           // one rank's rows
  static constexpr int DSX_OFF = DS_OFF + NDS * DS_BYTES;     // [2] staging: own rows, the other rank's queries
  static constexpr int DQ_STAGE_OFF = DSX_OFF + 2 * HALF_DS;  // NDQ tiles, fp32 [64 q][64 dims]
  static constexpr int DQ_STAGE_BYTES = 64 * 64 * 4;
  static constexpr int LD_OFF = DQ_STAGE_OFF + NDQ * DQ_STAGE_BYTES;  // per stage: -lse2 (256 B), delta (256 B)
  static constexpr int BAR_OFF = LD_OFF + NST * 512;
  static constexpr int B_KV_FULL = 0;                   // own K, V, K^T landed
  static constexpr int B_QDO_FULL = 1;                  // [NST] own stage (tiles, -lse2, delta) landed
  static constexpr int B_QDO_EMPTY = 1 + NST;           // [NST] committed to both
  static constexpr int B_QDO_PEER = 1 + 2 * NST;        // [NST] rank 0: rank 1's stage landed (relay)
  static constexpr int B_KV_PEER = 1 + 3 * NST;         // rank 0: rank 1's K, V, K^T landed (relay)
  static constexpr int B_S_FULL = 2 + 3 * NST;          // committed to both
  static constexpr int B_DS_READY = B_S_FULL + 1;       // rank 0: 16 warp arrivals (8 per CTA): P^T, dS^T written
  static constexpr int B_PD_FREE = B_S_FULL + 2;        // committed to both
  static constexpr int B_DQ_FULL = B_S_FULL + 3;        // committed to both
  static constexpr int B_DQ_FREE = B_S_FULL + 4;        // rank 0: 8 warp arrivals (4 per CTA)
  static constexpr int B_D_FINAL = B_S_FULL + 5;        // committed to both
  static constexpr int B_DRAIN = B_S_FULL + 6;          // rank 0
  static constexpr int B_EXIT = B_S_FULL + 7;           // one arrival from the other CTA
  static constexpr int B_DSX_FULL = B_S_FULL + 8;       // [2] 4 warp arrivals: staging tile written
  static constexpr int B_DSX_FREE = B_DSX_FULL + 2;     // [2] its bulk copy has read it
  static constexpr int B_DS_IN = B_DSX_FREE + 2;        // [NDS] the other rank's rows have landed (8 KB of tx)
  static constexpr int B_DS_PEER = B_DS_IN + NDS;       // [NDS] rank 0: rank 1's operand complete (relay)
  static constexpr int B_STAGED = B_DS_PEER + NDS;      // [NDQ] 4 warp arrivals
  static constexpr int B_STAGE_FREE = B_STAGED + NDQ;   // [NDQ]
  static constexpr int N_BARS = B_STAGE_FREE + NDQ;
  static constexpr int TMEM_SLOT_OFF = BAR_OFF + 8 * N_BARS;
  static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 4;
  static constexpr int TICKET_OFF = ABORT_OFF + 4;
  static constexpr int SMEM_USED = TICKET_OFF + 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(DS_OFF % 1024 == 0 && DSX_OFF % 1024 == 0 && DQ_STAGE_OFF % 1024 == 0, "operand alignment");
  // tensor memory columns: S^T 64 | dP^T 64 | P^T 32 | dS^T 32 | dV 128 | dK 128 | dQ^T 32
  static constexpr uint32_t X_COL = 0;
  static constexpr uint32_t Y_COL = 64;
  static constexpr uint32_t P_COL = 128;
  static constexpr uint32_t DS_COL = 160;
  static constexpr uint32_t DV_COL = 192;
  static constexpr uint32_t DK_COL = 320;
  // dQ^T: each CTA's 64 x 64 part occupies 128 lanes x 32 columns -- lane l < 64
  // holds head dim 64 r + l for queries 0-31, lane 64 + l the same dim for queries 32-63
  static constexpr uint32_t DQ_COL = 448;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 512;
  static constexpr int WARP_TMA = 12, WARP_MMA = 13, WARP_RED = 14, WARP_XCHG = 15;
};

template <bool CAUSAL, bool DET>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(BwdPairLayout<DET>::THREADS, 1)
    attn_bwd_pair_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_q32, const __grid_constant__ CUtensorMap tm_do32,
                         const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
                         const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using L = BwdPairLayout<DET>;
  constexpr int D = L::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const sptr = smem_raw + (sbase - raw);
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  auto bar = [&](int slot) -> uint32_t { return sbase + L::BAR_OFF + 8u * slot; };
  // the same barrier in rank 0 / in the other CTA (shared::cluster addresses)
  auto lbar = [&](int slot) -> uint32_t { return mapa_shared(bar(slot), 0u); };
  auto pbar = [&](int slot) -> uint32_t { return mapa_shared(bar(slot), peer); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L::ABORT_OFF);
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // timeline build only (events per query block, as in the one-CTA pass: 0 S^T/dP^T
  // issued, 1 S^T ready at the softmax, 2 dS^T published, 3 dS^T seen by the issuer,
  // 4 dV/dK issued, 5 dQ^T issued, 6 dQ^T ready at the staging warps, 7 dQ tile
  // staged, 8 reduce-add issued, 9 its source read (fixed order: done, turn passed on),
  // 10 fixed order: turn received; and 11 dS^T half sent to the other CTA, 12 the
  // issuer has both CTAs' dS^T halves and the previous dQ^T read out, 13 (rank 1)
  // the other CTA's half landed; the issuer's events in rank 0 only)
  [[maybe_unused]] const bool tl = ATTN_TL_ON();
  ATTN_TL_T0(tl);

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::N_BARS; ++i) {
      uint32_t cnt = 1u;
      if (i == L::B_DS_READY) cnt = 16u;
      if (i == L::B_DQ_FREE) cnt = 8u;
      if (i == L::B_DSX_FULL || i == L::B_DSX_FULL + 1) cnt = 4u;
      if (i >= L::B_STAGED && i < L::B_STAGED + L::NDQ) cnt = 4u;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_mbar_init();
    // Work item of the pair: the cluster index, or in the deterministic instance a
    // ticket that rank 0 takes and hands to rank 1 (see the one-CTA pass).
    if (DET && rank == 0) {
      const int t = atomicAdd(p.ticket, 1);
      *reinterpret_cast<volatile int*>(sptr + L::TICKET_OFF) = t;
      st_shared_cl_u32(mapa_shared(sbase + L::TICKET_OFF, 1u), static_cast<uint32_t>(t));
    }
  }
  if (warp == L::WARP_MMA) {
    tmem_alloc_pair(sbase + L::TMEM_SLOT_OFF, L::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == L::WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q32);
    tma_prefetch_desc(&tm_do32);
    tma_prefetch_desc(&tm_q64);
    tma_prefetch_desc(&tm_do64);
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, the ticket published
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sptr + L::TMEM_SLOT_OFF);

  // ---- work decode (per pair): groups of bh_group (batch, kv head) pairs, and in
  // a group the pairs of low key tiles (most query blocks when causal) first
  const int n_clusters = static_cast<int>(gridDim.x >> 1);
  const int item = DET ? *reinterpret_cast<volatile int*>(sptr + L::TICKET_OFF) : static_cast<int>(blockIdx.x >> 1);
  const bool live = item < n_clusters;
  if (!live && threadIdx.x == 0) atomicExch(p.status, kDevWaitTimeout);
  const int n_pt = (p.n_kv_tiles + 1) >> 1;  // tile pairs per (batch, kv head)
  const int BH = p.B * p.H_kv;
  const int per_group = p.bh_group * n_pt;
  const int grp = item / per_group;
  const int within = item - grp * per_group;
  const int gs = min(p.bh_group, BH - grp * p.bh_group);
  const int pj = DET ? n_pt - 1 - within / gs : within / gs;  // pair index
  const int bh = grp * p.bh_group + (within % gs);
  const int b = bh / p.H_kv;
  const int hkv = bh - b * p.H_kv;
  const int G = p.H_q / p.H_kv;
  const int pk0 = pj * 2 * L::BN;                        // the pair's first key
  const int k0 = pk0 + static_cast<int>(rank) * L::BN;   // this CTA's first key
  const int diag = p.S_k - p.S_q;
  const int n_qb = p.S_pad / L::BQ;
  int qb0 = 0;
  if (CAUSAL) {
    const int first_q = pk0 - diag;
    qb0 = first_q <= 0 ? 0 : min(n_qb, first_q / L::BQ);
  }
  const int per_head = n_qb - qb0;
  const int m = live ? G * per_head : 0;

  if (warp == L::WARP_TMA) {
    // ===================== TMA producer (both CTAs, own barriers) =====================
    if (lane == 0) {
      const uint32_t kv_bar = bar(L::B_KV_FULL);
      mbar_arrive_expect_tx(kv_bar, 6 * L::BOX);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        tma_load_4d(sbase + L::K_OFF + x * L::BOX, &tm_k, kv_bar, x * 64, hkv, k0, b);
        tma_load_4d(sbase + L::V_OFF + x * L::BOX, &tm_v, kv_bar, x * 64, hkv, k0, b);
      }
#pragma unroll
      for (int t = 0; t < 2; ++t)
        tma_load_4d(sbase + L::KT_OFF + t * L::BOX, &tm_k, kv_bar, static_cast<int>(rank) * 64, hkv,
                    pk0 + t * L::BN, b);
      int issued = 0;
      for (int i = 0; i < m; ++i) {
        const int st = i % L::NST;
        if (i >= L::NST && !mbar_wait(bar(L::B_QDO_EMPTY + st), ((i / L::NST) - 1) & 1, ctl)) break;
        const int h = hkv * G + i / per_head;
        const int q0 = (qb0 + i % per_head) * L::BQ;
        const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
        const uint32_t fb = bar(L::B_QDO_FULL + st);
        mbar_arrive_expect_tx(fb, L::STAGE_BYTES + 512);
        const int qr = q0 + 32 * static_cast<int>(rank);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          tma_load_4d(sb + L::ST_QH + x * L::HBOX, &tm_q32, fb, x * 64, h, qr, b);
          tma_load_4d(sb + L::ST_DOH + x * L::HBOX, &tm_do32, fb, x * 64, h, qr, b);
        }
        tma_load_4d(sb + L::ST_QB, &tm_q64, fb, static_cast<int>(rank) * 64, h, q0, b);
        tma_load_4d(sb + L::ST_DOB, &tm_do64, fb, static_cast<int>(rank) * 64, h, q0, b);
        const size_t r = (static_cast<size_t>(b) * p.H_q + h) * p.S_pad + q0;
        bulk_load(sbase + L::LD_OFF + st * 512, p.nlse2 + r, 256, fb);
        bulk_load(sbase + L::LD_OFF + st * 512 + 256, p.delta + r, 256, fb);
        issued = i + 1;
      }
      // drain: every copy this CTA issued has landed before it leaves
      mbar_wait_drain(kv_bar, 0, 1000000000ull);
      for (int st = 0; st < L::NST && st < issued; ++st) {
        const int uses = (issued - 1 - st) / L::NST + 1;
        mbar_wait_drain(bar(L::B_QDO_FULL + st), (uses - 1) & 1, 1000000000ull);
      }
    }
  } else if (warp == L::WARP_MMA && rank == 1) {
    // ===================== relay (rank 1): own tiles landed -> rank 0's barriers =====================
    if (lane == 0) {
      bool ok = mbar_wait(bar(L::B_KV_FULL), 0, ctl);
      if (ok) mbar_arrive_cl(lbar(L::B_KV_PEER));
      for (int i = 0; ok && i < m; ++i) {
        const int st = i % L::NST;
        ok = mbar_wait(bar(L::B_QDO_FULL + st), (i / L::NST) & 1, ctl);
        if (ok) mbar_arrive_cl(lbar(L::B_QDO_PEER + st));
      }
    }
  } else if (warp == L::WARP_MMA) {
    // ===================== MMA issuer (rank 0) =====================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(256, L::BQ, false, false);  // S^T, dP^T
      constexpr uint32_t IDESC_G = idesc_bf16_f32(256, D, false, true);       // dV, dK (A in TMEM)
      constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, L::BQ, true, true);    // dQ^T over 256 keys
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      constexpr uint32_t HI64 = sdesc_sw64_hi(512);
      const uint32_t k_lo = sdesc_lo(sbase + L::K_OFF, 16), v_lo = sdesc_lo(sbase + L::V_OFF, 16);
      const uint32_t kt_lo = sdesc_lo(sbase + L::KT_OFF, L::BOX);
      const uint32_t s_full0 = bar(L::B_S_FULL), s_full1 = pbar(L::B_S_FULL);
      auto issue_s_dp = [&](int st) {
        const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
        const uint32_t qh_lo = sdesc_lo(sb + L::ST_QH, 16), doh_lo = sdesc_lo(sb + L::ST_DOH, 16);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * L::BOX + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * L::HBOX + (kk & 3) * 32;
          umma2_ss_h(tmem + L::X_COL, k_lo + (ao >> 4), HI, qh_lo + (bo >> 4), HI, IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * L::BOX + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * L::HBOX + (kk & 3) * 32;
          umma2_ss_h(tmem + L::Y_COL, v_lo + (ao >> 4), HI, doh_lo + (bo >> 4), HI, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma2_commit(s_full0);
        umma2_commit(s_full1);
      };
      // DS_IN[db] expects the other rank's 8 KB of block i; the thread that waits on
      // it arms its next use only after that wait, so it never runs a phase ahead
      for (int i = 0; i < L::NDS && i < m; ++i) mbar_arrive_expect_tx(bar(L::B_DS_IN + i), L::HALF_DS);
      bool ok = mbar_wait(bar(L::B_KV_FULL), 0, ctl) && mbar_wait(bar(L::B_KV_PEER), 0, ctl);
      if (ok && m > 0) {
        ok = mbar_wait(bar(L::B_QDO_FULL), 0, ctl) && mbar_wait(bar(L::B_QDO_PEER), 0, ctl);
        if (ok) {
          tc_fence_after();
          issue_s_dp(0);
          ATTN_TL(tl, 0, 0);
        }
      }
      for (int i = 0; ok && i < m; ++i) {
        const int st = i % L::NST;
        const int st1 = (i + 1) % L::NST;
        const int db = i % L::NDS;
        const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
        if (!mbar_wait(bar(L::B_DS_READY), i & 1, ctl)) {
          ok = false;
          break;
        }
        ATTN_TL(tl, 3, i);
        tc_fence_after();
        if (i + 1 < m) {
          const uint32_t par = ((i + 1) / L::NST) & 1;
          if (!mbar_wait(bar(L::B_QDO_FULL + st1), par, ctl) || !mbar_wait(bar(L::B_QDO_PEER + st1), par, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s_dp(st1);
          ATTN_TL(tl, 0, i + 1);
        }
        // dV += P^T dO_i ; dK += dS^T Q_i  (16 queries per MMA: 8 TMEM columns, 2 KB of the column box)
        const uint32_t dob_lo = sdesc_lo(sb + L::ST_DOB, L::QBOX), qb_lo = sdesc_lo(sb + L::ST_QB, L::QBOX);
#pragma unroll
        for (int kk = 0; kk < L::BQ / 16; ++kk)
          umma2_ts_h(tmem + L::DV_COL, tmem + L::P_COL + kk * 8, dob_lo + kk * 128, HI, IDESC_G,
                     (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < L::BQ / 16; ++kk)
          umma2_ts_h(tmem + L::DK_COL, tmem + L::DS_COL + kk * 8, qb_lo + kk * 128, HI, IDESC_G,
                     (i > 0 || kk > 0) ? 1u : 0u);
        umma2_commit(bar(L::B_PD_FREE));
        umma2_commit(pbar(L::B_PD_FREE));
        umma2_commit(bar(L::B_QDO_EMPTY + st));
        umma2_commit(pbar(L::B_QDO_EMPTY + st));
        ATTN_TL(tl, 4, i);
        // dQ^T_i needs both CTAs' dS^T operands complete and dQ^T_{i-1} read out
        const uint32_t dpar = (i / L::NDS) & 1;
        if (!mbar_wait(bar(L::B_DS_IN + db), dpar, ctl) || !mbar_wait(bar(L::B_DS_PEER + db), dpar, ctl) ||
            (i >= 1 && !mbar_wait(bar(L::B_DQ_FREE), (i - 1) & 1, ctl))) {
          ok = false;
          break;
        }
        ATTN_TL(tl, 12, i);
        if (i + L::NDS < m) mbar_arrive_expect_tx(bar(L::B_DS_IN + db), L::HALF_DS);
        tc_fence_after();
        // dQ_i^T = K^T dS_i^T over the pair's 256 keys: 16 keys per MMA = 2 KB of K^T, 1 KB of dS^T
        const uint32_t ds_lo = sdesc_lo(sbase + L::DS_OFF + db * L::DS_BYTES, L::DS_BYTES);
#pragma unroll
        for (int kk = 0; kk < 2 * L::BN / 16; ++kk)
          umma2_ss_h(tmem + L::DQ_COL, kt_lo + kk * 128, HI, ds_lo + kk * 64, HI64, IDESC_Q, kk > 0 ? 1u : 0u);
        umma2_commit(bar(L::B_DQ_FULL));
        umma2_commit(pbar(L::B_DQ_FULL));
        ATTN_TL(tl, 5, i);
      }
      if (ok) {
        umma2_commit(bar(L::B_D_FINAL));
        umma2_commit(pbar(L::B_D_FINAL));
      }
      umma2_commit(bar(L::B_DRAIN));
      mbar_wait_drain(bar(L::B_DRAIN), 0, 1000000000ull);
    }
  } else if (warp < 8) {
    // ===================== softmax / dS: thread = (own key row, half of the 64 queries) =====================
    const int r = threadIdx.x & 127;   // key row == TMEM lane
    const int hc = threadIdx.x >> 7;   // query half: columns [32 hc, 32 hc + 32); warp-uniform
    const bool own_half = hc == static_cast<int>(rank);  // dS^T goes straight into the operand
    const int key = k0 + r;
    const bool valid_key = live && key < p.S_k;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    // this thread's dS^T row: row rank * 128 + r of the operand, or row r of the staging tile
    // (the same swizzle phase: 128 is a multiple of 8)
    const uint32_t row_off = static_cast<uint32_t>(own_half ? L::DS_OFF + (static_cast<int>(rank) * L::BN + r) * 64
                                                            : L::DSX_OFF + r * 64);
    const int sw = (r >> 1) & 3;
    const uint32_t ds_ready = lbar(L::B_DS_READY);
    bool ok = true;
    for (int i = 0; i < m; ++i) {
      const int st = i % L::NST;
      const int q0 = (qb0 + i % per_head) * L::BQ;
      ok = mbar_wait(bar(L::B_S_FULL), i & 1, ctl);
      if (threadIdx.x == 0) ATTN_TL(tl, 1, i);
      if (ok) ok = mbar_wait(bar(L::B_QDO_FULL + st), (i / L::NST) & 1, ctl);  // -lse2, delta
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[32], dp[32];
      tmem_ld32(tmem + lane_addr + L::X_COL + 32 * hc, sv);
      tmem_ld32(tmem + lane_addr + L::Y_COL + 32 * hc, dp);
      tmem_ld_wait(sv);
      tmem_ld_wait(dp);
      const float4* nl4 = reinterpret_cast<const float4*>(sptr + L::LD_OFF + st * 512) + 8 * hc;
      const float4* dl4 = reinterpret_cast<const float4*>(sptr + L::LD_OFF + st * 512 + 256) + 8 * hc;
      const int c_first = (!valid_key ? L::BQ : (CAUSAL ? key - diag - q0 : 0)) - 32 * hc;
      const bool masked = __any_sync(0xffffffffu, c_first > 0);
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 nlv = nl4[c4];
        const float4 dlv = dl4[c4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int cp = 2 * c4 + h2;
          const float na = h2 ? nlv.z : nlv.x, nb = h2 ? nlv.w : nlv.y;
          const float da = h2 ? dlv.z : dlv.x, dbv = h2 ? dlv.w : dlv.y;
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[2 * cp]), __uint_as_float(sv[2 * cp + 1])), c2,
                                     f2_pack(na, nb));
          float x0, x1;
          f2_unpack(x2, x0, x1);
          float p0 = exp2_mufu(x0), p1 = exp2_mufu(x1);
          if (masked) {
            if (2 * cp < c_first) p0 = 0.f;
            if (2 * cp + 1 < c_first) p1 = 0.f;
          }
          const uint64_t g2 = f2_sub(f2_pack(__uint_as_float(dp[2 * cp]), __uint_as_float(dp[2 * cp + 1])),
                                     f2_pack(da, dbv));
          float d0, d1;
          f2_unpack(f2_mul(f2_pack(p0, p1), g2), d0, d1);
          pp[cp] = pack_bf16x2(p0, p1);
          pd[cp] = pack_bf16x2(d0, d1);
        }
      }
      // the destination of this block's dS^T row is free:
      //  * deterministic instance (one operand buffer): dQ^T_{i-1} has completed;
      //    otherwise buffer i % 2 was last read by dQ^T_{i-2}, complete before S_FULL(i)
      //  * staging tile i % 2: the bulk copy of block i - 2 has read it
      if (DET && i >= 1) {
        ok = mbar_wait(bar(L::B_DQ_FULL), (i - 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      if (!own_half && i >= 2) {
        ok = mbar_wait(bar(L::B_DSX_FREE + (i & 1)), ((i >> 1) - 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      uint8_t* dsrow = sptr + row_off + (own_half ? (i % L::NDS) * L::DS_BYTES : (i & 1) * L::HALF_DS);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(dsrow + ((c ^ sw) << 4)) = make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2],
                                                                          pd[4 * c + 3]);
      fence_proxy_async_smem();
      if (!own_half) mbar_arrive_warp(bar(L::B_DSX_FULL + (i & 1)));
      if (i >= 1) {  // dV_{i-1}, dK_{i-1} have read the previous P^T, dS^T
        ok = mbar_wait(bar(L::B_PD_FREE), (i - 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st16(tmem + lane_addr + L::P_COL + 16 * hc, pp);
      tmem_st16(tmem + lane_addr + L::DS_COL + 16 * hc, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive_cl_warp(ds_ready);
      if (threadIdx.x == 0) ATTN_TL(tl, 2, i);
    }
    // ---- epilogue: dV, dK (scaled) -> bf16; this thread writes head dims [64 hc, 64 hc + 64)
    if (ok && m > 0) {
      ok = mbar_wait(bar(L::B_D_FINAL), 0, ctl);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const size_t rowoff = ((static_cast<size_t>(b) * p.S_k + key) * p.H_kv + hkv) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? L::DV_COL : L::DK_COL;
        const float sc = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + rowoff;
#pragma unroll 1
        for (int ch = 2 * hc; ch < 2 * (hc + 1); ++ch) {
          uint32_t v[32];
          if (m > 0) {
            tmem_ld32(tmem + lane_addr + col + ch * 32, v);
            tmem_ld_wait(v);
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            pk[t] = pack_bf16x2(__uint_as_float(v[2 * t]) * sc, __uint_as_float(v[2 * t + 1]) * sc);
          if (valid_key) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
            for (int t = 0; t < 4; ++t) d4[t] = make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
          }
        }
      }
    }
  } else if (warp < 12) {
    // ===================== dQ staging: thread = (head dim, query half) =====================
    // TMEM lane l = 32 (warp % 4) + lane: head dim 64 rank + (l % 64), queries 32 (l / 64) + [0, 32)
    const int tml = (warp & 3) * 32 + lane;
    const int dl = tml & 63;
    const int qh = tml >> 6;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t dq_free = lbar(L::B_DQ_FREE);
    for (int i = 0; i < m; ++i) {
      bool ok = mbar_wait(bar(L::B_DQ_FULL), i & 1, ctl);
      if (threadIdx.x == 256) ATTN_TL(tl, 6, i);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_addr + L::DQ_COL, v);
      tmem_ld_wait(v);
      tc_fence_before();
      mbar_arrive_cl_warp(dq_free);
      const int buf = i % L::NDQ;
      if (i >= L::NDQ) {
        ok = mbar_wait(bar(L::B_STAGE_FREE + buf), ((i / L::NDQ) - 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      float* stage = reinterpret_cast<float*>(sptr + L::DQ_STAGE_OFF + buf * L::DQ_STAGE_BYTES);
#pragma unroll
      for (int c = 0; c < 32; ++c) stage[(qh * 32 + c) * 64 + dl] = __uint_as_float(v[c]);
      fence_proxy_async_smem();
      mbar_arrive_warp(bar(L::B_STAGED + buf));
      if (threadIdx.x == 256) ATTN_TL(tl, 7, i);
    }
  } else if (warp == L::WARP_RED) {
    // ===================== dQ reduce issue: one 64 x 64 TMA reduce-add per block =====================
    if (lane == 0) {
      for (int i = 0; i < m; ++i) {
        const int buf = i % L::NDQ;
        if (!mbar_wait(bar(L::B_STAGED + buf), (i / L::NDQ) & 1, ctl)) break;
        const int h = hkv * G + i / per_head;
        const int qb = qb0 + i % per_head;
        // Deterministic mode: the pairs that see query block qb are 0..J, and they add
        // in the order J, J - 1, ..., 0 (both CTAs of a pair after both of the pair
        // before; each CTA adds its own half of the head dims).
        int* sem = p.dq_sem + (static_cast<size_t>(b) * p.H_q + h) * (p.S_pad / 64) + qb;
        if (DET) {
          const int Jt = CAUSAL ? min(p.n_kv_tiles - 1, (64 * qb + 63 + (p.S_k - p.S_q)) / 128) : p.n_kv_tiles - 1;
          if (!sem_wait_ge(sem, 2 * (Jt / 2 - pj), ctl)) break;
          ATTN_TL(tl, 10, i);
          fence_proxy_async_global();
        }
        tma_reduce_add_4d(&tm_dqacc, sbase + L::DQ_STAGE_OFF + buf * L::DQ_STAGE_BYTES, static_cast<int>(rank) * 64,
                          h, qb * L::BQ, b);
        bulk_commit_group();
        ATTN_TL(tl, 8, i);
        if (DET) {
          bulk_wait_all();
          fence_proxy_async_global();
          __threadfence();
          sem_release_add(sem);
        } else {
          bulk_wait_read_all();
        }
        ATTN_TL(tl, 9, i);
        mbar_arrive(bar(L::B_STAGE_FREE + buf));
      }
      bulk_wait_all();
    }
  } else if (warp == L::WARP_XCHG) {
    // ===================== dS^T exchange: staging tile -> the other CTA's operand =====================
    if (lane == 0) {
      if (rank == 1)  // rank 1's operand expects rank 0's 8 KB (armed as in the issuer)
        for (int i = 0; i < L::NDS && i < m; ++i) mbar_arrive_expect_tx(bar(L::B_DS_IN + i), L::HALF_DS);
      for (int i = 0; i < m; ++i) {
        const int db = i % L::NDS;
        const int x = i & 1;
        if (!mbar_wait(bar(L::B_DSX_FULL + x), (i >> 1) & 1, ctl)) break;
        bulk_copy_to_peer(mapa_shared(sbase + L::DS_OFF + db * L::DS_BYTES + static_cast<int>(rank) * L::HALF_DS, peer),
                          sbase + L::DSX_OFF + x * L::HALF_DS, L::HALF_DS, pbar(L::B_DS_IN + db));
        bulk_commit_group();
        ATTN_TL(tl, 11, i);
        bulk_wait_read_all();
        mbar_arrive(bar(L::B_DSX_FREE + x));
        if (rank == 1) {  // tell rank 0 that rank 1's operand is complete for block i
          if (!mbar_wait(bar(L::B_DS_IN + db), (i / L::NDS) & 1, ctl)) break;
          ATTN_TL(tl, 13, i);
          if (i + L::NDS < m) mbar_arrive_expect_tx(bar(L::B_DS_IN + db), L::HALF_DS);
          mbar_arrive_cl(lbar(L::B_DS_PEER + db));
        }
      }
      bulk_wait_all();  // the copies have landed in the other CTA before this one leaves
    }
  }

  // Exit: each CTA tells the other it no longer touches the other's shared or
  // tensor memory and waits (bounded) for the same word from it; then the pair's
  // tensor memory is freed.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_cl_release(pbar(L::B_EXIT));
    if (!mbar_wait_cl_drain(bar(L::B_EXIT), 0, 2000000000ull)) atomicExch(p.status, kDevWaitTimeout);
  }
  __syncthreads();
  if (warp == L::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, L::TMEM_COLS);
  }
}

}  // namespace attn

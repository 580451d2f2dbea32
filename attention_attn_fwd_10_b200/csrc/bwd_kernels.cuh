// Backward attention kernels for sm_100a: dQ, dK, dV of L = sum(dO * O).
//
// Three launches on one stream:
//   1. attn_bwd_preprocess_kernel  delta_i = sum_d dO_id O_id (fp32), -lse_i*log2(e)
//                                  into padded rows, and dQ_acc = 0
//   2. attn_bwd_kernel             KV-stationary main pass (below)
//   3. attn_bwd_convert_kernel     dQ = scale * dQ_acc -> bf16
//
// Main pass: a CTA owns one 128-key tile (K_j, V_j) of one (batch, kv head) at
// a time and visits every 64-query block (Q_i, dO_i) of every query head of the
// group that sees it.  In the normal dQ order the CTA is persistent: a scheduler
// warp claims the tile of a CTA that has not started (cluster launch control)
// when the current tile's last loads are issued, and the new tile's K and V load
// once the old tile's last MMAs have read theirs (KV_EMPTY), while the old tile's
// dK and dV are written out; the new tile's first dV/dK MMA waits for that
// epilogue to have read the accumulators (D_EMPTY).  P is recomputed from lse rather than stored
// ("AI Infra series ch. 6, GPU performance engineering (II)", section 5,
// recomputation).  Per query block, all on tcgen05 with fp32 accumulation:
//   S^T  = K_j Q_i^T      (128 x 64, TMEM X)     dP^T = V_j dO_i^T   (TMEM Y)
//   P^T  = 2^(S^T c - lse2_i),  dS^T = P^T o (dP^T - delta_i)     (softmax warpgroup)
//          P^T and dS^T (bf16) are written to their own TMEM columns -- the
//          intermediates stay in tensor memory (section 7, item 3) -- and
//          dS^T also goes to shared memory for the dQ product
//   dV_j += P^T dO_i     (A from TMEM X)         dK_j += dS^T Q_i    (A from TMEM Y)
//   dQ_i^T = K_j^T dS^T  (128 x 64: both operands MN-major in shared memory)
// dV_j, dK_j accumulate in TMEM over all query blocks.  dQ_i^T goes to a TMEM
// buffer, a warpgroup copies it into a shared-memory staging tile, and a
// separate warp adds the tile into the fp32 dQ accumulator with one TMA
// reduce-add (the "atomic reductions" of section 7, item 3).  Every MMA has
// M = 128 except dQ^T at D = 64 (M = 64).
// Tensor-pipe order per block i: S^T_{i+1}, dP^T_{i+1}, dV_i, dK_i, dQ^T_i, so
// the softmax of block i+1 overlaps dV_i, dK_i and dQ^T_i.  Barriers: the
// softmax writes P^T_{i+1}, dS^T_{i+1} only after dV_i, dK_i completed
// (PD_FREE); dQ^T_{i+1} waits for the dQ warpgroup to have read dQ^T_i.
// Deterministic instance (DET): the additions into each (b, h, 64-query block)
// of the accumulator happen in a fixed order of key tiles, through bounded turn
// counters in global memory.
//
// Warp roles (512 threads): warps 0-7 softmax / dS and the dK, dV epilogue
// (thread = key row = TMEM lane, two warps per row, 32 queries each: P^T and dS^T
// need no row reduction, so the row splits freely); warps 8-11 dQ staging
// (thread = head-dim row of dQ^T; at D = 64 dQ^T is an M = 64 accumulator whose
// rows 16w..16w+15 sit in lanes 32w..32w+15, so half of each warp is idle);
// warp 12 TMA producer; warp 13 TMEM allocator and MMA issuer; warp 14 issues
// the dQ reduce-adds; warp 15 work scheduler.  Head dims 64 and 128.
#pragma once

#include "sm100_common.cuh"

namespace attn {

struct BwdParams {
  const __nv_bfloat16* o;   // [B, S_q, H_q, D]
  const __nv_bfloat16* dO;  // [B, S_q, H_q, D]
  const float* lse;         // [B, H_q, S_q] natural log
  float* dq_acc;            // [B, S_q, H_q, D] fp32 (workspace)
  float* nlse2;             // [B, H_q, S_pad] = -lse * log2(e); -inf for padding / empty rows (workspace)
  float* delta;             // [B, H_q, S_pad] (workspace)
  int* dq_sem;              // [B, H_q, S_pad / 64] dQ turn counters (workspace; deterministic mode)
  int* ticket;              // work-item counter of the deterministic main pass (workspace)
  // Main pass, normal dQ order: persistent CTAs (after its key tile a CTA takes over
  // the tile of a CTA that has not started, by cluster launch control, loading the new
  // tile's K and V while it finishes the old one's epilogue).  0 = one CTA per tile.
  int persistent;
  __nv_bfloat16* dq;        // [B, S_q, H_q, D]
  __nv_bfloat16* dk;        // [B, S_k, H_kv, D]
  __nv_bfloat16* dv;        // [B, S_k, H_kv, D]
  int B, H_q, H_kv, S_q, S_k, S_pad;
  int n_kv_tiles;           // ceil(S_k / 128)
  int bh_group;             // main-pass grid order: (batch, kv head) pairs per group
  float scale, scale_log2;
  int* status;
  uint64_t wait_limit_ns;
};

// ---------------------------------------------------------------------------
// 1. preprocess: D / 8 lanes per (b, q, h) row (8 bf16 per lane)
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(const BwdParams p) {
  constexpr int LANES = D / 8;          // lanes per row (8 bf16 each)
  constexpr int ROWS_PER_WARP = 32 / LANES;
  const long long rows = static_cast<long long>(p.B) * p.S_pad * p.H_q;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const long long warp_id = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  // whole warps iterate together (the row reduction below shuffles across the warp)
  for (long long r0 = warp_id * ROWS_PER_WARP; r0 < rows; r0 += n_warps * ROWS_PER_WARP) {
    const long long row = r0 + lane / LANES;
    const bool in_range = row < rows;
    const int h = static_cast<int>(row % p.H_q);
    const long long bq = row / p.H_q;
    const int q = static_cast<int>(bq % p.S_pad);
    const int b = static_cast<int>(bq / p.S_pad);
    float dot = 0.f;
    if (in_range && q < p.S_q) {
      const size_t base = ((static_cast<size_t>(b) * p.S_q + q) * p.H_q + h) * D + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(p.o + base);
      const uint4 dv = *reinterpret_cast<const uint4*>(p.dO + base);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 of = __bfloat1622float2(o2[i]);
        const float2 df = __bfloat1622float2(d2[i]);
        dot = fmaf(of.x, df.x, dot);
        dot = fmaf(of.y, df.y, dot);
      }
      float4* acc = reinterpret_cast<float4*>(p.dq_acc + base);
      acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      acc[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = LANES / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off, LANES);
    if (in_range && sub == 0 && (q & 63) == 0)
      p.dq_sem[(static_cast<size_t>(b) * p.H_q + h) * (p.S_pad / 64) + q / 64] = 0;
    if (r0 == 0 && lane == 0) *p.ticket = 0;
    if (in_range && sub == 0) {
      const size_t r = (static_cast<size_t>(b) * p.H_q + h) * p.S_pad + q;
      float nl = -INFINITY;  // padding rows and rows that saw no key give P = 0
      if (q < p.S_q) {
        const float l = p.lse[(static_cast<size_t>(b) * p.H_q + h) * p.S_q + q];
        if (l > -INFINITY) nl = -l * 1.4426950408889634f;
      }
      p.nlse2[r] = nl;
      p.delta[r] = q < p.S_q ? dot : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// 3. convert: dQ = scale * dQ_acc, 8 elements per thread
__global__ void __launch_bounds__(256) attn_bwd_convert_kernel(const BwdParams p, long long n8, int D) {
  (void)D;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc) + 2 * i;
    const float4 a = src[0], b = src[1];
    uint4 r;
    r.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    r.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    r.z = pack_bf16x2(b.x * p.scale, b.y * p.scale);
    r.w = pack_bf16x2(b.z * p.scale, b.w * p.scale);
    reinterpret_cast<uint4*>(p.dq)[i] = r;
  }
}

// ---------------------------------------------------------------------------
// 2. main pass.  DET = deterministic dQ order; it trades the third Q/dO stage
// for a second dQ staging tile, so a tile can wait for its turn while the next
// block is staged.
template <int D, bool DET>
struct BwdLayout {
  static constexpr int BN = 128;                  // keys per CTA
  static constexpr int BQ = 64;                   // queries per block
  static constexpr int NBOX = D / 64;
  static constexpr int KBOX_BYTES = 128 * 128;    // 128 rows x 128 B
  static constexpr int QBOX_BYTES = 64 * 128;     // 64 rows x 128 B
  static constexpr int KV_TILE = 128 * D * 2;
  static constexpr int Q_TILE = 64 * D * 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KV_TILE;
  static constexpr int NST = DET ? 2 : 3;         // Q/dO ring depth
  static constexpr int NDQ = DET ? 2 : 1;         // dQ staging tiles
  static constexpr int STAGE_OFF = V_OFF + KV_TILE;
  // one stage: Q_i, dO_i (1024-aligned); their -lse2_i and delta_i (64 fp32 each) sit in LD_OFF
  static constexpr int ST_Q = 0, ST_DO = Q_TILE;
  static constexpr int STAGE_BYTES = 2 * Q_TILE;
  static constexpr int DS_OFF = STAGE_OFF + NST * STAGE_BYTES;  // two dS^T buffers, 128 x 64 bf16
  static constexpr int DS_BYTES = 128 * 64 * 2;
  static constexpr int DQ_STAGE_OFF = DS_OFF + 2 * DS_BYTES;  // NDQ dQ_i staging tiles, fp32 [64 q][D]
  static constexpr int DQ_STAGE_BYTES = 64 * D * 4;
  static constexpr int LD_OFF = DQ_STAGE_OFF + NDQ * DQ_STAGE_BYTES;  // per stage: -lse2 (256 B), delta (256 B)
  static constexpr int BAR_OFF = LD_OFF + NST * 512;
  static constexpr int B_KV_FULL = 0;
  static constexpr int B_QDO_FULL = 1;            // [NST]
  static constexpr int B_QDO_EMPTY = 1 + NST;     // [NST]
  static constexpr int B_S_FULL = 1 + 2 * NST;    // S^T_i and dP^T_i in TMEM
  static constexpr int B_DS_READY = B_S_FULL + 1; // 8 warp arrivals: P^T_i, dS^T_i written
  static constexpr int B_PD_FREE = B_S_FULL + 2;  // dV_i, dK_i have read P^T_i, dS^T_i
  static constexpr int B_DQ_FULL = B_S_FULL + 3;  // dQ^T_i in TMEM
  static constexpr int B_DQ_FREE = B_S_FULL + 4;  // 4 warp arrivals: dQ^T_i read out
  static constexpr int B_D_FINAL = B_S_FULL + 5;
  static constexpr int B_DRAIN = B_S_FULL + 6;
  static constexpr int B_STAGED = B_S_FULL + 7;   // [NDQ] 4 warp arrivals: dQ_i staged in tile i % NDQ
  static constexpr int B_STAGE_FREE = B_S_FULL + 7 + NDQ;  // [NDQ] the reduce of that tile has read it
  static constexpr int B_KV_EMPTY = B_S_FULL + 7 + 2 * NDQ;  // the tile's last MMAs have read K, V
  static constexpr int B_D_EMPTY = B_KV_EMPTY + 1;  // 8 warp arrivals: the epilogue has read dV, dK
  static constexpr int B_ITEM_FULL = B_KV_EMPTY + 2;  // [u % 2] the scheduler published tile u's item
  static constexpr int B_ITEM_READ = B_KV_EMPTY + 4;  // every role read the current item (15 arrivals)
  static constexpr int B_CLC = B_KV_EMPTY + 5;        // cluster launch control response written
  static constexpr int N_BARS = B_KV_EMPTY + 6;
  static constexpr int ITEM_READERS = 15;  // TMA, MMA, 8 softmax warps, 4 dQ staging warps, reduce
  static constexpr int CLC_OFF = (BAR_OFF + 8 * N_BARS + 15) / 16 * 16;  // 16-byte response
  static constexpr int ITEM_OFF = CLC_OFF + 16;                         // items of tiles u % 2
  static constexpr int TMEM_SLOT_OFF = ITEM_OFF + 8;
  static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 4;
  static constexpr int SMEM_USED = ABORT_OFF + 4;
  static constexpr int SMEM_BYTES = (SMEM_USED + 1024) > 122880 ? (SMEM_USED + 1024) : 122880;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // tensor memory columns (512): S^T 64 | dP^T 64 | P^T 32 | dS^T 32 | dV D | dK D | dQ^T 64
  static constexpr uint32_t X_COL = 0;              // S^T (fp32, 64 query columns)
  static constexpr uint32_t Y_COL = 64;             // dP^T (fp32)
  static constexpr uint32_t P_COL = 128;            // P^T (bf16 pairs)
  static constexpr uint32_t DS_COL = 160;           // dS^T (bf16 pairs)
  static constexpr uint32_t DV_COL = 192;           // D columns
  static constexpr uint32_t DK_COL = 192 + D;       // D columns
  static constexpr uint32_t DQ_COL = 192 + 2 * D;   // 64 columns
  static constexpr uint32_t TMEM_COLS = 512;
  // warps 0-7 softmax / dS (two warps per key row, 32 queries each), 8-11 dQ
  // staging, 12 TMA, 13 TMEM + MMA, 14 dQ reduce issue, 15 work scheduler; 128
  // registers per thread.
  static constexpr int THREADS = 512;
  static constexpr int WARP_TMA = 12, WARP_MMA = 13, WARP_RED = 14, WARP_SCHED = 15;
};

template <int D, bool CAUSAL, bool DET>
__global__ void __launch_bounds__(BwdLayout<D, DET>::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using L = BwdLayout<D, DET>;
  static_assert(D == 64 || D == 128, "head dim 64 or 128");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const sptr = smem_raw + (sbase - raw);
  auto bar = [&](int slot) -> uint32_t { return sbase + L::BAR_OFF + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L::ABORT_OFF);
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // timeline build only (events per query block: 0 S^T/dP^T issued, 1 S^T ready at
  // the softmax, 2 dS^T published, 3 dS^T seen by the issuer, 4 dV/dK issued, 5 dQ^T
  // issued, 6 dQ^T ready at the staging warps, 7 dQ tile staged, 8 reduce-add issued,
  // 9 its source read (fixed dQ order: its additions done and the turn passed on),
  // 10 fixed dQ order: the turn received)
  [[maybe_unused]] const bool tl = ATTN_TL_ON();
  ATTN_TL_T0(tl);

  // Work items: key tiles.  The first is the block index, or in the deterministic
  // instance a ticket taken from a global counter when the CTA starts.  Items are
  // ordered so that the dQ additions an item waits for belong to items with smaller
  // numbers; with tickets those items were claimed by CTAs that had already started,
  // so every wait ends whatever order the hardware dispatches the blocks in.  With
  // persistent CTAs (normal dQ order only), the scheduler warp then claims the item
  // of a block that has not started (cluster launch control, the hardware's launch
  // order) once every role has read the current one; -1 = no more work.
  volatile int* item_slot = reinterpret_cast<volatile int*>(sptr + L::ITEM_OFF);
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::N_BARS; ++i)
      mbar_init(bar(i), i == L::B_DS_READY || i == L::B_D_EMPTY ? 8u
                        : (i == L::B_DQ_FREE || (i >= L::B_STAGED && i < L::B_STAGED + L::NDQ)) ? 4u
                        : i == L::B_ITEM_READ ? static_cast<uint32_t>(L::ITEM_READERS) : 1u);
    *abort_flag = 0;
    item_slot[0] = DET ? atomicAdd(p.ticket, 1) : static_cast<int>(blockIdx.x);
    fence_mbar_init();
    mbar_arrive(bar(L::B_ITEM_FULL));
  }
  if (warp == L::WARP_MMA) {
    tmem_alloc(sbase + L::TMEM_SLOT_OFF, L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == L::WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sptr + L::TMEM_SLOT_OFF);

  // ---- work decode: groups of bh_group (batch, kv head) pairs run together, so
  // the dQ accumulator rows and Q / dO tiles they share stay in L2; inside a
  // group, causal tiles with the most query blocks (low key index) come first
  struct Item {
    bool live;  // a ticket beyond the grid (the counter was not reset) touches nothing
    int b, hkv, j, k0, qb0, per_head, m;  // m: query blocks this tile visits
  };
  const int G = p.H_q / p.H_kv;
  const int diag = p.S_k - p.S_q;  // key k visible to query q iff k <= q + diag
  auto decode = [&](int item) {
    Item w;
    w.live = item < static_cast<int>(gridDim.x);
    const int BH = p.B * p.H_kv;
    const int per_group = p.bh_group * p.n_kv_tiles;
    const int grp = item / per_group;
    const int within = item - grp * per_group;
    const int gs = min(p.bh_group, BH - grp * p.bh_group);
    // deterministic instance: highest key tile first (see the dQ reduce below)
    w.j = DET ? p.n_kv_tiles - 1 - within / gs : within / gs;
    const int bh = grp * p.bh_group + (within % gs);
    w.b = bh / p.H_kv;
    w.hkv = bh - w.b * p.H_kv;
    w.k0 = w.j * L::BN;
    const int n_qb = p.S_pad / L::BQ;
    w.qb0 = 0;
    if (CAUSAL) {
      const int first_q = w.k0 - diag;  // first query that sees key k0
      w.qb0 = first_q <= 0 ? 0 : min(n_qb, first_q / L::BQ);
    }
    w.per_head = n_qb - w.qb0;
    w.m = w.live ? G * w.per_head : 0;
    return w;
  };
  // Tile u's item (-1 = no more work), or -2 once a wait was abandoned.
  auto read_item = [&](int u) -> int {
    if (!mbar_wait(bar(L::B_ITEM_FULL + (u & 1)), (u >> 1) & 1, ctl)) return -2;
    return item_slot[u & 1];
  };
  if (threadIdx.x == 0 && item_slot[0] >= static_cast<int>(gridDim.x)) atomicExch(p.status, kDevWaitTimeout);

  if (warp == L::WARP_SCHED) {
    // ===================== work scheduler =====================
    if (lane == 0) {
      int item = item_slot[0];
      uint32_t clc_phase = 0;
      for (int u = 0;; ++u) {
        if (!mbar_wait(bar(L::B_ITEM_READ), u & 1, ctl)) break;
        int next = -1;
        if (p.persistent && !DET && item >= 0) {
          mbar_arrive_expect_tx(bar(L::B_CLC), 16);
          clc_try_cancel(sbase + L::CLC_OFF, bar(L::B_CLC));
          if (!mbar_wait(bar(L::B_CLC), clc_phase, ctl)) break;
          clc_phase ^= 1;
          next = clc_cancelled_block(sbase + L::CLC_OFF);
        }
        item_slot[(u + 1) & 1] = next;
        mbar_arrive(bar(L::B_ITEM_FULL + ((u + 1) & 1)));
        item = next;
        if (next < 0) break;
      }
    }
  } else if (warp == L::WARP_TMA) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      int g = 0;   // Q/dO blocks loaded (all tiles): ring stage g % NST
      int nkv = 0; // K/V tiles loaded
      bool ok = true;
      for (int u = 0; ok; ++u) {
        const int item = read_item(u);
        if (item < 0) {
          if (item == -1) mbar_arrive(bar(L::B_ITEM_READ));
          break;
        }
        const Item w = decode(item);
        if (w.m == 0) mbar_arrive(bar(L::B_ITEM_READ));
        // the previous tile's last MMAs have read its K and V
        if (nkv > 0 && !(ok = mbar_wait(bar(L::B_KV_EMPTY), (nkv - 1) & 1, ctl))) break;
        mbar_arrive_expect_tx(bar(L::B_KV_FULL), 2 * L::KV_TILE);
#pragma unroll
        for (int x = 0; x < L::NBOX; ++x) {
          tma_load_4d(sbase + L::K_OFF + x * L::KBOX_BYTES, &tm_k, bar(L::B_KV_FULL), x * 64, w.hkv, w.k0, w.b);
          tma_load_4d(sbase + L::V_OFF + x * L::KBOX_BYTES, &tm_v, bar(L::B_KV_FULL), x * 64, w.hkv, w.k0, w.b);
        }
        ++nkv;
        for (int i = 0; i < w.m; ++i, ++g) {
          const int st = g % L::NST;
          if (g >= L::NST && !(ok = mbar_wait(bar(L::B_QDO_EMPTY + st), ((g / L::NST) - 1) & 1, ctl))) break;
          const int h = w.hkv * G + i / w.per_head;
          const int q0 = (w.qb0 + i % w.per_head) * L::BQ;
          const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
          const uint32_t fb = bar(L::B_QDO_FULL + st);
          mbar_arrive_expect_tx(fb, 2 * L::Q_TILE + 512);
#pragma unroll
          for (int x = 0; x < L::NBOX; ++x) {
            tma_load_4d(sb + L::ST_Q + x * L::QBOX_BYTES, &tm_q, fb, x * 64, h, q0, w.b);
            tma_load_4d(sb + L::ST_DO + x * L::QBOX_BYTES, &tm_do, fb, x * 64, h, q0, w.b);
          }
          const size_t r = (static_cast<size_t>(w.b) * p.H_q + h) * p.S_pad + q0;
          bulk_load(sbase + L::LD_OFF + st * 512, p.nlse2 + r, 256, fb);
          bulk_load(sbase + L::LD_OFF + st * 512 + 256, p.delta + r, 256, fb);
          // the next tile is claimed when this one's last loads are issued, so a CTA
          // does not hold on to pending work while it still has much of its own
          if (i == w.m - 1) mbar_arrive(bar(L::B_ITEM_READ));
        }
      }
      // Drain: every load this thread issued has landed before the CTA may exit.
      if (nkv > 0) mbar_wait_drain(bar(L::B_KV_FULL), (nkv - 1) & 1, 1000000000ull);
      for (int i = 0; i < L::NST && i < g; ++i) {
        const int n = g - 1 - i;
        mbar_wait_drain(bar(L::B_QDO_FULL + n % L::NST), (n / L::NST) & 1, 1000000000ull);
      }
    }
  } else if (warp == L::WARP_MMA) {
    // ===================== MMA issuer =====================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, L::BQ, false, false);   // S^T, dP^T
      constexpr uint32_t IDESC_G = idesc_bf16_f32(128, D, false, true);        // dV, dK (A in TMEM)
      constexpr uint32_t IDESC_Q = idesc_bf16_f32(D, L::BQ, true, true);       // dQ^T
      // shared-memory descriptors as (low, high) halves: the descriptor of base + off is
      // the base's low half plus off / 16 (one 32-bit add per MMA)
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      const uint32_t k_lo = sdesc_lo(sbase + L::K_OFF, 16), v_lo = sdesc_lo(sbase + L::V_OFF, 16);
      const uint32_t kT_lo = sdesc_lo(sbase + L::K_OFF, L::KBOX_BYTES);  // K^T: MN-major view of K
      auto issue_s_dp = [&](int st) {
        const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * L::KBOX_BYTES + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * L::QBOX_BYTES + (kk & 3) * 32;
          umma_ss_h(tmem + L::X_COL, k_lo + (ao >> 4), HI, sdesc_lo(sb + L::ST_Q, 16) + (bo >> 4), HI, IDESC_S,
                    kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk >> 2) * L::KBOX_BYTES + (kk & 3) * 32;
          const uint32_t bo = (kk >> 2) * L::QBOX_BYTES + (kk & 3) * 32;
          umma_ss_h(tmem + L::Y_COL, v_lo + (ao >> 4), HI, sdesc_lo(sb + L::ST_DO, 16) + (bo >> 4), HI, IDESC_S,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(L::B_S_FULL));
      };
      int g = 0;  // query blocks processed (all tiles): the per-block barriers' phases
      bool ok = true;
      for (int u = 0; ok; ++u) {
        const int item = read_item(u);
        if (item != -2) mbar_arrive(bar(L::B_ITEM_READ));
        if (item < 0) break;
        const Item w = decode(item);
        if (!(ok = mbar_wait(bar(L::B_KV_FULL), u & 1, ctl))) break;
        if (w.m > 0) {
          if (!(ok = mbar_wait(bar(L::B_QDO_FULL + g % L::NST), (g / L::NST) & 1, ctl))) break;
          tc_fence_after();
          issue_s_dp(g % L::NST);
          ATTN_TL(tl, 0, g);
        }
        // dV, dK of the previous tile have been read out by its epilogue
        if (u > 0 && !(ok = mbar_wait(bar(L::B_D_EMPTY), (u - 1) & 1, ctl))) break;
        for (int i = 0; i < w.m; ++i, ++g) {
          const int st = g % L::NST;        // Q/dO stage of block g
          const int st1 = (g + 1) % L::NST;
          const int db = g & 1;             // dS^T buffer of block g
          const uint32_t sb = sbase + L::STAGE_OFF + st * L::STAGE_BYTES;
          if (!(ok = mbar_wait(bar(L::B_DS_READY), g & 1, ctl))) break;
          ATTN_TL(tl, 3, g);
          tc_fence_after();
          // the next block's S^T, dP^T first: the softmax warpgroup starts on them while
          // the tensor pipe runs dV_i, dK_i, dQ^T_i
          if (i + 1 < w.m) {
            if (!(ok = mbar_wait(bar(L::B_QDO_FULL + st1), ((g + 1) / L::NST) & 1, ctl))) break;
            tc_fence_after();
            issue_s_dp(st1);
            ATTN_TL(tl, 0, g + 1);
          }
          // dV += P^T dO_i ; dK += dS^T Q_i   (16 queries per MMA: 8 TMEM columns, 2048 B of the stage)
#pragma unroll
          for (int kk = 0; kk < L::BQ / 16; ++kk)
            umma_ts_h(tmem + L::DV_COL, tmem + L::P_COL + kk * 8, sdesc_lo(sb + L::ST_DO, L::QBOX_BYTES) + kk * 128,
                      HI, IDESC_G, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < L::BQ / 16; ++kk)
            umma_ts_h(tmem + L::DK_COL, tmem + L::DS_COL + kk * 8, sdesc_lo(sb + L::ST_Q, L::QBOX_BYTES) + kk * 128,
                      HI, IDESC_G, (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar(L::B_PD_FREE));
          umma_commit(bar(L::B_QDO_EMPTY + st));
          ATTN_TL(tl, 4, g);
          if (g >= 1) {
            if (!(ok = mbar_wait(bar(L::B_DQ_FREE), (g - 1) & 1, ctl))) break;
            tc_fence_after();
          }
          // dQ_i^T = K_j^T dS_i^T : 16 keys per MMA = 2048 B of K_j and of dS^T
          const uint32_t ds = sbase + L::DS_OFF + db * L::DS_BYTES;
#pragma unroll
          for (int kk = 0; kk < L::BN / 16; ++kk)
            umma_ss_h(tmem + L::DQ_COL, kT_lo + kk * 128, HI, sdesc_lo(ds, L::DS_BYTES) + kk * 128, HI, IDESC_Q,
                      kk > 0 ? 1u : 0u);
          umma_commit(bar(L::B_DQ_FULL));
          ATTN_TL(tl, 5, g);
        }
        if (!ok) break;
        umma_commit(bar(L::B_D_FINAL));   // dV, dK of this tile complete
        umma_commit(bar(L::B_KV_EMPTY));  // its K, V read by every MMA
      }
      umma_commit(bar(L::B_DRAIN));
      mbar_wait_drain(bar(L::B_DRAIN), 0, 1000000000ull);
    }
  } else if (warp < 8) {
    // ===================== softmax / dS =====================
    // Warp w covers TMEM lanes (key rows) of quadrant w % 4 and query half hc = w / 4.
    // Each thread holds 4 key rows x 8 queries (shape 16x256b): rows 32 (w % 4) + 16 h +
    // lane/4 + 8 v (h, v in {0, 1}), queries 32 hc + 8 k + 2 (lane % 4) + {0, 1} (k < 4),
    // so it needs only 8 of the per-query terms -lse2 and delta, which the warp reads
    // with one 8-byte load per term and k (4 distinct addresses: one wavefront).
    const int r = threadIdx.x & 127;   // epilogue: key row == TMEM lane
    const int hc = threadIdx.x >> 7;   // query half: columns [32 hc, 32 hc + 32)
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int t0 = lane & 3, t1 = lane >> 2;
    const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
    int g = 0;  // query blocks processed (all tiles): the per-block barriers' phases
    bool ok = true;
    for (int u = 0; ok; ++u) {
      const int item = read_item(u);
      if (item != -2) mbar_arrive_warp(bar(L::B_ITEM_READ));
      if (item < 0) break;
      const Item w = decode(item);
      const int key = w.k0 + r;
      const bool valid_key = w.live && key < p.S_k;
      int row_key[4];  // [2 h + v]: the key of this thread's row (h, v)
#pragma unroll
      for (int hv = 0; hv < 4; ++hv) row_key[hv] = w.k0 + (warp & 3) * 32 + 16 * (hv >> 1) + t1 + 8 * (hv & 1);
      for (int i = 0; i < w.m; ++i, ++g) {
        const int st = g % L::NST;  // Q/dO stage (its -lse2, delta)
        const int db = g & 1;       // dS^T buffer
        const int q0 = (w.qb0 + i % w.per_head) * L::BQ;
        // S_FULL(g) is committed after dQ^T_{g-2}, so dS^T buffer `db` is free as well.
        ok = mbar_wait(bar(L::B_S_FULL), g & 1, ctl);
        if (threadIdx.x == 0) ATTN_TL(tl, 1, g);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[32], dp[32];  // [16 h + 4 k + 2 v + j]
        tmem_ld16x256_x4(tmem + lane_addr + L::X_COL + 32 * hc, sv);
        tmem_ld16x256_x4(tmem + lane_addr + (16u << 16) + L::X_COL + 32 * hc, sv + 16);
        tmem_ld16x256_x4(tmem + lane_addr + L::Y_COL + 32 * hc, dp);
        tmem_ld16x256_x4(tmem + lane_addr + (16u << 16) + L::Y_COL + 32 * hc, dp + 16);
        const float2* nl2 = reinterpret_cast<const float2*>(sptr + L::LD_OFF + st * 512) + 16 * hc + t0;
        const float2* dl2 = reinterpret_cast<const float2*>(sptr + L::LD_OFF + st * 512 + 256) + 16 * hc + t0;
        float2 nlk[4], dlk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          nlk[k] = nl2[4 * k];
          dlk[k] = dl2[4 * k];
        }
        tmem_ld_wait16(sv);
        tmem_ld_wait16(sv + 16);
        tmem_ld_wait16(dp);
        tmem_ld_wait16(dp + 16);
        // causal: key visible to query q0 + c iff c >= key - diag - q0; keys past S_k see nothing.
        // c_first is relative to this thread's first query column 32 hc + 2 (lane % 4).
        int c_first[4];
        bool any_mask = false;
#pragma unroll
        for (int hv = 0; hv < 4; ++hv) {
          const bool vk = w.live && row_key[hv] < p.S_k;
          c_first[hv] = (!vk ? L::BQ : (CAUSAL ? row_key[hv] - diag - q0 : 0)) - 32 * hc - 2 * t0;
          any_mask |= c_first[hv] > 0;
        }
        const bool masked = __any_sync(0xffffffffu, any_mask);
        uint32_t pp[16], pd[16];  // [8 h + 2 k + v]: the bf16 pair (queries 2 j) of row (h, v)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int e = 16 * h + 4 * k + 2 * v;
              const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), c2,
                                         f2_pack(nlk[k].x, nlk[k].y));
              float x0, x1;
              f2_unpack(x2, x0, x1);
              float p0 = exp2_mufu(x0), p1 = exp2_mufu(x1);
              if (masked) {
                const int cf = c_first[2 * h + v];
                if (8 * k < cf) p0 = 0.f;
                if (8 * k + 1 < cf) p1 = 0.f;
              }
              const uint64_t g2 = f2_sub(f2_pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                         f2_pack(dlk[k].x, dlk[k].y));
              float d0, d1;
              f2_unpack(f2_mul(f2_pack(p0, p1), g2), d0, d1);
              pp[8 * h + 2 * k + v] = pack_bf16x2(p0, p1);
              pd[8 * h + 2 * k + v] = pack_bf16x2(d0, d1);
            }
          }
        }
        // dS^T rows into the 128B-swizzled MN-major operand: the 4-byte pair of queries
        // 32 hc + 8 k + 2 (lane % 4) sits in 16-byte chunk 4 hc + k of its row, and chunk c of
        // row R at chunk c ^ (R % 8).  A warp's store covers 8 rows x 16 B: conflict-free.
        uint8_t* dsb = sptr + L::DS_OFF + db * L::DS_BYTES;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int R = (warp & 3) * 32 + 16 * h + t1 + 8 * v;
            uint8_t* row = dsb + R * 128 + 4 * t0;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint32_t*>(row + (((4 * hc + k) ^ (R & 7)) << 4)) = pd[8 * h + 2 * k + v];
          }
        }
        fence_proxy_async_smem();
        if (g >= 1) {  // dV, dK of the previous block have read the previous P^T, dS^T
          ok = mbar_wait(bar(L::B_PD_FREE), (g - 1) & 1, ctl);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
        }
        // P^T, dS^T (bf16 pairs; column = query / 2) with shape 16x128b: packed column
        // 16 hc + 4 k + lane % 4 of rows (h, v)
        tmem_st16x128_x4(tmem + lane_addr + L::P_COL + 16 * hc, pp);
        tmem_st16x128_x4(tmem + lane_addr + (16u << 16) + L::P_COL + 16 * hc, pp + 8);
        tmem_st16x128_x4(tmem + lane_addr + L::DS_COL + 16 * hc, pd);
        tmem_st16x128_x4(tmem + lane_addr + (16u << 16) + L::DS_COL + 16 * hc, pd + 8);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive_warp(bar(L::B_DS_READY));
        if (threadIdx.x == 0) ATTN_TL(tl, 2, g);
      }
      if (!ok) break;
      // ---- epilogue: dV, dK (scaled) -> bf16; this thread writes head dims [D/2 hc, D/2 (hc + 1))
      ok = mbar_wait(bar(L::B_D_FINAL), u & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const size_t rowoff = ((static_cast<size_t>(w.b) * p.S_k + key) * p.H_kv + w.hkv) * D;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const uint32_t col = which == 0 ? L::DV_COL : L::DK_COL;
          const float sc = which == 0 ? 1.f : p.scale;
          __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + rowoff;
#pragma unroll 1
          for (int ch = (D / 64) * hc; ch < (D / 64) * (hc + 1); ++ch) {
            uint32_t v[32];
            if (w.m > 0) {
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
      // dV, dK read out: the next tile's first dV, dK MMAs may overwrite them
      tc_fence_before();
      mbar_arrive_warp(bar(L::B_D_EMPTY));
    }
  } else if (warp < 12) {
    // ===================== dQ reduction warpgroup: thread = head-dim index =====================
    // dQ_i^T (TMEM) -> fp32 [64 q][D] tile in shared memory (NDQ tiles, used in
    // turn); warp WARP_RED adds each tile into the dQ accumulator.
    // dQ^T has M = D rows.  For D = 128 row d is TMEM lane d.  For D = 64 (an M = 64
    // accumulator) rows 16g..16g+15 sit in lanes 32g..32g+15: only the low 16 lanes
    // of each warp hold a row.
    const int wl = (warp & 3) * 32 + lane;  // this thread's TMEM lane
    const int d = D == 128 ? wl : ((lane < 16) ? (warp & 3) * 16 + lane : -1);
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int g = 0;  // query blocks processed (all tiles)
    bool ok = true;
    for (int u = 0; ok; ++u) {
      const int item = read_item(u);
      if (item != -2) mbar_arrive_warp(bar(L::B_ITEM_READ));
      if (item < 0) break;
      const int m = decode(item).m;
      for (int i = 0; i < m; ++i, ++g) {
        ok = mbar_wait(bar(L::B_DQ_FULL), g & 1, ctl);
        if (wl == 0) ATTN_TL(tl, 6, g);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[64];
        tmem_ld32(tmem + lane_addr + L::DQ_COL, v);
        tmem_ld32(tmem + lane_addr + L::DQ_COL + 32, v + 32);
        tmem_ld_wait(v);
        tmem_ld_wait(v + 32);
        tc_fence_before();
        mbar_arrive_warp(bar(L::B_DQ_FREE));
        const int buf = g % L::NDQ;
        if (g >= L::NDQ) {  // the reduce of block g - NDQ has read this tile
          ok = mbar_wait(bar(L::B_STAGE_FREE + buf), ((g / L::NDQ) - 1) & 1, ctl);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        float* stage = reinterpret_cast<float*>(sptr + L::DQ_STAGE_OFF + buf * L::DQ_STAGE_BYTES);
#pragma unroll
        for (int c = 0; c < L::BQ; ++c)
          if (d >= 0) stage[c * D + d] = __uint_as_float(v[c]);
        fence_proxy_async_smem();
        mbar_arrive_warp(bar(L::B_STAGED + buf));
        if (wl == 0) ATTN_TL(tl, 7, g);
      }
    }
  } else if (warp == L::WARP_RED) {
    // ===================== dQ reduce issue: one TMA reduce-add per staged tile =====================
    if (lane == 0) {
      int g = 0;  // query blocks processed (all tiles)
      bool ok = true;
      for (int u = 0; ok; ++u) {
        const int item = read_item(u);
        if (item != -2) mbar_arrive(bar(L::B_ITEM_READ));
        if (item < 0) break;
        const Item w = decode(item);
        for (int i = 0; i < w.m; ++i, ++g) {
          const int buf = g % L::NDQ;
          if (!(ok = mbar_wait(bar(L::B_STAGED + buf), (g / L::NDQ) & 1, ctl))) break;
          const int h = w.hkv * G + i / w.per_head;
          const int qb = w.qb0 + i % w.per_head;
          // Deterministic mode: the key tiles that see query block qb are 0..J (lower
          // keys are visible to more queries).  They add their parts in the order J,
          // J - 1, ..., 0 -- the order in which they reach the block, since tile j
          // starts its sweep two blocks before tile j - 1 -- so tile j waits for
          // J - j others.  High tiles have the smaller work-item numbers, so tile
          // j + 1's item was claimed by a CTA that started before this one: it is
          // running or done, and the wait always ends.
          int* sem = p.dq_sem + (static_cast<size_t>(w.b) * p.H_q + h) * (p.S_pad / 64) + qb;
          if (DET) {
            // J: the last tile whose first visited block, max(0, (128 J - diag) / 64), is <= qb
            const int J = CAUSAL ? min(p.n_kv_tiles - 1, (64 * qb + 63 + (p.S_k - p.S_q)) / 128) : p.n_kv_tiles - 1;
            if (!(ok = sem_wait_eq(sem, J - w.j, ctl))) break;
            ATTN_TL(tl, 10, g);
            fence_proxy_async_global();
          }
          tma_reduce_add_4d(&tm_dqacc, sbase + L::DQ_STAGE_OFF + buf * L::DQ_STAGE_BYTES, 0, h, qb * L::BQ, w.b);
          bulk_commit_group();
          ATTN_TL(tl, 8, g);
          if (DET) {
            bulk_wait_all();  // the additions are performed
            fence_proxy_async_global();
            __threadfence();
            sem_release_add(sem);
          } else {
            bulk_wait_read_all();  // the tile has been read
          }
          ATTN_TL(tl, 9, g);
          mbar_arrive(bar(L::B_STAGE_FREE + buf));
        }
      }
      bulk_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace attn

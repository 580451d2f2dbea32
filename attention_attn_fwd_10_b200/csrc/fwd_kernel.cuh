// Forward attention kernel for sm_100a:  O = softmax(scale * Q K^T [+ causal]) V, lse.
//
// One CTA owns a work unit of 256 query rows of one (batch, query head) -- two
// 128-row Q tiles, A and B -- and streams the key/value blocks they can see;
// each K_j / V_j block is loaded once and used by both tiles.  For short S_q the
// query heads of one kv group share the tiles instead (row r = position r / gp
// of head r % gp), so K / V are streamed once for the whole group.  Warp roles:
//   warps 0-3   softmax warpgroup of tile A (thread t owns row t: TMEM lane t)
//   warps 4-7   softmax warpgroup of tile B
//   warp  8     TMA producer: Q_A, Q_B once, then K_j into a 3-stage ring
//   warp  9     TMEM allocator and single-thread tcgen05.mma issuer
//   warp  10    TMA producer: V_j into a 2-stage ring
//   warp  11    work scheduler: with persistent CTAs, claims the unit of a CTA
//               that has not started (cluster launch control) for this one
// A non-causal grid whose last wave would hold at most half as many units as there
// are SMs leaves those units to a second launch of this kernel, two CTAs per unit,
// each running the dual stream on 128 of its rows (FwdParams::unit_base).
// K_j is released as soon as both tiles' S(j) have completed and V_j once both
// PV(j) have, so the next loads start a full MMA group earlier than with a
// shared K/V stage.
// Tensor memory (32-bit columns): S_A, S_B (128 x 128 fp32 scores each),
// O_A, O_B (128 x D fp32).  The softmax writes P_t (bf16, two per column)
// over the first 64 columns of S_t, and the PV MMA reads it from there.
// Tensor-pipe issue order per key block j:  PV_A(j), PV_B(j), S_A(j+1),
// S_B(j+1); S_t(j+1) is issued only once PV_t(j) has completed (it overwrites
// P_t(j)).  While one tile's softmax runs, the tensor pipe works on the other
// tile's MMAs: the fully asynchronous MMA pipeline with softmax/MMA overlap of
// FlashAttention-4 ("AI Infra series ch. 6, GPU performance engineering (II)",
// section 7; "NVIDIA's strongest B200 wastes 60%", second move).
//
// Softmax (per row, base-2 units t = s * scale * log2 e):
//   m_new = max(m_used, rowmax(t)); the running max actually used for the
//   exponentials, m_used, moves only when m_new - m_used > tau (conditional
//   rescaling, same article section 7 item 2); then O and l are rescaled by
//   2^(m_used_old - m_new).  Between rescales p = 2^(t - m_used) <= 2^tau.
//   The final O / l and lse = (m_used + log2 l) * ln 2 are exact whatever tau is.
//   A fixed subset of columns uses the FMA-pipe cubic 2^x, the rest MUFU ex2
//   (same article section 7 item 1; the hybrid of "NVIDIA's strongest B200
//   wastes 60%", first move).
#pragma once

#include <type_traits>

#include "sm100_common.cuh"


namespace attn {

struct FwdParams {
  __nv_bfloat16* o;  // [B, S_q, H_q, D]
  float* lse;        // [B, H_q, S_q]
  int B, H_q, H_kv, S_q, S_k;
  int n_units;       // work units per (batch, head pack): ceil(S_q / (256 / gp))
  int bh_group;      // grid order: (batch, head pack) pairs per group
  // Head packing: gp query heads of one kv group share a tile, tile row r holding
  // query position r / gp of head r % gp (gp = 1: one head per tile).  Used for
  // short S_q, where a tile of one head would be mostly empty; K / V are then
  // streamed once per pack instead of once per head.
  int gp, gp_log2;
  // Split-KV: each (unit, batch, head) is processed by n_splits CTAs, split s
  // taking key blocks [s * split_blocks, (s + 1) * split_blocks).  With
  // n_splits > 1 the kernel writes O_s (normalized within the split, fp32,
  // [n_splits, B, S_q, H_q, D]) and lse_s ([n_splits, B, H_q, S_q]) for
  // attn_fwd_combine_kernel instead of o and lse.
  int n_splits, split_blocks;
  float* o_part;
  float* lse_part;
  // Dual stream (used when one tile holds every query row of the unit): tile B
  // takes the odd key blocks of the CTA's range for the same rows as tile A, so
  // the two tiles' softmax/MMA chains overlap; tile A merges the two partial
  // results by the log-sum-exp identity in the epilogue.
  int dual;
  // Persistent CTAs: after its work item a CTA claims the item of a CTA that has
  // not started yet (cluster launch control) and processes it with the barriers,
  // rings and tensor memory it already holds.  Not with the dual stream.
  int persistent;
  // Tail launch (>= 0): this grid runs, as the dual stream, the work units from item
  // unit_base on of a grid launched just before it with the same parameters; its item
  // n is the 128-row half n % 2 of that grid's item unit_base + n / 2.  -1 otherwise.
  int unit_base;
  float scale_log2;  // scale * log2(e)
  float tau;         // rescale threshold (base-2 units); 0 = rescale on every increase
  int* status;       // device status word
  unsigned long long* rescale_count;  // optional: number of (row, block) rescales of O
  uint64_t wait_limit_ns;
};

// QK8: Q and K are e4m3 (1 byte per element; head dim 128 only), S = Q K^T runs
// as kind::f8f6f4; V, P and O stay bf16.  PV8 (with QK8): V is e4m3 too and P is
// rounded to e4m3 in tensor memory, so O += P V runs as kind::f8f6f4 as well.
template <int D, bool QK8 = false, bool PV8 = false>
struct FwdLayout {
  static constexpr int BM = 128;                 // query rows per tile
  static constexpr int UNIT = 256;               // query rows per work unit (two tiles)
  static constexpr int BN = 128;                 // keys per block
  static constexpr int KST = 3;                  // K ring depth (released after the last S MMA of a block)
  static constexpr int VST = 2;                  // V ring depth (released after the last PV MMA of a block)
  // In the dual stream tile B reads tile A's Q, and (bf16 Q, where a Q tile is
  // exactly a V tile) tile B's Q buffer becomes a third V slot: each step then
  // uses two V blocks and a third can be loading.
  static constexpr int VST_DUAL = (QK8 && !PV8) ? 2 : 3;
  static constexpr int NBOX = D / 64;            // 64-element (128 B) TMA boxes per row block
  static constexpr int BOX_BYTES = 128 * 128;    // one 128 x 64 bf16 box
  static constexpr int TILE_BYTES = 128 * D * 2; // one 128 x D bf16 tile
  static_assert(!QK8 || D == 128, "8-bit Q/K: head dim 128 (one 128-byte row per key)");
  static constexpr int QK_BYTES = QK8 ? 128 * D : TILE_BYTES;  // one Q or K tile
  static constexpr int QK_NBOX = QK8 ? 1 : NBOX;                // 128-byte TMA boxes per Q / K row
  static_assert(!PV8 || QK8, "8-bit V and P come with 8-bit Q and K");
  static constexpr int V_BYTES = PV8 ? 128 * D : TILE_BYTES;    // one V tile
  static constexpr int V_NBOX = PV8 ? 1 : NBOX;                 // 128-byte TMA boxes per V row
  static constexpr int Q_OFF = 0;                // two Q tiles
  static constexpr int K_OFF = Q_OFF + 2 * QK_BYTES;
  static constexpr int V_OFF = K_OFF + KST * QK_BYTES;
  static constexpr int BAR_OFF = V_OFF + VST * V_BYTES;
  // barrier slots (8 bytes each); [t] = per Q tile, [s] = per ring stage
  static constexpr int B_Q_FULL = 0;                    // [t]
  static constexpr int B_K_FULL = B_Q_FULL + 2;        // [ks]
  static constexpr int B_K_EMPTY = B_K_FULL + KST;     // [ks]
  static constexpr int B_V_FULL = B_K_EMPTY + KST;     // [vs], up to 3
  static constexpr int B_V_EMPTY = B_V_FULL + 3;       // [vs], up to 3
  static constexpr int B_S_FULL = B_V_EMPTY + 3;       // [t]
  static constexpr int B_P_FULL = B_S_FULL + 2;         // [t][half]  (one arrival per softmax warp)
  static constexpr int B_O_FINAL = B_P_FULL + 4;        // [t]
  static constexpr int B_DRAIN = B_O_FINAL + 2;
  static constexpr int B_XCHG = B_DRAIN + 1;            // dual stream: tile B's row statistics written (4 warps)
  static constexpr int B_Q_EMPTY = B_XCHG + 1;          // [t] the unit's last S_t has read Q_t
  static constexpr int B_ITEM_FULL = B_Q_EMPTY + 2;     // [u % 2] the scheduler published unit u's work item
  static constexpr int B_ITEM_READ = B_ITEM_FULL + 2;   // every role read the current item (11 arrivals)
  static constexpr int B_CLC = B_ITEM_READ + 1;         // cluster launch control response written
  static constexpr int N_BARS = B_CLC + 1;
  static constexpr int ITEM_READERS = 11;  // 8 softmax warps, the two producers, the issuer
  static constexpr int XCHG_OFF = BAR_OFF + 8 * N_BARS;  // dual stream: tile B's running max, sum per row (2 x 128 fp32)
  static constexpr int CLC_OFF = (XCHG_OFF + 1024 + 15) / 16 * 16;  // 16-byte cluster launch control response
  static constexpr int ITEM_OFF = CLC_OFF + 16;                     // work items of units u % 2
  static constexpr int TMEM_SLOT_OFF = ITEM_OFF + 8;
  static constexpr int ABORT_OFF = TMEM_SLOT_OFF + 4;
  static constexpr int SMEM_USED = ABORT_OFF + 4;
  // 1 KiB of slack to align the base to 1024 bytes (128-byte swizzle atoms);
  // at least 120 KiB so a single CTA occupies an SM (its TMEM request is 512 columns).
  static constexpr int SMEM_BYTES = (SMEM_USED + 1024) > 122880 ? (SMEM_USED + 1024) : 122880;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // tensor memory columns
  __device__ static constexpr uint32_t s_col(int t) { return static_cast<uint32_t>(t) * 128u; }
  __device__ static constexpr uint32_t o_col(int t) { return 256u + static_cast<uint32_t>(t) * D; }
  // shared-memory offset of V slot s (slot 2 only in the dual stream: tile B's Q buffer)
  __device__ static constexpr int v_off(int s) { return s < 2 ? V_OFF + s * V_BYTES : Q_OFF + QK_BYTES; }
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int WARP_TMA = 8, WARP_MMA = 9, WARP_TMA_V = 10, WARP_SCHED = 11;
  // Register split: launched at 168 per thread (384 x 168 = 64512); the two
  // softmax warpgroups grow to 216 and the third (producers, MMA issuer,
  // scheduler) shrinks to 72: 2 x 128 x 216 + 128 x 72 = 64512, the launch's total.
  static constexpr int REG_SOFTMAX = 216, REG_OTHER = 72;
};

// p = 2^(s * c - m) for one 128-column score row, packed to bf16 pairs; returns
// the fp32 sum of the unrounded p.  Column pair cp (columns 2cp, 2cp+1) takes
// the FMA-pipe cubic when cp % POLY_EVERY == POLY_EVERY - 1, MUFU ex2 otherwise.
// P8: the p values are packed as e4m3, four per word (16 words per half) instead
// of bf16 pairs (32 words).
template <int POLY_EVERY, bool P8 = false>
__device__ __forceinline__ float exp_half(const uint32_t* sr, float c, float m, uint32_t* pk, int half) {
  const uint64_t c2 = f2_pack(c, c);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t acc[4];  // 4 independent packed partial sums (8 lanes of accumulation)
  float pe0 = 0.f, pe1 = 0.f;  // P8: the previous pair, packed with the next one
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = 0ull;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int cp = 32 * half + q;
    const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sr[2 * cp]), __uint_as_float(sr[2 * cp + 1])), c2, nm2);
    float x0, x1, e0, e1;
    f2_unpack(x2, x0, x1);
    if (POLY_EVERY > 0 && (cp % (POLY_EVERY > 0 ? POLY_EVERY : 1)) == POLY_EVERY - 1) {
      exp2_poly_x2(x2, e0, e1);
    } else {
      e0 = exp2_mufu(x0);
      e1 = exp2_mufu(x1);
    }
    acc[q & 3] = f2_add(acc[q & 3], f2_pack(e0, e1));
    if constexpr (P8) {
      if (q & 1) pk[q >> 1] = pack_e4m3x4(pe0, pe1, e0, e1);
      pe0 = e0;
      pe1 = e1;
    } else {
      pk[q] = pack_bf16x2(e0, e1);
    }
  }
  float a0, a1;
  f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
  return a0 + a1;
}

// Maximum of a 128-column score row: 8 independent 3-input-max chains plus a tree.
__device__ __forceinline__ float row_max128(const uint32_t* sr) {
  const float* s = reinterpret_cast<const float*>(sr);
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(s[i], s[8 + i]);
#pragma unroll
  for (int cc = 16; cc < 128; cc += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmax3(m[i], s[cc + i], s[cc + 8 + i]);
  }
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Number of key blocks the query positions [row0, row0 + rows) of a tile can see
// (0 if the tile has no valid row, or none of its rows sees a key).
__device__ __forceinline__ int tile_blocks(int row0, int rows, int S_q, int S_k, bool causal, int BN) {
  if (row0 >= S_q) return 0;
  const int n_kv = (S_k + BN - 1) / BN;
  if (!causal) return n_kv;
  const int last_key = min(row0 + rows - 1, S_q - 1) + (S_k - S_q);
  return last_key < 0 ? 0 : min(n_kv, last_key / BN + 1);
}

template <int D, bool CAUSAL, int POLY_EVERY, bool QK8 = false, bool PV8 = false>
__global__ void __launch_bounds__(FwdLayout<D, QK8, PV8>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D, QK8, PV8>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* const sptr = smem_raw + (sbase - raw);
  auto bar = [&](int slot) -> uint32_t { return sbase + L::BAR_OFF + 8u * slot; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L::ABORT_OFF);
  volatile int* item_slot = reinterpret_cast<volatile int*>(sptr + L::ITEM_OFF);
  const WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool dual = p.dual != 0;
  // timeline build only (events: 0/1 S_t ready at the softmax, 2/3 row max done,
  // 4/5 P_t published, 6/7 PV_t issued, 8/9 next S_t issued, 10 V block ready at the
  // issuer, 15 V block load issued, per block of the tile; 11/12 O_t final at the
  // softmax, 13/14 epilogue done, per unit)
  [[maybe_unused]] const bool tl = ATTN_TL_ON();
  ATTN_TL_T0(tl);
  const int tile_pos = L::BM >> p.gp_log2;  // query positions per tile
  // A programmatic dependent may start launching now: the merge of split ranges (it
  // waits on the device for this grid's results) or the tail launch (independent work).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int diag = p.S_k - p.S_q;           // bottom-right causal: key j visible to row i iff j <= i + diag

  // ---- work items.  Item n is the work of block n of a one-CTA-per-unit grid:
  // groups of bh_group (batch, head pack) pairs run together, so the K / V rows
  // they read stay in L2 (heads of one kv group are adjacent); inside a group the
  // longest units come first for causal (the hardware starts blocks, and hands
  // out pending blocks to persistent CTAs, in index order: longest first); the
  // splits of one unit are adjacent.
  struct Unit {
    int b, h0, hkv, q0, j0, split;
    int nb0, nb1;     // steps of tile A, tile B
    int n_loads;      // K / V blocks the producers load, in order j0, j0 + 1, ...
    int n_blocks;     // max(nb0, nb1)
    bool ql0, ql1;    // Q tiles loaded: one per tile, or only tile A's in the dual stream
    __device__ int nblk(int t) const { return t == 0 ? nb0 : nb1; }
    __device__ bool q_loaded(int t) const { return t == 0 ? ql0 : ql1; }
  };
  auto decode = [&](int item) {
    Unit w;
    int sub = 0;  // tail launch: which 128-row half of the 256-row unit
    if (p.unit_base >= 0) {
      sub = item & 1;
      item = p.unit_base + (item >> 1);
    }
    const int BH = p.B * (p.H_q >> p.gp_log2);  // (batch, head pack) pairs
    w.split = item % p.n_splits;
    const int cta = item / p.n_splits;
    const int per_group = p.bh_group * p.n_units;
    const int grp = cta / per_group;
    const int within = cta - grp * per_group;
    const int gs = min(p.bh_group, BH - grp * p.bh_group);
    int u = within / gs;
    const int bh = grp * p.bh_group + (within - u * gs);
    if (CAUSAL) u = p.n_units - 1 - u;
    w.b = bh / (p.H_q >> p.gp_log2);
    w.h0 = (bh - w.b * (p.H_q >> p.gp_log2)) << p.gp_log2;  // first query head of the pack
    w.hkv = w.h0 / (p.H_q / p.H_kv);
    w.q0 = (2 * u + sub) * tile_pos;  // first query position of the unit
    // Key block of tile t's step j: j0 + j (both tiles take the same blocks), or in the
    // dual stream j0 + 2j + t.
    w.j0 = w.split * p.split_blocks;
    if (dual) {
      const int nb_all = min(max(tile_blocks(w.q0, tile_pos, p.S_q, p.S_k, CAUSAL, L::BN) - w.j0, 0), p.split_blocks);
      w.nb0 = (nb_all + 1) / 2;
      w.nb1 = nb_all / 2;
      w.n_loads = nb_all;
    } else {
      w.nb0 = min(max(tile_blocks(w.q0, tile_pos, p.S_q, p.S_k, CAUSAL, L::BN) - w.j0, 0), p.split_blocks);
      w.nb1 = min(max(tile_blocks(w.q0 + tile_pos, tile_pos, p.S_q, p.S_k, CAUSAL, L::BN) - w.j0, 0), p.split_blocks);
      w.n_loads = max(w.nb0, w.nb1);
    }
    w.n_blocks = max(w.nb0, w.nb1);
    w.ql0 = w.nb0 > 0;
    w.ql1 = w.nb1 > 0 && !dual;
    return w;
  };
  // Unit u's item (-1 = no more work) sits in slot u % 2 once ITEM_FULL[u % 2]
  // completes; every role arrives on ITEM_READ when it has read it, and only then
  // does the scheduler claim the next unit (one unit ahead of the slowest role).
  auto read_item = [&](int u) -> int {
    if (!mbar_wait(bar(L::B_ITEM_FULL + (u & 1)), (u >> 1) & 1, ctl)) return -2;
    return item_slot[u & 1];
  };

  // ---- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::N_BARS; ++i)
      mbar_init(bar(i), ((i >= L::B_P_FULL && i < L::B_P_FULL + 4) || i == L::B_XCHG) ? 4u
                        : i == L::B_ITEM_READ ? static_cast<uint32_t>(L::ITEM_READERS) : 1u);
    *abort_flag = 0;
    item_slot[0] = static_cast<int>(blockIdx.x);  // unit 0: this block's own item
    fence_mbar_init();
    mbar_arrive(bar(L::B_ITEM_FULL));
  }
  if (warp == L::WARP_MMA) {
    tmem_alloc(sbase + L::TMEM_SLOT_OFF, L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == L::WARP_TMA && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sptr + L::TMEM_SLOT_OFF);
  static_assert(2 * 128 * L::REG_SOFTMAX + 128 * L::REG_OTHER <= L::THREADS * 168, "register split");

  if (warp >= 8) {
    // Each role's register budget is set inside its own branch, so the
    // register allocator sees the budget that dominates the role's code.
    setmaxnreg_dec<L::REG_OTHER>();
  }
  if (warp == L::WARP_TMA) {
    // ===================== TMA producer: Q, K =====================
    if (lane == 0) {
      int kn = 0;              // K blocks loaded (all units)
      int qn0 = 0, qn1 = 0;    // Q_A, Q_B tiles loaded
      bool ok = true;
      for (int u = 0; ok; ++u) {
        const int item = read_item(u);
        mbar_arrive(bar(L::B_ITEM_READ));
        if (item < 0) break;
        const Unit w = decode(item);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok || !w.q_loaded(t)) continue;
          int& qn = t == 0 ? qn0 : qn1;
          // the previous unit's last S_t has read Q_t
          if (qn > 0 && !(ok = mbar_wait(bar(L::B_Q_EMPTY + t), (qn - 1) & 1, ctl))) break;
          mbar_arrive_expect_tx(bar(L::B_Q_FULL + t), L::QK_BYTES);
#pragma unroll
          for (int x = 0; x < L::QK_NBOX; ++x)
            tma_load_4d(sbase + L::Q_OFF + t * L::QK_BYTES + x * L::BOX_BYTES, &tm_q, bar(L::B_Q_FULL + t),
                        x * 64, w.h0, w.q0 + t * tile_pos, w.b);
          ++qn;
        }
        for (int j = 0; ok && j < w.n_loads; ++j) {
          const int s = kn % L::KST;
          if (kn >= L::KST && !(ok = mbar_wait(bar(L::B_K_EMPTY + s), ((kn / L::KST) - 1) & 1, ctl))) break;
          mbar_arrive_expect_tx(bar(L::B_K_FULL + s), L::QK_BYTES);
#pragma unroll
          for (int x = 0; x < L::QK_NBOX; ++x)
            tma_load_4d(sbase + L::K_OFF + s * L::QK_BYTES + x * L::BOX_BYTES, &tm_k, bar(L::B_K_FULL + s),
                        x * 64, w.hkv, (w.j0 + j) * L::BN, w.b);
          ++kn;
        }
      }
      // Drain: every load this thread issued has landed before the CTA may exit.
      if (qn0 > 0) mbar_wait_drain(bar(L::B_Q_FULL), (qn0 - 1) & 1, 1000000000ull);
      if (qn1 > 0) mbar_wait_drain(bar(L::B_Q_FULL + 1), (qn1 - 1) & 1, 1000000000ull);
      for (int i = 0; i < L::KST && i < kn; ++i) {
        const int n = kn - 1 - i;
        mbar_wait_drain(bar(L::B_K_FULL + n % L::KST), (n / L::KST) & 1, 1000000000ull);
      }
    }
  } else if (warp == L::WARP_TMA_V) {
    // ===================== TMA producer: V =====================
    if (lane == 0) {
      // V slots in use: VST, or VST_DUAL in the dual stream (the same for every unit)
      auto load_v = [&](auto nv_c) {
        constexpr int nv = decltype(nv_c)::value;
        int vn = 0;  // V blocks loaded (all units)
        bool ok = true;
        for (int u = 0; ok; ++u) {
          const int item = read_item(u);
          mbar_arrive(bar(L::B_ITEM_READ));
          if (item < 0) break;
          const Unit w = decode(item);
          for (int j = 0; ok && j < w.n_loads; ++j) {
            const int s = vn % nv;
            if (vn >= nv && !(ok = mbar_wait(bar(L::B_V_EMPTY + s), ((vn / nv) - 1) & 1, ctl))) break;
            mbar_arrive_expect_tx(bar(L::B_V_FULL + s), L::V_BYTES);
#pragma unroll
            for (int x = 0; x < L::V_NBOX; ++x)
              tma_load_4d(sbase + L::v_off(s) + x * L::BOX_BYTES, &tm_v, bar(L::B_V_FULL + s),
                          x * 64, w.hkv, (w.j0 + j) * L::BN, w.b);
            ATTN_TL(tl, 15, vn);
            ++vn;
          }
        }
        for (int i = 0; i < nv && i < vn; ++i) {
          const int n = vn - 1 - i;
          mbar_wait_drain(bar(L::B_V_FULL + n % nv), (n / nv) & 1, 1000000000ull);
        }
      };
      if (dual)
        load_v(std::integral_constant<int, L::VST_DUAL>{});
      else
        load_v(std::integral_constant<int, L::VST>{});
    }
  } else if (warp == L::WARP_MMA) {
    // ===================== MMA issuer =====================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
      // The shared-memory base goes through an opaque move in each call, so the MMA
      // descriptors are computed where they are used rather than hoisted out of the
      // unit and block loops (this warp has 72 registers).
      auto opaque = [](uint32_t x) {
        uint32_t y;
        asm volatile("mov.b32 %0, %1;" : "=r"(y) : "r"(x));
        return y;
      };
      // Descriptors as (low, high) halves: the high half is a constant, and the
      // descriptor of base + off is the base's low half plus off / 16, one 32-bit add
      // per MMA.
      constexpr uint32_t HI = sdesc_sw128_hi(1024);
      auto issue_s = [&](int t, int stage) {
        const uint32_t base = opaque(sbase);
        const uint32_t qd = sdesc_lo(base + L::Q_OFF + (dual ? 0 : t) * L::QK_BYTES, 16);
        const uint32_t kd = sdesc_lo(base + L::K_OFF + stage * L::QK_BYTES, 16);
        if constexpr (QK8) {
          // 32 head dims (32 bytes of the 128-byte row) per MMA
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            umma_ss_f8_h(tmem + L::s_col(t), qd + (kk * 32 >> 4), HI, kd + (kk * 32 >> 4), HI,
                         idesc_e4m3_f32(128, 128), kk > 0 ? 1u : 0u);
          umma_commit(bar(L::B_S_FULL + t));
          return;
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::BOX_BYTES + (kk & 3) * 32;
          umma_ss_h(tmem + L::s_col(t), qd + (off >> 4), HI, kd + (off >> 4), HI, IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(L::B_S_FULL + t));
      };
      // PV_t(j) in two halves of 64 keys, each issued once its half of P_t(j) is in TMEM
      auto issue_pv_half = [&](int t, int stage, bool acc, int hf) {
        const uint32_t v_base = opaque(sbase) + L::v_off(stage);
        if constexpr (PV8) {
          // 32 keys per MMA: 8 columns of e4m3 P (4 per column), 32 rows of 128 B of V
          // (MN-major, one 128-byte column block: LBO unused)
          constexpr uint32_t IDESC_PV8 = idesc_e4m3_f32(128, D) | (1u << 16);
          const uint32_t vd = sdesc_lo(v_base, 16);
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int kk = 2 * hf + k2;
            umma_ts_f8_h(tmem + L::o_col(t), tmem + L::s_col(t) + kk * 8, vd + (kk * 4096 >> 4), HI, IDESC_PV8,
                         (acc || kk > 0) ? 1u : 0u);
          }
          return;
        }
        const uint32_t vd = sdesc_lo(v_base, L::BOX_BYTES);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * hf + k4;
          // 16 keys = 16 rows of 128 B = 2048 bytes; 64-wide d blocks are BOX_BYTES apart.
          umma_ts_h(tmem + L::o_col(t), tmem + L::s_col(t) + kk * 8, vd + (kk * 2048 >> 4), HI, IDESC_PV,
                    (acc || kk > 0) ? 1u : 0u);
        }
      };
      // K / V blocks consumed (all units): ring slot n % KST and n % VST (VST_DUAL in the
      // dual stream), phase n / KST and n / VST
      int kc = 0, vc = 0;
      int qc0 = 0, qc1 = 0;  // Q_A, Q_B tiles consumed
      int pc0 = 0, pc1 = 0;  // blocks of tile A, tile B processed (S_FULL / P_FULL phases)
      bool ok = true;
      for (int u = 0; ok; ++u) {
        const int item = read_item(u);
        mbar_arrive(bar(L::B_ITEM_READ));
        if (item < 0) break;
        const Unit w = decode(item);
        if (w.n_blocks == 0) continue;
        if (dual) {
          // Dual stream: tile t takes key blocks j0 + 2j + t.  Load n = 2j + t of the unit
          // is used by one tile only; the S and the PV MMAs each consume their ring in
          // load order.
          for (int t = 0; ok && t < 2; ++t) {
            if (w.nblk(t) == 0) continue;
            ok = mbar_wait(bar(L::B_K_FULL + kc % L::KST), (kc / L::KST) & 1, ctl);
            if (ok && t == 0) ok = mbar_wait(bar(L::B_Q_FULL), qc0 & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            issue_s(t, kc % L::KST);
            umma_commit(bar(L::B_K_EMPTY + kc % L::KST));
            ++kc;
          }
          // both tiles read Q_A: release it after the unit's last S
          if (ok && w.n_loads <= 2) umma_commit(bar(L::B_Q_EMPTY));
          for (int j = 0; ok && j < w.n_blocks; ++j) {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok || j >= w.nblk(t)) continue;
              const int vs = vc % L::VST_DUAL;
              ok = mbar_wait(bar(L::B_V_FULL + vs), (vc / L::VST_DUAL) & 1, ctl);
              ATTN_TL(tl, 10, vc);
              ok = ok && mbar_wait(bar(L::B_P_FULL + 2 * t), ((t == 0 ? pc0 : pc1) + j) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv_half(t, vs, j > 0, 0);
              ok = mbar_wait(bar(L::B_P_FULL + 2 * t + 1), ((t == 0 ? pc0 : pc1) + j) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv_half(t, vs, j > 0, 1);
              ATTN_TL(tl, 6 + t, (t == 0 ? pc0 : pc1) + j);
              if (j == w.nblk(t) - 1) umma_commit(bar(L::B_O_FINAL + t));
              umma_commit(bar(L::B_V_EMPTY + vs));
              ++vc;
              if (j + 1 < w.nblk(t)) {
                const int ks = kc % L::KST;
                ok = mbar_wait(bar(L::B_K_FULL + ks), (kc / L::KST) & 1, ctl);
                if (!ok) break;
                issue_s(t, ks);
                umma_commit(bar(L::B_K_EMPTY + ks));
                // the unit's last S reads Q_A (both tiles use it): release it after that one
                if (2 * (j + 1) + t == w.n_loads - 1) umma_commit(bar(L::B_Q_EMPTY));
                ++kc;
              }
            }
          }
        } else {
          // S_t(0) of both tiles on K_0 of the unit.  This overwrites S_t / P_t of the
          // previous unit, whose PV MMAs this thread issued first.
          ok = mbar_wait(bar(L::B_K_FULL + kc % L::KST), (kc / L::KST) & 1, ctl);
          for (int t = 0; ok && t < 2; ++t) {
            if (w.nblk(t) == 0) continue;
            ok = mbar_wait(bar(L::B_Q_FULL + t), (t == 0 ? qc0 : qc1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            issue_s(t, kc % L::KST);
            if (w.nblk(t) == 1) umma_commit(bar(L::B_Q_EMPTY + t));  // the unit's last S_t has been issued
          }
          if (!ok) break;
          umma_commit(bar(L::B_K_EMPTY + kc % L::KST));  // K_0 released once both S(0) complete
          ++kc;
          // Per key block j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1).  S_t(j+1) overwrites
          // P_t(j), which PV_t(j) reads: the MMAs of this one issuing thread execute
          // in issue order, so PV_t(j) has read P_t(j) before S_t(j+1) writes there.
          // The first PV_t of a unit overwrites O_t: the softmax publishes P_t(0) only
          // after its epilogue has read the previous unit's O_t.
          for (int j = 0; ok && j < w.n_blocks; ++j) {
            const int vs = vc % L::VST;
            const int ks1 = kc % L::KST;
            if (!(ok = mbar_wait(bar(L::B_V_FULL + vs), (vc / L::VST) & 1, ctl))) break;
            ATTN_TL(tl, 10, vc);
            bool k_next_ready = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              if (!ok || j >= w.nblk(t)) continue;
              ok = mbar_wait(bar(L::B_P_FULL + 2 * t), ((t == 0 ? pc0 : pc1) + j) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv_half(t, vs, j > 0, 0);
              ok = mbar_wait(bar(L::B_P_FULL + 2 * t + 1), ((t == 0 ? pc0 : pc1) + j) & 1, ctl);
              if (!ok) break;
              tc_fence_after();
              issue_pv_half(t, vs, j > 0, 1);
              ATTN_TL(tl, 6 + t, (t == 0 ? pc0 : pc1) + j);
              if (j == w.nblk(t) - 1) umma_commit(bar(L::B_O_FINAL + t));
              if (j + 1 < w.nblk(t)) {
                if (!k_next_ready) {
                  ok = mbar_wait(bar(L::B_K_FULL + ks1), (kc / L::KST) & 1, ctl);
                  if (!ok) break;
                  k_next_ready = true;
                }
                issue_s(t, ks1);
                ATTN_TL(tl, 8 + t, (t == 0 ? pc0 : pc1) + j + 1);
                if (j + 2 == w.nblk(t)) umma_commit(bar(L::B_Q_EMPTY + t));  // the unit's last S_t
              }
            }
            if (!ok) break;
            umma_commit(bar(L::B_V_EMPTY + vs));
            ++vc;
            if (k_next_ready) {
              umma_commit(bar(L::B_K_EMPTY + ks1));
              ++kc;
            }
          }
        }
        pc0 += w.nb0;
        pc1 += w.nb1;
        qc0 += w.ql0 ? 1 : 0;
        qc1 += w.ql1 ? 1 : 0;
      }
      // Drain: no MMA may still be writing TMEM when it is released.
      umma_commit(bar(L::B_DRAIN));
      mbar_wait_drain(bar(L::B_DRAIN), 0, 1000000000ull);
    }
  } else if (warp == L::WARP_SCHED) {
    // ===================== work scheduler =====================
    // Unit u + 1's item: once every role has read unit u's, the next pending block of
    // the grid (the hardware's launch order) is cancelled and its item taken over.
    // Without the persistent mode, or once no block is left, the item is -1.
    if (lane == 0) {
      int item = static_cast<int>(blockIdx.x);
      uint32_t clc_phase = 0;
      for (int u = 0;; ++u) {
        if (!mbar_wait(bar(L::B_ITEM_READ), u & 1, ctl)) break;
        int next = -1;
        if (p.persistent && item >= 0) {
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
  } else if (warp < 8) {
    // ===================== softmax warpgroups (warps 0-3: tile A, 4-7: tile B) =====================
    setmaxnreg_inc<L::REG_SOFTMAX>();
    const int t = warp >> 2;
    const int row = threadIdx.x & 127;  // == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float c = p.scale_log2;
    int sc = 0;  // blocks of this tile processed (S_FULL / P_FULL phases)
    int oc = 0;  // O_FINAL phases consumed
    bool ok = true;
    for (int u = 0; ok; ++u) {
      const int item = read_item(u);
      if (item < 0) {
        mbar_arrive_warp(bar(L::B_ITEM_READ));
        break;
      }
      int nb, kb0, lim, lim_tile;  // the key-block loop needs only these (the rest is decoded again after it)
      bool idle;                   // every row of this warp is padding (past S_q)
      {
        const Unit w = decode(item);
        const int row0 = w.q0 + (dual ? 0 : t * tile_pos);  // first query position of the tile
        const int qi = row0 + (row >> p.gp_log2);           // this row's query position
        nb = w.nblk(t);
        kb0 = w.j0 * L::BN;
        lim = min(qi + (CAUSAL ? diag : p.S_k), p.S_k - 1);  // last visible key of this row
        lim_tile = CAUSAL ? row0 + diag : p.S_k - 1;         // last key every row of the tile sees
        // rows are query-major (row r: position r / gp), so a decode tile's real rows are
        // its first gp * S_q: the warps past them have nothing to compute
        idle = row0 + ((((warp & 3) * 32)) >> p.gp_log2) >= p.S_q;
      }
      float m_used = -INFINITY;
      float l = 0.f;
      unsigned rescales = 0;
      // The next unit is claimed once every role has read this one; the softmax
      // warps count as having read it only when they start the unit's 8th-last block:
      // early enough for the next unit's Q and first K/V tiles to arrive before this
      // unit ends, late enough that a CTA does not hold on to pending work while it
      // still has much of its own.
      if (nb == 0) mbar_arrive_warp(bar(L::B_ITEM_READ));
      for (int j = 0; j < nb; ++j) {
        if (j == (nb > 8 ? nb - 8 : 0)) mbar_arrive_warp(bar(L::B_ITEM_READ));
        ok = mbar_wait(bar(L::B_S_FULL + t), (sc + j) & 1, ctl);
        if (row == 0) ATTN_TL(tl, 0 + t, sc + j);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (idle) {
          // no row to compute: publish both halves of P(j) (their rows only ever reach
          // padding rows of O) at the pace of S(j), like the tile's other warps
          mbar_arrive_warp(bar(L::B_P_FULL + 2 * t));
          mbar_arrive_warp(bar(L::B_P_FULL + 2 * t + 1));
          continue;
        }
        tc_fence_after();
        uint32_t sr[128];
        const uint32_t s_addr = tmem + lane_addr + L::s_col(t);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32(s_addr + ch * 32, sr + ch * 32);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld_wait(sr + ch * 32);

        float* s = reinterpret_cast<float*>(sr);
        const int kbase = kb0 + (dual ? 2 * j + t : j) * L::BN;
        const bool need_mask = (kbase + L::BN - 1 > lim_tile) || (kbase + L::BN > p.S_k);
        if (need_mask) {
          const int lim_c = lim - kbase;
#pragma unroll
          for (int cc = 0; cc < 128; ++cc)
            if (cc > lim_c) s[cc] = -INFINITY;
        }
        const float mx = row_max128(sr);
        const float m_new = fmaxf(m_used, mx * c);
        const bool resc = (m_new - m_used) > p.tau;  // false for NaN (-inf - -inf)
        float alpha = 1.f;
        if (resc) {
          alpha = exp2_mufu(m_used - m_new);  // 0 when m_used = -inf
          m_used = m_new;
          l *= alpha;
          if (j > 0) ++rescales;
        }
        const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
        if (row == 0) ATTN_TL(tl, 2 + t, sc + j);
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          // PV_t(j-1) completed before S_t(j) was issued, so O_t is final up to block
          // j-1; it is rescaled before any part of P_t(j) is published.
          const uint32_t o_addr = tmem + lane_addr + L::o_col(t);
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t orr[32];
            tmem_ld32(o_addr + ch * 32, orr);
            tmem_ld_wait(orr);
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(o_addr + ch * 32, orr);
          }
        }
        // P_t(j) over the first 64 columns of S_t (32 for e4m3 P), published in two
        // halves (keys 0-63, then 64-127) so the PV MMA starts on the first while the
        // second is computed.
        // Masked blocks take MUFU ex2 only: it maps -inf to an exact 0.
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t pk[32];
          l += need_mask ? exp_half<0, PV8>(sr, c, m_eff, pk, hf) : exp_half<POLY_EVERY, PV8>(sr, c, m_eff, pk, hf);
          if constexpr (PV8)
            tmem_st16(s_addr + 16 * hf, pk);  // 64 keys as e4m3: 16 columns
          else
            tmem_st32(s_addr + 32 * hf, pk);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive_warp(bar(L::B_P_FULL + 2 * t + hf));
        }
        if (row == 0) ATTN_TL(tl, 4 + t, sc + j);
      }
      sc += nb;
      if (p.rescale_count != nullptr && rescales) atomicAdd(p.rescale_count, (unsigned long long)rescales);
      const Unit w = decode(item);
      const int qi = w.q0 + (dual ? 0 : t * tile_pos) + (row >> p.gp_log2);  // this row's query position
      const int h = w.h0 + (row & (p.gp - 1));                                 // and query head

      // ---- epilogue: O / l -> bf16 (or the split's fp32 O_s), lse
      if (ok && nb > 0) {
        ok = mbar_wait(bar(L::B_O_FINAL + t), oc & 1, ctl);
        if (row == 0) ATTN_TL(tl, 11 + t, u);
        ok = __all_sync(0xffffffffu, ok);
        ++oc;
      }
      float* xch = reinterpret_cast<float*>(sptr + L::XCHG_OFF);
      if (dual && t == 1) {
        // tile B hands its row statistics to tile A, which merges both halves
        xch[row] = m_used;
        xch[128 + row] = l;
        mbar_arrive_warp(bar(L::B_XCHG));
      } else if (ok) {
        // Row result = (w_A O_A + w_B O_B) / (w_A l_A + w_B l_B), w = 2^(m - max m): the
        // log-sum-exp merge of the two key halves in the dual stream; only this tile's
        // O (w = 1) otherwise.  A half that saw no key has l = 0 and weight 0, and its O
        // columns are never read into the result (select, not multiply).
        float m_b = -INFINITY, l_b = 0.f;
        const bool have_b = dual && w.nblk(1) > 0;
        if (dual) {
          ok = mbar_wait(bar(L::B_XCHG), 0, ctl);
          if (ok && have_b) ok = mbar_wait(bar(L::B_O_FINAL + 1), 0, ctl);
          ok = __all_sync(0xffffffffu, ok);
          m_b = xch[row];
          l_b = xch[128 + row];
        }
        if (ok) {
          tc_fence_after();
          const float mx = fmaxf(m_used, m_b);
          const float w_a = l > 0.f ? exp2_mufu(m_used - mx) : 0.f;
          const float w_b = l_b > 0.f ? exp2_mufu(m_b - mx) : 0.f;
          const float lsum = l * w_a + l_b * w_b;
          const float inv_l = lsum > 0.f ? 1.f / lsum : 0.f;
          const float c_a = w_a * inv_l, c_b = w_b * inv_l;
          const float lse_v = lsum > 0.f ? (mx + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
          const bool valid = qi < p.S_q;
          const uint32_t oa_addr = tmem + lane_addr + L::o_col(t);
          const uint32_t ob_addr = tmem + lane_addr + L::o_col(1);
          const size_t part = static_cast<size_t>(w.split) * p.B + w.b;
#pragma unroll 1
          for (int ch = 0; ch < D / 16; ++ch) {  // 16 columns at a time
            uint32_t orr[16], obr[16];
            if (nb > 0) {
              tmem_ld16(oa_addr + ch * 16, orr);
              tmem_ld_wait16(orr);
            }
            if (have_b) {
              tmem_ld16(ob_addr + ch * 16, obr);
              tmem_ld_wait16(obr);
            }
            float* ov = reinterpret_cast<float*>(orr);  // the result, in place
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float v = (nb > 0 && w_a > 0.f) ? __uint_as_float(orr[i]) * c_a : 0.f;
              if (have_b && w_b > 0.f) v += __uint_as_float(obr[i]) * c_b;
              ov[i] = v;
            }
            if (!valid) continue;
            if (p.n_splits > 1) {
              // partial result of this split: fp32 O_s
              float4* dst = reinterpret_cast<float4*>(p.o_part + ((part * p.S_q + qi) * p.H_q + h) * D + ch * 16);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_float4(ov[4 * i], ov[4 * i + 1], ov[4 * i + 2], ov[4 * i + 3]);
            } else {
              uint32_t pkd[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) pkd[i] = pack_bf16x2(ov[2 * i], ov[2 * i + 1]);
              __nv_bfloat16* dst = p.o + ((static_cast<size_t>(w.b) * p.S_q + qi) * p.H_q + h) * D + ch * 16;
              // Non-causal units are short enough that the epilogue is a visible share of
              // them: one 256-bit store per chunk when O is 32-byte aligned (every row
              // chunk then is).  The causal kernel keeps two 16-byte stores, which
              // measured faster there.
              bool wide = false;
              if constexpr (!CAUSAL) wide = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
              if (wide) {
                st_global_v8(dst, pkd);
              } else {
                uint4* d4 = reinterpret_cast<uint4*>(dst);
                d4[0] = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
                d4[1] = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
              }
            }
          }
          if (valid) {
            if (p.n_splits > 1)
              p.lse_part[(part * p.H_q + h) * p.S_q + qi] = lse_v;
            else
              p.lse[(static_cast<size_t>(w.b) * p.H_q + h) * p.S_q + qi] = lse_v;
          }
          if (row == 0) ATTN_TL(tl, 13 + t, u);
        }
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == L::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// Split-KV combine, one warp per (b, q, h) row.  Split s saw a disjoint key range
// and produced O_s (normalized over its keys) and lse_s = log sum over its keys
// of exp(scale * s_ij); then, exactly,
//   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s,
// evaluated with the largest lse_s factored out.  Rows that saw no key in any
// split (every lse_s = -inf) give O = 0 and lse = -inf, as the unsplit kernel.
// The row's lse_s values are loaded by the lanes at once (lane s holds split s, 32
// at a time) and reduced across the warp; the O_s rows are then streamed with
// independent loads, so the row costs a few memory round trips, not one per split.
template <int D>
__global__ void __launch_bounds__(256) attn_fwd_combine_kernel(const FwdParams p) {
  constexpr int PER = D / 32;  // values per lane
  static_assert(PER == 2 || PER == 4, "head dim 64 or 128");
  const long long rows = static_cast<long long>(p.B) * p.S_q * p.H_q;
  const int lane = threadIdx.x & 31;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < rows; w += n_warps) {
    // w = (b * S_q + q) * H_q + h, the row of O; the split-s row of o_part is s * rows + w
    const int h = static_cast<int>(w % p.H_q);
    const long long bq = w / p.H_q;
    const int q = static_cast<int>(bq % p.S_q);
    const int b = static_cast<int>(bq / p.S_q);
    const size_t lse_stride = static_cast<size_t>(p.B) * p.H_q * p.S_q;
    const size_t lse_row = (static_cast<size_t>(b) * p.H_q + h) * p.S_q + q;
    float m = -INFINITY;
    for (int s0 = 0; s0 < p.n_splits; s0 += 32) {
      const float ls = s0 + lane < p.n_splits ? p.lse_part[(s0 + lane) * lse_stride + lse_row] : -INFINITY;
      m = fmaxf(m, ls);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float sum = 0.f;
    if (m > -INFINITY) {
      for (int s0 = 0; s0 < p.n_splits; s0 += 32) {
        const int ns = min(32, p.n_splits - s0);
        const float ls = lane < ns ? p.lse_part[(s0 + lane) * lse_stride + lse_row] : -INFINITY;
        const float wl = ls == -INFINITY ? 0.f : exp2_mufu((ls - m) * 1.4426950408889634f);  // lane's split weight
        float part = wl;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        sum += part;
#pragma unroll 4
        for (int s = 0; s < ns; ++s) {
          const float wgt = __shfl_sync(0xffffffffu, wl, s);
          const float* src = p.o_part + (static_cast<size_t>(s0 + s) * rows + w) * D + lane * PER;
          if constexpr (PER == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            acc[0] += wgt * v.x;
            acc[1] += wgt * v.y;
            acc[2] += wgt * v.z;
            acc[3] += wgt * v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2*>(src);
            acc[0] += wgt * v.x;
            acc[1] += wgt * v.y;
          }
        }
      }
    }
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + w * D + lane * PER);
#pragma unroll
    for (int i = 0; i < PER / 2; ++i) dst[i] = pack_bf16x2(acc[2 * i] * inv, acc[2 * i + 1] * inv);
    if (lane == 0) p.lse[lse_row] = sum > 0.f ? m + logf(sum) : -INFINITY;
  }
}

// Merge of the ranges for few output rows (decode shapes): one CTA per row, its 8
// warps taking the ranges in turn, so a row's partials load in parallel instead of
// one range after another.  Same identity as attn_fwd_combine_kernel:
//   lse = log sum_s exp(lse_s),   O = sum_s exp(lse_s - lse) O_s.
template <int D>
__global__ void __launch_bounds__(256) attn_fwd_merge_rows_kernel(const FwdParams p) {
  constexpr int PER = D / 32;
  __shared__ float red_m[8], red_w[8], lse_s[128];
  __shared__ __align__(16) float red_o[8][D];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // launched as a programmatic dependent of the forward: wait for its results
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long rows = static_cast<long long>(p.B) * p.S_q * p.H_q;
  const size_t lse_stride = static_cast<size_t>(p.B) * p.H_q * p.S_q;
  for (long long w = blockIdx.x; w < rows; w += gridDim.x) {
    const int h = static_cast<int>(w % p.H_q);
    const long long bq = w / p.H_q;
    const int q = static_cast<int>(bq % p.S_q);
    const int b = static_cast<int>(bq / p.S_q);
    const size_t lse_row = (static_cast<size_t>(b) * p.H_q + h) * p.S_q + q;
    // the row's largest lse_s (thread t holds range t; at most 128 ranges)
    const float ls = tid < p.n_splits ? p.lse_part[tid * lse_stride + lse_row] : -INFINITY;
    if (tid < 128) lse_s[tid] = ls;
    float m = ls;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red_m[warp] = m;
    __syncthreads();
    m = red_m[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) m = fmaxf(m, red_m[k]);
    // warp k: ranges k, k + 8, ...
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    if (m > -INFINITY) {
      // ranges warp, warp + 8, ... (at most 16 per warp), in groups of 4 whose loads
      // are all issued (predicated) before any of them is used
#pragma unroll 1
      for (int s0 = warp; s0 < p.n_splits; s0 += 32) {
        float4 v4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = s0 + 8 * u;
          v4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (s < p.n_splits) {
            const float* src = p.o_part + (static_cast<size_t>(s) * rows + w) * D + lane * PER;
            if constexpr (PER == 4) {
              v4[u] = *reinterpret_cast<const float4*>(src);
            } else {
              const float2 v = *reinterpret_cast<const float2*>(src);
              v4[u] = make_float4(v.x, v.y, 0.f, 0.f);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = s0 + 8 * u;
          const float lss = s < p.n_splits ? lse_s[s] : -INFINITY;
          const float wgt = lss == -INFINITY ? 0.f : exp2_mufu((lss - m) * 1.4426950408889634f);
          wsum += wgt;
          acc[0] += wgt * v4[u].x;
          acc[1] += wgt * v4[u].y;
          if constexpr (PER == 4) {
            acc[2] += wgt * v4[u].z;
            acc[3] += wgt * v4[u].w;
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) red_o[warp][lane * PER + i] = acc[i];
    if (lane == 0) red_w[warp] = wsum;
    __syncthreads();
    if (warp == 0) {
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) sum += red_w[k];
      float o[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        o[i] = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) o[i] += red_o[k][lane * PER + i];
      }
      const float inv = sum > 0.f ? 1.f / sum : 0.f;
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + w * D + lane * PER);
#pragma unroll
      for (int i = 0; i < PER / 2; ++i) dst[i] = pack_bf16x2(o[2 * i] * inv, o[2 * i + 1] * inv);
      if (lane == 0) p.lse[lse_row] = sum > 0.f ? m + logf(sum) : -INFINITY;
    }
    __syncthreads();  // red_* are reused by the next row
  }
}

}  // namespace attn

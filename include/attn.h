/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library (libattn.so).
 *
 * What it computes (forward):
 *     S   = scale * Q K^T            (per batch b and query head h; K, V of head h / (H_q / H_kv))
 *     S_ij = -inf where causal and j > i + (S_k - S_q)   (bottom-right alignment)
 *     P   = softmax(S) row-wise,  O = P V,  lse_i = log(sum_j exp(S_ij))   (natural log)
 * This is the attention kernel that "AI Infra series ch. 6, GPU performance
 * engineering (II)" analyses in its section 1 (GEMMs plus softmax
 * exponentials, quoting the FlashAttention-4 paper) and whose Blackwell
 * techniques its section 7 lists (asynchronous MMA pipeline, software
 * exponential, conditional rescaling, 2-CTA MMA with TMEM intermediates).
 * The backward returns dQ, dK, dV of L = sum(dO * O) using the forward's O
 * and lse (P is recomputed, same article section 5, "recomputation").
 *
 * Tensors (all device pointers, caller-owned, never retained after a call returns):
 *   q, o, dO, dq : bf16 [B, S_q, H_q, D]   contiguous ("BSHD", D innermost)
 *   k, v, dk, dv : bf16 [B, S_k, H_kv, D]  contiguous
 *   lse          : fp32 [B, H_q, S_q]
 * Every pointer must be 16-byte aligned.  D is 64 or 128; H_q % H_kv == 0;
 * S_q, S_k >= 1; scale finite and > 0; causal is 0 or 1.  Every device pointer
 * of a call must point into the memory of the calling thread's current device
 * (cudaSetDevice), and `stream` must belong to that device: the kernels run there
 * and read their operands with TMA, which must never be handed another GPU's
 * memory.
 *
 * Execution: calls enqueue work on `stream` (a cudaStream_t; NULL = legacy
 * default stream) and return without synchronising.  The return value reports
 * argument and launch errors only.  A kernel that gives up on an internal wait
 * (it never spins without a bound) records ATTN_ERR_DEVICE_TIMEOUT in a device
 * status word that attn_device_status() reads.  The library allocates no
 * device memory on any call: scratch space (the backward's workspace) is
 * passed in by the caller.  All entry points are thread-safe.
 *
 * Per-device state: the library caches, per device, the device addresses of
 * its own __device__ variables and each kernel's shared-memory opt-in.  Both
 * belong to the device's CUDA context; when the current context is no longer
 * the one they were set up in (e.g. after cudaDeviceReset) the next call sets
 * them up again.
 */
#ifndef ATTN_B200_ATTN_H_
#define ATTN_B200_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,    /* a size, scale, causal flag or pointer is invalid */
  ATTN_ERR_UNSUPPORTED = 2,    /* a valid request this build does not serve (e.g. D not in {64,128}) */
  ATTN_ERR_MISALIGNED = 3,     /* a tensor pointer is not 16-byte aligned */
  ATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed (no device, launch failure ...) */
  ATTN_ERR_DEVICE_TIMEOUT = 5, /* a kernel abandoned a bounded internal wait (see attn_device_status) */
  ATTN_ERR_SCRATCH_TOO_SMALL = 6 /* attn_bwd_noalloc: the problem needs more than its fixed scratch */
} attn_status_t;

/* Version of this ABI (bumped on any incompatible change; 2: attn_bwd_options_t gained
 * `deterministic`, the split-KV and 8-bit Q/K forwards were added; 3: the backward
 * workspace gained the deterministic mode's work-item counter, attn_fwd_qkv8; 4:
 * attn_fwd_options_t gained `persistent`, attn_bwd_options_t gained `cta_mode`). */
int attn_abi_version(void);

/* Human-readable name of a status code (static storage). */
const char* attn_status_string(attn_status_t s);

/*
 * Forward pass.  Writes o [B,S_q,H_q,D] (bf16) and lse [B,H_q,S_q] (fp32).
 * Rows that see no key (only possible when causal and S_q > S_k) get O = 0, lse = -inf.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                       int H_kv, int S_q, int S_k, int D, int causal, float scale, void* stream);

/*
 * Tunables and diagnostics of the forward; none of them changes the exact
 * result, only rounding.
 *   rescale_threshold : tau, in base-2 units of the scores.  O is rescaled only
 *                       when a row's running max grows by more than tau
 *                       ("conditional softmax rescaling", AI Infra series ch. 6
 *                       section 7 item 2).  0 = rescale on every increase.
 *                       Must be in [0, 16].  Default 8.
 *   poly_exp_every    : of every `poly_exp_every` column pairs of a score block,
 *                       one pair takes the FMA-pipe cubic 2^x instead of the
 *                       MUFU unit (same section, item 1: 10-25 % of the
 *                       exponentials).  Allowed: 0 (MUFU only), 4 (25 %),
 *                       8 (12.5 %).  Default 8.
 *   rescale_count     : optional device pointer to an unsigned 64-bit counter;
 *                       the kernel adds the number of (row, key block) O rescales
 *                       it performed after a row's first block.  NULL = off.
 *   persistent        : 1 (default) = persistent CTAs: a CTA that finishes its
 *                       work unit (256 query rows of one head, or a key range of
 *                       one in the split forward) claims the unit of a CTA that
 *                       has not started yet -- the grid lists units longest first
 *                       for causal -- and runs it with the barriers, rings and
 *                       tensor memory it holds, loading the next unit's tiles
 *                       while it finishes the current one (a persistent tile
 *                       scheduler; Blackwell cluster launch control).  With it,
 *                       a non-causal forward whose units leave a last wave of at
 *                       most half the SMs runs those units in a second launch,
 *                       two CTAs per unit (each on 128 rows, its two tiles
 *                       splitting the keys), started as the first launch's CTAs
 *                       finish.  0 = one CTA per unit.  Ignored when one tile
 *                       holds every query row (the two tiles then split the keys
 *                       instead).
 */
typedef struct {
  float rescale_threshold;
  int poly_exp_every;
  unsigned long long* rescale_count;
  int persistent;
} attn_fwd_options_t;

/* Fills `opt` with the defaults above. */
void attn_fwd_default_options(attn_fwd_options_t* opt);

/* attn_fwd with explicit options (`opt` NULL = defaults). */
attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                          int H_kv, int S_q, int S_k, int D, int causal, float scale,
                          const attn_fwd_options_t* opt, void* stream);

/*
 * Forward with 8-bit Q and K: q and k hold float8 e4m3 values (one byte per
 * element, the same BSHD layout); v and o are bf16.  S = scale * Q K^T runs on
 * the tensor cores' 8-bit path (kind::f8f6f4, fp32 accumulation, twice the
 * bf16 rate); the softmax, P (bf16) and O += P V are as in attn_fwd.  The
 * result is the attention of the e4m3 values themselves: the caller's
 * quantisation of q and k is the only precision change (the "reduce precision"
 * lever of AI Infra series ch. 6, GPU performance engineering (II), section 5).
 * Head dim 128 only (else ATTN_ERR_UNSUPPORTED); options and errors as
 * attn_fwd_ex.
 */
attn_status_t attn_fwd_qk8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                           int H_kv, int S_q, int S_k, int D, int causal, float scale,
                           const attn_fwd_options_t* opt, void* stream);

/*
 * Forward with 8-bit Q, K and V: q, k and v hold float8 e4m3 values (one byte per
 * element, BSHD); o is bf16, lse fp32.  Both products run on the tensor cores'
 * 8-bit path (kind::f8f6f4): S = scale * Q K^T as in attn_fwd_qk8, and O += P V
 * with the unnormalised weights p = 2^(scale log2(e) s - m) (m the row's running
 * max, p <= 2^rescale_threshold) rounded to e4m3 in tensor memory.  The row sums
 * and lse use the unrounded p, so lse is as accurate as attn_fwd_qk8's; O differs
 * from the exact attention of the e4m3 inputs by the rounding of p: per element
 * at most 2^-4 sum_k P_ik |v_k| (three mantissa bits, round to nearest) plus
 * 2^-10 sum_k |v_k| / L_i for weights in e4m3's subnormal range (L_i = sum_k
 * exp(s_ik - max_k s_ik)), plus the bf16 rounding of O (the "reduce precision"
 * lever of AI Infra series ch. 6, GPU performance engineering (II), section 5,
 * applied to the whole forward).  Head dim 128 only; options and errors as
 * attn_fwd_ex, except that rescale_threshold must be <= 8 (ATTN_ERR_INVALID_ARG
 * otherwise): p <= 2^rescale_threshold must stay below e4m3's largest value, 448.
 */
attn_status_t attn_fwd_qkv8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                            int H_kv, int S_q, int S_k, int D, int causal, float scale,
                            const attn_fwd_options_t* opt, void* stream);

/*
 * Split-KV forward for shapes with few query rows and many keys (decoding
 * shapes: S_q << S_k), where one CTA per 256 query rows of each (batch, head)
 * would leave most of the 148 SMs idle.  The pages describe no such variant;
 * it computes the same O and lse as attn_fwd.  The ceil(S_k / 128) key blocks
 * are cut into ranges of ceil(blocks / n_splits) blocks (trailing empty ranges
 * are dropped).  Each range is processed by its own CTAs with the attn_fwd
 * kernel, which writes the range's O_s (normalized over its keys, fp32) and
 * lse_s into `workspace`.  A second kernel merges them with the log-sum-exp
 * identity lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.  Causal
 * masking is bottom-right as in attn_fwd.  Default attn_fwd options.
 *
 *   n_splits  : 0 = attn_fwd_split_count(...); 1 = plain attn_fwd (workspace may
 *               be NULL); 2..128 = at most that many ranges.
 *   workspace : device, 16-byte aligned, attn_fwd_split_workspace_size(B, H_q,
 *               S_q, D, n_splits) bytes for the n_splits passed (or chosen);
 *               owned by the caller, unused when only one range results.
 * Errors as attn_fwd; ATTN_ERR_INVALID_ARG also for n_splits outside [0, 128]
 * or a NULL workspace when more than one range results.
 */
attn_status_t attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                             int B, int H_q, int H_kv, int S_q, int S_k, int D, int causal, float scale,
                             int n_splits, void* stream);

/* attn_fwd_split with 8-bit Q and K as in attn_fwd_qk8 (q, k e4m3; v, o bf16; head
 * dim 128): for decoding shapes, where the step is bound by streaming K and V,
 * e4m3 K moves half the bytes of bf16 K.  Arguments, workspace and errors as
 * attn_fwd_split. */
attn_status_t attn_fwd_split_qk8(const void* q, const void* k, const void* v, void* o, float* lse,
                                 void* workspace, int B, int H_q, int H_kv, int S_q, int S_k, int D, int causal,
                                 float scale, int n_splits, void* stream);

/* The n_splits attn_fwd_split uses for n_splits = 0: 1 when the forward's CTAs
 * (one per 256 query rows of a (batch, head), or of a pack of the query heads of one
 * kv group when S_q <= 128) already fill the 148 SMs; otherwise the count (at most
 * 128) that minimises waves of CTAs x (key blocks per range + 2), the 2 standing
 * for a CTA's fixed cost. */
int attn_fwd_split_count(int B, int H_q, int H_kv, int S_q, int S_k, int causal);

/* Bytes of workspace attn_fwd_split needs for n_splits ranges: fp32 O_s
 * [n_splits, B, S_q, H_q, D] and lse_s [n_splits, B, H_q, S_q]; 0 for n_splits = 1
 * or invalid sizes. */
size_t attn_fwd_split_workspace_size(int B, int H_q, int S_q, int D, int n_splits);

/*
 * Bytes of device workspace attn_bwd needs: an fp32 dQ accumulator
 * [B, S_q, H_q, D], two fp32 row-term arrays [B, H_q, S_pad] (S_pad =
 * S_q rounded up to 64): -lse_i * log2(e) and delta_i = sum_d dO_id O_id,
 * one int per (b, h, 64-query block) for the deterministic mode's turn counters,
 * and one int for its work-item counter (each part 256-byte aligned).
 * Returns 0 for invalid sizes.
 */
size_t attn_bwd_workspace_size(int B, int H_q, int S_q, int D);

/*
 * Backward pass.  q, k, v, o, lse as produced/consumed by attn_fwd with the
 * same arguments; dO is the gradient of the loss w.r.t. o.  Writes dq, dk, dv
 * (bf16).  `workspace` must hold attn_bwd_workspace_size(...) bytes, 16-byte
 * aligned; its contents on entry are ignored.  The dQ parts of the key tiles are
 * added into an fp32 accumulator in the order the tiles finish, so dQ may differ
 * in the last bits from run to run (attn_bwd_ex with deterministic = 1 fixes the
 * order).  D = 64 or 128.
 */
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv, void* workspace, int B, int H_q,
                       int H_kv, int S_q, int S_k, int D, int causal, float scale, void* stream);

/*
 * Options of the backward.
 *   main_pass_start / main_pass_stop : optional cudaEvent_t handles (created by
 *       the caller) that the library records on `stream` immediately before and
 *       after the main-pass kernel, so the caller can time that kernel alone.
 *       NULL = not recorded.
 *   deterministic : 0 (default) = each key tile adds its dQ part for a query
 *       block as soon as it has it, so the fp32 sums (and the bf16 dQ) may
 *       differ in the last bits between runs.  1 = the parts for each (b, h,
 *       64-query block) are added in a fixed key-tile order, one tile waiting
 *       (bounded) for the previous one's addition to complete.  The CTAs take
 *       their work items from a counter as they start, so that a tile only ever
 *       waits for tiles whose CTAs started before it: progress does not depend
 *       on the order in which the hardware dispatches the blocks.  dQ is then
 *       bitwise identical from run to run (the pages' atomic reductions, section
 *       7 item 3, leave the order open); dK, dV are deterministic in both modes.
 *       With CTA pairs the order is over pairs of key tiles.
 *   cta_mode : how the main pass maps key tiles to CTAs.  0 (default) = the
 *       faster kernel of each mode on B200: CTA pairs for the deterministic
 *       instance at D = 128, one CTA per tile otherwise.  1 = one CTA per
 *       128-key tile (every MMA on one SM); in the normal dQ order these CTAs
 *       are persistent: a CTA that finishes its tile takes over the tile of a
 *       CTA that has not started (cluster launch control) and loads its K and V
 *       while it writes the old tile's dK and dV.  2 = CTA pairs (clusters of two CTAs on
 *       adjacent key tiles whose tensor cores execute each MMA together,
 *       cta_group::2: "AI Infra series ch. 6", section 7 item 3): half of each
 *       B operand per CTA and half the dQ reduce-adds, at the cost of a dS^T
 *       exchange between the two CTAs and a dQ^T product of M = 128 per pair.
 *       D = 128 only; other D return ATTN_ERR_INVALID_ARG.  Results agree to
 *       rounding; only the summation order of dQ differs.
 */
typedef struct {
  void* main_pass_start;
  void* main_pass_stop;
  int deterministic;
  int cta_mode;
} attn_bwd_options_t;

/* attn_bwd with explicit options (`opt` NULL = all fields 0). */
attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, void* workspace, int B, int H_q,
                          int H_kv, int S_q, int S_k, int D, int causal, float scale,
                          const attn_bwd_options_t* opt, void* stream);

/*
 * attn_bwd for callers that cannot allocate device memory: the same backward,
 * with its scratch taken from a buffer built into the library instead of a
 * caller-provided workspace.  (The pages describe no such variant; it serves
 * integrations where allocation is not available at the call site -- code that
 * runs under a framework's memory pool it may not grow, inside a plug-in or a
 * callback with no allocator handle, or in a latency path that must never
 * reach cudaMalloc.)
 *
 * The buffer is a file-scope device array of 32 MiB (33554432 bytes) that
 * every GPU which loads the library holds until the process exits.  Problems
 * whose attn_bwd_workspace_size() exceeds it return ATTN_ERR_SCRATCH_TOO_SMALL
 * before anything is launched.  The first call on a device looks up the
 * buffer's device address (cudaGetSymbolAddress); make that first call before
 * any stream capture.  The address is kept per device and context: after the
 * device's context is replaced (cudaDeviceReset) the next call looks it up
 * again, so that call too should come before any capture.  No call allocates
 * or frees device memory.  All calls share the one buffer and it keeps the last call's
 * contents (each call clears what must start at zero): calls that may overlap
 * on the GPU -- on different streams, or from different host threads -- race
 * on it and must be serialised by the caller.  Arguments and results as attn_bwd.
 */
attn_status_t attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dO, void* dq, void* dk, void* dv, int B, int H_q, int H_kv,
                               int S_q, int S_k, int D, int causal, float scale, void* stream);

/*
 * Reads and clears the current device's status word in one atomic step, on
 * `stream` (so after every kernel enqueued on it before), then synchronises
 * `stream` and returns the value read: ATTN_OK, or ATTN_ERR_DEVICE_TIMEOUT if a
 * kernel gave up on a wait since the last read, or ATTN_ERR_CUDA if a CUDA call
 * failed.  There is one status word per device, shared by every stream: a
 * timeout recorded by a kernel on another stream is reported by whichever read
 * comes first after it, and a kernel still running on another stream may record
 * one after this call returns.
 */
attn_status_t attn_device_status(void* stream);

/*
 * Upper bound, in nanoseconds, of any single internal wait of the kernels
 * (default 4e9).  Tests lower it to exercise the timeout path without a hang.
 * 0 restores the default.
 */
void attn_set_wait_limit_ns(unsigned long long ns);

/*
 * Diagnostic: y[i] = the kernels' FMA-pipe cubic 2^x applied to x[i]
 * (device pointers, n >= 0), for checking its error bound.
 */
attn_status_t attn_exp2_poly_eval(const float* x, float* y, long long n, void* stream);

/*
 * Diagnostic: reads `bytes` bytes at device pointer x once (16-byte loads, four
 * in flight per thread, four CTAs of 512 threads per SM) and folds them into the
 * device word *sink, so the caller can time a plain read of as many bytes as a
 * bytes-bound call moves: the yardstick for the split-KV forward on decoding
 * shapes.  x and sink 16- and 8-byte aligned, bytes >= 0 and a multiple of 16;
 * otherwise ATTN_ERR_INVALID_ARG.
 */
attn_status_t attn_read_probe(const void* x, long long bytes, unsigned long long* sink, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H_ */

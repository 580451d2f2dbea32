// C-ABI entry points of libattn.so (declared in include/attn.h): argument
// validation, TMA descriptor encoding, kernel selection and launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "bwd_kernels.cuh"
#include "bwd_pair_kernel.cuh"
#include "fwd_kernel.cuh"
#include "sm100_common.cuh"

namespace attn {

// Device status word: kernels record kDevWaitTimeout here when they abandon a wait.
__device__ int g_status = 0;
// Where attn_device_status() puts the word it read (and cleared) in one atomic step.
__device__ int g_status_taken = 0;

// Fixed scratch for attn_bwd_noalloc: every device that loads this library
// holds these bytes until the process exits.  Host code must not pass the
// symbol itself to a kernel (on the host it is only a stand-in); it looks up
// the device address with cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

namespace {

constexpr unsigned long long kDefaultWaitLimitNs = 4000000000ull;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

// Grid order of the forward and of the backward main pass: (batch, head) pairs
// per group of CTAs that run together and share L2.
#ifndef ATTN_FWD_BH_GROUP
#define ATTN_FWD_BH_GROUP 8
#endif
#ifndef ATTN_BWD_BH_GROUP
#define ATTN_BWD_BH_GROUP 8
#endif
constexpr int kFwdBhGroup = ATTN_FWD_BH_GROUP;
constexpr int kBwdBhGroup = ATTN_BWD_BH_GROUP;

constexpr int kNumSms = 148;     // B200
constexpr int kMaxSplits = 128;  // key splits of the split-KV forward

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 BSHD tensor viewed as (D, H, S, B); boxes of 64 x 1 x box_rows x 1, 128-byte swizzle.
bool make_bshd_map(CUtensorMap* map, const void* ptr, int B, int S, int H, int D, int box_rows = 128,
                   int box_heads = 1, int elem_bytes = 2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(B)};
  const cuuint64_t eb = static_cast<cuuint64_t>(elem_bytes);
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * eb, static_cast<cuuint64_t>(H) * D * eb,
                                 static_cast<cuuint64_t>(S) * H * D * eb};
  // 128-byte rows: 64 bf16 or 128 one-byte elements
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(box_heads),
                             static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estride[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(map, dt, 4, const_cast<void*>(ptr), dims, strides, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [B, S, H, D] dQ accumulator viewed as (D, H, S, B); boxes of box_d x 1 x 64 x 1
// (whole 64-query blocks; all D dims, or half of them for a CTA of a pair), no
// swizzle: the target of the backward's TMA reduce-adds.
bool make_dqacc_map(CUtensorMap* map, void* ptr, int B, int S, int H, int D, int box_d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(H) * D * 4,
                                 static_cast<cuuint64_t>(S) * H * D * 4};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_d), 1, 64, 1};
  const cuuint32_t estride[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The calling thread's current CUDA context (the runtime's primary context of
// the current device once the runtime has initialised it), or nullptr.
CUcontext current_ctx() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

constexpr int kMaxDevices = 64;

// Per-device state of the library: device addresses of its __device__ symbols,
// valid in the context they were looked up in.  A device reset (or anything else
// that replaces the device's context) invalidates them; they are looked up again
// when the current context is not the recorded one.
struct DevState {
  CUcontext ctx = nullptr;
  int* status = nullptr;  // g_status
  int* taken = nullptr;   // g_status_taken
  void* scratch = nullptr;  // g_bwd_scratch (looked up on first use)
};
std::mutex g_dev_mu;
DevState g_dev[kMaxDevices];

// Current device's state, refreshed if the context changed.  `with_scratch` also
// resolves the no-allocation backward's scratch buffer.
bool device_state(DevState* out, bool with_scratch = false) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DevState& s = g_dev[dev];
  CUcontext ctx = current_ctx();
  if (ctx == nullptr || ctx != s.ctx) {
    void* st = nullptr;
    void* tk = nullptr;
    if (cudaGetSymbolAddress(&st, g_status) != cudaSuccess) return false;
    if (cudaGetSymbolAddress(&tk, g_status_taken) != cudaSuccess) return false;
    s = DevState{};
    s.status = static_cast<int*>(st);
    s.taken = static_cast<int*>(tk);
    s.ctx = current_ctx();  // the lookup above initialised the context if it was not yet
  }
  if (with_scratch && s.scratch == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess) return false;
    s.scratch = ptr;
  }
  *out = s;
  return true;
}

int* status_ptr() {
  DevState s;
  return device_state(&s) ? s.status : nullptr;
}

// Device address of g_bwd_scratch on the current device (looked up once per
// device and context).
void* noalloc_scratch_ptr() {
  DevState s;
  return device_state(&s, true) ? s.scratch : nullptr;
}

// The dynamic shared-memory opt-in of a kernel is an attribute of the current
// device's context: set it once per (kernel, context).  `seen` is the kernel's
// own record of the contexts it was set in, one slot per device.
std::mutex g_attr_mu;
template <typename Kern>
cudaError_t smem_opt_in(Kern kern, int bytes, CUcontext* seen) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  const CUcontext ctx = current_ctx();
  if (ctx != nullptr && seen[dev] == ctx) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) seen[dev] = current_ctx();
  return e;
}

attn_status_t check_common(int B, int H_q, int H_kv, int S_q, int S_k, int D, int causal, float scale) {
  if (B < 1 || H_q < 1 || H_kv < 1 || S_q < 1 || S_k < 1) return ATTN_ERR_INVALID_ARG;
  if (H_q % H_kv != 0) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  // index arithmetic inside the kernels is 32-bit per head row; keep products in range
  const double rows = static_cast<double>(B) * (S_q > S_k ? S_q : S_k);
  if (rows * (H_q > H_kv ? H_q : H_kv) * D >= 9.0e18 || static_cast<double>(B) * H_q * ((S_q + 127) / 128) >= 2.0e9)
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

template <int D, bool CAUSAL, int POLY, bool QK8, bool PV8 = false>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p,
                       unsigned grid, cudaStream_t st) {
  using L = FwdLayout<D, QK8, PV8>;
  auto kern = attn_fwd_kernel<D, CAUSAL, POLY, QK8, PV8>;
  static CUcontext seen[kMaxDevices] = {};
  const cudaError_t attr_err = smem_opt_in(kern, L::SMEM_BYTES, seen);
  if (attr_err != cudaSuccess) return attr_err;
  if (p.unit_base < 0) {
    kern<<<grid, L::THREADS, L::SMEM_BYTES, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
  }
  // the tail launch: a programmatic dependent of the grid before it, so its CTAs take
  // the SMs that grid leaves as its last CTAs finish (it reads none of that grid's results)
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p);
}

template <int D, bool CAUSAL, bool QK8 = false, bool PV8 = false>
cudaError_t launch_fwd_poly(int poly, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const FwdParams& p, unsigned grid, cudaStream_t st) {
  switch (poly) {
    case 0: return launch_fwd<D, CAUSAL, 0, QK8, PV8>(mq, mk, mv, p, grid, st);
    case 4: return launch_fwd<D, CAUSAL, 4, QK8, PV8>(mq, mk, mv, p, grid, st);
    default: return launch_fwd<D, CAUSAL, 8, QK8, PV8>(mq, mk, mv, p, grid, st);
  }
}

template <int D, bool CAUSAL, bool DET>
cudaError_t launch_bwd(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mq, const CUtensorMap& mdo,
                       const CUtensorMap& mdq, const BwdParams& p, unsigned grid, cudaStream_t st) {
  using L = BwdLayout<D, DET>;
  auto kern = attn_bwd_kernel<D, CAUSAL, DET>;
  static CUcontext seen[kMaxDevices] = {};
  const cudaError_t attr_err = smem_opt_in(kern, L::SMEM_BYTES, seen);
  if (attr_err != cudaSuccess) return attr_err;
  kern<<<grid, L::THREADS, L::SMEM_BYTES, st>>>(mk, mv, mq, mdo, mdq, p);
  return cudaGetLastError();
}

template <bool CAUSAL, bool DET>
cudaError_t launch_bwd_pair(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mq32,
                            const CUtensorMap& mdo32, const CUtensorMap& mq64, const CUtensorMap& mdo64,
                            const CUtensorMap& mdq, const BwdParams& p, unsigned grid, cudaStream_t st) {
  using L = BwdPairLayout<DET>;
  auto kern = attn_bwd_pair_kernel<CAUSAL, DET>;
  static CUcontext seen[kMaxDevices] = {};
  const cudaError_t attr_err = smem_opt_in(kern, L::SMEM_BYTES, seen);
  if (attr_err != cudaSuccess) return attr_err;
  // the kernel is declared with a cluster size of two: grid is a multiple of two
  kern<<<grid, L::THREADS, L::SMEM_BYTES, st>>>(mk, mv, mq32, mdo32, mq64, mdo64, mdq, p);
  return cudaGetLastError();
}

// Reads and clears the status word in one atomic step (a timeout recorded by a
// kernel on another stream is never lost between a read and a clear).
__global__ void take_status_kernel(int* status, int* taken) { *taken = atomicExch(status, 0); }

// One plain pass over n16 16-byte words, four loads in flight per thread; the
// XOR of everything read goes to a branch that keeps the loads alive (its
// condition is practically never true).
__global__ void read_probe_kernel(const uint4* __restrict__ x, long long n16, unsigned long long* sink) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 a = __ldg(x + i), b = __ldg(x + i + stride), c = __ldg(x + i + 2 * stride), d = __ldg(x + i + 3 * stride);
    acc ^= (a.x ^ a.y ^ a.z ^ a.w) ^ (b.x ^ b.y ^ b.z ^ b.w) ^ (c.x ^ c.y ^ c.z ^ c.w) ^ (d.x ^ d.y ^ d.z ^ d.w);
  }
  for (; i < n16; i += stride) {
    const uint4 a = __ldg(x + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  if (acc == 0x9E3779B9u) atomicAdd(sink, 1ull);
}

// Evaluates the kernels' packed-pair cubic on x[2i], x[2i+1] (the last element of
// an odd-length array is paired with itself).
__global__ void exp2_poly_eval_kernel(const float* x, float* y, long long n) {
  const long long pairs = (n + 1) / 2;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < pairs;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float a = x[2 * i];
    const float b = 2 * i + 1 < n ? x[2 * i + 1] : a;
    float ea, eb;
    exp2_poly_x2(f2_pack(a, b), ea, eb);
    y[2 * i] = ea;
    if (2 * i + 1 < n) y[2 * i + 1] = eb;
  }
}

// Query heads packed into one forward tile: the whole kv group when S_q is short
// (a tile of one head would be mostly empty) and the group size is a power of two
// that leaves at least one query position per tile; else 1.
int fwd_head_pack(int H_q, int H_kv, int S_q) {
  const int G = H_q / H_kv;
  if (S_q > 128 || G < 2 || G > 64 || (G & (G - 1)) != 0) return 1;
  return G;
}

// Forward (unsplit when n_splits == 1); with n_splits > 1 the kernel writes
// per-split partial results into `workspace` and a combine kernel merges them.
attn_status_t run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace, int B,
                      int H_q, int H_kv, int S_q, int S_k, int D, int causal, float scale,
                      const attn_fwd_options_t* opt_in, int n_splits, void* stream, bool qk8 = false,
                      bool pv8 = false) {
  attn_fwd_options_t opt;
  attn_fwd_default_options(&opt);
  if (opt_in) opt = *opt_in;
  attn_status_t st = check_common(B, H_q, H_kv, S_q, S_k, D, causal, scale);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if ((qk8 || pv8) && D != 128) return ATTN_ERR_UNSUPPORTED;
  // split ranges: split_blocks key blocks each; trailing splits that would be empty are dropped
  const int n_kv = (S_k + 127) / 128;
  const int split_blocks = (n_kv + n_splits - 1) / n_splits;
  n_splits = (n_kv + split_blocks - 1) / split_blocks;
  if (n_splits > 1 && (!workspace || !aligned16(workspace))) return workspace ? ATTN_ERR_MISALIGNED : ATTN_ERR_INVALID_ARG;
  if (!(opt.rescale_threshold >= 0.f && opt.rescale_threshold <= 16.f)) return ATTN_ERR_INVALID_ARG;
  // e4m3 weights: p <= 2^tau must stay below e4m3's largest value, 448
  if (pv8 && opt.rescale_threshold > 8.f) return ATTN_ERR_INVALID_ARG;
  if (opt.poly_exp_every != 0 && opt.poly_exp_every != 4 && opt.poly_exp_every != 8) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return ATTN_ERR_MISALIGNED;

  const int gp = fwd_head_pack(H_q, H_kv, S_q);
  int gp_log2 = 0;
  while ((1 << gp_log2) < gp) ++gp_log2;
  CUtensorMap mq, mk, mv;
  const int qk_bytes = qk8 ? 1 : 2;
  if (!make_bshd_map(&mq, q, B, S_q, H_q, D, 128 / gp, gp, qk_bytes) ||
      !make_bshd_map(&mk, k, B, S_k, H_kv, D, 128, 1, qk_bytes) ||
      !make_bshd_map(&mv, v, B, S_k, H_kv, D, 128, 1, pv8 ? 1 : 2))
    return ATTN_ERR_CUDA;
  int* status = status_ptr();
  if (!status) return ATTN_ERR_CUDA;

  FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.S_q = S_q;
  p.S_k = S_k;
  p.gp = gp;
  p.gp_log2 = gp_log2;
  p.n_units = (S_q + 256 / gp - 1) / (256 / gp);
  p.bh_group = kFwdBhGroup < B * (H_q / gp) ? kFwdBhGroup : B * (H_q / gp);
  p.n_splits = n_splits;
  p.split_blocks = split_blocks;
  // one tile holds every query row: tile B takes half of the key blocks instead of idling
  p.dual = S_q <= 128 / gp ? 1 : 0;
  p.persistent = (opt.persistent && !p.dual) ? 1 : 0;
  p.unit_base = -1;
  if (n_splits > 1) {
    const size_t rows = static_cast<size_t>(n_splits) * B * H_q * S_q;
    p.o_part = static_cast<float*>(workspace);
    p.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + (rows * D * sizeof(float) + 255) / 256 * 256);
  }
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.tau = opt.rescale_threshold;
  p.status = status;
  p.rescale_count = opt.rescale_count;
  p.wait_limit_ns = g_wait_limit_ns.load();
  const long long grid_ll = static_cast<long long>(p.n_units) * B * (H_q / gp) * n_splits;
  if (grid_ll > 2147483647LL) return ATTN_ERR_UNSUPPORTED;  // one CTA per (unit, head pack, range)
  // Last wave: equal-length (non-causal) units fill ceil(units / SMs) waves, the last
  // one partly.  When it holds at most half as many units as there are SMs, those
  // units go to a second launch as the dual stream (both tiles on one 128-row half,
  // odd and even key blocks), two CTAs per unit, so they finish in about half a wave.
  int tail = 0;
  if (p.persistent && !causal && n_splits == 1 && gp == 1 && grid_ll > kNumSms) {
    const int r = static_cast<int>(grid_ll % kNumSms);
    if (r > 0 && r <= kNumSms / 2) tail = r;
  }
  const unsigned grid = static_cast<unsigned>(grid_ll - tail);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto launch = [&](const FwdParams& pl, unsigned g) {
    if (pv8)
      return causal ? launch_fwd_poly<128, true, true, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s)
                    : launch_fwd_poly<128, false, true, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s);
    if (qk8)
      return causal ? launch_fwd_poly<128, true, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s)
                    : launch_fwd_poly<128, false, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s);
    if (D == 128)
      return causal ? launch_fwd_poly<128, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s)
                    : launch_fwd_poly<128, false>(opt.poly_exp_every, mq, mk, mv, pl, g, s);
    return causal ? launch_fwd_poly<64, true>(opt.poly_exp_every, mq, mk, mv, pl, g, s)
                  : launch_fwd_poly<64, false>(opt.poly_exp_every, mq, mk, mv, pl, g, s);
  };
  cudaError_t err = launch(p, grid);
  if (err == cudaSuccess && tail > 0) {
    FwdParams pt = p;
    pt.dual = 1;
    pt.persistent = 0;
    pt.unit_base = static_cast<int>(grid);
    err = launch(pt, 2u * static_cast<unsigned>(tail));
  }
  if (err != cudaSuccess) return ATTN_ERR_CUDA;
  if (n_splits > 1) {
    const long long rows = static_cast<long long>(B) * S_q * H_q;
    if (rows <= kNumSms * 8) {
      // few rows (decode): one CTA per row, launched as a programmatic dependent so its
      // launch overlaps the forward's tail; it waits on the device for the results
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(static_cast<unsigned>(rows));
      cfg.blockDim = dim3(256);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const cudaError_t me = D == 128 ? cudaLaunchKernelEx(&cfg, attn_fwd_merge_rows_kernel<128>, p)
                                      : cudaLaunchKernelEx(&cfg, attn_fwd_merge_rows_kernel<64>, p);
      if (me != cudaSuccess) return ATTN_ERR_CUDA;
    } else {
      const long long blocks = (rows + 7) / 8;  // one warp per row
      const unsigned g = static_cast<unsigned>(blocks < kNumSms * 16 ? blocks : kNumSms * 16);
      if (D == 128)
        attn_fwd_combine_kernel<128><<<g, 256, 0, s>>>(p);
      else
        attn_fwd_combine_kernel<64><<<g, 256, 0, s>>>(p);
      if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
  }
  return ATTN_OK;
}

// Range count of the tensor-core split-KV forward: time ~ waves of CTAs x (key
// blocks per range + ~2 blocks of per-CTA fixed cost).
int tc_split_count(int B, int H_q, int H_kv, int S_q, int S_k) {
  if (B < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0 || S_q < 1 || S_k < 1) return 1;
  const int gp = fwd_head_pack(H_q, H_kv, S_q);
  const long long ctas = static_cast<long long>((S_q + 256 / gp - 1) / (256 / gp)) * B * (H_q / gp);
  const int n_kv = (S_k + 127) / 128;
  if (ctas >= kNumSms) return 1;
  int best = 1;
  long long best_cost = -1;
  for (int n = 1; n <= std::min(kMaxSplits, n_kv); ++n) {
    const long long per = (n_kv + n - 1) / n;
    const long long ranges = (n_kv + per - 1) / per;
    const long long waves = (ctas * ranges + kNumSms - 1) / kNumSms;
    const long long cost = waves * (per + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = static_cast<int>(ranges);
    }
  }
  return best;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" {

int attn_abi_version(void) { return 4; }

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG: invalid size, scale, causal flag or null pointer";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED: request not served by this build (D must be 64 or 128)";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED: tensor pointers must be 16-byte aligned";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: a CUDA call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT: a kernel abandoned a bounded wait";
    case ATTN_ERR_SCRATCH_TOO_SMALL:
      return "ATTN_ERR_SCRATCH_TOO_SMALL: the problem needs more scratch than attn_bwd_noalloc's fixed 32 MiB buffer";
  }
  return "ATTN_ERR_UNKNOWN";
}

void attn_fwd_default_options(attn_fwd_options_t* opt) {
  if (!opt) return;
  opt->rescale_threshold = 8.0f;
  opt->poly_exp_every = 8;
  opt->rescale_count = nullptr;
  opt->persistent = 1;
}

attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                          int H_kv, int S_q, int S_k, int D, int causal, float scale,
                          const attn_fwd_options_t* opt_in, void* stream) {
  return run_fwd(q, k, v, o, lse, nullptr, B, H_q, H_kv, S_q, S_k, D, causal, scale, opt_in, 1, stream);
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q, int H_kv,
                       int S_q, int S_k, int D, int causal, float scale, void* stream) {
  return attn_fwd_ex(q, k, v, o, lse, B, H_q, H_kv, S_q, S_k, D, causal, scale, nullptr, stream);
}

int attn_fwd_split_count(int B, int H_q, int H_kv, int S_q, int S_k, int causal) {
  (void)causal;
  if (B < 1 || H_q < 1 || H_kv < 1 || H_q % H_kv != 0 || S_q < 1 || S_k < 1) return 1;
  return attn::tc_split_count(B, H_q, H_kv, S_q, S_k);
}

attn_status_t attn_fwd_qk8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                           int H_kv, int S_q, int S_k, int D, int causal, float scale,
                           const attn_fwd_options_t* opt, void* stream) {
  return run_fwd(q, k, v, o, lse, nullptr, B, H_q, H_kv, S_q, S_k, D, causal, scale, opt, 1, stream, true);
}

attn_status_t attn_fwd_qkv8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H_q,
                            int H_kv, int S_q, int S_k, int D, int causal, float scale,
                            const attn_fwd_options_t* opt, void* stream) {
  return run_fwd(q, k, v, o, lse, nullptr, B, H_q, H_kv, S_q, S_k, D, causal, scale, opt, 1, stream, true, true);
}

attn_status_t attn_fwd_split_qk8(const void* q, const void* k, const void* v, void* o, float* lse,
                                 void* workspace, int B, int H_q, int H_kv, int S_q, int S_k, int D, int causal,
                                 float scale, int n_splits, void* stream) {
  if (n_splits < 0 || n_splits > kMaxSplits) return ATTN_ERR_INVALID_ARG;
  if (n_splits == 0) n_splits = attn::tc_split_count(B, H_q, H_kv, S_q, S_k);
  return run_fwd(q, k, v, o, lse, workspace, B, H_q, H_kv, S_q, S_k, D, causal, scale, nullptr, n_splits, stream,
                 true);
}

size_t attn_fwd_split_workspace_size(int B, int H_q, int S_q, int D, int n_splits) {
  if (B < 1 || H_q < 1 || S_q < 1 || (D != 64 && D != 128) || n_splits < 1 || n_splits > kMaxSplits) return 0;
  if (n_splits == 1) return 0;
  const size_t rows = static_cast<size_t>(n_splits) * B * H_q * S_q;
  return (rows * D * sizeof(float) + 255) / 256 * 256 + (rows * sizeof(float) + 255) / 256 * 256;
}

attn_status_t attn_fwd_split(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                             int B, int H_q, int H_kv, int S_q, int S_k, int D, int causal, float scale,
                             int n_splits, void* stream) {
  if (n_splits < 0 || n_splits > kMaxSplits) return ATTN_ERR_INVALID_ARG;
  if (n_splits == 0) n_splits = attn_fwd_split_count(B, H_q, H_kv, S_q, S_k, causal);
  return run_fwd(q, k, v, o, lse, workspace, B, H_q, H_kv, S_q, S_k, D, causal, scale, nullptr, n_splits, stream);
}



size_t attn_bwd_workspace_size(int B, int H_q, int S_q, int D) {
  if (B < 1 || H_q < 1 || S_q < 1 || (D != 64 && D != 128)) return 0;
  const size_t s_pad = (static_cast<size_t>(S_q) + 63) / 64 * 64;
  const size_t dq_acc = static_cast<size_t>(B) * S_q * H_q * D * sizeof(float);
  const size_t rows = static_cast<size_t>(B) * H_q * s_pad * sizeof(float);
  const size_t sems = static_cast<size_t>(B) * H_q * (s_pad / 64) * sizeof(int);
  return (dq_acc + 255) / 256 * 256 + 2 * ((rows + 255) / 256 * 256) + (sems + 255) / 256 * 256 + 256;
}

attn_status_t attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, void* workspace, int B, int H_q, int H_kv,
                          int S_q, int S_k, int D, int causal, float scale, const attn_bwd_options_t* opt,
                          void* stream) {
  attn_status_t st = check_common(B, H_q, H_kv, S_q, S_k, D, causal, scale);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, static_cast<const void*>(lse), dO, static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv), static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return ATTN_ERR_MISALIGNED;
  int* status = status_ptr();
  if (!status) return ATTN_ERR_CUDA;

  const int s_pad = (S_q + 63) / 64 * 64;
  BwdParams p{};
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t dq_bytes = (static_cast<size_t>(B) * S_q * H_q * D * sizeof(float) + 255) / 256 * 256;
  const size_t row_bytes = (static_cast<size_t>(B) * H_q * s_pad * sizeof(float) + 255) / 256 * 256;
  p.dq_acc = reinterpret_cast<float*>(ws);
  p.nlse2 = reinterpret_cast<float*>(ws + dq_bytes);
  p.delta = reinterpret_cast<float*>(ws + dq_bytes + row_bytes);
  p.dq_sem = reinterpret_cast<int*>(ws + dq_bytes + 2 * row_bytes);
  const size_t sem_bytes = (static_cast<size_t>(B) * H_q * (s_pad / 64) * sizeof(int) + 255) / 256 * 256;
  p.ticket = reinterpret_cast<int*>(ws + dq_bytes + 2 * row_bytes + sem_bytes);
  const bool det = opt && opt->deterministic;
  const int cta_mode = opt ? opt->cta_mode : 0;
  if (cta_mode < 0 || cta_mode > 2 || (cta_mode == 2 && D != 128)) return ATTN_ERR_INVALID_ARG;
  // default: CTA pairs for the deterministic instance at D = 128 (its turn waits halve
  // with the number of dQ adders), one CTA per tile otherwise -- the faster kernel of
  // each mode on B200
  const bool pairs = cta_mode == 2 || (cta_mode == 0 && det && D == 128);
  p.persistent = det ? 0 : 1;  // the one-CTA-per-tile pass in the normal dQ order
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.B = B;
  p.H_q = H_q;
  p.H_kv = H_kv;
  p.S_q = S_q;
  p.S_k = S_k;
  p.S_pad = s_pad;
  p.n_kv_tiles = (S_k + 127) / 128;
  p.bh_group = kBwdBhGroup < B * H_kv ? kBwdBhGroup : B * H_kv;
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.status = status;
  p.wait_limit_ns = g_wait_limit_ns.load();

  CUtensorMap mk, mv, mq, mdo, mdq, mq32, mdo32;
  if (!make_bshd_map(&mk, k, B, S_k, H_kv, D, 128) || !make_bshd_map(&mv, v, B, S_k, H_kv, D, 128) ||
      !make_bshd_map(&mq, q, B, S_q, H_q, D, 64) || !make_bshd_map(&mdo, dO, B, S_q, H_q, D, 64) ||
      !make_dqacc_map(&mdq, p.dq_acc, B, S_q, H_q, D, pairs ? D / 2 : D))
    return ATTN_ERR_CUDA;
  if (pairs && (!make_bshd_map(&mq32, q, B, S_q, H_q, D, 32) || !make_bshd_map(&mdo32, dO, B, S_q, H_q, D, 32)))
    return ATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // 1. preprocess
  {
    const long long rows = static_cast<long long>(B) * s_pad * H_q;
    const long long blocks = (rows * (D / 8) + 255) / 256;
    const unsigned g = static_cast<unsigned>(blocks < 148 * 64 ? blocks : 148 * 64);
    if (D == 128)
      attn_bwd_preprocess_kernel<128><<<g, 256, 0, s>>>(p);
    else
      attn_bwd_preprocess_kernel<64><<<g, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // 2. main pass
  if (opt && opt->main_pass_start && cudaEventRecord(static_cast<cudaEvent_t>(opt->main_pass_start), s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  {
    const unsigned grid = static_cast<unsigned>(p.n_kv_tiles) * B * H_kv;
    const unsigned grid_pairs = 2u * static_cast<unsigned>((p.n_kv_tiles + 1) / 2) * B * H_kv;
    cudaError_t err;
    if (pairs)
      err = det ? (causal ? launch_bwd_pair<true, true>(mk, mv, mq32, mdo32, mq, mdo, mdq, p, grid_pairs, s)
                          : launch_bwd_pair<false, true>(mk, mv, mq32, mdo32, mq, mdo, mdq, p, grid_pairs, s))
                : (causal ? launch_bwd_pair<true, false>(mk, mv, mq32, mdo32, mq, mdo, mdq, p, grid_pairs, s)
                          : launch_bwd_pair<false, false>(mk, mv, mq32, mdo32, mq, mdo, mdq, p, grid_pairs, s));
    else if (D == 128)
      err = det ? (causal ? launch_bwd<128, true, true>(mk, mv, mq, mdo, mdq, p, grid, s)
                          : launch_bwd<128, false, true>(mk, mv, mq, mdo, mdq, p, grid, s))
                : (causal ? launch_bwd<128, true, false>(mk, mv, mq, mdo, mdq, p, grid, s)
                          : launch_bwd<128, false, false>(mk, mv, mq, mdo, mdq, p, grid, s));
    else
      err = det ? (causal ? launch_bwd<64, true, true>(mk, mv, mq, mdo, mdq, p, grid, s)
                          : launch_bwd<64, false, true>(mk, mv, mq, mdo, mdq, p, grid, s))
                : (causal ? launch_bwd<64, true, false>(mk, mv, mq, mdo, mdq, p, grid, s)
                          : launch_bwd<64, false, false>(mk, mv, mq, mdo, mdq, p, grid, s));
    if (err != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (opt && opt->main_pass_stop && cudaEventRecord(static_cast<cudaEvent_t>(opt->main_pass_stop), s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  // 3. dQ convert
  {
    const long long n8 = static_cast<long long>(B) * S_q * H_q * D / 8;
    const long long blocks = (n8 + 255) / 256;
    attn_bwd_convert_kernel<<<static_cast<unsigned>(blocks < 148 * 64 ? blocks : 148 * 64), 256, 0, s>>>(p, n8, D);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                       void* dq, void* dk, void* dv, void* workspace, int B, int H_q, int H_kv, int S_q, int S_k,
                       int D, int causal, float scale, void* stream) {
  return attn_bwd_ex(q, k, v, o, lse, dO, dq, dk, dv, workspace, B, H_q, H_kv, S_q, S_k, D, causal, scale, nullptr,
                     stream);
}

attn_status_t attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dO, void* dq, void* dk, void* dv, int B, int H_q, int H_kv, int S_q,
                               int S_k, int D, int causal, float scale, void* stream) {
  attn_status_t st = check_common(B, H_q, H_kv, S_q, S_k, D, causal, scale);
  if (st != ATTN_OK) return st;
  const size_t need = attn_bwd_workspace_size(B, H_q, S_q, D);
  if (need == 0) return ATTN_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return ATTN_ERR_SCRATCH_TOO_SMALL;
  void* scratch = noalloc_scratch_ptr();
  if (scratch == nullptr) return ATTN_ERR_CUDA;
  return attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, scratch, B, H_q, H_kv, S_q, S_k, D, causal, scale, stream);
}

attn_status_t attn_device_status(void* stream) {
  // One caller at a time: the read-out slot g_status_taken is shared.
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DevState ds;
  if (!device_state(&ds)) return ATTN_ERR_CUDA;
  take_status_kernel<<<1, 1, 0, s>>>(ds.status, ds.taken);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  int host = 0;
  if (cudaMemcpyAsync(&host, ds.taken, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  return host == 0 ? ATTN_OK : static_cast<attn_status_t>(host);
}

void attn_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns ? ns : kDefaultWaitLimitNs); }

attn_status_t attn_exp2_poly_eval(const float* x, float* y, long long n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return ATTN_ERR_INVALID_ARG;
  if (n == 0) return ATTN_OK;
  const long long blocks_ll = (n + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(blocks_ll < 148 * 16 ? blocks_ll : 148 * 16);
  exp2_poly_eval_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_read_probe(const void* x, long long bytes, unsigned long long* sink, void* stream) {
  if (bytes < 0 || (bytes & 15) || (bytes > 0 && (!x || !sink)) || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(sink) & 7))
    return ATTN_ERR_INVALID_ARG;
  if (bytes == 0) return ATTN_OK;
  read_probe_kernel<<<kNumSms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(x),
                                                                                  bytes / 16, sink);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

#ifdef ATTN_TIMELINE
// Timeline build only (include/attn_timeline.h).
attn_status_t attn_timeline_read(long long* events, long long* t0, int next_cta) {
  if (!events || !t0) return ATTN_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(events, attn::g_timeline, sizeof(attn::g_timeline)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(t0, attn::g_timeline_t0, sizeof(long long)) != cudaSuccess) return ATTN_ERR_CUDA;
  static long long zeros[attn::kTimelineEvents][attn::kTimelineBlocks];
  if (cudaMemcpyToSymbol(attn::g_timeline, zeros, sizeof(zeros)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyToSymbol(attn::g_timeline_cta, &next_cta, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}
#endif

}  // extern "C"

// sdpa_b200.cu -- host side of libsdpa_b200.so: argument checks, TMA
// descriptors, launch configuration and the extern "C" entry points declared
// in include/sdpa_b200.h.  Device code lives in prefill.cuh and decode.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sdpa_b200.h"
#include "decode.cuh"
#include "prefill.cuh"
#include "rope.cuh"
#include "backward.cuh"

namespace sdpa {
constexpr int kMaxDeviceSlots = 64;
namespace {

constexpr int kMaxDevices = kMaxDeviceSlots;
constexpr int kMaxSeq = 1 << 30;

// ------------------------------------------------------------ checks
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

attn_status_t check_common(const void* q, const void* k, const void* v, const void* o, const float* lse, int B,
                           int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Sq < 0 || Sk < 0 || d <= 0) return ATTN_ERR_SHAPE;
  if (Sq > kMaxSeq || Sk > kMaxSeq) return ATTN_ERR_SHAPE;
  if (static_cast<int64_t>(B) * Hq > INT_MAX / 4) return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_GQA;
  if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
  if (causal < ATTN_CAUSAL_NONE || causal > ATTN_CAUSAL_BOTTOM_RIGHT) return ATTN_ERR_CAUSAL;
  if (!(scale >= 0.f) || std::isinf(scale)) return ATTN_ERR_SCALE;  // also rejects NaN
  const bool empty = (B == 0 || Sq == 0);
  if (!empty) {
    if (q == nullptr || o == nullptr) return ATTN_ERR_NULL;
    if (Sk > 0 && (k == nullptr || v == nullptr)) return ATTN_ERR_NULL;
    if (!aligned(q, 16) || !aligned(o, 16)) return ATTN_ERR_ALIGN;
    if (Sk > 0 && (!aligned(k, 16) || !aligned(v, 16))) return ATTN_ERR_ALIGN;
    if (lse != nullptr && !aligned(lse, 4)) return ATTN_ERR_ALIGN;
  }
  return ATTN_OK;
}

// The optional inputs of the *_ex entry points (nullptr: none of them).
attn_status_t check_extras(const attn_extras_t* ex, int B, int Hq, bool allow_seqlens_q) {
  if (ex == nullptr) return ATTN_OK;
  if (ex->seqlens_q != nullptr && (!allow_seqlens_q || !aligned(ex->seqlens_q, 4)))
    return allow_seqlens_q ? ATTN_ERR_ALIGN : ATTN_ERR_SHAPE;
  if (ex->seqlens_k != nullptr && !aligned(ex->seqlens_k, 4)) return ATTN_ERR_ALIGN;
  if (ex->layout != ATTN_LAYOUT_BHSD && ex->layout != ATTN_LAYOUT_BSHD) return ATTN_ERR_SHAPE;
  if (ex->bias != nullptr) {
    if (!(ex->bias_b == 1 || ex->bias_b == B) || !(ex->bias_h == 1 || ex->bias_h == Hq)) return ATTN_ERR_SHAPE;
    if (!aligned(ex->bias, 2)) return ATTN_ERR_ALIGN;
  }
  return ATTN_OK;
}

// Element strides of a bias [bias_b, bias_h, Sq, Sk]: 0 along a broadcast dim.
void bias_strides(const attn_extras_t* ex, int Sq, int Sk, int64_t* sb, int64_t* sh) {
  const int64_t plane = static_cast<int64_t>(Sq) * Sk;
  *sh = (ex->bias_h == 1) ? 0 : plane;
  *sb = (ex->bias_b == 1) ? 0 : plane * ex->bias_h;
}

float effective_scale(float scale, int d) { return scale == 0.f ? 1.f / std::sqrt(static_cast<float>(d)) : scale; }

int causal_offset(int causal, int Sq, int Sk) { return causal == ATTN_CAUSAL_BOTTOM_RIGHT ? Sk - Sq : 0; }

// ------------------------------------------------------------ device info
struct DeviceInfo {
  bool probed = false;
  bool ok = false;
  int sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

attn_status_t current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    di.probed = true;
    di.ok = (major == 10 && minor == 0);
    di.sms = sms;
  }
  if (!di.ok) return ATTN_ERR_ARCH;
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = di.sms;
  return ATTN_OK;
}

// Best-effort SM count for size queries that may run without a device.
int sm_count_or_default() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
    return sms;
  cudaGetLastError();  // clear a sticky "no device" error from the probe
  return 148;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D bf16 map over a contiguous [outer][rows][d] tensor; box = {64, box_rows, 1},
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* map, const void* base, int d, int rows, int64_t outer, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(outer)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Element strides (batch, head, row) of a [B, H, S, d] tensor in `layout`.
struct Strides {
  int64_t b, h, r;
};
Strides layout_strides(int layout, int H, int S, int d) {
  if (layout == ATTN_LAYOUT_BSHD) return {static_cast<int64_t>(S) * H * d, d, static_cast<int64_t>(H) * d};
  return {static_cast<int64_t>(H) * S * d, static_cast<int64_t>(S) * d, d};
}

// 4-D bf16 map (d, S, H, B) over a [B, H, S, d] tensor stored in `layout`;
// box = {64, box_rows, 1, 1}, 128-byte swizzle, zero fill outside the tensor.
bool make_map4(CUtensorMap* map, const void* base, int layout, int B, int H, int S, int d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const Strides st = layout_strides(layout, H, S, d);
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.r) * 2, static_cast<cuuint64_t>(st.h) * 2,
                                 static_cast<cuuint64_t>(st.b) * 2};
  const cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D bf16 map (Sk, Sq, Hb, Bb) over an additive bias [Bb][Hb][Sq][Sk] (Hb, Bb
// are 1 where it broadcasts); box {64 keys, 128 rows, 1, 1}, 128-byte
// swizzle, zero fill outside.  Sk % 8 == 0 and a 16-byte aligned base
// (checked by the caller) make the row stride a multiple of 16 bytes.
bool make_bias_map(CUtensorMap* map, const void* base, int Bb, int Hb, int Sq, int Sk) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(Sk), static_cast<cuuint64_t>(Sq), static_cast<cuuint64_t>(Hb),
                              static_cast<cuuint64_t>(Bb)};
  const cuuint64_t row = static_cast<cuuint64_t>(Sk) * 2;
  const cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(Sq),
                                 row * static_cast<cuuint64_t>(Sq) * static_cast<cuuint64_t>(Hb)};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------ kernels' config
constexpr int kStagesD128 = 5;
constexpr int kStagesD64 = 8;
// The bias variant stages a 32 KB bias tile in shared memory, which leaves
// room for 4 K/V slots at d = 128.
constexpr int kStagesD128Bias = 4;
constexpr int kDecStages = 3;   // 3 x 32 KB ring: two decode CTAs fit on one SM
constexpr int kDecCtasPerSm = 2;

template <typename K>
bool set_smem(K kernel, int bytes, int dev, bool* done) {
  if (done[dev]) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done[dev] = true;
  return true;
}

// Fill o with zeros and lse with -inf (rows with no visible key, Sk == 0).
__global__ void fill_empty_kernel(uint16_t* o, float* lse, int64_t rows, int d) {
  const int64_t n = rows * d;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    o[i] = 0;
    if (lse != nullptr && i % d == 0) lse[i / d] = -INFINITY;
  }
}

attn_status_t launch_fill_empty(void* o, float* lse, int64_t rows, int d, cudaStream_t st) {
  const int64_t n = rows * d;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096));
  fill_empty_kernel<<<blocks, 256, 0, st>>>(static_cast<uint16_t*>(o), lse, rows, d);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Fill a bf16 buffer with zeros (gradients of inputs no row depends on).
__global__ void fill_zero_kernel(uint16_t* x, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    x[i] = 0;
}

attn_status_t launch_fill_zero(void* x, int64_t n, cudaStream_t st) {
  if (n <= 0) return ATTN_OK;
  const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 4096));
  fill_zero_kernel<<<blocks, 256, 0, st>>>(static_cast<uint16_t*>(x), n);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, int NS, bool BIAS>
attn_status_t launch_prefill(const PrefillParams& prm, int grid, int dev, cudaStream_t st) {
  static bool smem_done[kMaxDevices] = {};
  static std::mutex mu;
  using Cfg = PrefillCfg<D, NS, BIAS>;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!smem_done[dev]) {
      // The kernel's in-kernel register split (setmaxnreg) adds up to exactly
      // kLaunchRegs per thread; launching with any other allocation could make
      // setmaxnreg.inc wait forever, so refuse instead.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, prefill_kernel<D, NS, BIAS>) != cudaSuccess || fa.numRegs != kLaunchRegs)
        return ATTN_ERR_CUDA;
    }
    if (!set_smem(prefill_kernel<D, NS, BIAS>, Cfg::kSmemBytes, dev, smem_done)) return ATTN_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPrefillThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, prefill_kernel<D, NS, BIAS>, prm) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ------------------------------------------------------------ decode split policy
// Pick tiles-per-split by a model of an HBM-bound grid of equal CTAs (fitted
// to B200 measurements of the decode workload over 4..32 splits): a wave of n
// resident CTAs with t tiles each takes t * max(n, kSatCtas) tile-times --
// the CTAs share the HBM bandwidth, but fewer than kSatCtas CTAs cannot keep
// it busy -- plus a fixed start-up/drain cost per wave.  In practice this
// prefers one full wave (every CTA resident) over a short trailing wave.
constexpr double kSatCtas = 75.0;     // CTAs that saturate HBM (per-CTA rate ~ 1/75 of the device's)
constexpr double kWaveFixed = 330.0;  // per-wave start-up and drain, in tile-times of the whole device

double decode_grid_cost(int64_t ctas, int t, int64_t slots) {
  const int64_t full = ctas / slots, rem = ctas - full * slots;
  double cost = static_cast<double>(full) * (t * std::max(static_cast<double>(slots), kSatCtas) + kWaveFixed);
  if (rem > 0) cost += t * std::max(static_cast<double>(rem), kSatCtas) + kWaveFixed;
  return cost;
}

// Each split count s is tried once, with the fewest tiles per split that give
// exactly s splits, in increasing order (ties go to more splits: more CTAs in
// flight).  Counts above kMaxAutoSplitsPerSlot * slots never win under the
// model (one full wave already keeps every slot busy; more only adds waves),
// so the search stops there and stays short for caches of any length.
constexpr int kMaxAutoSplitsPerSlot = 4;

int decode_tiles_per_split(int64_t pairs, int total_tiles, int sms, int requested_splits) {
  if (total_tiles <= 0) return 1;
  if (requested_splits > 0) {
    const int s = std::min(requested_splits, total_tiles);
    return (total_tiles + s - 1) / s;
  }
  const int64_t slots = static_cast<int64_t>(sms) * kDecCtasPerSm;
  const int64_t max_s = std::min<int64_t>(total_tiles, kMaxAutoSplitsPerSlot * slots);
  int best_t = total_tiles;
  double best = 1e300;
  for (int64_t s = 1; s <= max_s; ++s) {
    const int t = static_cast<int>((total_tiles + s - 1) / s);
    if ((total_tiles + t - 1) / t != s) continue;  // s splits are not reachable exactly
    const double cost = decode_grid_cost(pairs * s, t, slots);
    if (cost <= best * (1.0 + 1e-9)) {
      best = cost;
      best_t = t;
    }
  }
  return best_t;
}

bool decode_shape(int B, int Hq, int Hkv, int Sq, int Sk, int d, int num_splits, int sms, int* tiles_per_split,
                  int* nsplit, int* row_groups) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Sk <= 0 || (d != 64 && d != 128) || Hq % Hkv != 0) return false;
  if (Sq > kMaxSeq || Sk > kMaxSeq || num_splits < 0) return false;
  const int group = Hq / Hkv;
  const int64_t rows = static_cast<int64_t>(group) * Sq;
  if (rows > INT_MAX) return false;  // the kernel indexes a KV head's query rows in int
  const int rg = static_cast<int>((rows + kDecRows - 1) / kDecRows);
  const int total_tiles = (Sk + kDecKeys - 1) / kDecKeys;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv * rg;
  const int t = decode_tiles_per_split(pairs, total_tiles, sms, num_splits);
  *tiles_per_split = t;
  *nsplit = (total_tiles + t - 1) / t;
  *row_groups = rg;
  return true;
}

// Workspace: fp32 partial outputs and (max, sum) pairs of every (kv head,
// slot, query row).
size_t decode_ws_bytes(int B, int Hq, int Sq, int d, int nsplit) {
  const size_t rows = static_cast<size_t>(B) * Hq * Sq;
  const size_t po = rows * nsplit * d * sizeof(float);
  return po + rows * nsplit * sizeof(float2);
}

template <int D>
attn_status_t launch_decode(const DecodeParams& prm, int grid, void* o, float* lse, int64_t rows, int dev,
                            cudaStream_t st) {
  static bool smem_done[kMaxDevices] = {};
  static std::mutex mu;
  using Cfg = DecodeCfg<D, kDecStages>;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_smem(decode_split_kernel<D, kDecStages>, Cfg::kSmemBytes, dev, smem_done)) return ATTN_ERR_CUDA;
  }
  // The split kernel is itself a programmatic dependent of whatever precedes
  // it in the stream: its CTAs can be resident while that kernel finishes and
  // wait (griddepcontrol.wait) before touching global memory, which hides the
  // launch between back-to-back decode calls.
  cudaLaunchAttribute sattr[1];
  sattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  sattr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = sattr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_split_kernel<D, kDecStages>, prm) != cudaSuccess) return ATTN_ERR_CUDA;
  // The combine is a programmatic dependent launch: it may be scheduled while
  // the split kernel's last CTAs run and waits (griddepcontrol.wait) for the
  // split grid to complete before reading the partials.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t ccfg = {};
  ccfg.gridDim = dim3(static_cast<unsigned>((rows + 3) / 4));
  ccfg.blockDim = dim3(128);
  ccfg.dynamicSmemBytes = 0;
  ccfg.stream = st;
  ccfg.attrs = attr;
  ccfg.numAttrs = 1;
  CombineParams cp;
  cp.part_o = prm.part_o;
  cp.part_ml = prm.part_ml;
  cp.seqlens_k = prm.seqlens_k;
  cp.out = static_cast<uint16_t*>(o);
  cp.lse = lse;
  cp.rows = rows;
  cp.B = prm.B;
  cp.Hq = prm.Hq;
  cp.Sq = prm.Sq;
  cp.Sk = prm.Sk;
  cp.group = prm.group;
  cp.nsplit = prm.nsplit;
  cp.slots = prm.B * prm.nsplit;
  // q and o share the layout (q's strides are the caller's choice of layout)
  cp.sb = prm.q_sb;
  cp.sh = prm.q_sh;
  cp.sr = prm.q_sr;
  return cudaLaunchKernelEx(&ccfg, decode_combine_kernel<D>, cp) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// The three backward kernels, in stream order: prep (D, LSE in log2), then
// dK/dV over key tiles, then dQ over query tiles.
template <int D>
attn_status_t launch_bwd(const BwdParams& prm, int dev, cudaStream_t st) {
  static bool smem_done_kv[kMaxDevices] = {};
  static bool smem_done_q[kMaxDevices] = {};
  static std::mutex mu;
  using Cfg = BwdCfg<D>;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_smem(bwd_dkdv_kernel<D>, Cfg::kSmemLaunch, dev, smem_done_kv) ||
        !set_smem(bwd_dq_kernel<D>, Cfg::kDqSmemLaunch, dev, smem_done_q))
      return ATTN_ERR_CUDA;
  }
  const int64_t prep_rows = static_cast<int64_t>(prm.B) * prm.Hq * prm.Sq_pad;
  bwd_prep_kernel<D><<<static_cast<unsigned>((prep_rows + 7) / 8), 256, 0, st>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  const int64_t g_kv = static_cast<int64_t>(prm.B) * prm.Hkv * prm.n_kt;
  const int64_t g_q = static_cast<int64_t>(prm.B) * prm.Hq * prm.n_qt;
  if (g_kv > 0) {
    bwd_dkdv_kernel<D><<<static_cast<unsigned>(g_kv), kBwdThreads, Cfg::kSmemLaunch, st>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  if (g_q > 0) {
    bwd_dq_kernel<D><<<static_cast<unsigned>(g_q), kBwdThreads, Cfg::kDqSmemLaunch, st>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// Blocks for the rotary/append kernel: one per token, at most one resident
// wave (kRopeBlocksPerSm per SM); the blocks stride over the remaining tokens.
// When total_lens overlaps past_lens (lengths advanced in place) the append
// kernel leaves it alone and a second kernel, ordered after it on the stream,
// writes it.
template <int D>
attn_status_t launch_rope(const RopeParams& prm, int sms, cudaStream_t st) {
  const int64_t wave = static_cast<int64_t>(sms) * kRopeBlocksPerSm;
  const int grid = static_cast<int>(std::min<int64_t>(std::max(prm.tokens, 1), wave));
  const uintptr_t pl = reinterpret_cast<uintptr_t>(prm.past_lens), tl = reinterpret_cast<uintptr_t>(prm.total_lens);
  const uintptr_t n = static_cast<uintptr_t>(prm.B) * sizeof(int);
  const bool overlap = prm.total_lens != nullptr && pl < tl + n && tl < pl + n;
  RopeParams main = prm;
  if (overlap) main.total_lens = nullptr;
  rope_append_kernel<D><<<grid, kRopeWarps * 32, 0, st>>>(main);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  if (overlap) {
    rope_lengths_kernel<<<static_cast<unsigned>((prm.B + 255) / 256), 256, 0, st>>>(prm.past_lens, prm.total_lens,
                                                                                    prm.B, prm.S_new);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace

// Whether the current device can run the library's kernels (ATTN_ERR_ARCH if not).
attn_status_t current_device_status() { return current_device(nullptr, nullptr); }
}  // namespace sdpa

using namespace sdpa;

extern "C" {

static attn_status_t fwd_impl(const void* q, const void* k, const void* v, const attn_extras_t* ex, void* o,
                              float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal,
                              void* stream) {
  attn_status_t s = check_common(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
  if (s != ATTN_OK) return s;
  if ((s = check_extras(ex, B, Hq, true)) != ATTN_OK) return s;
  const bool has_bias = ex != nullptr && ex->bias != nullptr;
  // the forward reads bias rows with 16-byte loads: rows must be 16-byte aligned
  if (has_bias && (Sk % 8 != 0 || !aligned(ex->bias, 16))) return ATTN_ERR_ALIGN;
  if (B == 0 || Sq == 0) return ATTN_OK;
  int dev = 0, sms = 0;
  if ((s = current_device(&dev, &sms)) != ATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Sq;
  if (Sk == 0) return launch_fill_empty(o, lse, rows, d, st);

  const float sc = effective_scale(scale, d);
  PrefillParams prm;
  std::memset(&prm, 0, sizeof(prm));
  const int layout = ex ? ex->layout : ATTN_LAYOUT_BHSD;
  if (!make_map4(&prm.tm_q, q, layout, B, Hq, Sq, d, kBlockM) ||
      !make_map4(&prm.tm_k, k, layout, B, Hkv, Sk, d, kBlockN) ||
      !make_map4(&prm.tm_v, v, layout, B, Hkv, Sk, d, kBlockN))
    return ATTN_ERR_CUDA;
  prm.o = static_cast<uint16_t*>(o);
  const Strides os = layout_strides(layout, Hq, Sq, d);
  prm.o_sb = os.b;
  prm.o_sh = os.h;
  prm.o_sr = os.r;
  prm.lse = lse;
  prm.seqlens_q = ex ? ex->seqlens_q : nullptr;
  prm.seqlens_k = ex ? ex->seqlens_k : nullptr;
  if (has_bias) {
    prm.bias = static_cast<const uint16_t*>(ex->bias);
    bias_strides(ex, Sq, Sk, &prm.bias_sb, &prm.bias_sh);
    prm.bias_per_b = ex->bias_b == 1 ? 0 : 1;
    prm.bias_per_h = ex->bias_h == 1 ? 0 : 1;
    if (!make_bias_map(&prm.tm_bias, ex->bias, ex->bias_b, ex->bias_h, Sq, Sk)) return ATTN_ERR_CUDA;
  }
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.group = Hq / Hkv;
  prm.causal = causal;
  prm.causal_offset = causal_offset(causal, Sq, Sk);
  prm.num_units = (Sq + 2 * kBlockM - 1) / (2 * kBlockM);
  prm.lpt = causal != ATTN_CAUSAL_NONE ? 1 : 0;
  prm.scale = sc;
  prm.scale_log2 = sc * 1.4426950408889634f;
  prm.inv_scale = 1.f / sc;
  const int64_t units = static_cast<int64_t>(B) * Hq * prm.num_units;
  if (units > INT_MAX / 2) return ATTN_ERR_SHAPE;
  prm.total_units = static_cast<int>(units);
  prm.div_bh = make_fastdiv(static_cast<uint32_t>(std::max(B * Hq, 1)));
  prm.div_hq = make_fastdiv(static_cast<uint32_t>(std::max(Hq, 1)));
  prm.div_group = make_fastdiv(static_cast<uint32_t>(std::max(prm.group, 1)));
  prm.div_units = make_fastdiv(static_cast<uint32_t>(std::max(prm.num_units, 1)));
  // Non-causal fixed lengths (units of equal cost): persistent grid, one CTA
  // per SM (the kernel's shared memory allows one), units dealt statically.
  // Per-batch lengths and causal masks (units of unequal cost): one CTA per
  // unit, running CTAs take over the units of CTAs that have not started (see
  // prefill.cuh), which balances the tail better than the static heaviest-
  // first deal (measured on B200: causal seq 512 / 1024 / 2048 / 4096
  // +4.0 / +5.8 / +0.8 / +0.3 %).
  prm.dynamic = (prm.seqlens_q != nullptr || prm.seqlens_k != nullptr || causal != ATTN_CAUSAL_NONE) ? 1 : 0;
  const int64_t grid = prm.dynamic ? units : std::min<int64_t>(units, sms);
  if (d == 128) {
    return has_bias ? launch_prefill<128, kStagesD128Bias, true>(prm, static_cast<int>(grid), dev, st)
                    : launch_prefill<128, kStagesD128, false>(prm, static_cast<int>(grid), dev, st);
  }
  return has_bias ? launch_prefill<64, kStagesD64, true>(prm, static_cast<int>(grid), dev, st)
                  : launch_prefill<64, kStagesD64, false>(prm, static_cast<int>(grid), dev, st);
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Sq, int Sk, int d, float scale, int causal, void* stream) {
  return fwd_impl(q, k, v, nullptr, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, stream);
}

attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                          int Sq, int Sk, int d, float scale, int causal, const attn_extras_t* extras,
                          void* stream) {
  return fwd_impl(q, k, v, extras, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, stream);
}

attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, const int* seqlens_q,
                              const int* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv, int Sq_max,
                              int Sk_max, int d, float scale, int causal, void* stream) {
  if (B > 0 && Sq_max > 0) {
    if (seqlens_q == nullptr || seqlens_k == nullptr) return ATTN_ERR_NULL;
    if (!aligned(seqlens_q, 4) || !aligned(seqlens_k, 4)) return ATTN_ERR_ALIGN;
  }
  attn_extras_t ex;
  std::memset(&ex, 0, sizeof(ex));
  ex.seqlens_q = seqlens_q;
  ex.seqlens_k = seqlens_k;
  return fwd_impl(q, k, v, &ex, o, lse, B, Hq, Hkv, Sq_max, Sk_max, d, scale, causal, stream);
}

int attn_decode_num_splits(int B, int Hq, int Hkv, int Sq, int Sk, int d) {
  int t = 0, ns = 0, rg = 0;
  if (!decode_shape(B, Hq, Hkv, Sq, Sk, d, 0, sm_count_or_default(), &t, &ns, &rg)) return 0;
  return ns;
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int d, int num_splits) {
  int t = 0, ns = 0, rg = 0;
  const int sms = num_splits > 0 ? 148 : sm_count_or_default();
  if (!decode_shape(B, Hq, Hkv, Sq, Sk, d, num_splits, sms, &t, &ns, &rg)) return 0;
  return decode_ws_bytes(B, Hq, Sq, d, ns);
}

static attn_status_t decode_impl(const void* q, const void* k_cache, const void* v_cache, const attn_extras_t* ex,
                                 void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale,
                                 int causal, int num_splits, void* workspace, size_t workspace_bytes, void* stream,
                                 bool withhold_loads = false) {
  attn_status_t s = check_common(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
  if (s != ATTN_OK) return s;
  if ((s = check_extras(ex, B, Hq, false)) != ATTN_OK) return s;
  const int* seqlens_k = ex ? ex->seqlens_k : nullptr;
  if (num_splits < 0) return ATTN_ERR_SHAPE;
  if (B == 0 || Sq == 0) return ATTN_OK;
  int dev = 0, sms = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Sk == 0) {
    if ((s = current_device(&dev, &sms)) != ATTN_OK) return s;
    return launch_fill_empty(o, lse, static_cast<int64_t>(B) * Hq * Sq, d, st);
  }
  int t = 0, ns = 0, rg = 0;
  // The split policy must not depend on the device when the caller fixed the count.
  const int sms_for_policy = num_splits > 0 ? 148 : sm_count_or_default();
  if (!decode_shape(B, Hq, Hkv, Sq, Sk, d, num_splits, sms_for_policy, &t, &ns, &rg)) return ATTN_ERR_SHAPE;
  const size_t need = decode_ws_bytes(B, Hq, Sq, d, ns);
  if (workspace == nullptr || !aligned(workspace, 16) || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if ((s = current_device(&dev, &sms)) != ATTN_OK) return s;

  const float sc = effective_scale(scale, d);
  const int64_t rows = static_cast<int64_t>(B) * Hq * Sq;
  DecodeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!make_map(&prm.tm_k, k_cache, d, Sk, static_cast<int64_t>(B) * Hkv, kDecKeys) ||
      !make_map(&prm.tm_v, v_cache, d, Sk, static_cast<int64_t>(B) * Hkv, kDecKeys))
    return ATTN_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_o = reinterpret_cast<float*>(ws);
  float2* part_ml = reinterpret_cast<float2*>(ws + rows * ns * d * sizeof(float));
  prm.q = static_cast<const uint16_t*>(q);
  const int layout = ex ? ex->layout : ATTN_LAYOUT_BHSD;
  const Strides qs = layout_strides(layout, Hq, Sq, d);
  prm.q_sb = qs.b;
  prm.q_sh = qs.h;
  prm.q_sr = qs.r;
  prm.seqlens_k = seqlens_k;
  if (ex != nullptr && ex->bias != nullptr) {
    prm.bias = static_cast<const uint16_t*>(ex->bias);
    bias_strides(ex, Sq, Sk, &prm.bias_sb, &prm.bias_sh);
  }
  prm.part_o = part_o;
  prm.part_ml = part_ml;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.group = Hq / Hkv;
  prm.causal = causal;
  prm.causal_offset = causal_offset(causal, Sq, Sk);
  prm.nsplit = ns;
  prm.tiles_per_split = t;
  prm.row_groups = rg;
  prm.scale = sc;
  prm.scale_log2 = sc * 1.4426950408889634f;
  prm.inv_scale = 1.f / sc;
  prm.withhold_loads = withhold_loads ? 1 : 0;
  const int64_t grid = static_cast<int64_t>(B) * Hkv * ns * rg;
  if (grid > INT_MAX || (rows + 3) / 4 > INT_MAX) return ATTN_ERR_SHAPE;
  if (d == 128) return launch_decode<128>(prm, static_cast<int>(grid), o, lse, rows, dev, st);
  return launch_decode<64>(prm, static_cast<int>(grid), o, lse, rows, dev, st);
}

attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                                  int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal,
                                  int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(q, k_cache, v_cache, nullptr, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, num_splits,
                     workspace, workspace_bytes, stream);
}

attn_status_t attn_decode_splitkv_varlen(const void* q, const void* k_cache, const void* v_cache,
                                         const int* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv, int Sq,
                                         int Sk_capacity, int d, float scale, int causal, int num_splits,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  if (B > 0 && Sq > 0 && Sk_capacity > 0) {
    if (seqlens_k == nullptr) return ATTN_ERR_NULL;
    if (!aligned(seqlens_k, 4)) return ATTN_ERR_ALIGN;
  }
  attn_extras_t ex;
  std::memset(&ex, 0, sizeof(ex));
  ex.seqlens_k = seqlens_k;
  return decode_impl(q, k_cache, v_cache, &ex, o, lse, B, Hq, Hkv, Sq, Sk_capacity, d, scale, causal, num_splits,
                     workspace, workspace_bytes, stream);
}

attn_status_t attn_decode_splitkv_ex(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                                     int B, int Hq, int Hkv, int Sq, int Sk, int d, float scale, int causal,
                                     int num_splits, void* workspace, size_t workspace_bytes,
                                     const attn_extras_t* extras, void* stream) {
  return decode_impl(q, k_cache, v_cache, extras, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, num_splits,
                     workspace, workspace_bytes, stream);
}

attn_status_t attn_selftest_decode_wait_timeout(const void* q, const void* k_cache, const void* v_cache, void* o,
                                                float* lse, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                                                void* workspace, size_t workspace_bytes, void* stream) {
  if (B <= 0 || Sq <= 0 || Sk <= 0) return ATTN_ERR_SHAPE;  // the kernel must have something to wait for
  return decode_impl(q, k_cache, v_cache, nullptr, o, lse, B, Hq, Hkv, Sq, Sk, d, 0.f, ATTN_CAUSAL_BOTTOM_RIGHT, 0,
                     workspace, workspace_bytes, stream, /*withhold_loads=*/true);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Sq) {
  if (B < 0 || Hq <= 0 || Sq < 0 || Sq > kMaxSeq) return 0;
  const int64_t sq_pad = (static_cast<int64_t>(Sq) + 127) / 128 * 128;
  return static_cast<size_t>(2 * static_cast<int64_t>(B) * Hq * sq_pad * 4);
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk, int d,
                       float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  attn_status_t s = check_common(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
  if (s != ATTN_OK) return s;
  if (B == 0) return ATTN_OK;
  const bool have_q = Sq > 0, have_k = Sk > 0;
  if (have_q && (dq == nullptr || dout == nullptr)) return ATTN_ERR_NULL;
  if (have_k && (dk == nullptr || dv == nullptr || k == nullptr || v == nullptr)) return ATTN_ERR_NULL;
  if ((have_q && (!aligned(dq, 16) || !aligned(dout, 16))) || (have_k && (!aligned(dk, 16) || !aligned(dv, 16))))
    return ATTN_ERR_ALIGN;
  int dev = 0, sms = 0;
  if ((s = current_device(&dev, &sms)) != ATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // no query rows: nothing depends on k, v; no keys: o = 0 does not depend on q
  if (!have_q) return launch_fill_zero(dk, static_cast<int64_t>(B) * Hkv * Sk * d, st) == ATTN_OK
                          ? launch_fill_zero(dv, static_cast<int64_t>(B) * Hkv * Sk * d, st)
                          : ATTN_ERR_CUDA;
  if (!have_k) return launch_fill_zero(dq, static_cast<int64_t>(B) * Hq * Sq * d, st);
  if (lse == nullptr || o == nullptr) return ATTN_ERR_NULL;
  const size_t need = attn_bwd_workspace_size(B, Hq, Sq);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)) return ATTN_ERR_WORKSPACE;

  BwdParams prm;
  std::memset(&prm, 0, sizeof(prm));
  if (!make_map4(&prm.tm_q, q, ATTN_LAYOUT_BHSD, B, Hq, Sq, d, 128) ||
      !make_map4(&prm.tm_k, k, ATTN_LAYOUT_BHSD, B, Hkv, Sk, d, 128) ||
      !make_map4(&prm.tm_v, v, ATTN_LAYOUT_BHSD, B, Hkv, Sk, d, 128) ||
      !make_map4(&prm.tm_do, dout, ATTN_LAYOUT_BHSD, B, Hq, Sq, d, 128))
    return ATTN_ERR_CUDA;
  const int sq_pad = (Sq + 127) / 128 * 128;
  prm.o = static_cast<const uint16_t*>(o);
  prm.dout = static_cast<const uint16_t*>(dout);
  prm.lse = lse;
  prm.l2 = static_cast<float*>(workspace);
  prm.dvec = prm.l2 + static_cast<int64_t>(B) * Hq * sq_pad;
  prm.dq = static_cast<uint16_t*>(dq);
  prm.dk = static_cast<uint16_t*>(dk);
  prm.dv = static_cast<uint16_t*>(dv);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.Sq = Sq;
  prm.Sk = Sk;
  prm.Sq_pad = sq_pad;
  prm.group = Hq / Hkv;
  prm.causal = causal;
  prm.coff = causal_offset(causal, Sq, Sk);
  prm.n_qt = sq_pad / 128;
  prm.n_kt = (Sk + 127) / 128;
  prm.scale = effective_scale(scale, d);
  prm.scale_log2 = prm.scale * 1.4426950408889634f;
  return d == 128 ? launch_bwd<128>(prm, dev, st) : launch_bwd<64>(prm, dev, st);
}

attn_status_t attn_rope_append(const void* packed_qkv, const float* cos_table, const float* sin_table, int max_pos,
                               const int* past_lens, void* q_out, void* k_cache, void* v_cache, int* total_lens,
                               int B, int S_new, int Hq, int Hkv, int cap, int d, int layout, void* stream) {
  if (B < 0 || S_new < 0 || Hq <= 0 || Hkv <= 0 || cap <= 0 || max_pos <= 0) return ATTN_ERR_SHAPE;
  if (S_new > kMaxSeq || cap > kMaxSeq || max_pos > kMaxSeq) return ATTN_ERR_SHAPE;
  if (static_cast<int64_t>(B) * (Hq + 2 * static_cast<int64_t>(Hkv)) > INT_MAX / 4) return ATTN_ERR_SHAPE;
  if (static_cast<int64_t>(B) * S_new > INT_MAX || Hq + 2 * static_cast<int64_t>(Hkv) > INT_MAX / 128)
    return ATTN_ERR_SHAPE;
  if (Hq % Hkv != 0) return ATTN_ERR_GQA;
  if (d != 64 && d != 128) return ATTN_ERR_HEADDIM;
  if (layout != ATTN_LAYOUT_BHSD && layout != ATTN_LAYOUT_BSHD) return ATTN_ERR_SHAPE;
  if (B == 0) return ATTN_OK;
  if (past_lens == nullptr) return ATTN_ERR_NULL;
  if (!aligned(past_lens, 4) || (total_lens != nullptr && !aligned(total_lens, 4))) return ATTN_ERR_ALIGN;
  if (S_new > 0) {
    if (packed_qkv == nullptr || cos_table == nullptr || sin_table == nullptr || q_out == nullptr ||
        k_cache == nullptr || v_cache == nullptr)
      return ATTN_ERR_NULL;
    if (!aligned(packed_qkv, 16) || !aligned(cos_table, 16) || !aligned(sin_table, 16) || !aligned(q_out, 16) ||
        !aligned(k_cache, 16) || !aligned(v_cache, 16))
      return ATTN_ERR_ALIGN;
  } else if (total_lens == nullptr) {
    return ATTN_OK;  // nothing to write
  }
  int dev = 0, sms = 0;
  attn_status_t s = current_device(&dev, &sms);
  if (s != ATTN_OK) return s;
  RopeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.packed = static_cast<const uint16_t*>(packed_qkv);
  prm.cos_t = cos_table;
  prm.sin_t = sin_table;
  prm.past_lens = past_lens;
  prm.q_out = static_cast<uint16_t*>(q_out);
  prm.k_cache = static_cast<uint16_t*>(k_cache);
  prm.v_cache = static_cast<uint16_t*>(v_cache);
  prm.total_lens = total_lens;
  const Strides qs = layout_strides(layout, Hq, S_new, d);
  const Strides cs = layout_strides(layout, Hkv, cap, d);
  prm.q_sb = qs.b;
  prm.q_sh = qs.h;
  prm.q_sr = qs.r;
  prm.c_sb = cs.b;
  prm.c_sh = cs.h;
  prm.c_sr = cs.r;
  prm.tokens = B * S_new;
  prm.B = B;
  prm.S_new = S_new;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.cap = cap;
  prm.max_pos = max_pos;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_rope<128>(prm, sms, st) : launch_rope<64>(prm, sms, st);
}

const char* attn_status_string(attn_status_t status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_NULL: return "a required pointer is NULL";
    case ATTN_ERR_SHAPE: return "invalid or unsupported size";
    case ATTN_ERR_GQA: return "Hq is not a multiple of Hkv";
    case ATTN_ERR_HEADDIM: return "head_dim must be 64 or 128";
    case ATTN_ERR_ALIGN: return "pointer not aligned (16 bytes; lse 4 bytes)";
    case ATTN_ERR_CAUSAL: return "unknown causal mode";
    case ATTN_ERR_WORKSPACE: return "decode workspace missing, misaligned or too small";
    case ATTN_ERR_CUDA: return "a CUDA runtime call failed";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel gave up";
    case ATTN_ERR_ARCH: return "the current device is not sm_100 (B200)";
    case ATTN_ERR_SCALE: return "scale must be 0 (default) or finite and > 0";
    case ATTN_ERR_SCRATCH_LIMIT: return "problem needs more than the library's static decode scratch (16 MiB)";
    case ATTN_ERR_SEQLEN: return "a per-batch length or position was outside its range (clamped or skipped)";
  }
  return "unknown status";
}

attn_status_t attn_check_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, sdpa::g_error_word, sizeof(word)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(sdpa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
    return (word & sdpa::kErrWaitTimeout) ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_ERR_SEQLEN;
  }
  return ATTN_OK;
}

int attn_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------- allocation-free decode
// Scratch for attn_decode_splitkv_static: a file-scope device array, so the
// library never allocates on behalf of callers that may not allocate.  Every
// device that loads the library holds it until the process exits.
namespace {
static __device__ __align__(256) unsigned char g_decode_static_scratch[ATTN_STATIC_SCRATCH_BYTES];

void* g_static_scratch_addr[sdpa::kMaxDeviceSlots] = {};
std::mutex g_static_scratch_mu;

// Device address of the scratch array on the current device (looked up once per
// device, with that device current).  Host code cannot use the symbol itself:
// on the host it names a stand-in, not device memory.  The cached address
// assumes the device's primary context lives as long as the process; a caller
// that resets the device (cudaDeviceReset) must not call this entry point
// again in that process.
attn_status_t static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sdpa::kMaxDeviceSlots) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_static_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return ATTN_OK;
}
}  // namespace

extern "C" attn_status_t attn_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache,
                                                    void* o, float* lse, int B, int Hq, int Hkv, int Sq, int Sk,
                                                    int d, float scale, int causal, int num_splits, void* stream) {
  attn_status_t s = check_common(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal);
  if (s != ATTN_OK) return s;
  if (num_splits < 0) return ATTN_ERR_SHAPE;
  // the device must be a B200 before its copy of the scratch is looked up
  if (B > 0 && Sq > 0 && (s = sdpa::current_device_status()) != ATTN_OK) return s;
  if (B > 0 && Sq > 0 && Sk > 0) {
    const size_t need = attn_decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits);
    if (need == 0) return ATTN_ERR_SHAPE;
    if (need > ATTN_STATIC_SCRATCH_BYTES) return ATTN_ERR_SCRATCH_LIMIT;
  }
  void* scratch = nullptr;
  if (B > 0 && Sq > 0 && (s = static_scratch_address(&scratch)) != ATTN_OK) return s;
  return attn_decode_splitkv(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, num_splits, scratch,
                             ATTN_STATIC_SCRATCH_BYTES, stream);
}

// backward.cuh -- gradients of the fused attention forward for sm_100a.
//
// For a loss L with dO = dL/dO, the forward's P = softmax(scale Q K^T + mask)
// and O = P V give (one query row i, key j):
//   dP_ij = dO_i . V_j,   dS_ij = P_ij (dP_ij - D_i),   D_i = sum_j P_ij dP_ij
//   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i,   dV_j = sum_i P_ij dO_i
// and D_i also equals dO_i . O_i, since O_i = sum_j P_ij V_j.  The pages
// report the FlashAttention-2 backward's speed ("FlashAttention-2" notes) but
// give no algorithm; this file is this library's own design: P is recomputed
// from the forward's LSE (P_ij = exp(scale q_i.k_j - LSE_i)), so nothing of
// size Sq x Sk is ever stored.
//
// Three kernels:
//   bwd_prep_kernel   D_i = dO_i . O_i and LSE_i in log2 units, into the
//                     caller's workspace (rows padded to whole 128-row tiles:
//                     padding has D = 0 and LSE = +inf, i.e. P = 0).
//   bwd_dkdv_kernel   one CTA per 128-key tile of a (batch, KV head): K and V
//                     stay in shared memory while the query tiles of every
//                     query head of the group stream through a 2-stage ring.
//                     Per query tile: S^T = K Q^T and dP^T = V dO^T (tcgen05,
//                     into TMEM), P^T and dS^T by eight compute warps (two per
//                     key row, one for each half of the 128 query columns;
//                     each half's bf16 results overwrite that half's first
//                     32 columns of S^T and dP^T), then dV += P^T dO and
//                     dK += dS^T Q with P^T, dS^T read from TMEM.  The next
//                     tile's S^T is issued right after dV and its dP^T after
//                     dK, each with its own commit, so its P^T (the
//                     exponentials) is under way while dK and dP^T run.
//   bwd_dq_kernel     one CTA per 128-row query tile: Q and dO stay in shared
//                     memory while the key tiles stream through a ring of
//                     single K and V slots (V_j freed after dP_j, K_j after
//                     dS_j K_j, so the next tiles land early); S = Q K^T and
//                     dP = dO V^T, dS by the compute warps into TMEM columns
//                     of its own, dQ += dS K.  With dS apart from S, the next
//                     tile's S and dP are issued before this tile's dS K, and
//                     S and dP have commits of their own: the compute warps
//                     take the exponentials of S while dP and dS K run.
// Fully masked key tiles are skipped (causal).  TMEM holds every accumulator
// (dK and dV for the whole query loop, dQ for the whole key loop).  Every
// wait is bounded; a timeout sets the device error word and the kernel exits.
#pragma once
#include "prefill.cuh"

namespace sdpa {

struct BwdParams {
  // 4-D maps (d, S, H, B) over q, k, v, dO (BHSD); box {64, 128, 1, 1}, 128-byte swizzle.
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_do;
  const uint16_t* o;    // forward output, bf16 [B, Hq, Sq, d]
  const uint16_t* dout;  // dO, bf16 [B, Hq, Sq, d]
  const float* lse;     // forward LSE (natural log) [B, Hq, Sq]
  float* l2;            // workspace [B*Hq][Sq_pad]: LSE * log2(e), +inf where P = 0
  float* dvec;          // workspace [B*Hq][Sq_pad]: D = rowsum(dO * O)
  uint16_t* dq;         // bf16 [B, Hq, Sq, d]
  uint16_t* dk;         // bf16 [B, Hkv, Sk, d]
  uint16_t* dv;         // bf16 [B, Hkv, Sk, d]
  int B, Hq, Hkv, Sq, Sk, Sq_pad, group;
  int causal;    // 0 none, 1 top-left, 2 bottom-right
  int coff;      // key j visible to row i iff j <= i + coff (causal)
  int n_qt, n_kt;  // query / key tiles of 128
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
};

constexpr int kBwdThreads = 320;  // warps 0-7 compute, 8 MMA issuer (+ TMEM owner), 9 TMA producer
constexpr int kBwdComputeWarps = 8;
constexpr int kBwdMmaWarp = 8;
constexpr int kBwdLoadWarp = 9;
constexpr int kBwdStages = 2;
constexpr int kBwdHeadGroup = 8;  // heads dealt together under a causal mask (see lpt_coords)

// Under a causal mask the CTAs' work differs up to n-fold (a key tile near
// the start is seen by every query tile, one near the end by few), and CTAs
// are dispatched in blockIdx order: in head-major order the heaviest tiles of
// the last heads would start last and run on alone.  So CTA idx takes, within
// groups of kBwdHeadGroup heads (whose K, V, Q and dO stay in L2 together),
// the tiles heaviest first: rank 0 = heaviest.  Covers [0, n_t * heads).
__device__ __forceinline__ void lpt_coords(int idx, int n_t, int heads, int& rank, int& head) {
  const int per_group = n_t * kBwdHeadGroup;
  const int g = idx / per_group;
  const int rem = idx - g * per_group;
  const int gh = min(kBwdHeadGroup, heads - g * kBwdHeadGroup);
  rank = rem / gh;
  head = g * kBwdHeadGroup + (rem - rank * gh);
}
constexpr float kLog2e = 1.4426950408889634f;

// 1-D bulk copy global -> shared (no tensor map), completion counted on `bar`.
// Both addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t smem_dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// 32 lanes x 16 consecutive 32-bit TMEM columns from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

template <int D>
struct BwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;   // one 128-row bf16 tile
  static constexpr int kBlocks = D / 64;            // 64-column swizzle blocks per tile
  static constexpr int kBlockBytes = 128 * 128;     // 16 KB per swizzle block
  static constexpr int kVecBytes = 128 * 4;         // 128 fp32 (L2 or D of one query tile)
  // smem: two resident tiles, then per stage two streamed tiles and two vectors
  static constexpr int kStageBytes = 2 * kTileBytes + 2 * kVecBytes;
  // res_full, st_full[2], st_empty[2], s_full, p_full, done, then dK/dV: dp_full
  // (and ds_full); dQ: ds_free (the previous dS has been read), dp_full, s_free,
  // dp_free (S / dP read out of TMEM)
  static constexpr int kNumBars = 1 + 2 * kBwdStages + 7;
  static constexpr int kSmemBytes = 2 * kTileBytes + kBwdStages * kStageBytes + kNumBars * 8 + 16 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
  // dQ kernel: Q, dO resident, then a ring of kDqSlots single tiles (K_0, V_0,
  // K_1, V_1, ...): V_j's slot is free once dP_j is done and K_j's once
  // dQ += dS_j K_j is, so the next tiles start landing a whole tile earlier
  // than with K and V in one stage; then res_full, kv_full[kDqSlots],
  // kv_empty[kDqSlots], s_full, p_full, done, ds_free, dp_full, s_free, dp_free
  static constexpr int kDqSlots = D == 128 ? 5 : 8;
  static constexpr int kDqNumBars = 1 + 2 * kDqSlots + 7;
  static constexpr int kDqSmemBytes = (2 + kDqSlots) * kTileBytes + kDqNumBars * 8 + 16 + 1024;
  static_assert(kDqSmemBytes <= 227 * 1024, "shared memory per block");
  static constexpr int kDqSmemLaunch = kDqSmemBytes > 116 * 1024 ? kDqSmemBytes : 116 * 1024;
  static constexpr uint32_t kTmemCols = 512;
  // Each CTA takes all 512 TMEM columns, and tcgen05.alloc waits without a
  // bound for columns another CTA holds: launch with more than half of the
  // SM's 228 KB of shared memory, so that no two CTAs share an SM.
  static constexpr int kSmemLaunch = kSmemBytes > 116 * 1024 ? kSmemBytes : 116 * 1024;
};

// -------------------------------------------------------------- prep kernel
// One warp per padded row: D = dO . O (fp32) and LSE * log2(e).  A row that
// saw no key has LSE = -inf and a padding row has none: both get +inf, so
// that exp2(x - l2) = 0 for them.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ BwdParams p) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(p.B) * p.Hq * p.Sq_pad) return;
  const int i = static_cast<int>(w % p.Sq_pad);
  const int64_t bh = w / p.Sq_pad;
  float dsum = 0.f, l2 = INFINITY;
  if (i < p.Sq) {
    const int64_t row = (bh * p.Sq + i) * D;
    constexpr int kPer = D / 32;  // bf16 elements per lane: 4 (d=128) or 2 (d=64)
    const uint16_t* orow = p.o + row + lane * kPer;
    const uint16_t* grow = p.dout + row + lane * kPer;
#pragma unroll
    for (int e = 0; e < kPer; ++e) dsum += bf16_bits_to_float(__ldg(orow + e)) * bf16_bits_to_float(__ldg(grow + e));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    const float lse = __ldg(p.lse + bh * p.Sq + i);
    l2 = (lse == -INFINITY) ? INFINITY : lse * kLog2e;
  }
  if (lane == 0) {
    p.dvec[w] = dsum;
    p.l2[w] = l2;
  }
}

// P^T and dS^T for 32 query columns col0 .. col0+31 of one key row, in two
// passes, so that P^T can be computed as soon as S^T is in TMEM, before dP^T
// is: P (fp32, kept for the second pass) and P^T as bf16 pairs from S^T
// (sv) and the query tile's LSE*log2(e) (l2v); then dS^T from P, dP^T (dp)
// and D (ddv).  Columns before cmin do not see the key.
__device__ __forceinline__ void p_chunk(const uint32_t (&sv)[32], const float* l2v, int col0, int cmin, float c,
                                        float (&pr)[32], uint32_t (&pk)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 lv = *reinterpret_cast<const float4*>(l2v + col0 + e);
    const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float x = fmaf(__uint_as_float(sv[e + u]), c, -lq[u]);
      pr[e + u] = (col0 + e + u >= cmin) ? ex2_approx(x) : 0.f;
    }
    pk[e / 2] = pack_bf16x2(pr[e], pr[e + 1]);
    pk[e / 2 + 1] = pack_bf16x2(pr[e + 2], pr[e + 3]);
  }
}

__device__ __forceinline__ void ds_chunk(const float (&pr)[32], const uint32_t (&dp)[32], const float* ddv, int col0,
                                         uint32_t (&dk16)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const float4 dv4 = *reinterpret_cast<const float4*>(ddv + col0 + e);
    const float dq4[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
    float ds[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) ds[u] = pr[e + u] * (__uint_as_float(dp[e + u]) - dq4[u]);
    dk16[e / 2] = pack_bf16x2(ds[0], ds[1]);
    dk16[e / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
  }
}

// ------------------------------------------------------------ dK, dV kernel
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // K | V | stage 0: Q, dO, L2, D | stage 1: ... | barriers
  const uint32_t sK = smem_u32(smem);
  const uint32_t sV = sK + Cfg::kTileBytes;
  auto sQ = [&](int st) { return sK + 2 * Cfg::kTileBytes + st * Cfg::kStageBytes; };
  auto sDO = [&](int st) { return sQ(st) + Cfg::kTileBytes; };
  const float* vec_base = reinterpret_cast<const float*>(smem + 2 * Cfg::kTileBytes + 2 * Cfg::kTileBytes);
  auto l2_at = [&](int st) { return vec_base + st * (Cfg::kStageBytes / 4); };
  auto dd_at = [&](int st) { return vec_base + st * (Cfg::kStageBytes / 4) + 128; };
  const uint32_t bar0 = sK + 2 * Cfg::kTileBytes + kBwdStages * Cfg::kStageBytes;
  const uint32_t res_full = bar0;
  auto st_full = [&](int st) { return bar0 + 8u * (1 + st); };
  auto st_empty = [&](int st) { return bar0 + 8u * (1 + kBwdStages + st); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * kBwdStages);  // S^T of the current query tile done
  const uint32_t p_full = s_full + 8u;
  const uint32_t done = p_full + 8u;
  const uint32_t dp_full = done + 8u;  // dP^T of the current query tile done
  const uint32_t ds_full = dp_full + 8u;  // dS^T of the current query tile written (p_full: P^T)
  uint8_t* bar_ptr = smem + 2 * Cfg::kTileBytes + kBwdStages * Cfg::kStageBytes;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * Cfg::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int kt, bkv;
  if (p.causal) {
    lpt_coords(static_cast<int>(blockIdx.x), p.n_kt, p.B * p.Hkv, kt, bkv);  // early key tiles are heaviest
  } else {
    kt = static_cast<int>(blockIdx.x % p.n_kt);
    bkv = static_cast<int>(blockIdx.x / p.n_kt);
  }
  const int b = bkv / p.Hkv;
  const int hkv = bkv - b * p.Hkv;
  const int k0 = kt * 128;
  // query tiles that see any key of this tile: rows i >= k0 - coff (causal)
  const int qt0 = p.causal ? max(0, (k0 - p.coff) / 128) : 0;
  const int per_head = max(0, p.n_qt - qt0);
  const int n_it = per_head * p.group;

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int st = 0; st < kBwdStages; ++st) {
      mbar_init(st_full(st), 1);
      mbar_init(st_empty(st), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kBwdComputeWarps);  // one arrive per compute warp
    mbar_init(done, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdComputeWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S^T [0,128) | dP^T [128,256) | dV [256,256+D) | dK [256+D,256+2D)
  constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

  if (warp == kBwdLoadWarp) {
    if (lane == 0 && n_it > 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_do);
      mbar_arrive_expect_tx(res_full, 2 * Cfg::kTileBytes);
      for (int blk = 0; blk < Cfg::kBlocks; ++blk) {
        tma_load_4d(sK + blk * Cfg::kBlockBytes, &p.tm_k, blk * 64, k0, hkv, b, res_full);
        tma_load_4d(sV + blk * Cfg::kBlockBytes, &p.tm_v, blk * 64, k0, hkv, b, res_full);
      }
      int it = 0;
      for (; it < n_it; ++it) {
        const int st = it % kBwdStages;
        if (!mbar_wait(st_empty(st), ((it / kBwdStages) & 1) ^ 1, abort_flag)) break;
        const int hq = hkv * p.group + it / per_head;
        const int qt = qt0 + it % per_head;
        mbar_arrive_expect_tx(st_full(st), 2 * Cfg::kTileBytes + 2 * Cfg::kVecBytes);
        for (int blk = 0; blk < Cfg::kBlocks; ++blk) {
          tma_load_4d(sQ(st) + blk * Cfg::kBlockBytes, &p.tm_q, blk * 64, qt * 128, hq, b, st_full(st));
          tma_load_4d(sDO(st) + blk * Cfg::kBlockBytes, &p.tm_do, blk * 64, qt * 128, hq, b, st_full(st));
        }
        const int64_t vec = (static_cast<int64_t>(b) * p.Hq + hq) * p.Sq_pad + qt * 128;
        bulk_load(smem_u32(l2_at(st)), p.l2 + vec, Cfg::kVecBytes, st_full(st));
        bulk_load(smem_u32(dd_at(st)), p.dvec + vec, Cfg::kVecBytes, st_full(st));
      }
      // copies in flight must land before the CTA may exit
      mbar_wait_drain(res_full, 0);
      for (int i = max(0, it - kBwdStages); i < it; ++i) mbar_wait_drain(st_full(i % kBwdStages), (i / kBwdStages) & 1);
    }
    __syncwarp();
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0 && n_it > 0) {
      const uint64_t hi = static_cast<uint64_t>(sdesc_hi(1024)) << 32;
      const uint64_t dk_k = hi | sdesc_lo(sK, 16);  // K, K-major (A of S^T)
      const uint64_t dv_k = hi | sdesc_lo(sV, 16);  // V, K-major (A of dP^T)
      bool ok = mbar_wait(res_full, 0, abort_flag);
      // Per query tile it (stage st): S^T = K Q^T and dP^T = V dO^T (M = 128
      // keys, N = 128 queries, K = D); dV += P^T dO once the compute warps
      // have left P^T in TMEM, and dK += dS^T Q once they have left dS^T
      // (M = 128 keys, N = D, K = 128 queries; A from TMEM, B the query-side
      // tile, MN-major).  The next tile's S^T goes right after dV (which read
      // the P^T it overwrites) and its dP^T right after dK, so the compute
      // warps' dS^T overlaps dV and the next S^T, and their next exponentials
      // overlap dK and the next dP^T.  One thread issues everything, in order.
      auto issue_s = [&](int st) {
        issue_qk<D>(tmem + kColS, dk_k, hi | sdesc_lo(sQ(st), 16));
        mma_commit(s_full);
      };
      auto issue_dp = [&](int st) {
        issue_qk<D>(tmem + kColDP, dv_k, hi | sdesc_lo(sDO(st), 16));
        mma_commit(dp_full);
      };
      if (ok && mbar_wait(st_full(0), 0, abort_flag)) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      } else {
        ok = false;
      }
      for (int it = 0; ok && it < n_it; ++it) {
        const int st = it % kBwdStages;
        const bool next = it + 1 < n_it;
        const int st1 = (it + 1) % kBwdStages;
        if (!mbar_wait(p_full, it & 1, abort_flag)) break;
        if (next && !mbar_wait(st_full(st1), ((it + 1) / kBwdStages) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t ddo_mn = hi | sdesc_lo(sDO(st), Cfg::kBlockBytes);
        const uint64_t dq_mn = hi | sdesc_lo(sQ(st), Cfg::kBlockBytes);
        // P^T, dS^T of queries 0..63 are at columns 0..31 of S^T / dP^T and of
        // queries 64..127 at 64..95: issue_pv reads keys 16 kk.. at column 8 kk
        // of its base, so the second half's base is 32 columns further.
        issue_pv<D, 0>(tmem + kColDV, tmem + kColS, ddo_mn, it > 0);
        issue_pv<D, 1>(tmem + kColDV, tmem + kColS + 32, ddo_mn, true);
        if (next) issue_s(st1);
        if (!mbar_wait(ds_full, it & 1, abort_flag)) break;
        tc_fence_after();
        issue_pv<D, 0>(tmem + kColDK, tmem + kColDP, dq_mn, it > 0);
        issue_pv<D, 1>(tmem + kColDK, tmem + kColDP + 32, dq_mn, true);
        mma_commit(st_empty(st));
        if (next) issue_dp(st1);
      }
      mma_commit(done);
      mbar_wait_drain(done, 0);
    }
    __syncwarp();
  } else if (warp < kBwdComputeWarps) {
    // ------------------------------------ compute: two warps per key row (column halves)
    // Warpgroup wg takes query columns 64 wg .. 64 wg + 63 (chunks 2 wg, 2 wg + 1)
    // of TMEM lane quarter `quarter` and writes their bf16 results over its
    // own first 32 columns (64 wg .. 64 wg + 31 of S^T and of dP^T), which it
    // has already read: the two warpgroups never touch each other's columns.
    // The dV/dK MMAs read queries 0..63 at column 0 and 64..127 at column 64.
    const int wg = warp >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int j = k0 + r;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_bits + kColS + 64 * wg;
    const uint32_t tDP = tmem + lane_bits + kColDP + 64 * wg;
    const float c = p.scale_log2;
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int st = it % kBwdStages;
      const int qt = qt0 + it % per_head;
      // query columns c < cmin do not see key j (causal); keys past Sk see nothing
      const int cmin = (j >= p.Sk) ? INT_MAX : (p.causal ? j - p.coff - qt * 128 : INT_MIN);
      // S^T/dP^T ready; the stage's L2/D vectors landed (the wait on the
      // stage's own barrier makes the bulk copy's writes visible here).
      // Warp-uniform: the tcgen05.ld/st below are collective over the warp.
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag) &&
                                       mbar_wait(st_full(st), (it / kBwdStages) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float* l2v = l2_at(st);
      const float* ddv = dd_at(st);
      // pass 1, once S^T is in: P (kept) and P^T over S^T's columns 16 h ..
      // 16 h + 15 of this half (read in step 0 already)
      float pr[2][32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sv[32], pk[16];
        tmem_ld32(tS + 32 * h, sv);
        tmem_wait_ld();
        p_chunk(sv, l2v, 64 * wg + 32 * h, cmin, c, pr[h], pk);
        tmem_st16(tS + 16 * h, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);  // P^T written: dV may run
      // pass 2, once dP^T is in: dS^T over dP^T's columns the same way
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dp[32], dk16[16];
        tmem_ld32(tDP + 32 * h, dp);
        tmem_wait_ld();
        ds_chunk(pr[h], dp, ddv, 64 * wg + 32 * h, dk16);
        tmem_st16(tDP + 16 * h, dk16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);  // dS^T written: dK may run
    }
    // ---- epilogue: dK = scale * acc, dV = acc -> bf16 rows.  The TMEM loads
    // are collective: the whole warp runs them (warp-uniform `have`); only
    // the stores depend on the lane's row.
    const bool have = __all_sync(0xffffffffu, ok && n_it > 0 && mbar_wait(done, 0, abort_flag));
    if (have) tc_fence_after();
    {
      const int64_t row = ((static_cast<int64_t>(b) * p.Hkv + hkv) * p.Sk + j) * D;
#pragma unroll 1
      for (int q = wg * (D / 64); q < (wg + 1) * (D / 64); ++q) {  // this warpgroup's half of the columns
        uint32_t a[32], g[32];
        if (have) {
          tmem_ld32(tmem + lane_bits + kColDV + q * 32, a);
          tmem_ld32(tmem + lane_bits + kColDK + q * 32, g);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = g[e] = 0u;
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint4 wv, wk;
          wv.x = pack_bf16x2(__uint_as_float(a[c8 * 8 + 0]), __uint_as_float(a[c8 * 8 + 1]));
          wv.y = pack_bf16x2(__uint_as_float(a[c8 * 8 + 2]), __uint_as_float(a[c8 * 8 + 3]));
          wv.z = pack_bf16x2(__uint_as_float(a[c8 * 8 + 4]), __uint_as_float(a[c8 * 8 + 5]));
          wv.w = pack_bf16x2(__uint_as_float(a[c8 * 8 + 6]), __uint_as_float(a[c8 * 8 + 7]));
          wk.x = pack_bf16x2(__uint_as_float(g[c8 * 8 + 0]) * p.scale, __uint_as_float(g[c8 * 8 + 1]) * p.scale);
          wk.y = pack_bf16x2(__uint_as_float(g[c8 * 8 + 2]) * p.scale, __uint_as_float(g[c8 * 8 + 3]) * p.scale);
          wk.z = pack_bf16x2(__uint_as_float(g[c8 * 8 + 4]) * p.scale, __uint_as_float(g[c8 * 8 + 5]) * p.scale);
          wk.w = pack_bf16x2(__uint_as_float(g[c8 * 8 + 6]) * p.scale, __uint_as_float(g[c8 * 8 + 7]) * p.scale);
          if (j < p.Sk) {
            *reinterpret_cast<uint4*>(p.dv + row + q * 32 + c8 * 8) = wv;
            *reinterpret_cast<uint4*>(p.dk + row + q * 32 + c8 * 8) = wk;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ----------------------------------------------------------------- dQ kernel
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using Cfg = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Q | dO | ring of kDqSlots tiles: position 2j holds K_j, 2j + 1 holds V_j | barriers
  constexpr int NSL = Cfg::kDqSlots;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sDO = sQ + Cfg::kTileBytes;
  auto slot_addr = [&](int pos) { return sQ + (2 + pos % NSL) * Cfg::kTileBytes; };
  const uint32_t bar0 = sQ + (2 + NSL) * Cfg::kTileBytes;
  const uint32_t res_full = bar0;
  auto kv_full = [&](int pos) { return bar0 + 8u * (1 + pos % NSL); };
  auto kv_empty = [&](int pos) { return bar0 + 8u * (1 + NSL + pos % NSL); };
  auto kv_par = [&](int pos) { return static_cast<uint32_t>((pos / NSL) & 1); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * NSL);
  const uint32_t p_full = s_full + 8u;
  const uint32_t done = p_full + 8u;
  const uint32_t ds_free = done + 8u;     // dQ += dS K of the previous key tile is done
  const uint32_t dp_full = ds_free + 8u;  // dP of the current key tile done
  const uint32_t s_free = dp_full + 8u;   // every compute warp has read S of the current key tile
  const uint32_t dp_free = s_free + 8u;   // ... and dP
  uint8_t* bar_ptr = smem + (2 + NSL) * Cfg::kTileBytes;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * Cfg::kDqNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int qt, bh;
  if (p.causal) {
    int rank;
    lpt_coords(static_cast<int>(blockIdx.x), p.n_qt, p.B * p.Hq, rank, bh);
    qt = p.n_qt - 1 - rank;  // late query tiles are heaviest
  } else {
    qt = static_cast<int>(blockIdx.x % p.n_qt);
    bh = static_cast<int>(blockIdx.x / p.n_qt);
  }
  const int b = bh / p.Hq;
  const int hq = bh - b * p.Hq;
  const int hkv = hq / p.group;
  const int i0 = qt * 128;
  // key tiles this query tile sees: keys j <= last row + coff (causal)
  int n_it = p.n_kt;
  if (p.causal) {
    const int last_key = min(i0 + 127, p.Sq - 1) + p.coff;
    n_it = last_key < 0 ? 0 : min(p.n_kt, last_key / 128 + 1);
  }

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int sl = 0; sl < NSL; ++sl) {
      mbar_init(kv_full(sl), 1);
      mbar_init(kv_empty(sl), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, kBwdComputeWarps);
    mbar_init(done, 1);
    mbar_init(ds_free, 1);
    mbar_init(dp_full, 1);
    mbar_init(s_free, kBwdComputeWarps);
    mbar_init(dp_free, kBwdComputeWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S [0,128) | dP [128,256) | dQ [256,256+D) | dS [384,448) (bf16 pairs)
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDS = 384;

  if (warp == kBwdLoadWarp) {
    if (lane == 0 && n_it > 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(res_full, 2 * Cfg::kTileBytes);
      for (int blk = 0; blk < Cfg::kBlocks; ++blk) {
        tma_load_4d(sQ + blk * Cfg::kBlockBytes, &p.tm_q, blk * 64, i0, hq, b, res_full);
        tma_load_4d(sDO + blk * Cfg::kBlockBytes, &p.tm_do, blk * 64, i0, hq, b, res_full);
      }
      int pos = 0;  // ring positions issued: K_j at 2j, V_j at 2j + 1
      for (; pos < 2 * n_it; ++pos) {
        if (!mbar_wait(kv_empty(pos), kv_par(pos) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(kv_full(pos), Cfg::kTileBytes);
        const CUtensorMap* tm = (pos & 1) ? &p.tm_v : &p.tm_k;
        for (int blk = 0; blk < Cfg::kBlocks; ++blk)
          tma_load_4d(slot_addr(pos) + blk * Cfg::kBlockBytes, tm, blk * 64, (pos >> 1) * 128, hkv, b, kv_full(pos));
      }
      mbar_wait_drain(res_full, 0);
      for (int i = max(0, pos - NSL); i < pos; ++i) mbar_wait_drain(kv_full(i), kv_par(i));
    }
    __syncwarp();
  } else if (warp == kBwdMmaWarp) {
    if (lane == 0 && n_it > 0) {
      const uint64_t hi = static_cast<uint64_t>(sdesc_hi(1024)) << 32;
      const uint64_t dq_k = hi | sdesc_lo(sQ, 16);
      const uint64_t ddo_k = hi | sdesc_lo(sDO, 16);
      // Key tile it+1's S = Q K^T (M = 128 queries, N = 128 keys, K = D) is
      // issued as soon as the compute warps have read tile it's S out of TMEM
      // (they keep P in registers), its dP = dO V^T once they have read tile
      // it's dP, and dQ += dS K for tile it once its dS is written: the
      // tensor core computes the next tile's S while the compute warps still
      // take this tile's exponentials.
      // S(j) reads K_j (ring position 2j), dP(j) V_j (2j + 1), dQ(j) K_j
      // again; V_j's slot is released after dP(j), K_j's after dQ(j).
      auto issue_s = [&](int j) {
        issue_qk<D>(tmem + kColS, dq_k, hi | sdesc_lo(slot_addr(2 * j), 16));
        mma_commit(s_full);
      };
      auto issue_dp = [&](int j) {
        issue_qk<D>(tmem + kColDP, ddo_k, hi | sdesc_lo(slot_addr(2 * j + 1), 16));
        mma_commit(dp_full);
        mma_commit(kv_empty(2 * j + 1));
      };
      bool ok = mbar_wait(res_full, 0, abort_flag) && mbar_wait(kv_full(0), kv_par(0), abort_flag) &&
                mbar_wait(kv_full(1), kv_par(1), abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int it = 0; ok && it < n_it; ++it) {
        const bool next = it + 1 < n_it;
        if (next) {
          if (!mbar_wait(s_free, it & 1, abort_flag) ||
              !mbar_wait(kv_full(2 * it + 2), kv_par(2 * it + 2), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(it + 1);
          if (!mbar_wait(dp_free, it & 1, abort_flag) ||
              !mbar_wait(kv_full(2 * it + 3), kv_par(2 * it + 3), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_dp(it + 1);
        }
        // dS(it) written
        if (!mbar_wait(p_full, it & 1, abort_flag)) break;
        tc_fence_after();
        // dQ += dS K (M = 128 queries, N = D, K = 128 keys; dS from TMEM, K MN-major)
        const uint64_t dk_mn = hi | sdesc_lo(slot_addr(2 * it), Cfg::kBlockBytes);
        issue_pv<D, 0>(tmem + kColDQ, tmem + kColDS, dk_mn, it > 0);
        issue_pv<D, 1>(tmem + kColDQ, tmem + kColDS, dk_mn, true);
        mma_commit(ds_free);
        mma_commit(kv_empty(2 * it));
      }
      mma_commit(done);
      mbar_wait_drain(done, 0);
    }
    __syncwarp();
  } else if (warp < kBwdComputeWarps) {
    // ------------------------------------ compute: two warps per query row (column halves)
    const int wg = warp >> 2;  // key columns 64 wg .. 64 wg + 63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int i = i0 + r;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    const int64_t vec = static_cast<int64_t>(bh) * p.Sq_pad + i;
    const float l2 = __ldg(p.l2 + vec);   // +inf for rows past Sq or that saw no key
    const float dd = __ldg(p.dvec + vec);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      // key columns past Sk, or (causal) past row i + coff, are masked
      const int jlim = min(p.Sk - 1, p.causal ? i + p.coff : INT_MAX) - it * 128;  // last visible column
      // (warp-uniform: the tcgen05.ld/st below are collective over the warp)
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // pass 1, once S is in: P (fp32)
      float pr[2][32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int ch = 2 * wg + h;
        uint32_t sv[32];
        tmem_ld32(tmem + lane_bits + kColS + ch * 32, sv);
        tmem_wait_ld();
        if (h == 1) {  // this warp's part of S is read: the next key tile's S may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int col = ch * 32 + e;
          pr[h][e] = (col <= jlim) ? ex2_approx(fmaf(__uint_as_float(sv[e]), c, -l2)) : 0.f;
        }
      }
      // pass 2, once dP is in: dS = P (dP - D)
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, it & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t pk[2][16];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int ch = 2 * wg + h;
        uint32_t dp[32];
        tmem_ld32(tmem + lane_bits + kColDP + ch * 32, dp);
        tmem_wait_ld();
        if (h == 1) {  // this warp's part of dP is read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dp_free);
        }
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pk[h][e / 2] = pack_bf16x2(pr[h][e] * (__uint_as_float(dp[e]) - dd),
                                     pr[h][e + 1] * (__uint_as_float(dp[e + 1]) - dd));
      }
      // the dS columns are free once dQ += dS K of the previous key tile is done
      if (it > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(ds_free, (it - 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st16(tmem + lane_bits + kColDS + (2 * wg) * 16, pk[0]);
      tmem_st16(tmem + lane_bits + kColDS + (2 * wg + 1) * 16, pk[1]);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---- epilogue: dQ = scale * acc -> bf16 row (collective TMEM loads by
    // the whole warp; only the stores depend on the lane's row)
    const bool have = __all_sync(0xffffffffu, ok && n_it > 0 && mbar_wait(done, 0, abort_flag));
    if (have) tc_fence_after();
    {
      uint16_t* dst = p.dq + (static_cast<int64_t>(bh) * p.Sq + i) * D;
#pragma unroll 1
      for (int q = wg * (D / 64); q < (wg + 1) * (D / 64); ++q) {  // this warpgroup's half of the columns
        uint32_t a[32];
        if (have) {
          tmem_ld32(tmem + lane_bits + kColDQ + q * 32, a);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) a[e] = 0u;
        }
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(a[c8 * 8 + 0]) * p.scale, __uint_as_float(a[c8 * 8 + 1]) * p.scale);
          w.y = pack_bf16x2(__uint_as_float(a[c8 * 8 + 2]) * p.scale, __uint_as_float(a[c8 * 8 + 3]) * p.scale);
          w.z = pack_bf16x2(__uint_as_float(a[c8 * 8 + 4]) * p.scale, __uint_as_float(a[c8 * 8 + 5]) * p.scale);
          w.w = pack_bf16x2(__uint_as_float(a[c8 * 8 + 6]) * p.scale, __uint_as_float(a[c8 * 8 + 7]) * p.scale);
          if (i < p.Sq) *reinterpret_cast<uint4*>(dst + q * 32 + c8 * 8) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace sdpa

// prefill.cuh -- fused attention forward (prefill) for sm_100a.
//
// O = softmax(scale * Q K^T + causal mask) V, with LSE, bf16 in / bf16 out,
// fp32 accumulation.  The loop structure is the FlashAttention-2 forward
// ("FlashAttention-2" notes, algorithm overview): each query block keeps a
// running row max m and row sum l, walks the key/value blocks, and divides by
// l once at the end; fully masked causal blocks are never visited (same
// notes, causal masking); the parallel work items are (batch, head, query
// block) (same notes, improvement 2: sequence-length parallelism).
//
// B200 mapping (this file's own design, not the pages'):
//   * Work units (batch*head, pair of 128-row query tiles) in a list that, for
//     causal masks, holds the heaviest units (the last query tiles of each
//     head) first.  One CTA fits on an SM.  Fixed lengths: a persistent grid
//     of one CTA per SM deals the list round by round in snake order, which
//     balances units of known cost like longest-processing-time-first.
//     Per-batch lengths (units whose cost is only known on the device, many
//     of them empty): the grid has one CTA per unit, and each running CTA,
//     when it has issued the loads of its unit, takes the next unit whose CTA
//     has not started by cancelling that CTA's launch (cluster launch
//     control), so the SMs pull units from the list as they free up.  Either
//     way one thread (the K/V producer) announces the CTA's units to the
//     other roles through a small ring in shared memory.  One unit's epilogue
//     overlaps the next unit's loads and first MMAs.
//   * One CTA = two query tiles sharing every K/V tile it loads; 12 warps:
//       warps 0-3  softmax group 0 (one thread per row of query tile 0)
//       warps 4-7  softmax group 1 (query tile 1)
//       warp  8    MMA issuer for query tile 0 (one elected thread) + TMEM owner
//       warp  9    TMA producer (one elected thread)
//       warp 10    MMA issuer for query tile 1
//       warp 11    bias tile loader (bias variant), else idle
//     Each query tile has its own MMA-issuing thread.  On B200 any
//     shared-memory access (an mbarrier wait included) by a thread that has
//     just issued tcgen05.mma stalls it for 120-210 cycles, while only about
//     one MMA of work is queued ahead: one issuer that waits between MMA
//     groups starves the tensor core.  With two issuers taking turns, each
//     one's waits overlap the other's MMAs.
//     The block launches at kLaunchRegs registers per thread (3 warps per SM
//     sub-partition); warpgroup 2 gives registers back (kCtrlRegs) and the
//     softmax warpgroups take them (kSoftmaxRegs) to hold a full 128-column S
//     row.  The split adds up to exactly the launch allocation:
//     256*kSoftmaxRegs + 128*kCtrlRegs == 384*kLaunchRegs.
//   * K/V arrive as 128-key tiles through an NS-slot shared-memory ring (K_j,
//     V_j in consecutive slots), 128-byte swizzled, filled by TMA, released by
//     tcgen05.commit when the MMAs reading them are done.  The ring's slot
//     sequence runs on across units.
//   * TMEM (512 columns) = S0 | S1 | O0 | O1.  P (bf16) is written over the
//     first 64 columns of its own S and read by the P.V MMA from TMEM.  The
//     two query tiles alternate on the tensor core: one tile's P.V and next S
//     run while the other tile's softmax works.
//   * Every MMA sequence is fully unrolled with compile-time descriptor
//     offsets: a 128x128x16 tcgen05.mma then issues about every 70 cycles,
//     the tensor core's own rate; a rolled loop around the issue costs more
//     than the MMA itself.
//   * Rescaling of O is skipped unless the running max grows by more than
//     2^8 in the exp2 domain (exact: the final O/l and LSE use the same m).
//   * Bias variant: warp 11 stages each (query tile, key tile) bias tile by TMA
//     into one 32 KB buffer that the two tiles' softmax steps use in turn
//     (tile 0 step j, tile 1 step j, tile 0 step j + 1, ...); the softmax
//     reads its row's 16-byte chunks at their 128-byte-swizzle positions.  The
//     buffer costs one K/V slot (4 instead of 5 at d = 128).
//   * The epilogue writes O/l from registers straight to global memory, so a
//     tile's Q buffer is free as soon as its last S MMA is done and the next
//     unit's Q can load while this unit finishes.
#pragma once
#include <climits>

#include "fastdiv.h"
#include "ptx.cuh"

namespace sdpa {

struct PrefillParams {
  // 4-D maps (d, S, H, B) over q, k, v whatever their layout (the strides
  // carry it); box {64, 128, 1, 1}, 128-byte swizzle.
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  // 4-D map (Sk, Sq, bias_h, bias_b) over the additive bias, box {64, 128, 1, 1},
  // 128-byte swizzle, zero fill outside (bias variant only)
  CUtensorMap tm_bias;
  uint16_t* o;       // bf16 bits; element (b, h, i, c) at b*o_sb + h*o_sh + i*o_sr + c
  int64_t o_sb, o_sh, o_sr;
  float* lse;        // [B*Hq*Sq] or nullptr
  const int* seqlens_q;  // [B] valid query rows of each batch (device), or nullptr: all Sq
  const int* seqlens_k;  // [B] valid keys of each batch (device), or nullptr: all Sk
  const uint16_t* bias;  // bf16 additive bias [bias_b][bias_h][Sq][Sk] (Sk % 8 == 0), or nullptr
  int64_t bias_sb, bias_sh;  // its batch and head strides in elements (0 where it broadcasts)
  int bias_per_b, bias_per_h;  // 1 where the bias has its own plane per batch / per query head
  float inv_scale;       // 1 / scale: the bias enters the raw scores as bias / scale
  int B, Hq, Hkv, Sq, Sk;
  int group;          // Hq / Hkv
  int causal;         // 0 none, 1 top-left, 2 bottom-right
  int causal_offset;  // key j visible to row i iff j <= i + causal_offset (fixed lengths)
  int num_units;      // ceil(Sq / 256): work units per (batch, head)
  int total_units;    // B * Hq * num_units
  int lpt;            // 1: heaviest units first (causal)
  int dynamic;        // 1: grid of one CTA per unit, units taken over at run time; 0: persistent snake deal
  float scale;        // softmax scale on q.k
  float scale_log2;   // scale * log2(e)
  // the same divisions by launch constants as multiply-highs (no division
  // instruction sequence at a unit boundary): by B*Hq, Hq, group, num_units
  FastDiv div_bh, div_hq, div_group, div_units;
};

constexpr int kBlockM = 128;  // query rows per tile
constexpr int kBlockN = 128;  // keys per TMA tile
constexpr int kHalfN = 64;    // keys per issue_pv call (half a tile)
constexpr int kPrefillThreads = 384;
constexpr int kMmaWarp = 8;    // query tile 0; also allocates and frees TMEM
constexpr int kLoadWarp = 9;
constexpr int kMmaWarp1 = 10;  // query tile 1
constexpr int kBiasWarp = 11;  // bias variant: loads the bias tiles
constexpr int kLaunchRegs = 168;  // 3 warps per SM sub-partition: 3*32*168 <= 16384
constexpr int kSoftmaxRegs = 216;
constexpr int kCtrlRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kCtrlRegs == kPrefillThreads * kLaunchRegs,
              "register split must equal the launch allocation");
// The bias variant's softmax holds a tile of bias besides the scores.
constexpr int kSoftmaxRegsBias = 224;
constexpr int kCtrlRegsBias = 56;
static_assert(256 * kSoftmaxRegsBias + 128 * kCtrlRegsBias == kPrefillThreads * kLaunchRegs,
              "register split must equal the launch allocation");
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest P kept unrescaled
constexpr int kUnitRing = 4;  // units announced ahead by the scheduling thread

template <int D, int NS, bool BIAS = false>
struct PrefillCfg {
  static constexpr int kTileBytes = kBlockM * D * 2;  // one Q, K or V tile (bf16)
  // bias variant: one 128-row x 128-key bf16 bias tile, staged by TMA, which
  // the two query tiles' softmax steps use in turn
  static constexpr int kBiasTileBytes = BIAS ? kBlockM * kBlockN * 2 : 0;
  static constexpr int kBlocks = D / 64;               // 64-column swizzle blocks per tile
  static constexpr int kBlockBytes = kBlockM * 128;    // 16 KB per swizzle block
  // q_full[2] q_empty[2] kv_full[NS] kv_empty[NS] s_full[2] p_full[2] o_full[2] turn[2] drain
  // unit_full[kUnitRing] unit_empty[kUnitRing] clc bias_full[2] bias_empty[2]
  static constexpr int kNumBars = 4 + 2 * NS + 2 + 2 + 2 + 2 + 1 + 2 * kUnitRing + 1 + 4;
  // after the barriers, 16-byte aligned: the cancel answer (16 bytes), the unit
  // ring (kUnitRing ints), the TMEM base and the abort flag
  static constexpr int kMiscOffset = (kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kSmemBytes =
      (2 + NS) * kTileBytes + kBiasTileBytes + kMiscOffset + 16 + 4 * kUnitRing + 8 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per block");
};

// Number of 128-key tiles the query tile starting at row0 must visit, for a
// batch with Lq valid query rows, Lk valid keys and causal offset coff.
__device__ __forceinline__ int kv_tiles_for(int causal, int Lq, int Lk, int coff, int row0) {
  if (row0 >= Lq || Lk <= 0) return 0;
  int last_key = Lk - 1;
  if (causal) {
    const int last_row = min(row0 + kBlockM - 1, Lq - 1);
    last_key = min(last_key, last_row + coff);
  }
  if (last_key < 0) return 0;
  return last_key / kBlockN + 1;
}

// The r-th work unit of CTA c in a persistent grid of G CTAs: round r deals
// list entries [r*G, r*G + G) in snake order (forward in even rounds,
// backward in odd).
__device__ __forceinline__ int unit_index(int r, int c, int G) { return r * G + ((r & 1) ? (G - 1 - c) : c); }

// Work-list entry -> (batch*head, pair index v of query tiles 2v, 2v+1).
__device__ __forceinline__ void unit_coords(const PrefillParams& p, int idx, int& bh, int& v) {
  const int BH = p.B * p.Hq;
  if (p.lpt) {
    const int r = static_cast<int>(fastdiv(static_cast<uint32_t>(idx), p.div_bh));
    v = p.num_units - 1 - r;
    bh = idx - r * BH;
  } else {
    bh = static_cast<int>(fastdiv(static_cast<uint32_t>(idx), p.div_units));
    v = idx - bh * p.num_units;
  }
}

struct Unit {
  int bh, b, hq, hkv, row0_0, n0, n1, n_max;
  int Lq, Lk, coff;  // this batch's valid query rows, valid keys, causal offset
};

// A per-batch length read from device memory, clamped to [0, cap].
__device__ __forceinline__ int batch_length(const int* lens, int b, int cap) {
  return lens == nullptr ? cap : min(max(__ldg(lens + b), 0), cap);
}

__device__ __forceinline__ Unit make_unit(const PrefillParams& p, int idx) {
  Unit u;
  int v;
  unit_coords(p, idx, u.bh, v);
  const int b = static_cast<int>(fastdiv(static_cast<uint32_t>(u.bh), p.div_hq));
  const int hq = u.bh - b * p.Hq;
  u.b = b;
  u.hq = hq;
  u.hkv = static_cast<int>(fastdiv(static_cast<uint32_t>(hq), p.div_group));
  u.row0_0 = v * 2 * kBlockM;
  u.Lq = batch_length(p.seqlens_q, b, p.Sq);
  u.Lk = batch_length(p.seqlens_k, b, p.Sk);
  u.coff = (p.seqlens_q == nullptr && p.seqlens_k == nullptr) ? p.causal_offset
                                                               : (p.causal == 2 ? u.Lk - u.Lq : 0);
  u.n0 = kv_tiles_for(p.causal, u.Lq, u.Lk, u.coff, u.row0_0);
  u.n1 = kv_tiles_for(p.causal, u.Lq, u.Lk, u.coff, u.row0_0 + kBlockM);
  u.n_max = max(u.n0, u.n1);
  return u;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// S_t = Q_t K^T: M=128, N=128, K=D in steps of 16.  Both operands K-major with
// 128-byte swizzle: step kk starts 32*(kk%4) bytes into a 128-byte row, and the
// next 64-column block is 16 KB further.  `dq`, `dk` are the tiles' base
// descriptors; the offsets are compile-time, added to the address field.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t dq, uint64_t dk) {
  constexpr uint32_t kId = idesc_bf16_f32(kBlockM, kBlockN, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kBlockM * 128 + (kk & 3) * 32) >> 4);
    mma_ss(d_tmem, dq + off, dk + off, kId, kk > 0 ? 1u : 0u);
  }
}

// O_t (+)= P_t[:, keys kb..kb+63] V[kb..kb+63, :]: M=128, N=D, K=64 in steps of
// 16 keys = 8 TMEM columns of packed bf16 P = 2048 bytes of V rows.  V is
// MN-major; its two 64-column blocks are 16 KB apart (leading byte offset in
// the base descriptor `dv`).
template <int D, int HALF>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, bool acc) {
  constexpr uint32_t kId = idesc_bf16_f32(kBlockM, D, true);
#pragma unroll
  for (int k4 = 0; k4 < kHalfN / 16; ++k4) {
    constexpr int kBase = HALF * (kHalfN / 16);
    const int kk = kBase + k4;
    const uint64_t off = static_cast<uint64_t>((kk * 2048) >> 4);
    mma_ts(o_tmem, p_tmem + kk * 8, dv + off, kId, (acc || kk > 0) ? 1u : 0u);
  }
}

// BIAS: add the additive attention bias to the scores (a separate
// instantiation, so the common path carries none of its loads).
template <int D, int NS, bool BIAS>
__global__ void __launch_bounds__(kPrefillThreads, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  using Cfg = PrefillCfg<D, NS, BIAS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Shared-memory map (32-bit shared addresses):
  //   sQ   2 query tiles, sKV NS key/value slots, (bias variant) sBias one bias
  //   tile, then the barriers.
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + 2 * Cfg::kTileBytes;
  const uint32_t sBias = sKV + NS * Cfg::kTileBytes;
  const uint32_t bar0 = sBias + Cfg::kBiasTileBytes;
  auto q_full = [&](int t) { return bar0 + 8u * t; };                   // Q_t landed
  auto q_empty = [&](int t) { return bar0 + 8u * (2 + t); };            // Q_t's last S MMA done
  auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };            // slot filled
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + NS + s); };      // slot released
  auto s_full = [&](int t) { return bar0 + 8u * (4 + 2 * NS + t); };    // S_t(j) ready
  auto p_full = [&](int t) { return bar0 + 8u * (6 + 2 * NS + t); };    // P_t(j) written
  auto o_full = [&](int t) { return bar0 + 8u * (8 + 2 * NS + t); };    // a unit's last P.V done
  auto turn = [&](int t) { return bar0 + 8u * (10 + 2 * NS + t); };     // tile t may issue
  const uint32_t drain = bar0 + 8u * (12 + 2 * NS);                     // every MMA done
  auto unit_full = [&](int k) { return bar0 + 8u * (13 + 2 * NS + k); };              // ring entry k written
  auto unit_empty = [&](int k) { return bar0 + 8u * (13 + 2 * NS + kUnitRing + k); }; // ring entry k read
  const uint32_t clc_bar = bar0 + 8u * (13 + 2 * NS + 2 * kUnitRing);                 // cancel answer landed
  auto bias_full = [&](int t) { return bar0 + 8u * (14 + 2 * NS + 2 * kUnitRing + t); };   // bias tile t landed
  auto bias_empty = [&](int t) { return bar0 + 8u * (16 + 2 * NS + 2 * kUnitRing + t); };  // bias tile t read
  uint8_t* bar_ptr = smem + 2 * Cfg::kTileBytes + NS * Cfg::kTileBytes + Cfg::kBiasTileBytes;
  uint8_t* misc = bar_ptr + Cfg::kMiscOffset;
  const uint32_t clc_resp = smem_u32(misc);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(misc + 16);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 16 + 4 * kUnitRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // The r-th unit of this CTA: wait for ring entry r, read it, release it.
  // -1 ends the sequence.  The caller's whole warp (or its lone thread) calls
  // it; one arrival per warp.
  auto next_unit = [&](int r, bool& ok) -> int {
    const int k = r % kUnitRing;
    ok = ok && mbar_wait(unit_full(k), (r / kUnitRing) & 1, abort_flag);
    if (!ok) return -1;
    const int idx = unit_ring[k];
    __syncwarp(__activemask());
    if ((threadIdx.x & 31) == 0 || __activemask() == 1u) mbar_arrive(unit_empty(k));
    return idx;
  };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(q_full(t), 1);
      mbar_init(q_empty(t), 1);
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 4);  // one arrive per softmax warp
      mbar_init(turn(t), 1);
      mbar_init(o_full(t), 1);
      mbar_init(bias_full(t), 1);
      mbar_init(bias_empty(t), 4);  // one arrive per softmax warp of tile t
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 2);  // released by both MMA threads
    }
    mbar_init(drain, 2);  // one commit per MMA thread
    for (int k = 0; k < kUnitRing; ++k) {
      mbar_init(unit_full(k), 1);
      mbar_init(unit_empty(k), 2 + 8 + (BIAS ? 1 : 0));  // MMA threads, softmax warps (bias loader)
    }
    mbar_init(clc_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    // Warpgroup 2 (control): every warp runs the same setmaxnreg first.
    regs_decrease<BIAS ? kCtrlRegsBias : kCtrlRegs>();
    if (warp == kLoadWarp) {
      // ------------------------------------------------------ TMA producer
      // Per unit: K_0, V_0 through the ring, then Q_0, Q_1 (each once the
      // previous unit's last S MMA on that buffer is done), then K_1, V_1, ...
      // Loading K_0 and V_0 first lets them land while the previous unit
      // finishes.
      if (lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        int it = 0;  // K/V tiles issued so far (ring position)
        int ui = 0;  // units started so far
        bool ok = true;
        // This thread also schedules: it announces the CTA's units in the
        // unit ring -- the persistent grid's snake deal, or (dynamic) its own
        // unit first, then each one it takes over from a CTA that has not
        // started -- and -1 when there is none left.
        int clc_asked = 0;      // cancel requests issued (clc_bar phase)
        bool clc_pending = false;
        auto announce = [&](int r, int v) -> bool {
          const int k = r % kUnitRing;
          if (r >= kUnitRing && !mbar_wait(unit_empty(k), ((r / kUnitRing) - 1) & 1, abort_flag)) return false;
          unit_ring[k] = v;
          mbar_arrive(unit_full(k));  // release: the entry is visible to whoever sees the phase
          return true;
        };
        const int cta = static_cast<int>(blockIdx.x);
        const int G = static_cast<int>(gridDim.x);
        int idx = p.dynamic ? cta : unit_index(0, cta, G);
        if (idx >= p.total_units) idx = -1;
        ok = announce(0, idx);
        // Q_0 and Q_1 of unit u, each once the previous unit's last S MMA on
        // that buffer is done (a tile with no key tiles only completes the phase).
        auto load_q = [&](const Unit& u) -> bool {
          for (int t = 0; t < 2; ++t) {
            if (ui > 0 && !mbar_wait(q_empty(t), (ui - 1) & 1, abort_flag)) return false;
            if ((t ? u.n1 : u.n0) > 0) {
              mbar_arrive_expect_tx(q_full(t), Cfg::kTileBytes);
              for (int blk = 0; blk < Cfg::kBlocks; ++blk)
                tma_load_4d(sQ + t * Cfg::kTileBytes + blk * Cfg::kBlockBytes, &p.tm_q, blk * 64,
                            u.row0_0 + t * kBlockM, u.hq, u.b, q_full(t));
            } else {
              mbar_arrive(q_full(t));
            }
          }
          return true;
        };
#pragma unroll 1
        for (int r = 0; ok && idx >= 0; ++r) {
          const Unit u = make_unit(p, idx);
          if (p.seqlens_q != nullptr || p.seqlens_k != nullptr) {
            const int b = static_cast<int>(fastdiv(static_cast<uint32_t>(u.bh), p.div_hq));
            const bool bad_q = p.seqlens_q != nullptr && __ldg(p.seqlens_q + b) != u.Lq;
            const bool bad_k = p.seqlens_k != nullptr && __ldg(p.seqlens_k + b) != u.Lk;
            if (bad_q || bad_k) atomicOr(&g_error_word, kErrSeqlen);
          }
          if (u.n_max <= 1) ok = load_q(u);
#pragma unroll 1
          for (int x = 0; ok && x < 2 * u.n_max; ++x, ++it) {  // K_0, V_0, K_1, V_1, ...
            if (x == 2 && !load_q(u)) {  // this unit's Q after its K_0, V_0
              ok = false;
              break;
            }
            const int slot = it % NS;
            if (!mbar_wait(kv_empty(slot), ((it / NS) & 1) ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(kv_full(slot), Cfg::kTileBytes);
            const CUtensorMap* tm = (x & 1) ? &p.tm_v : &p.tm_k;
            const uint32_t dst = sKV + slot * Cfg::kTileBytes;
            for (int blk = 0; blk < Cfg::kBlocks; ++blk)
              tma_load_4d(dst + blk * Cfg::kBlockBytes, tm, blk * 64, (x >> 1) * kBlockN, u.hkv, u.b,
                          kv_full(slot));
          }
          ++ui;
          if (!ok) break;
          // The next unit: the snake deal's, or (dynamic) the first one in the
          // list whose CTA has not started.
          int next = -1;
          if (!p.dynamic) {
            next = unit_index(r + 1, cta, G);
            if (next >= p.total_units) next = -1;
          } else if (clc_asked >= 0) {
            mbar_arrive_expect_tx(clc_bar, 16);
            clc_try_cancel(clc_resp, clc_bar);
            clc_pending = true;
            if (!mbar_wait(clc_bar, clc_asked & 1, abort_flag)) {
              ok = false;
              break;
            }
            clc_pending = false;
            ++clc_asked;
            next = clc_canceled_x(clc_resp);
            if (next < 0 || next >= p.total_units) {
              next = -1;
              clc_asked = -1;  // never ask again after a refusal
            }
          }
          if (!announce(r + 1, next)) {
            ok = false;
            break;
          }
          idx = next;
        }
        // An answer still on its way must land before the CTA may exit.
        if (clc_pending) mbar_wait_drain(clc_bar, clc_asked & 1);
        // Copies still in flight must land before the CTA may exit.
        if (ui > 0) {
          mbar_wait_drain(q_full(0), (ui - 1) & 1);
          mbar_wait_drain(q_full(1), (ui - 1) & 1);
        }
        for (int i = max(0, it - NS); i < it; ++i) mbar_wait_drain(kv_full(i % NS), (i / NS) & 1);
      }
      __syncwarp();
    } else if (BIAS && warp == kBiasWarp) {
      // ---------------------------------------------------- bias loader
      // The bias tile of (query tile t, key tile j) -- 128 rows x 128 keys,
      // two 64-key boxes -- into the bias buffer, in the order the softmax
      // steps use them (tile 0 step j, tile 1 step j, tile 0 step j + 1, ...),
      // each once the previous tile's softmax warps have read theirs; rows
      // and keys outside the bias read as zero (those scores are masked or
      // never written).
      if (lane == 0) {
        tma_prefetch_desc(&p.tm_bias);
        int loaded[2] = {0, 0};  // bias tiles loaded for each query tile
        int prev_t = -1;         // query tile of the previous load
        bool ok = true;
#pragma unroll 1
        for (int r = 0; ok; ++r) {
          const int idx = next_unit(r, ok);
          if (idx < 0) break;
          const Unit u = make_unit(p, idx);
          const int hb = p.bias_per_h ? u.hq : 0;
          const int bb = p.bias_per_b ? u.b : 0;
#pragma unroll 1
          for (int j = 0; ok && j < u.n_max; ++j) {
            for (int t = 0; t < 2 && ok; ++t) {
              if (j >= (t ? u.n1 : u.n0)) continue;
              if (prev_t >= 0 && !mbar_wait(bias_empty(prev_t), (loaded[prev_t] - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(bias_full(t), Cfg::kBiasTileBytes);
              const uint32_t dst = sBias;
              for (int blk = 0; blk < 2; ++blk)
                tma_load_4d(dst + blk * (kBlockM * 128), &p.tm_bias, j * kBlockN + blk * 64, u.row0_0 + t * kBlockM,
                            hb, bb, bias_full(t));
              ++loaded[t];
              prev_t = t;
            }
          }
        }
        // the last copy must land before the CTA may exit (the earlier ones
        // were all read)
        if (prev_t >= 0) mbar_wait_drain(bias_full(prev_t), (loaded[prev_t] - 1) & 1);
      }
      __syncwarp();
    } else if (warp == kMmaWarp || warp == kMmaWarp1) {
      // ---------------------------------------------- MMA issuer of tile t
      // Segment k of tile t in a unit is O_t += P_t(k-1) V_{k-1} (k >= 1)
      // followed by S_t(k) = Q_t K_k^T (k < n_t): 16 MMAs, issued back to back
      // once everything they read is ready.  The two issuers take turns (tile
      // 0 segment k, tile 1 segment k, tile 0 segment k+1, ...) through the
      // turn barriers, so the tensor core runs one tile's segment at a time --
      // a tile's softmax waits for its own segment only -- while the other
      // issuer's waits (for its P, its K/V slot, its turn) overlap the MMAs in
      // flight.  Both issuers walk all n_max + 1 segments of every unit and
      // release every K/V slot once, so kv_empty and turn see one arrival per
      // phase from each.
      const int t = (warp == kMmaWarp) ? 0 : 1;
      if (lane == 0) {
        const uint64_t hi = static_cast<uint64_t>(sdesc_hi(1024)) << 32;  // 8-row groups 1024 B apart
        const uint64_t dq = hi | sdesc_lo(sQ + t * Cfg::kTileBytes, 16);
        auto dk = [&](int slot) { return hi | sdesc_lo(sKV + slot * Cfg::kTileBytes, 16); };
        auto dv = [&](int slot) { return hi | sdesc_lo(sKV + slot * Cfg::kTileBytes, Cfg::kBlockBytes); };
        const uint32_t tS = tmem + t * kBlockN;
        const uint32_t tO = tmem + 2 * kBlockN + t * D;
        int it_base = 0;  // ring position of the unit's K_0
        int seg = 0;      // segments walked (the same count on both issuers)
        int pj = 0;       // P_t tiles consumed (p_full phase)
        int ui = 0;       // units walked (q_full phase)
        bool ok = true;
#pragma unroll 1
        for (int r = 0; ok; ++r) {
          const int idx = next_unit(r, ok);
          if (idx < 0) break;
          const Unit u = make_unit(p, idx);
          const int nt = t ? u.n1 : u.n0;  // n0 <= n1: tile 1's rows come later
          if (!mbar_wait(q_full(t), ui & 1, abort_flag)) break;
          if (nt == 0) mma_commit(q_empty(t));  // nothing reads Q_t in this unit
#pragma unroll 1
          for (int k = 0; k <= u.n_max; ++k, ++seg) {
            int slot_v = -1, slot_k = -1;
            if (k >= 1) {
              const int itv = it_base + 2 * k - 1;  // V_{k-1}
              slot_v = itv % NS;
              if (!mbar_wait(kv_full(slot_v), (itv / NS) & 1, abort_flag)) {
                ok = false;
                break;
              }
              if (k - 1 < nt && !mbar_wait(p_full(t), pj & 1, abort_flag)) {
                ok = false;
                break;
              }
            }
            if (k < u.n_max) {
              const int itk = it_base + 2 * k;  // K_k
              slot_k = itk % NS;
              if (!mbar_wait(kv_full(slot_k), (itk / NS) & 1, abort_flag)) {
                ok = false;
                break;
              }
            }
            if (t == 1) {
              if (!mbar_wait(turn(1), seg & 1, abort_flag)) {
                ok = false;
                break;
              }
            } else if (seg >= 1) {
              if (!mbar_wait(turn(0), (seg - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
            }
            tc_fence_after();
            if (k >= 1 && k - 1 < nt) {
              const uint64_t v_desc = dv(slot_v);
              issue_pv<D, 0>(tO, tS, v_desc, k > 1);
              issue_pv<D, 1>(tO, tS, v_desc, true);
              ++pj;
              if (k == nt) mma_commit(o_full(t));
            }
            if (k < nt) {
              issue_qk<D>(tS, dq, dk(slot_k));
              mma_commit(s_full(t));
              if (k == nt - 1) mma_commit(q_empty(t));
            }
            if (slot_v >= 0) mma_commit(kv_empty(slot_v));
            if (slot_k >= 0) mma_commit(kv_empty(slot_k));
            mbar_arrive(turn(1 - t));
          }
          it_base += 2 * u.n_max;
          ++ui;
        }
        // Every MMA this thread issued must finish before TMEM is released.
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
      __syncwarp();
    }
  } else {
    // Warpgroups 0 and 1: softmax / epilogue for query tile 0 and 1.
    regs_increase<BIAS ? kSoftmaxRegsBias : kSoftmaxRegs>();
    const int t = warp >> 2;      // query tile 0 or 1
    const int wq = warp & 3;      // TMEM lane quarter of this warp
    const int r_in_tile = wq * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_bits + t * kBlockN;
    const uint32_t tO = tmem + lane_bits + 2 * kBlockN + t * D;
    const float c = p.scale_log2;
    int sj = 0;  // S_t tiles consumed (s_full phase)
    int ou = 0;  // units whose O_t was read (o_full phase)
    bool ok = true;
#pragma unroll 1
    for (int r = 0; ok; ++r) {
      const int idx = next_unit(r, ok);  // warp-uniform
      if (idx < 0) break;
      const Unit u = make_unit(p, idx);
      const int row0 = u.row0_0 + t * kBlockM;
      const int row = row0 + r_in_tile;
      const int n = t ? u.n1 : u.n0;
      const int row_limit = p.causal ? row + u.coff : INT_MAX - kBlockN;
      float m_used = -INFINITY;
      float l = 0.f;

#pragma unroll 1
      for (int j = 0; j < n; ++j, ++sj) {
        if (!mbar_wait(s_full(t), sj & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[128];
        if constexpr (!BIAS) {
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld32(tS + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[q * 32]));
          tmem_wait_ld();
        } else {
          // S in two 64-column halves, each given its bias from the staged
          // bias tile: this thread's row, 16-byte chunks of 8 keys at the
          // 128-byte swizzle's position (chunk c of row r at c ^ (r mod 8)).
          const float2 is2 = make_float2(p.inv_scale, p.inv_scale);
          if (!mbar_wait(bias_full(t), sj & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t brow = sBias + static_cast<uint32_t>(r_in_tile) * 128u;
          const uint32_t bsw = static_cast<uint32_t>(r_in_tile & 7);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tmem_ld32(tS + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[half * 64]));
            tmem_ld32(tS + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[half * 64 + 32]));
            tmem_wait_ld();
#pragma unroll
            for (int c8 = half * 8; c8 < half * 8 + 8; ++c8) {
              const uint4 bz = ld_shared_u4(brow + half * (kBlockM * 128) + ((static_cast<uint32_t>(c8 & 7) ^ bsw) << 4));
              const uint32_t w[4] = {bz.x, bz.y, bz.z, bz.w};
#pragma unroll
              for (int u2 = 0; u2 < 4; ++u2) {
                const int e = c8 * 8 + u2 * 2;
                const float2 bb = make_float2(__uint_as_float(w[u2] << 16), __uint_as_float(w[u2] & 0xFFFF0000u));
                const float2 r =
                    __ffma2_rn(bb, is2, make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])));
                sv[e] = __float_as_uint(r.x);
                sv[e + 1] = __float_as_uint(r.y);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bias_empty(t));  // this warp's rows of the bias tile are read
        }
        const int k0 = j * kBlockN;
        const bool need_mask = (k0 + kBlockN > u.Lk) || (p.causal && k0 + kBlockN - 1 > row0 + u.coff);
        if (need_mask) {
          const int lim = min(u.Lk - 1, row_limit) - k0;  // last visible column
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > lim) sv[e] = __float_as_uint(-INFINITY);
        }
        // row max over the 128 scores: four independent chains of 3-input max
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          mx0 = max3f(mx0, __uint_as_float(sv[e + 0]), __uint_as_float(sv[e + 1]));
          mx1 = max3f(mx1, __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
          mx2 = max3f(mx2, __uint_as_float(sv[e + 4]), __uint_as_float(sv[e + 5]));
          mx3 = max3f(mx3, __uint_as_float(sv[e + 6]), __uint_as_float(sv[e + 7]));
        }
        const float m_new = max3f(m_used, max3f(mx0, mx1, mx2), mx3);
        // (m_new - m_used) is NaN while both are -inf: no rescale then.
        const bool rescale = (m_new - m_used) * c > kRescaleThreshold;
        float alpha = 1.f;
        if (rescale) {
          alpha = ex2_approx((m_used - m_new) * c);
          m_used = m_new;
          l *= alpha;
        }
        // O holds P.V of this unit's earlier tiles; the S wait above implies
        // they are done (S_t(j) is issued after P_t(j-1).V by the same thread).
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll 1
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + q * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 rr = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
              o[e] = __float_as_uint(rr.x);
              o[e + 1] = __float_as_uint(rr.y);
            }
            tmem_st32(tO + q * 32, o);
          }
        }
        const float mc = (m_used == -INFINITY) ? 0.f : m_used * c;
        const float2 c2 = make_float2(c, c);
        const float2 nmc2 = make_float2(-mc, -mc);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 64; e += 4) {
            const int i = half * 64 + e;
            const float2 x0 = __ffma2_rn(make_float2(__uint_as_float(sv[i]), __uint_as_float(sv[i + 1])), c2, nmc2);
            const float2 x1 =
                __ffma2_rn(make_float2(__uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3])), c2, nmc2);
            const float2 p0 = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
            const float2 p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
            acc0 = __fadd2_rn(acc0, p0);
            acc1 = __fadd2_rn(acc1, p1);
            pk[e / 2] = pack_bf16x2(p0.x, p0.y);
            pk[e / 2 + 1] = pack_bf16x2(p1.x, p1.y);
          }
          tmem_st32(tS + half * 32, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(t));
        l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
      }
      if (!ok) break;

      // ---- epilogue: O / l -> bf16 -> global.  Each thread normalises its own
      // row; then, per 64 columns, a transpose of row chunks between the lanes
      // of a small group (xor shuffles) makes every store instruction write
      // whole 128-byte row segments instead of 32 scattered pieces.  The
      // epilogue sits on the tile's path from one unit to the next, so its
      // cost counts once per unit (about 10 % of a causal seq-2048 unit).
      if (row0 < u.Lq) {
        if (n > 0) {
          if (!mbar_wait(o_full(t), ou & 1, abort_flag)) ok = false;
          ++ou;
        }
        tc_fence_after();
        // A row whose running max is still -inf saw no visible key: O = 0 and
        // LSE = -inf.
        const bool empty_row = (m_used == -INFINITY) || !(l > 0.f);
        const float inv_l = empty_row ? 0.f : 1.f / l;
        const bool have_o = __all_sync(0xffffffffu, ok && n > 0);  // collective loads: warp-uniform
        const int g = lane & 7;
        const int group_row0 = row0 + wq * 32 + (lane & ~7);  // first row of this lane's group of 8
        uint16_t* const o_head = p.o + u.b * p.o_sb + u.hq * p.o_sh;
        if ((reinterpret_cast<uintptr_t>(p.o) & 31u) == 0u) {
          // 32-byte aligned rows.  Per 64 columns (128 bytes of a row = four
          // 32-byte chunks), a 4 x 4 transpose of chunks inside each group of
          // 4 lanes (xor shuffles), after which every 32-byte store of the warp
          // writes eight whole 128-byte row segments.
          const int g4 = lane & 3;
          const int grp_row0 = row0 + wq * 32 + (lane & ~3);
          const float2 il2 = make_float2(inv_l, inv_l);
#pragma unroll 1
          for (int h = 0; h < D / 64; ++h) {
            uint32_t o0[32], o1[32];
            if (have_o) {
              tmem_ld32(tO + h * 64, o0);
              tmem_ld32(tO + h * 64 + 32, o1);
              tmem_wait_ld();
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) o0[e] = o1[e] = 0u;
            }
            uint32_t w[4][8];  // chunk c = columns 64 h + 16 c .. + 15 of this lane's row
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint32_t* f = (c < 2) ? &o0[c * 16] : &o1[(c - 2) * 16];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float2 x = __fmul2_rn(make_float2(__uint_as_float(f[2 * e]), __uint_as_float(f[2 * e + 1])), il2);
                w[c][e] = pack_bf16x2(x.x, x.y);
              }
            }
#pragma unroll
            for (int sft = 2; sft > 0; sft >>= 1) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                if (i & sft) continue;
                const int jj = i | sft;
                const bool upper = (g4 & sft) != 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const uint32_t x = upper ? w[i][e] : w[jj][e];
                  const uint32_t y = __shfl_xor_sync(0xffffffffu, x, sft);
                  if (upper) {
                    w[i][e] = y;
                  } else {
                    w[jj][e] = y;
                  }
                }
              }
            }
            // lane g4 now holds chunk g4 of rows grp_row0 + 0..3 in w[0..3]
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rr = grp_row0 + i;
              if (rr < u.Lq) st_global_v8(o_head + static_cast<int64_t>(rr) * p.o_sr + h * 64 + g4 * 16, w[i]);
            }
          }
        } else
#pragma unroll 1
        for (int h = 0; h < D / 64; ++h) {
          uint32_t o0[32], o1[32];
          if (have_o) {
            tmem_ld32(tO + h * 64, o0);
            tmem_ld32(tO + h * 64 + 32, o1);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o0[e] = o1[e] = 0u;
          }
          uint4 v[8];  // chunk c = columns 64 h + 8 c .. + 7 of this lane's row
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* f = (c < 4) ? &o0[c * 8] : &o1[(c - 4) * 8];
            v[c].x = pack_bf16x2(__uint_as_float(f[0]) * inv_l, __uint_as_float(f[1]) * inv_l);
            v[c].y = pack_bf16x2(__uint_as_float(f[2]) * inv_l, __uint_as_float(f[3]) * inv_l);
            v[c].z = pack_bf16x2(__uint_as_float(f[4]) * inv_l, __uint_as_float(f[5]) * inv_l);
            v[c].w = pack_bf16x2(__uint_as_float(f[6]) * inv_l, __uint_as_float(f[7]) * inv_l);
          }
          // butterfly: after it, lane g of a group holds chunk g of the
          // group's rows 0..7 in v[0..7]
#pragma unroll
          for (int sft = 4; sft > 0; sft >>= 1) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (i & sft) continue;
              const int jj = i | sft;
              const bool upper = (g & sft) != 0;
              const uint4 x = upper ? v[i] : v[jj];
              uint4 y;
              y.x = __shfl_xor_sync(0xffffffffu, x.x, sft);
              y.y = __shfl_xor_sync(0xffffffffu, x.y, sft);
              y.z = __shfl_xor_sync(0xffffffffu, x.z, sft);
              y.w = __shfl_xor_sync(0xffffffffu, x.w, sft);
              if (upper) {
                v[i] = y;
              } else {
                v[jj] = y;
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = group_row0 + i;
            if (rr < u.Lq) *reinterpret_cast<uint4*>(o_head + rr * p.o_sr + h * 64 + g * 8) = v[i];
          }
        }
        if (p.lse != nullptr && row < u.Lq) {
          const float lse = empty_row ? -INFINITY : (m_used * p.scale + lg2_approx(l) * 0.69314718055994531f);
          p.lse[static_cast<int64_t>(u.bh) * p.Sq + row] = lse;
        }
        // O_t may be overwritten by the next unit's first P.V only after every
        // warp of this group has read it: that P.V waits for this group's P of
        // the next unit, which each warp writes after its own reads here.
        tc_fence_before();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sdpa

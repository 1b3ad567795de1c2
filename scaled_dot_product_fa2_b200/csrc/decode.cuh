// decode.cuh -- split-KV decode attention and the log-sum-exp combine.
//
// The method is the fused decode of "[onnxruntime] WebGPU FlashAttention:
// kernel fusion and variable sequence length", section 1: one kernel computes,
// per KV split, Q K^T, the causal mask, a local softmax and the product with
// V, and writes a LOCALLY normalised partial output plus (local max, local
// sum) metadata; a second, reduce kernel rescales the partials with that
// metadata so the result equals full softmax(Q K^T) V.  Section 2 of the
// same page amortises one K/V load over several query rows (m_tile); here a
// CTA serves every query row that shares its KV head (G = Hq/Hkv heads times
// Sq rows, up to 16 per CTA).
//
// B200 mapping (this file's own design):
//   * grid = (kv head, slot, row group); 4 consumer warps + 1 TMA producer
//     warp; K/V tiles of 64 keys stream through an NSTAGE-deep ring of
//     128-byte-swizzled shared-memory tiles.
//   * A KV head has B * nsplit slots (CTAs).  With one cache length every
//     batch takes nsplit of them; with per-batch lengths (several splits, at
//     most kDealMaxBatch batches) the slots are dealt in proportion to each
//     batch's tiles (assign_slot), so a mix of long and short caches keeps
//     every CTA's share of the keys about equal.
//   * The work per byte is tiny (<= 16 query rows), so the contraction runs on
//     warp-level mma.sync m16n8k16 (bf16, fp32 accumulate): the kernel is
//     bound by HBM bandwidth, not by the tensor pipe.  Each warp owns 16 keys
//     of every tile and its own running (m, l, O); the four warps merge once
//     through shared memory at the end.
//   * The combine kernel is one warp per output row with 16-byte coalesced
//     loads of the fp32 partials, the (max, sum) pairs loaded with the first
//     eight partial rows; it is a programmatic dependent of the split kernel.
#pragma once
#include "ptx.cuh"

namespace sdpa {

struct DecodeParams {
  CUtensorMap tm_k;       // [B*Hkv][Sk][d] bf16, box {64, 64, 1}, 128-byte swizzle
  CUtensorMap tm_v;       // [B*Hkv][Sk][d]
  const uint16_t* q;      // bf16 bits; element (b, h, i, c) at b*q_sb + h*q_sh + i*q_sr + c
  int64_t q_sb, q_sh, q_sr;
  const int* seqlens_k;   // [B] valid keys of each batch's cache (device), or nullptr: all Sk
  const uint16_t* bias;   // bf16 additive bias [bias_b][bias_h][Sq][Sk], or nullptr
  int64_t bias_sb, bias_sh;  // its batch and head strides in elements (0 where it broadcasts)
  float inv_scale;        // 1 / scale: the bias enters the raw scores as bias / scale
  float* part_o;          // [Hkv][B*nsplit slots][G*Sq rows][d]  locally normalised partial outputs
  float2* part_ml;        // [Hkv][B*nsplit slots][G*Sq rows]     (local max of scale*q.k, local sum)
  int B, Hq, Hkv, Sq, Sk, group;
  int causal;             // 0 none, 1 top-left, 2 bottom-right
  int causal_offset;      // key j visible to row i iff j <= i + causal_offset (if causal; fixed-length caches)
  int nsplit;             // splits per (batch, kv head)
  int tiles_per_split;    // 64-key tiles per split
  int row_groups;         // ceil(group*Sq / 16)
  float scale, scale_log2;
  int withhold_loads;     // self-test only: the producer issues no copy, so every consumer
                          // wait runs out and the kernel exits through its timeout path
};

constexpr int kDecKeys = 64;          // keys per tile
constexpr int kDecRows = 16;          // query rows per CTA (mma M)
constexpr int kDecThreads = 160;      // 4 consumer warps + 1 producer warp
constexpr int kDecProducerWarp = 4;

template <int D, int NSTAGE>
struct DecodeCfg {
  static constexpr int kBoxBytes = kDecKeys * 128;         // one 64-key x 64-col swizzle block
  static constexpr int kHalfBytes = kBoxBytes * (D / 64);  // K or V tile
  static constexpr int kStageBytes = 2 * kHalfBytes;
  static constexpr int kMergeBytes = 4 * kDecRows * D * 4 + 2 * 4 * kDecRows * 4;
  static constexpr int kRingBytes = NSTAGE * kStageBytes > kMergeBytes ? NSTAGE * kStageBytes : kMergeBytes;
  static constexpr int kSmemBytes = kRingBytes + 2 * NSTAGE * 8 + 16 + 1024;
};

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of element (key r, column c) inside a 128-byte-swizzled tile of
// 64-column blocks with `rows` rows per block (16-byte chunk granularity).
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int block_bytes) {
  return (c >> 6) * block_bytes + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// Slot deal for per-batch key lengths.  A KV head has `slots` CTAs
// (B * nsplit).  Batch b has T_b = ceil(len_b / 64) tiles; the per-CTA quota
// q is the smallest number of tiles for which sum_b max(1, ceil(T_b / q))
// slots suffice, and batch b takes n_b = max(1, ceil(T_b / q)) consecutive
// slots, its k-th slot streaming tiles [k q, min(T_b, (k + 1) q)).  So the
// longest CTA does as little as whole tiles allow, whatever the length mix;
// an empty batch still gets one slot (it writes o = 0, lse = -inf).  The
// split kernel (slot -> batch) and the combine (batch -> slots) both derive
// the deal from the lengths; every lane of the calling warp gets the same
// answer.
__device__ __forceinline__ int len_tiles(const int* __restrict__ seqlens, int bb, int B, int Sk) {
  return bb < B ? (min(max(__ldg(seqlens + bb), 0), Sk) + kDecKeys - 1) / kDecKeys : 0;
}

// The deal holds the tile counts of up to kDealMaxBatch batches in registers
// (kDealChunks per lane); with more batches, or one split, each batch keeps
// nsplit CTAs and its tiles are spread evenly over them.
constexpr int kDealChunks = 4;
constexpr int kDealMaxBatch = 32 * kDealChunks;

__device__ __forceinline__ bool use_deal(int B, int nsplit) { return nsplit > 1 && B <= kDealMaxBatch; }

// Inclusive prefix sum over the warp.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += u;
  }
  return v;
}

// Tile counts of batches c*32 + lane, c < kDealChunks (0 beyond B).
struct DealTiles {
  int t[kDealChunks];
};

__device__ __forceinline__ int slot_quota(const int* __restrict__ seqlens, int B, int Sk, int slots, int lane,
                                          DealTiles& dt) {
  int64_t tot = 0;
  int mx = 0;
#pragma unroll
  for (int c = 0; c < kDealChunks; ++c) {
    dt.t[c] = len_tiles(seqlens, c * 32 + lane, B, Sk);
    tot += dt.t[c];
    mx = max(mx, dt.t[c]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  // For q >= ceil(tot / slots) the slot count is at most B + slots < 2^32.
  auto fits = [&](int q) {
    unsigned n = 0;
#pragma unroll
    for (int c = 0; c < kDealChunks; ++c)
      if (c * 32 + lane < B) n += static_cast<unsigned>(max(1, (dt.t[c] + q - 1) / q));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    return n <= static_cast<unsigned>(slots);
  };
  // No q below ceil(tot / slots) fits; q = max T_b always does (B <= slots),
  // and so does ceil(tot / (slots - B)), since max(1, ceil(T_b / q)) <= T_b / q + 1.
  // Equal lengths fit at the lower bound: it is tried first.
  const int64_t lo0 = (tot + slots - 1) / slots;
  int lo = lo0 > 1 ? static_cast<int>(lo0) : 1;
  int hi = max(1, mx);
  if (slots > B) hi = min(hi, max(lo, static_cast<int>((tot + (slots - B) - 1) / (slots - B))));
  if (lo < hi && fits(lo)) hi = lo;
  else if (lo < hi) ++lo;
  while (lo < hi) {
    const int mid = lo + ((hi - lo) >> 1);
    if (fits(mid)) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

struct SlotAssign {
  int b, k, quota;  // b = -1: a slot that no batch needs
};

// Requires use_deal(B, nsplit).
__device__ __forceinline__ SlotAssign assign_slot(const int* __restrict__ seqlens, int B, int Sk, int slots, int j,
                                                  int lane) {
  DealTiles dt;
  const int q = slot_quota(seqlens, B, Sk, slots, lane, dt);
  int start = 0;
#pragma unroll
  for (int c = 0; c < kDealChunks; ++c) {
    const int n = (c * 32 + lane < B) ? max(1, (dt.t[c] + q - 1) / q) : 0;
    const int incl = warp_incl_scan(n, lane);
    const int excl = incl - n;
    const unsigned hit = __ballot_sync(0xffffffffu, n > 0 && j >= start + excl && j < start + incl);
    if (hit != 0u) {
      const int src = __ffs(hit) - 1;
      return {c * 32 + src, j - start - __shfl_sync(0xffffffffu, excl, src), q};
    }
    start += __shfl_sync(0xffffffffu, incl, 31);
  }
  return {-1, 0, q};
}

// (first slot, slot count) of batch b.  Requires use_deal(B, nsplit).
__device__ __forceinline__ int2 batch_slots(const int* __restrict__ seqlens, int B, int Sk, int slots, int b,
                                            int lane) {
  DealTiles dt;
  const int q = slot_quota(seqlens, B, Sk, slots, lane, dt);
  int start = 0;
#pragma unroll
  for (int c = 0; c < kDealChunks; ++c) {
    const int n = (c * 32 + lane < B) ? max(1, (dt.t[c] + q - 1) / q) : 0;
    const int incl = warp_incl_scan(n, lane);
    if (b < c * 32 + 32) {
      const int src = b - c * 32;
      return make_int2(start + __shfl_sync(0xffffffffu, incl - n, src), __shfl_sync(0xffffffffu, n, src));
    }
    start += __shfl_sync(0xffffffffu, incl, 31);
  }
  return make_int2(0, 0);
}

template <int D, int NSTAGE>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using Cfg = DecodeCfg<D, NSTAGE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = smem_u32(smem);
  const uint32_t bar0 = ring + Cfg::kRingBytes;
  auto full = [&](int s) { return bar0 + 8u * s; };             // [NSTAGE] stage filled
  auto empty = [&](int s) { return bar0 + 8u * (NSTAGE + s); }; // [NSTAGE] stage released
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kRingBytes + 16 * NSTAGE);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Shared-memory set-up and the tensor-map prefetch touch no global memory
  // that an earlier kernel writes, so they run before the dependency wait.
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 4);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kDecProducerWarp && lane == 0) {
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  __syncthreads();  // the barriers are initialised; no CTA-wide barrier follows the length deal
  // Launched as a programmatic dependent of the previous kernel in the
  // stream (the previous call's combine, in a decode loop): this grid's CTAs
  // may be resident before that kernel ends, and wait here, before any global
  // memory access, for its completion and the visibility of its writes.
  grid_dependency_wait();

  // blockIdx.x = (kv head * slots + slot) * row_groups + row group
  const int slots = p.B * p.nsplit;  // CTAs per (kv head, row group)
  const int rg = static_cast<int>(blockIdx.x) % p.row_groups;
  const int j = (static_cast<int>(blockIdx.x) / p.row_groups) % slots;
  const int hkv = static_cast<int>(blockIdx.x) / (p.row_groups * slots);
  const int rows_total = p.group * p.Sq;  // query rows sharing this KV head
  // Batch of this slot, its index among the batch's slots and the tiles it
  // streams.  One cache length: nsplit slots per batch.  Per-batch lengths
  // (read here, on the device, so the grid never depends on them): slots are
  // dealt to batches in proportion to their tiles, and the mask is aligned to
  // each batch's own length.
  int b, k_in_batch, tile_begin, tile_end;
  int L = p.Sk;
  int coff = p.causal_offset;
  if (p.seqlens_k == nullptr) {
    b = j / p.nsplit;
    k_in_batch = j - b * p.nsplit;
    tile_begin = k_in_batch * p.tiles_per_split;
    tile_end = min((L + kDecKeys - 1) / kDecKeys, tile_begin + p.tiles_per_split);
  } else {
    int quota;
    if (use_deal(p.B, p.nsplit)) {
      const SlotAssign a = assign_slot(p.seqlens_k, p.B, p.Sk, slots, j, lane);
      if (a.b < 0) return;  // a slot no batch needs (every thread of the CTA leaves here)
      b = a.b;
      k_in_batch = a.k;
      quota = a.quota;
    } else {
      b = j / p.nsplit;
      k_in_batch = j - b * p.nsplit;
      quota = -1;
    }
    const int raw = __ldg(p.seqlens_k + b);
    L = min(max(raw, 0), p.Sk);
    if (raw != L && k_in_batch == 0 && rg == 0 && hkv == 0 && threadIdx.x == 0) atomicOr(&g_error_word, kErrSeqlen);
    const int tiles = (L + kDecKeys - 1) / kDecKeys;
    if (quota < 0) quota = (tiles + p.nsplit - 1) / p.nsplit;
    tile_begin = k_in_batch * quota;
    tile_end = min(tiles, tile_begin + quota);
    coff = (p.causal == 2) ? L - p.Sq : 0;
  }
  const int ntiles = max(0, tile_end - tile_begin);
  const int bhkv = b * p.Hkv + hkv;  // K/V head row of the tensor maps

  // Let the combine kernel (a programmatic dependent launch) be scheduled
  // as soon as every CTA of this grid has started; it waits for this grid's
  // completion before it reads anything.
  grid_dependency_trigger();

  if (warp == kDecProducerWarp) {
    if (lane == 0 && ntiles > 0 && !p.withhold_loads) {
      int issued = 0;
      for (int it = 0; it < ntiles; ++it) {
        const int st = it % NSTAGE;
        if (!mbar_wait(empty(st), ((it / NSTAGE) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(full(st), Cfg::kStageBytes);
        const uint32_t sk = ring + st * Cfg::kStageBytes;
        const uint32_t sv = sk + Cfg::kHalfBytes;
        const int key0 = (tile_begin + it) * kDecKeys;
#pragma unroll
        for (int blk = 0; blk < D / 64; ++blk) {
          tma_load_3d(sk + blk * Cfg::kBoxBytes, &p.tm_k, blk * 64, key0, bhkv, full(st));
          tma_load_3d(sv + blk * Cfg::kBoxBytes, &p.tm_v, blk * 64, key0, bhkv, full(st));
        }
        ++issued;
      }
      for (int it = max(0, issued - NSTAGE); it < issued; ++it) mbar_wait_drain(full(it % NSTAGE), (it / NSTAGE) & 1);
    }
    __syncwarp();
    named_bar_sync(1, kDecThreads);  // matches the consumers' barrier before the merge
    named_bar_sync(1, kDecThreads);  // matches the consumers' barrier after the merge writes
    return;
  }

  // ------------------------------------------------------------ consumers
  const float c = p.scale_log2;
  const int qr = lane >> 2;        // fragment row (and row + 8)
  const int qc = (lane & 3) * 2;   // fragment column pair
  // Query rows of this CTA: r in [0,16) -> local row rg*16 + r of this KV head.
  uint32_t qf[D / 16][4];
  {
    const int r_lo = rg * kDecRows + qr;
    const int r_hi = r_lo + 8;
    const bool v_lo = r_lo < rows_total, v_hi = r_hi < rows_total;
    // local row g*Sq + i of this KV head -> query head hkv*group + g, row i
    auto q_row = [&](int lr) {
      const int g = lr / p.Sq;
      return reinterpret_cast<const uint32_t*>(p.q + b * p.q_sb + (hkv * p.group + g) * p.q_sh +
                                               (lr - g * p.Sq) * p.q_sr);
    };
    const uint32_t* q_lo = q_row(v_lo ? r_lo : 0);
    const uint32_t* q_hi = q_row(v_hi ? r_hi : 0);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qf[ks][0] = v_lo ? q_lo[(ks * 16 + qc) >> 1] : 0u;
      qf[ks][1] = v_hi ? q_hi[(ks * 16 + qc) >> 1] : 0u;
      qf[ks][2] = v_lo ? q_lo[(ks * 16 + 8 + qc) >> 1] : 0u;
      qf[ks][3] = v_hi ? q_hi[(ks * 16 + 8 + qc) >> 1] : 0u;
    }
  }
  // causal limit per fragment row: the last key each row may see; and the
  // row of the bias (if any) that belongs to it
  int lim[2];
  const uint16_t* brow[2] = {nullptr, nullptr};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int lr = rg * kDecRows + qr + 8 * h;  // local row = g*Sq + i
    const int i = lr % p.Sq;
    lim[h] = p.causal ? min(L - 1, i + coff) : L - 1;
    if (p.bias != nullptr && lr < rows_total) {
      const int hq = hkv * p.group + lr / p.Sq;
      brow[h] = p.bias + b * p.bias_sb + hq * p.bias_sh + static_cast<int64_t>(i) * p.Sk;
    }
  }

  float o[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};
  float l[2] = {0.f, 0.f};
  bool ok = true;

  for (int it = 0; it < ntiles; ++it) {
    const int st = it % NSTAGE;
    // warp-uniform: a lane that gave up must not leave its warp's mma.sync
    if (!__all_sync(0xffffffffu, mbar_wait(full(st), (it / NSTAGE) & 1, abort_flag))) {
      ok = false;
      break;
    }
    const uint32_t sk = ring + st * Cfg::kStageBytes;
    const uint32_t sv = sk + Cfg::kHalfBytes;
    const int kb = warp * 16;  // this warp's 16 keys inside the tile
    // ---- S = Q K^T for 16 rows x 16 keys
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mi = lane >> 3;
      const int key = kb + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(sk + sw128_off(key, ks * 16 + (mi & 1) * 8, Cfg::kBoxBytes), b0, b1, b2, b3);
        mma_bf16_16816(sc[0], qf[ks], b0, b1);
        mma_bf16_16816(sc[1], qf[ks], b2, b3);
      }
    }
    // ---- bias, mask, online softmax (rows qr and qr+8 of this thread)
    const int key0 = (tile_begin + it) * kDecKeys + kb;
    if (p.bias != nullptr) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int key = key0 + nt * 8 + qc;  // this thread's keys key, key + 1
          if (brow[h] != nullptr) {
            if (key < p.Sk) sc[nt][2 * h] += bf16_bits_to_float(__ldg(brow[h] + key)) * p.inv_scale;
            if (key + 1 < p.Sk) sc[nt][2 * h + 1] += bf16_bits_to_float(__ldg(brow[h] + key + 1)) * p.inv_scale;
          }
        }
    }
    if (key0 + 15 > min(lim[0], lim[1])) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + nt * 8 + qc + (e & 1);
          if (key > lim[e >> 1]) sc[nt][e] = -INFINITY;
        }
    }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = fmaxf(fmaxf(sc[0][2 * h], sc[0][2 * h + 1]), fmaxf(sc[1][2 * h], sc[1][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m[h], mx);
      alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2_approx((m[h] - m_new) * c);
      m[h] = m_new;
    }
    uint32_t pa[4];
    {
      const float mc0 = (m[0] == -INFINITY) ? 0.f : m[0] * c;
      const float mc1 = (m[1] == -INFINITY) ? 0.f : m[1] * c;
      float p00 = ex2_approx(fmaf(sc[0][0], c, -mc0)), p01 = ex2_approx(fmaf(sc[0][1], c, -mc0));
      float p02 = ex2_approx(fmaf(sc[0][2], c, -mc1)), p03 = ex2_approx(fmaf(sc[0][3], c, -mc1));
      float p10 = ex2_approx(fmaf(sc[1][0], c, -mc0)), p11 = ex2_approx(fmaf(sc[1][1], c, -mc0));
      float p12 = ex2_approx(fmaf(sc[1][2], c, -mc1)), p13 = ex2_approx(fmaf(sc[1][3], c, -mc1));
      l[0] = l[0] * alpha[0] + (p00 + p01 + p10 + p11);
      l[1] = l[1] * alpha[1] + (p02 + p03 + p12 + p13);
      pa[0] = pack_bf16x2(p00, p01);
      pa[1] = pack_bf16x2(p02, p03);
      pa[2] = pack_bf16x2(p10, p11);
      pa[3] = pack_bf16x2(p12, p13);
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // ---- O += P V  (V^T fragments through ldmatrix.trans)
    {
      const int mi = lane >> 3;
      const int key = kb + (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int n = 0; n < D / 8; n += 2) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(sv + sw128_off(key, (n + (mi >> 1)) * 8, Cfg::kBoxBytes), b0, b1, b2, b3);
        mma_bf16_16816(o[n], pa, b0, b1);
        mma_bf16_16816(o[n + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(st));
  }

  // ---- merge the four warps' (m, l, O) through shared memory
  // (quad-reduce l first: each thread summed only its own columns)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
    l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
  }
  named_bar_sync(1, kDecThreads);  // every warp is past the ring: reuse it for the merge
  float* s_o = reinterpret_cast<float*>(smem);          // [4][16][D]
  float* s_m = s_o + 4 * kDecRows * D;                   // [4][16]
  float* s_l = s_m + 4 * kDecRows;                       // [4][16]
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    *reinterpret_cast<float2*>(&s_o[(warp * kDecRows + qr) * D + n * 8 + qc]) = make_float2(o[n][0], o[n][1]);
    *reinterpret_cast<float2*>(&s_o[(warp * kDecRows + qr + 8) * D + n * 8 + qc]) = make_float2(o[n][2], o[n][3]);
  }
  if ((lane & 3) == 0) {
    s_m[warp * kDecRows + qr] = m[0];
    s_m[warp * kDecRows + qr + 8] = m[1];
    s_l[warp * kDecRows + qr] = l[0];
    s_l[warp * kDecRows + qr + 8] = l[1];
  }
  named_bar_sync(1, kDecThreads);
  if (!ok) return;
  // thread t: row t/8, 16 (D=128) or 8 (D=64) consecutive columns
  {
    const int r = threadIdx.x >> 3;
    const int lr = rg * kDecRows + r;
    if (lr < rows_total) {
      constexpr int kCols = D / 8;
      const int c0 = (threadIdx.x & 7) * kCols;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w)
        if (s_l[w * kDecRows + r] > 0.f) M = fmaxf(M, s_m[w * kDecRows + r]);
      float wt[4];
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float lw = s_l[w * kDecRows + r];
        wt[w] = (lw > 0.f) ? ex2_approx((s_m[w * kDecRows + r] - M) * c) : 0.f;
        L += wt[w] * lw;
      }
      const float inv = (L > 0.f) ? 1.f / L : 0.f;
      // partial row [kv head][slot][local row]
      const int64_t pr = (static_cast<int64_t>(hkv) * slots + j) * rows_total + lr;
      float* dst = p.part_o + pr * D + c0;
#pragma unroll
      for (int cc = 0; cc < kCols; cc += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 v = *reinterpret_cast<const float4*>(&s_o[(w * kDecRows + r) * D + c0 + cc]);
          acc.x += wt[w] * v.x;
          acc.y += wt[w] * v.y;
          acc.z += wt[w] * v.z;
          acc.w += wt[w] * v.w;
        }
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
        *reinterpret_cast<float4*>(dst + cc) = acc;
      }
      if ((threadIdx.x & 7) == 0)
        p.part_ml[pr] = make_float2(L > 0.f ? M * p.scale : -INFINITY, L);
    }
  }
}

// One warp per output row: O = sum_s w_s O_s / sum_s w_s with
// w_s = l_s exp(m_s - M), M = max_s m_s; LSE = M + ln(sum_s w_s).  A split
// with l_s = 0 saw no visible key and gets weight 0; a row whose splits are
// all empty gets O = 0 and LSE = -inf.
//
// Lane s of the warp holds split s's weight (32 splits at a time); the
// partial rows are read kUnroll splits at a time with independent 16-byte
// loads, and with up to 32 splits the first kUnroll of them are loaded with
// the (max, sum) pairs, so a row of up to kUnroll splits costs one memory
// latency.
// The kernel is launched as a programmatic dependent of the split kernel: it
// may start while the split kernel's last CTAs run, and waits for that
// grid's completion (and the visibility of its writes) before reading.
struct CombineParams {
  const float* part_o;     // as DecodeParams
  const float2* part_ml;
  const int* seqlens_k;    // per-batch lengths (the slot deal of the split kernel when
                           // use_deal), or nullptr: nsplit slots from b * nsplit
  uint16_t* out;           // output row (b*Hq + h)*Sq + i at b*sb + h*sh + i*sr elements
  float* lse;              // [B*Hq*Sq] or nullptr
  int64_t rows;            // B*Hq*Sq
  int B, Hq, Sq, Sk, group, nsplit, slots;
  int64_t sb, sh, sr;
};

template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const __grid_constant__ CombineParams cp) {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  constexpr int kPer = D / 32;  // floats per lane: 4 (one 16-byte load) or 2
  constexpr int kUnroll = 8;
  constexpr float kLog2e = 1.4426950408889634f;
  // the next kernel in the stream (a programmatic dependent) may be scheduled now
  grid_dependency_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= cp.rows) {
    grid_dependency_wait();
    return;
  }
  const int64_t bh = row / cp.Sq;
  const int i = static_cast<int>(row - bh * cp.Sq);
  const int b = static_cast<int>(bh / cp.Hq);
  const int hq = static_cast<int>(bh - static_cast<int64_t>(b) * cp.Hq);
  const int hkv = hq / cp.group;
  const int rows_total = cp.group * cp.Sq;
  const int lr = (hq - hkv * cp.group) * cp.Sq + i;  // row among the kv head's query rows
  int first = b * cp.nsplit, nsplit = cp.nsplit;
  if (cp.seqlens_k != nullptr && use_deal(cp.B, cp.nsplit)) {
    // Read before the wait: this grid starts only after every CTA of the
    // split kernel has passed its own dependency wait, so whatever kernel
    // wrote the lengths has completed and its writes are visible.
    const int2 r = batch_slots(cp.seqlens_k, cp.B, cp.Sk, cp.slots, b, lane);
    first = r.x;
    nsplit = r.y;
  }
  grid_dependency_wait();
  // partial rows of this output row: [kv head][slot][local row], slot stride rows_total
  const int64_t pr0 = (static_cast<int64_t>(hkv) * cp.slots + first) * rows_total + lr;
  const int64_t pstride = rows_total;
  const float* po = cp.part_o + pr0 * D + lane * kPer;
  // lane's kPer columns of partial row s of this output row
  auto load_part = [&](int s, float (&x)[kPer]) {
    const float* src = po + s * pstride * D;
    if constexpr (kPer == 4) {
      const float4 t = *reinterpret_cast<const float4*>(src);
      x[0] = t.x;
      x[1] = t.y;
      x[2] = t.z;
      x[3] = t.w;
    } else {
      const float2 t = *reinterpret_cast<const float2*>(src);
      x[0] = t.x;
      x[1] = t.y;
    }
  };
  float M = -INFINITY;
  float acc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) acc[e] = 0.f;
  float W = 0.f;
  if (nsplit <= 32) {
    // One round trip: lane s's (m_s, l_s) and the first kUnroll partial rows
    // are loaded together, before the maximum is known.
    const float2 v = (lane < nsplit) ? cp.part_ml[pr0 + lane * pstride] : make_float2(-INFINITY, 0.f);
    float x[kUnroll][kPer];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (u < nsplit) load_part(u, x[u]);
    M = (v.y > 0.f) ? v.x : -INFINITY;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (M != -INFINITY) {
      const float w_lane = (v.y > 0.f) ? v.y * ex2_approx((v.x - M) * kLog2e) : 0.f;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const float w = __shfl_sync(0xffffffffu, w_lane, u);
        if (u < nsplit) {
#pragma unroll
          for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
        }
      }
      for (int i0 = kUnroll; i0 < nsplit; i0 += kUnroll) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (i0 + u < nsplit) load_part(i0 + u, x[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const float w = __shfl_sync(0xffffffffu, w_lane, (i0 + u) & 31);
          if (i0 + u < nsplit) {
#pragma unroll
            for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
          }
        }
      }
      W = w_lane;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
    }
  } else {
    for (int s = lane; s < nsplit; s += 32) {
      const float2 v = cp.part_ml[pr0 + s * pstride];
      if (v.y > 0.f) M = fmaxf(M, v.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (M != -INFINITY) {
      for (int s0 = 0; s0 < nsplit; s0 += 32) {
        const int n = min(32, nsplit - s0);
        float w_lane = 0.f;
        if (lane < n) {
          const float2 v = cp.part_ml[pr0 + (s0 + lane) * pstride];
          w_lane = (v.y > 0.f) ? v.y * ex2_approx((v.x - M) * kLog2e) : 0.f;
        }
        W += w_lane;
        for (int i0 = 0; i0 < n; i0 += kUnroll) {
          float x[kUnroll][kPer];
#pragma unroll
          for (int u = 0; u < kUnroll; ++u)
            if (i0 + u < n) load_part(s0 + i0 + u, x[u]);
#pragma unroll
          for (int u = 0; u < kUnroll; ++u) {
            const float w = __shfl_sync(0xffffffffu, w_lane, (i0 + u) & 31);
            if (i0 + u < n) {
#pragma unroll
              for (int e = 0; e < kPer; ++e) acc[e] = fmaf(w, x[u][e], acc[e]);
            }
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(0xffffffffu, W, off);
    }
  }
  const float inv = (W > 0.f) ? 1.f / W : 0.f;
  uint16_t* dst = cp.out + b * cp.sb + hq * cp.sh + i * cp.sr + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  }
  if (lane == 0 && cp.lse != nullptr)
    cp.lse[row] = (W > 0.f) ? M + lg2_approx(W) * 0.69314718055994531f : -INFINITY;
}

}  // namespace sdpa

// rope.cuh -- the step before the decode: split a packed QKV projection,
// apply the rotary embedding to q and k, append k and v to the KV cache.
//
// This is the fused "split packed QKV with rotary embedding and copy KV" step
// named by "[onnxruntime] WebGPU FlashAttention: kernel fusion and variable
// sequence length" (section 2), which gives no formula.  Reading taken: the
// non-interleaved rotary embedding -- for position p and i < d/2 the pair
// (x_i, x_{i+d/2}) becomes (x_i c - x_{i+d/2} s, x_{i+d/2} c + x_i s) with
// c = cos[p][i], s = sin[p][i] -- at the absolute position past_lens[b] + t of
// token t of batch b; k and v go to cache rows past_lens[b] .. + S_new - 1.
//
// A pure streaming kernel, bound by HBM bandwidth: every element of the packed
// input is read once and written once (the cos/sin rows stay in L2).  A block
// takes whole tokens (grid-stride over them), so the batch/token split and the
// position check happen once per token and each lane loads its slice of the
// token's cos/sin row once for all of the token's heads.  One row of d bf16 is
// held by d/8 lanes, 16 bytes each: a warp covers 2 (d=128) or 4 (d=64) head
// rows per pass, the block 8 times that, and every lane issues the loads of
// kRopeUnroll passes before it uses any, to keep enough bytes in flight.  The
// partner half of each rotated pair sits d/16 lanes away and comes over by
// shuffle.  Tokens are pipelined one deep: a block issues the loads of its
// next token's rows before it rotates and stores the current token's, so its
// loads never wait for its stores (at 64 registers, four blocks per SM).
#pragma once
#include <climits>

#include "ptx.cuh"

namespace sdpa {

struct RopeParams {
  const uint16_t* packed;  // [B][S_new][(Hq + 2*Hkv) * d] bf16
  const float* cos_t;      // [max_pos][d/2]
  const float* sin_t;      // [max_pos][d/2]
  const int* past_lens;    // [B]
  uint16_t* q_out;         // q rows, element (b, h, t, :) at b*q_sb + h*q_sh + t*q_sr
  uint16_t* k_cache;       // cache rows, element (b, h, pos, :) at b*c_sb + h*c_sh + pos*c_sr
  uint16_t* v_cache;
  int* total_lens;         // [B] past + S_new written by this kernel, or nullptr (none, or
                           // written by rope_lengths_kernel afterwards when it aliases past_lens)
  int64_t q_sb, q_sh, q_sr;
  int64_t c_sb, c_sh, c_sr;
  int tokens;              // B * S_new (< 2^31, checked on the host)
  int B, S_new, Hq, Hkv, cap, max_pos;
};

constexpr int kRopeWarps = 8;        // warps per block (256 threads)
constexpr int kRopeUnroll = 3;       // block passes over a token's head rows with loads in flight together
constexpr int kRopeBlocksPerSm = 4;  // resident blocks per SM

// past + S_new, saturated to the int range instead of wrapping (a corrupt
// past near INT_MAX gives INT_MAX, which a later decode clamps and reports).
__device__ __forceinline__ int rope_total_length(int past, int s_new) {
  const long long t = static_cast<long long>(past) + s_new;
  return t > INT_MAX ? INT_MAX : static_cast<int>(t);
}

// total_lens[b] = past_lens[b] + S_new as a second, stream-ordered step: used
// when the two arrays overlap (lengths updated in place), so that no block of
// the append kernel can read a past length another block has already advanced.
__global__ void rope_lengths_kernel(const int* past_lens, int* total_lens, int B, int s_new) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B; i += gridDim.x * blockDim.x) {
    const int past = past_lens[i];  // plain load: the array may be the one written
    total_lens[i] = rope_total_length(past, s_new);
  }
}

template <int D>
__global__ void __launch_bounds__(kRopeWarps * 32, kRopeBlocksPerSm)
    rope_append_kernel(const __grid_constant__ RopeParams p) {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  constexpr int kHalf = D / 2;
  constexpr int kLanesPerRow = D / 8;  // 16 bytes of the row per lane
  constexpr int kRowsPerPass = 32 / kLanesPerRow;
  constexpr int kBlockRows = kRopeWarps * kRowsPerPass;  // head rows per block pass
  constexpr int kPartner = kLanesPerRow / 2;             // lane distance between x_i and x_{i+d/2}
  const int lane = threadIdx.x & 31;
  const int sub = lane % kLanesPerRow;
  const int row_in_block = (threadIdx.x >> 5) * kRowsPerPass + lane / kLanesPerRow;
  // the partner's element enters with a minus sign in the first half
  // (x_i c - x_{i+d/2} s) and a plus sign in the second (x_{i+d/2} c + x_i s)
  const float sign = sub < kPartner ? -1.f : 1.f;
  const int i0 = (sub % kPartner) * 8;  // index within the half of this lane's 8 elements
  const int slots = p.Hq + 2 * p.Hkv;

  // Safe only because total_lens never overlaps past_lens here (the host
  // then leaves total_lens to rope_lengths_kernel, launched after this one).
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.B; i += gridDim.x * blockDim.x)
    if (p.total_lens != nullptr) p.total_lens[i] = rope_total_length(__ldg(p.past_lens + i), p.S_new);

  // Token bt's position, or -1 when it is out of range (reported, skipped).
  auto token_pos = [&](int bt, int& b, int& t) {
    b = bt / p.S_new;
    t = bt - b * p.S_new;
    const int past = __ldg(p.past_lens + b);
    // pos = past + t must lie in [0, min(cap, max_pos)); tested without
    // forming past + t, which overflows for a corrupt past near INT_MAX
    if (past < 0 || past > p.cap - 1 - t || past > p.max_pos - 1 - t) {
      if (threadIdx.x == 0) atomicOr(&g_error_word, kErrSeqlen);
      return -1;
    }
    return past + t;
  };
  // The loads of one token's head rows (kRopeUnroll block passes cover every
  // row when (Hq + 2 Hkv) <= kBlockRows * kRopeUnroll; more rows take further
  // rounds in process_token).
  auto load_rows = [&](int bt, int h0, uint4 (&x)[kRopeUnroll]) {
    const uint4* src = reinterpret_cast<const uint4*>(p.packed + static_cast<int64_t>(bt) * slots * D) + sub;
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int h = h0 + u * kBlockRows + row_in_block;
      x[u] = h < slots ? __ldg(src + h * (D / 8)) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // Rotate and store the rows of one round.
  auto store_rows = [&](int b, int t, int pos, int h0, const uint4 (&x)[kRopeUnroll], const float (&c)[8],
                        const float (&s)[8]) {
    uint16_t* const q_base = p.q_out + b * p.q_sb + t * p.q_sr;
    const int64_t c_off = b * p.c_sb + static_cast<int64_t>(pos) * p.c_sr;
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      // every lane of the warp takes part in the exchange; the partner lane
      // always belongs to the same row
      uint4 y;
      y.x = __shfl_xor_sync(0xffffffffu, x[u].x, kPartner);
      y.y = __shfl_xor_sync(0xffffffffu, x[u].y, kPartner);
      y.z = __shfl_xor_sync(0xffffffffu, x[u].z, kPartner);
      y.w = __shfl_xor_sync(0xffffffffu, x[u].w, kPartner);
      const int h = h0 + u * kBlockRows + row_in_block;
      if (h >= slots) continue;
      uint4 out = x[u];
      uint16_t* dst;
      if (h < p.Hq + p.Hkv) {
        dst = h < p.Hq ? q_base + h * p.q_sh : p.k_cache + c_off + (h - p.Hq) * p.c_sh;
        const uint32_t xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
        const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float xa = bf16_bits_to_float(static_cast<unsigned short>(xs[j] & 0xFFFFu));
          const float xb = bf16_bits_to_float(static_cast<unsigned short>(xs[j] >> 16));
          const float ya = bf16_bits_to_float(static_cast<unsigned short>(ys[j] & 0xFFFFu));
          const float yb = bf16_bits_to_float(static_cast<unsigned short>(ys[j] >> 16));
          o[j] = pack_bf16x2(fmaf(ya, s[2 * j], xa * c[2 * j]), fmaf(yb, s[2 * j + 1], xb * c[2 * j + 1]));
        }
        out = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        dst = p.v_cache + c_off + (h - p.Hq - p.Hkv) * p.c_sh;  // v: copied as is
      }
      reinterpret_cast<uint4*>(dst)[sub] = out;
    }
  };

  // Tokens are pipelined one deep: the first round of the next token's rows
  // is loaded before this token's rows are rotated and stored, so the loads
  // of a block never stop for its stores.
  int bt = blockIdx.x;  // block-uniform
  if (bt >= p.tokens) return;
  int b, t;
  int pos = token_pos(bt, b, t);
  uint4 x[kRopeUnroll];
  if (pos >= 0) load_rows(bt, 0, x);
  while (true) {
    const int nbt = bt + gridDim.x;
    int nb = 0, nt = 0, npos = -1;
    uint4 xn[kRopeUnroll];
    if (nbt < p.tokens) {
      npos = token_pos(nbt, nb, nt);
      if (npos >= 0) load_rows(nbt, 0, xn);
    }
    if (pos >= 0) {
      const float4* cr = reinterpret_cast<const float4*>(p.cos_t + static_cast<int64_t>(pos) * kHalf + i0);
      const float4* sr = reinterpret_cast<const float4*>(p.sin_t + static_cast<int64_t>(pos) * kHalf + i0);
      const float4 c0 = __ldg(cr), c1 = __ldg(cr + 1), s0 = __ldg(sr), s1 = __ldg(sr + 1);
      const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float s[8] = {s0.x * sign, s0.y * sign, s0.z * sign, s0.w * sign,
                          s1.x * sign, s1.y * sign, s1.z * sign, s1.w * sign};
      store_rows(b, t, pos, 0, x, c, s);
      for (int h0 = kBlockRows * kRopeUnroll; h0 < slots; h0 += kBlockRows * kRopeUnroll) {  // block-uniform
        uint4 xr[kRopeUnroll];
        load_rows(bt, h0, xr);
        store_rows(b, t, pos, h0, xr, c, s);
      }
    }
    if (nbt >= p.tokens) break;
    bt = nbt;
    b = nb;
    t = nt;
    pos = npos;
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) x[u] = xn[u];
  }
}

}  // namespace sdpa

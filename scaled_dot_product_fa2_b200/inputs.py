"""Seeded synthetic inputs and the named workloads.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic.  Both the CUDA path's tests/benchmark and the oracle
consume the tensors it returns, so the two sides always see identical inputs.

Recipe: ``torch.Generator('cpu').manual_seed(seed)``, then ``randn`` fp32
N(0, 1) for q, then k, then v (in that order), then a round-to-nearest-even
conversion to bf16.  ``seed = 1000 * family + shape_index``, family 1..5 in the
order the workloads are listed below.  The pages'
own benchmark draws ``randn`` inputs the same way ("FlashAttention-2" notes,
code example).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

CAUSAL_NONE, CAUSAL_TOP_LEFT, CAUSAL_BOTTOM_RIGHT = 0, 1, 2


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    d: int
    causal: int
    seed: int
    scale: float = 0.0  # 0 -> 1/sqrt(d)
    decode: bool = False

    @property
    def eff_scale(self) -> float:
        return self.scale if self.scale != 0.0 else 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """Algorithmic FLOPs: 4*B*Hq*Sq*Sk*d, halved for a causal prefill."""
        f = 4.0 * self.B * self.Hq * self.Sq * self.Sk * self.d
        return f / 2.0 if (self.causal and not self.decode) else f

    def decode_bytes(self) -> int:
        """Algorithmic bytes of a decode call: K+V cache, Q, O (bf16) and LSE (fp32)."""
        kv = 2 * self.B * self.Hkv * self.Sk * self.d * 2
        qo = 2 * self.B * self.Hq * self.Sq * self.d * 2
        return kv + qo + self.B * self.Hq * self.Sq * 4

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _prefill_sweep(family: int, causal: int):
    out = []
    for idx, seq in enumerate((512, 1024, 2048, 4096)):
        out.append(Workload(name=f"prefill_{'causal' if causal else 'noncausal'}_s{seq}",
                            B=16384 // seq, Hq=16, Hkv=16, Sq=seq, Sk=seq, d=128,
                            causal=causal, seed=1000 * family + idx))
    return out


#: tiny causal attention B=1 H=2 S=128 d=64 (fp32 inputs; rounded to bf16 for the GPU)
TINY = Workload("tiny_causal", B=1, Hq=2, Hkv=2, Sq=128, Sk=128, d=64,
                causal=CAUSAL_TOP_LEFT, seed=1000, scale=1.0 / 8.0)
#: non-causal prefill, d=128, H=16, seq 512..4096, 16k tokens per shape
PREFILL_NONCAUSAL = _prefill_sweep(2, CAUSAL_NONE)
#: the same shapes with a top-left causal mask
PREFILL_CAUSAL = _prefill_sweep(3, CAUSAL_TOP_LEFT)
#: GQA causal prefill, one long sequence (Hq=32, Hkv=8, S=16384)
GQA_LONG = Workload("gqa_causal_s16384", B=1, Hq=32, Hkv=8, Sq=16384, Sk=16384, d=128,
                    causal=CAUSAL_TOP_LEFT, seed=4000)
#: split-KV decode, 1 or 4 query rows at the end of an 8192-long cache
DECODE = [Workload(f"decode_sq{sq}", B=8, Hq=32, Hkv=8, Sq=sq, Sk=8192, d=128,
                   causal=CAUSAL_BOTTOM_RIGHT, seed=5000 + idx, decode=True)
          for idx, sq in enumerate((1, 4))]

ALL = [TINY, *PREFILL_NONCAUSAL, *PREFILL_CAUSAL, GQA_LONG, *DECODE]
BY_NAME = {w.name: w for w in ALL}


def make_qkv(B: int, Hq: int, Hkv: int, Sq: int, Sk: int, d: int, seed: int,
             dtype: torch.dtype = torch.bfloat16):
    """Seeded host tensors q[B,Hq,Sq,d], k[B,Hkv,Sk,d], v[B,Hkv,Sk,d].

    Drawn as fp32 N(0,1) in the order q, k, v from one CPU generator, then
    converted to ``dtype`` (round-to-nearest-even for bf16).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, Sq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, Sk, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, Sk, d), generator=g, dtype=torch.float32)
    if dtype != torch.float32:
        q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    return q, k, v


def workload_inputs(w: Workload, dtype: torch.dtype = torch.bfloat16):
    return make_qkv(w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.d, w.seed, dtype)


def decode_lengths(w: Workload) -> list[int]:
    """Seeded per-batch valid cache lengths for the variable-length decode:
    batch 0 uses the whole capacity w.Sk, batch 1 a single key, the others are
    uniform in [1, w.Sk] from a CPU generator seeded with w.seed + 77."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) + 77)
    lens = torch.randint(1, w.Sk + 1, (w.B,), generator=g, dtype=torch.int64).tolist()
    lens[0] = w.Sk
    if w.B > 1:
        lens[1] = 1
    return [int(x) for x in lens]


#: variable-length causal prefill: 8 sequences padded to 4096 (d=128, H=16),
#: query and key lengths equal per sequence, drawn by ``prefill_lengths``
PREFILL_VARLEN = Workload("prefill_varlen_causal_max4096", B=8, Hq=16, Hkv=16, Sq=4096, Sk=4096, d=128,
                          causal=CAUSAL_TOP_LEFT, seed=6000)


def prefill_lengths(w: Workload) -> list[int]:
    """Seeded per-sequence lengths for the variable-length prefill: uniform in
    [w.Sq // 8, w.Sq] from a CPU generator seeded with w.seed + 77; the first
    sequence uses the full w.Sq."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed) + 77)
    lens = torch.randint(w.Sq // 8, w.Sq + 1, (w.B,), generator=g, dtype=torch.int64).tolist()
    lens[0] = w.Sq
    return [int(x) for x in lens]


#: the step before a decode: split a packed QKV of one new token per sequence,
#: rotate q and k, append k and v to a cache of 8192 rows (the decode's shape)
ROPE_DECODE = Workload("rope_append_decode_b8_hq32_hkv8", B=8, Hq=32, Hkv=8, Sq=1, Sk=8192, d=128,
                       causal=CAUSAL_NONE, seed=7000)
#: the same step over a whole 4096-token prompt (the prefill's shape), into an
#: empty cache of 4096 rows
ROPE_PROMPT = Workload("rope_append_prompt_b8_s4096_h16", B=8, Hq=16, Hkv=16, Sq=4096, Sk=4096, d=128,
                       causal=CAUSAL_NONE, seed=7001)


def rope_bytes(w: Workload) -> int:
    """Algorithmic bytes of one rotary/append call: the packed projection read
    once, q written once, k and v written once into the cache (bf16).  The
    cos/sin rows (4*d bytes a token, about 2% of the rest) are left out: they
    are shared across sequences and heads and stay in L2."""
    per_token = (w.Hq + 2 * w.Hkv) * w.d * 2
    return 2 * w.B * w.Sq * per_token


def rope_tables(max_pos: int, d: int, base: float = 10000.0):
    """cos/sin tables [max_pos, d/2] fp32 of the usual rotary frequencies:
    angle(p, i) = p * base^(-2i/d), evaluated in fp64 and rounded to fp32.
    The kernel and the oracle both take these tables as inputs."""
    p = torch.arange(max_pos, dtype=torch.float64)[:, None]
    i = torch.arange(d // 2, dtype=torch.float64)[None, :]
    ang = p * torch.pow(torch.tensor(base, dtype=torch.float64), -2.0 * i / d)
    return torch.cos(ang).float().contiguous(), torch.sin(ang).float().contiguous()


def make_rope_inputs(B: int, S_new: int, Hq: int, Hkv: int, d: int, cap: int, seed: int,
                     past_lens: list[int] | None = None, layout: int = 0):
    """Seeded host tensors for the rotary/append step.

    packed [B, S_new, (Hq+2*Hkv)*d], then k_cache and v_cache (their existing
    contents; [B, Hkv, cap, d], or [B, cap, Hkv, d] for layout 1), all fp32
    N(0, 1) from one CPU generator in that order and rounded to bf16; then,
    unless given, past_lens uniform in [0, cap - S_new] from the same
    generator with past_lens[0] = cap - S_new (a cache filled to capacity).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    packed = torch.randn((B, S_new, (Hq + 2 * Hkv) * d), generator=g, dtype=torch.float32).bfloat16()
    shape = (B, cap, Hkv, d) if layout == 1 else (B, Hkv, cap, d)
    kc = torch.randn(shape, generator=g, dtype=torch.float32).bfloat16()
    vc = torch.randn(shape, generator=g, dtype=torch.float32).bfloat16()
    if past_lens is None:
        past_lens = torch.randint(0, cap - S_new + 1, (B,), generator=g, dtype=torch.int64).tolist()
        if B > 0:
            past_lens[0] = cap - S_new
    return packed, kc, vc, torch.tensor(past_lens, dtype=torch.int32)

"""fp64 CPU oracle for scaled-dot-product attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product library never does,
and this package imports nothing from the product.

The arithmetic lives in ``sdpa_oracle.c`` (plain C, fp64, no fast-math); this
module compiles it with gcc on first use and wraps it with ctypes.  Every
function takes and returns numpy float64 arrays in the [B, H, S, d] layout.

Sources followed (page title and section):
  * "PyTorch attention profiling: Flash, cuDNN, Math backends", section 1
    (naive attention, five steps) and "math backend" (_safe_softmax)
      -> attn_fwd, attn_rows
  * "FlashAttention-2" notes, "algorithm overview" (online-softmax loop)
      -> online_attn  (used only as a pin of the plain definition)
  * "[onnxruntime] WebGPU FlashAttention: kernel fusion ...", section 1
    (fused decode partial with (max, sum) metadata, VxReduce rescale)
      -> split_partials, split_combine
  * same page, same section: additive attention bias applied with the causal
    mask, two leading dims broadcasting over batch and heads
      -> attn_fwd(..., bias=...), attn_rows(..., bias=...)
  * same page, section 2: the fused split of a packed QKV projection with
    rotary embedding and copy into the KV cache (plain numpy, fp64)
      -> rope_append
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdpa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsdpa_oracle.so")
_lock = threading.Lock()
_lib = None

CAUSAL_NONE, CAUSAL_TOP_LEFT, CAUSAL_BOTTOM_RIGHT = 0, 1, 2

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_I32 = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile sdpa_oracle.c into libsdpa_oracle.so (gcc, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-shared", "-fPIC",
                        "-pthread", _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    i, d = ctypes.c_int, ctypes.c_double
    lib.oracle_attn_fwd.argtypes = [_D, _D, _D, _D, _D, i, i, i, i, i, i, d, i, i]
    lib.oracle_attn_rows.argtypes = [_D, _D, _D, i, i, i, i, i, i, d, i,
                                     _I64, ctypes.c_int64, _D, _D, i]
    lib.oracle_attn_fwd_bias.argtypes = [_D, _D, _D, _D, i, i, _D, _D, i, i, i, i, i, i, d, i, i]
    lib.oracle_attn_rows_bias.argtypes = [_D, _D, _D, _D, i, i, i, i, i, i, i, i, d, i,
                                          _I64, ctypes.c_int64, _D, _D, i]
    lib.oracle_online_attn.argtypes = [_D, _D, _D, _D, _D, i, i, i, i, i, i, d, i, i, i]
    lib.oracle_attn_bwd.argtypes = [_D, _D, _D, _D, _D, _D, _D, i, i, i, i, i, i, d, i, i]
    lib.oracle_split_partials.argtypes = [_D, _D, _D, i, i, i, i, i, i, d, i,
                                          _I32, i, _D, _D, _D]
    lib.oracle_split_combine.argtypes = [_D, _D, _D, ctypes.c_int64, i, i, _D, _D]
    for f in (lib.oracle_attn_fwd, lib.oracle_attn_rows, lib.oracle_attn_fwd_bias, lib.oracle_attn_rows_bias,
              lib.oracle_online_attn,
              lib.oracle_split_partials, lib.oracle_split_combine):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
    return _lib


def _f64(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_D)


def _dims(q, k, v):
    B, Hq, Sq, d = q.shape
    Bk, Hkv, Sk, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k disagree on batch or head_dim")
    if v.shape != k.shape:
        raise ValueError("v must have the shape of k")
    return B, Hq, Hkv, Sq, Sk, d


def _threads(nthreads):
    return int(nthreads) if nthreads else (os.cpu_count() or 1)


def _bias(bias, B, Hq, Sq, Sk):
    """The bias as a contiguous fp64 [bias_b, bias_h, Sq, Sk] array and its two
    broadcast dims (each 1 or the full size)."""
    b = _f64(bias)
    if b.ndim != 4 or b.shape[2:] != (Sq, Sk) or b.shape[0] not in (1, B) or b.shape[1] not in (1, Hq):
        raise ValueError(f"bias must be [1|B, 1|Hq, Sq, Sk], got {b.shape}")
    return b, int(b.shape[0]), int(b.shape[1])


def attn_fwd(q, k, v, scale: float, causal: int = CAUSAL_NONE, nthreads: int | None = None, bias=None):
    """The five naive steps for every row (the bias, if given, is added to the
    scaled scores before the mask).  Returns (o[B,Hq,Sq,d], lse[B,Hq,Sq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    o = np.zeros((B, Hq, Sq, d))
    lse = np.zeros((B, Hq, Sq))
    if bias is None:
        st = _load().oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                     B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal),
                                     _threads(nthreads))
    else:
        bb, nb, nh = _bias(bias, B, Hq, Sq, Sk)
        st = _load().oracle_attn_fwd_bias(_ptr(q), _ptr(k), _ptr(v), _ptr(bb), nb, nh, _ptr(o), _ptr(lse),
                                          B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal),
                                          _threads(nthreads))
    if st != 0:
        raise ValueError(f"oracle_attn_fwd failed ({st})")
    return o, lse


def attn_bwd(q, k, v, dout, scale: float, causal: int = CAUSAL_NONE, nthreads: int | None = None):
    """Gradients (dq, dk, dv) of a loss whose gradient with respect to the
    output o = attn_fwd(q, k, v, scale, causal) is ``dout`` ([B, Hq, Sq, d]).

    The pages report the backward pass's speed but give no algorithm; this is
    the chain rule through the five naive steps (sdpa_oracle.c,
    oracle_attn_bwd), in fp64.  dk and dv of a KV head sum over the query heads
    that share it.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    if g.shape != q.shape:
        raise ValueError("dout must have q's shape")
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    st = _load().oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dq), _ptr(dk), _ptr(dv),
                                 B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), _threads(nthreads))
    if st != 0:
        raise RuntimeError(f"oracle_attn_bwd failed ({st})")
    return dq, dk, dv


def attn_rows(q, k, v, scale: float, causal: int, rows, nthreads: int | None = None, bias=None):
    """The five naive steps for selected rows.

    ``rows`` are flattened indices (b*Hq + hq)*Sq + i.  Returns (o[n,d], lse[n]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = rows.shape[0]
    o = np.zeros((n, d))
    lse = np.zeros((n,))
    if bias is None:
        st = _load().oracle_attn_rows(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Sk, d,
                                      float(scale), int(causal), rows.ctypes.data_as(_I64), n,
                                      _ptr(o), _ptr(lse), _threads(nthreads))
    else:
        bb, nb, nh = _bias(bias, B, Hq, Sq, Sk)
        st = _load().oracle_attn_rows_bias(_ptr(q), _ptr(k), _ptr(v), _ptr(bb), nb, nh, B, Hq, Hkv, Sq, Sk, d,
                                           float(scale), int(causal), rows.ctypes.data_as(_I64), n,
                                           _ptr(o), _ptr(lse), _threads(nthreads))
    if st != 0:
        raise ValueError(f"oracle_attn_rows failed ({st})")
    return o, lse


def online_attn(q, k, v, scale: float, causal: int, block_q: int, block_k: int):
    """The FlashAttention-2 online-softmax recurrence in fp64 (a pin, not a product)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    o = np.zeros((B, Hq, Sq, d))
    lse = np.zeros((B, Hq, Sq))
    st = _load().oracle_online_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                    B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal),
                                    int(block_q), int(block_k))
    if st != 0:
        raise ValueError(f"oracle_online_attn failed ({st})")
    return o, lse


def split_partials(q, k, v, scale: float, causal: int, bounds):
    """Per-split locally normalised partials and (max, sum) metadata.

    ``bounds`` is a list [0, b1, ..., Sk] of split boundaries over the keys.
    Returns (part_o[B,Hq,Sq,ns,d], part_m[B,Hq,Sq,ns], part_l[B,Hq,Sq,ns]).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Hkv, Sq, Sk, d = _dims(q, k, v)
    b = np.ascontiguousarray(np.asarray(bounds, dtype=np.int32))
    ns = b.shape[0] - 1
    po = np.zeros((B, Hq, Sq, ns, d))
    pm = np.zeros((B, Hq, Sq, ns))
    pl = np.zeros((B, Hq, Sq, ns))
    st = _load().oracle_split_partials(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Sk, d,
                                       float(scale), int(causal), b.ctypes.data_as(_I32), ns,
                                       _ptr(po), _ptr(pm), _ptr(pl))
    if st != 0:
        raise ValueError(f"oracle_split_partials failed ({st})")
    return po, pm, pl


def split_combine(part_o, part_m, part_l):
    """Combine split partials.  part_o is [..., ns, d]; returns (o[..., d], lse[...])."""
    po, pm, pl = _f64(part_o), _f64(part_m), _f64(part_l)
    lead = po.shape[:-2]
    ns, d = po.shape[-2], po.shape[-1]
    n = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (d,))
    lse = np.zeros(lead)
    st = _load().oracle_split_combine(_ptr(po), _ptr(pm), _ptr(pl), n, ns, d,
                                      _ptr(o), _ptr(lse))
    if st != 0:
        raise ValueError(f"oracle_split_combine failed ({st})")
    return o, lse


# --------------------------------------------------------- rotary + KV append

def rope_append(packed_qkv, cos, sin, past_lens, k_cache, v_cache, Hq: int, Hkv: int):
    """The step before the decode, in plain fp64 loops: split a packed
    [B, S_new, (Hq + 2*Hkv) * d] projection into q, k, v heads (q heads first,
    then k, then v), rotate q and k by their absolute position, and append k, v
    to the caches at rows past_lens[b] .. past_lens[b] + S_new - 1.

    Follows the fused "split packed QKV with rotary embedding and copy KV" step
    named by "[onnxruntime] WebGPU FlashAttention: kernel fusion and variable
    sequence length" (section 2).  The page gives no formula; reading taken:
    the non-interleaved rotary embedding -- for position p and i < d/2,
    (x_i, x_{i+d/2}) -> (x_i cos[p,i] - x_{i+d/2} sin[p,i],
                         x_{i+d/2} cos[p,i] + x_i sin[p,i]).
    Returns (q [B, Hq, S_new, d], new k_cache, new v_cache [B, Hkv, cap, d],
    total_lens [B] = past_lens + S_new).  Inputs are not modified.
    """
    x = _f64(packed_qkv)
    cos, sin = _f64(cos), _f64(sin)
    kc, vc = _f64(k_cache).copy(), _f64(v_cache).copy()
    past = [int(p) for p in np.asarray(past_lens).reshape(-1)]
    B, S_new, width = x.shape
    d = width // (Hq + 2 * Hkv)
    half = d // 2
    q = np.zeros((B, Hq, S_new, d))

    def rotate(vec, pos):
        out = np.empty(d)
        for i in range(half):
            c, s = cos[pos, i], sin[pos, i]
            out[i] = vec[i] * c - vec[i + half] * s
            out[i + half] = vec[i + half] * c + vec[i] * s
        return out

    for b in range(B):
        for s in range(S_new):
            pos = past[b] + s
            row = x[b, s]
            for h in range(Hq):
                q[b, h, s] = rotate(row[h * d:(h + 1) * d], pos)
            for h in range(Hkv):
                kc[b, h, pos] = rotate(row[(Hq + h) * d:(Hq + h + 1) * d], pos)
                vc[b, h, pos] = row[(Hq + Hkv + h) * d:(Hq + Hkv + h + 1) * d]
    return q, kc, vc, np.asarray([p + S_new for p in past], dtype=np.int64)

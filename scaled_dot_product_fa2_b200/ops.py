"""Torch-facing wrappers over the C ABI (argument marshalling only).

Every computation happens in the CUDA kernels of libsdpa_b200.so; these
functions only check dtypes/devices, allocate outputs with torch and pass raw
pointers plus the current CUDA stream.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

CAUSAL_NONE, CAUSAL_TOP_LEFT, CAUSAL_BOTTOM_RIGHT = 0, 1, 2
LAYOUT_BHSD, LAYOUT_BSHD = 0, 1


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_tensor(name: str, t: torch.Tensor, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shapes(q, k, v, q_layout=LAYOUT_BHSD, kv_layout=LAYOUT_BHSD):
    """(B, Hq, Hkv, Sq, Sk, d) of q [B,Hq,Sq,d] (or [B,Sq,Hq,d] for BSHD) and
    k, v [B,Hkv,Sk,d] (or [B,Sk,Hkv,d])."""
    _check_tensor("q", q, torch.bfloat16, 4)
    _check_tensor("k", k, torch.bfloat16, 4)
    _check_tensor("v", v, torch.bfloat16, 4)
    if q_layout == LAYOUT_BSHD:
        B, Sq, Hq, d = q.shape
    else:
        B, Hq, Sq, d = q.shape
    if kv_layout == LAYOUT_BSHD:
        Bk, Sk, Hkv, dk = k.shape
    else:
        Bk, Hkv, Sk, dk = k.shape
    if Bk != B or dk != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    return B, Hq, Hkv, Sq, Sk, d


def _outputs(q, out, lse, want_lse, layout=LAYOUT_BHSD):
    if layout == LAYOUT_BSHD:
        B, Sq, Hq, d = q.shape
    else:
        B, Hq, Sq, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_tensor("out", out, torch.bfloat16, 4)
        if tuple(out.shape) != tuple(q.shape) or out.device != q.device:
            raise ValueError("out must have the shape of q, on q's device")
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    elif lse is not None:
        _check_tensor("lse", lse, torch.float32, 3)
        if tuple(lse.shape) != (B, Hq, Sq) or lse.device != q.device:
            raise ValueError("lse must be [B, Hq, Sq] on q's device")
    return out, lse


def _bias_extras(bias, B, Hq, Sq, Sk, device, ex=None):
    """attn_extras_t carrying a bf16 bias [1|B, 1|Hq, Sq, Sk] (or None)."""
    ex = ex if ex is not None else _lib.Extras()
    if bias is None:
        return ex
    _check_tensor("bias", bias, torch.bfloat16, 4)
    if (bias.shape[0] not in (1, B) or bias.shape[1] not in (1, Hq) or tuple(bias.shape[2:]) != (Sq, Sk)
            or bias.device != device):
        raise ValueError(f"bias must be [1|B, 1|Hq, Sq, Sk] on q's device, got {tuple(bias.shape)}")
    ex.bias = bias.data_ptr()
    ex.bias_b = int(bias.shape[0])
    ex.bias_h = int(bias.shape[1])
    return ex


def attn_fwd(q, k, v, causal: int = CAUSAL_NONE, scale: float = 0.0, out=None, lse=None,
             return_lse: bool = True, bias=None, layout: int = LAYOUT_BHSD):
    """O = softmax(scale * q k^T + bias + mask) v through the C ABI.

    q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] bf16 contiguous CUDA tensors ([B,S,H,d]
    for all four with ``layout=LAYOUT_BSHD``); ``scale=0`` means 1/sqrt(d);
    ``bias`` an optional bf16 [1|B, 1|Hq, Sq, Sk] tensor (``attn_fwd_ex``).
    Returns (o, lse) with o shaped like q and lse fp32 [B,Hq,Sq] (None when
    ``return_lse`` is False and no ``lse`` buffer was given).
    """
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k, v, layout, layout)
    out, lse = _outputs(q, out, lse, return_lse, layout)
    lib = _lib.get()
    with torch.cuda.device(q.device):
        args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr() if lse is not None else None,
                B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal))
        if bias is None and layout == LAYOUT_BHSD:
            st = lib.attn_fwd(*args, _stream_handle(q.device))
        else:
            ex = _bias_extras(bias, B, Hq, Sq, Sk, q.device)
            ex.layout = int(layout)
            st = lib.attn_fwd_ex(*args, ctypes.byref(ex), _stream_handle(q.device))
    _lib.check(st, "attn_fwd")
    return out, lse


def _check_lengths(name, t, B, device):
    if not isinstance(t, torch.Tensor) or t.dtype != torch.int32 or t.dim() != 1:
        raise TypeError(f"{name} must be an int32 tensor [B]")
    if tuple(t.shape) != (B,) or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B] tensor on q's device")


def attn_fwd_varlen(q, k, v, seqlens_q, seqlens_k, causal: int = CAUSAL_NONE, scale: float = 0.0, out=None,
                    lse=None, return_lse: bool = True):
    """Forward over padded sequences of per-batch lengths (``attn_fwd_varlen``).

    q [B,Hq,Sq_max,d], k/v [B,Hkv,Sk_max,d]; ``seqlens_q``/``seqlens_k`` int32
    CUDA tensors [B] read on the device.  Padding rows of the outputs are not
    written (a new ``out`` is zero-filled so they read as 0).  Returns (o, lse).
    """
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k, v)
    _check_lengths("seqlens_q", seqlens_q, B, q.device)
    _check_lengths("seqlens_k", seqlens_k, B, q.device)
    if out is None:
        out = torch.zeros_like(q)
    out, lse = _outputs(q, out, lse, return_lse)
    lib = _lib.get()
    with torch.cuda.device(q.device):
        st = lib.attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), seqlens_q.data_ptr(),
                                 seqlens_k.data_ptr(), out.data_ptr(), lse.data_ptr() if lse is not None else None,
                                 B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), _stream_handle(q.device))
    _lib.check(st, "attn_fwd_varlen")
    return out, lse


def decode_num_splits(B, Hq, Hkv, Sq, Sk, d) -> int:
    return int(_lib.get().attn_decode_num_splits(B, Hq, Hkv, Sq, Sk, d))


def decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits: int = 0) -> int:
    return int(_lib.get().attn_decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits))


def bwd_workspace_size(B, Hq, Sq) -> int:
    """Bytes of workspace ``attn_bwd`` needs (``attn_bwd_workspace_size``)."""
    return int(_lib.get().attn_bwd_workspace_size(B, Hq, Sq))


def decode_workspace(q, k_cache, num_splits: int = 0) -> torch.Tensor:
    """A caller-owned workspace buffer sized for ``attn_decode_splitkv``."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k_cache.shape[1], k_cache.shape[2]
    with torch.cuda.device(q.device):
        n = decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)


def attn_decode_splitkv(q, k_cache, v_cache, causal: int = CAUSAL_BOTTOM_RIGHT, scale: float = 0.0,
                        num_splits: int = 0, workspace=None, out=None, lse=None, return_lse: bool = True,
                        bias=None, seqlens_k=None, layout: int = LAYOUT_BHSD):
    """Split-KV decode through the C ABI (``attn_decode_splitkv``, or
    ``attn_decode_splitkv_ex`` when a bf16 ``bias`` [1|B, 1|Hq, Sq, Sk], an
    int32 ``seqlens_k`` [B] or ``layout=LAYOUT_BSHD`` (q and o as [B,Sq,Hq,d];
    the cache stays [B,Hkv,Sk,d]) is given).  Returns (o, lse)."""
    if bias is not None or seqlens_k is not None or layout != LAYOUT_BHSD:
        return _decode_ex(q, k_cache, v_cache, causal, scale, num_splits, workspace, out, lse, return_lse, bias,
                          seqlens_k, layout)
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k_cache, v_cache)
    out, lse = _outputs(q, out, lse, return_lse)
    if workspace is None:
        workspace = decode_workspace(q, k_cache, num_splits)
    if workspace.device != q.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous buffer on q's device")
    lib = _lib.get()
    with torch.cuda.device(q.device):
        st = lib.attn_decode_splitkv(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                     lse.data_ptr() if lse is not None else None,
                                     B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), int(num_splits),
                                     workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                     _stream_handle(q.device))
    _lib.check(st, "attn_decode_splitkv")
    return out, lse


def _decode_ex(q, k_cache, v_cache, causal, scale, num_splits, workspace, out, lse, return_lse, bias, seqlens_k,
               layout=LAYOUT_BHSD):
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k_cache, v_cache, layout, LAYOUT_BHSD)
    ex = _bias_extras(bias, B, Hq, Sq, Sk, q.device)
    ex.layout = int(layout)
    if seqlens_k is not None:
        _check_lengths("seqlens_k", seqlens_k, B, q.device)
        ex.seqlens_k = seqlens_k.data_ptr()
    out, lse = _outputs(q, out, lse, return_lse, layout)
    if workspace is None:
        with torch.cuda.device(q.device):
            n = decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, num_splits)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    if workspace.device != q.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous buffer on q's device")
    lib = _lib.get()
    with torch.cuda.device(q.device):
        st = lib.attn_decode_splitkv_ex(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                        lse.data_ptr() if lse is not None else None,
                                        B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), int(num_splits),
                                        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                        ctypes.byref(ex), _stream_handle(q.device))
    _lib.check(st, "attn_decode_splitkv_ex")
    return out, lse


def attn_decode_splitkv_varlen(q, k_cache, v_cache, seqlens_k, causal: int = CAUSAL_BOTTOM_RIGHT,
                               scale: float = 0.0, num_splits: int = 0, workspace=None, out=None, lse=None,
                               return_lse: bool = True):
    """Split-KV decode over caches with per-batch valid lengths (``attn_decode_splitkv_varlen``).

    ``k_cache``/``v_cache`` are [B, Hkv, capacity, d]; ``seqlens_k`` is an int32
    CUDA tensor [B] of valid keys per batch, read on the device only.
    Returns (o, lse).
    """
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k_cache, v_cache)
    _check_lengths("seqlens_k", seqlens_k, B, q.device)
    out, lse = _outputs(q, out, lse, return_lse)
    if workspace is None:
        workspace = decode_workspace(q, k_cache, num_splits)
    if workspace.device != q.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous buffer on q's device")
    lib = _lib.get()
    with torch.cuda.device(q.device):
        st = lib.attn_decode_splitkv_varlen(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                            seqlens_k.data_ptr(), out.data_ptr(),
                                            lse.data_ptr() if lse is not None else None,
                                            B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), int(num_splits),
                                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                            _stream_handle(q.device))
    _lib.check(st, "attn_decode_splitkv_varlen")
    return out, lse


def attn_decode_splitkv_static(q, k_cache, v_cache, causal: int = CAUSAL_BOTTOM_RIGHT, scale: float = 0.0,
                               num_splits: int = 0, out=None, lse=None, return_lse: bool = True):
    """Split-KV decode without a workspace (``attn_decode_splitkv_static``).

    For callers that cannot hand the library device memory: the partials live
    in the library's fixed 16 MiB scratch array.  Output tensors are still the
    caller's (allocated here with torch when not given).  Calls that may
    overlap on the GPU share that scratch and race; issue them on one stream.
    """
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k_cache, v_cache)
    out, lse = _outputs(q, out, lse, return_lse)
    lib = _lib.get()
    with torch.cuda.device(q.device):
        st = lib.attn_decode_splitkv_static(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(),
                                            lse.data_ptr() if lse is not None else None,
                                            B, Hq, Hkv, Sq, Sk, d, float(scale), int(causal), int(num_splits),
                                            _stream_handle(q.device))
    _lib.check(st, "attn_decode_splitkv_static")
    return out, lse


def attn_bwd(q, k, v, o, lse, dout, causal: int = CAUSAL_NONE, scale: float = 0.0, dq=None, dk=None, dv=None,
             workspace=None):
    """Gradients (dq, dk, dv) of the forward ``o, lse = attn_fwd(q, k, v, causal, scale)``
    for ``dout`` = dL/do (``attn_bwd``).  BHSD tensors, bf16; lse fp32 from the forward.

    P is recomputed from ``lse``; nothing of size Sq x Sk is stored.  dk and dv
    of a KV head sum over the query heads that share it.
    """
    B, Hq, Hkv, Sq, Sk, d = _shapes(q, k, v)
    _check_tensor("o", o, torch.bfloat16, 4)
    _check_tensor("dout", dout, torch.bfloat16, 4)
    _check_tensor("lse", lse, torch.float32, 3)
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must have q's shape")
    if tuple(lse.shape) != (B, Hq, Sq):
        raise ValueError("lse must be [B, Hq, Sq]")
    if not (o.device == dout.device == lse.device == q.device):
        raise ValueError("o, lse and dout must be on q's device")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, ref in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        _check_tensor(name, t, torch.bfloat16, 4)
        if tuple(t.shape) != tuple(ref.shape) or t.device != q.device:
            raise ValueError(f"{name} must match {tuple(ref.shape)} on q's device")
    lib = _lib.get()
    if workspace is None:
        workspace = torch.empty(max(bwd_workspace_size(B, Hq, Sq), 16), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Sq, Sk, d, float(scale),
                          int(causal), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          _stream_handle(q.device))
    _lib.check(st, "attn_bwd")
    return dq, dk, dv


def attn_rope_append(packed_qkv, cos, sin, past_lens, k_cache, v_cache, Hq: int, Hkv: int,
                     layout: int = LAYOUT_BHSD, q_out=None, total_lens=None):
    """Split a packed QKV projection, rotate q and k, append k and v to the cache
    (``attn_rope_append``).

    packed_qkv [B, S_new, (Hq + 2*Hkv) * d] bf16 (q heads, then k, then v);
    cos, sin [max_pos, d/2] fp32; past_lens [B] int32; k_cache, v_cache
    [B, Hkv, cap, d] bf16 ([B, cap, Hkv, d] for LAYOUT_BSHD), updated in place.
    Returns (q [B, Hq, S_new, d] -- [B, S_new, Hq, d] for LAYOUT_BSHD --,
    total_lens [B] int32 = past_lens + S_new).  A token whose position is out
    of range is skipped and reported by check_device_error().
    """
    _check_tensor("packed_qkv", packed_qkv, torch.bfloat16, 3)
    _check_tensor("k_cache", k_cache, torch.bfloat16, 4)
    _check_tensor("v_cache", v_cache, torch.bfloat16, 4)
    _check_tensor("cos", cos, torch.float32, 2)
    _check_tensor("sin", sin, torch.float32, 2)
    B, S_new, width = packed_qkv.shape
    if Hq <= 0 or Hkv <= 0 or width % (Hq + 2 * Hkv) != 0:
        raise ValueError("packed_qkv's last dim must be (Hq + 2*Hkv) * d")
    d = width // (Hq + 2 * Hkv)
    if layout == LAYOUT_BSHD:
        cap = k_cache.shape[1]
        cache_shape, q_shape = (B, cap, Hkv, d), (B, S_new, Hq, d)
    elif layout == LAYOUT_BHSD:
        cap = k_cache.shape[2]
        cache_shape, q_shape = (B, Hkv, cap, d), (B, Hq, S_new, d)
    else:
        raise ValueError(f"unknown layout {layout}")
    if tuple(k_cache.shape) != cache_shape or tuple(v_cache.shape) != cache_shape:
        raise ValueError(f"k_cache and v_cache must be {cache_shape}")
    if tuple(cos.shape) != tuple(sin.shape) or cos.shape[1] != d // 2:
        raise ValueError("cos and sin must both be [max_pos, d/2]")
    dev = packed_qkv.device
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache), ("cos", cos), ("sin", sin)):
        if t.device != dev:
            raise ValueError(f"{name} must be on packed_qkv's device")
    _check_lengths("past_lens", past_lens, B, dev)
    if q_out is None:
        q_out = torch.empty(q_shape, dtype=torch.bfloat16, device=dev)
    else:
        _check_tensor("q_out", q_out, torch.bfloat16, 4)
        if tuple(q_out.shape) != q_shape or q_out.device != dev:
            raise ValueError(f"q_out must be {q_shape} on packed_qkv's device")
    if total_lens is None:
        total_lens = torch.empty(B, dtype=torch.int32, device=dev)
    else:
        _check_lengths("total_lens", total_lens, B, dev)
    lib = _lib.get()
    with torch.cuda.device(dev):
        st = lib.attn_rope_append(packed_qkv.data_ptr(), cos.data_ptr(), sin.data_ptr(), int(cos.shape[0]),
                                  past_lens.data_ptr(), q_out.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                  total_lens.data_ptr(), B, S_new, Hq, Hkv, cap, d, int(layout),
                                  _stream_handle(dev))
    _lib.check(st, "attn_rope_append")
    return q_out, total_lens


def check_device_error(device=None) -> None:
    """Synchronize the current stream and raise if a kernel gave up on a bounded wait."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    with torch.cuda.device(dev):
        st = _lib.get().attn_check_device_error(_stream_handle(dev))
    _lib.check(st, "attn_check_device_error")

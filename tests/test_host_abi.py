"""Host-side checks of the C ABI that need no GPU.

The library must load on a machine without a GPU, export every function the
header declares, and reject bad arguments on the host before touching CUDA.
"""
import ctypes
import os
import re

import pytest

from scaled_dot_product_fa2_b200 import _lib, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sdpa_b200.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.get()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for required in ("attn_fwd", "attn_decode_splitkv", "attn_decode_workspace_size",
                     "attn_status_string", "attn_check_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in sdpa_b200.h but not exported"
    assert set(_lib.EXPORTS) <= set(names)


def test_status_strings(lib):
    for code in range(14):
        assert lib.attn_status_string(code)
    assert lib.attn_status_string(0) == b"ok"


# Fake, well-aligned device addresses: validation must fail before any use.
P = 1 << 20


def fwd(lib, q=P, k=P, v=P, o=P, lse=None, B=1, Hq=2, Hkv=2, Sq=8, Sk=8, d=128, scale=0.0, causal=0):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Sq, Sk, d, scale, causal, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(k=None), 1), (dict(v=None), 1),
    (dict(B=-1), 2), (dict(Sq=-3), 2), (dict(Sk=-1), 2), (dict(Hq=0), 2), (dict(Hkv=0), 2),
    (dict(Sq=(1 << 30) + 1), 2),
    (dict(Hq=6, Hkv=4), 3),
    (dict(d=96), 4), (dict(d=256), 4), (dict(d=32), 4),
    (dict(q=P + 8), 5), (dict(k=P + 2), 5), (dict(o=P + 4), 5), (dict(lse=P + 2), 5),
    (dict(causal=3), 6), (dict(causal=-1), 6),
    (dict(scale=-0.5), 11), (dict(scale=float("nan")), 11), (dict(scale=float("inf")), 11),
])
def test_fwd_rejects_bad_arguments_on_host(lib, kw, status):
    assert fwd(lib, **kw) == status


def test_fwd_empty_problem_is_ok_without_launch(lib):
    assert fwd(lib, B=0, q=None, k=None, v=None, o=None) == 0
    assert fwd(lib, Sq=0, q=None, k=None, v=None, o=None) == 0


def test_decode_workspace_size_formula(lib):
    # fixed split count: rows * splits * (d floats + 2 floats)
    B, Hq, Hkv, Sq, Sk, d = 8, 32, 8, 4, 8192, 128
    for splits in (1, 2, 7, 128):
        n = lib.attn_decode_workspace_size(B, Hq, Hkv, Sq, Sk, d, splits)
        tiles = (Sk + 63) // 64
        t = -(-tiles // min(splits, tiles))
        eff = -(-tiles // t)
        assert n == B * Hq * Sq * eff * (d + 2) * 4
    # more splits than tiles are clamped to one tile per split
    assert lib.attn_decode_workspace_size(1, 1, 1, 1, 100, 64, 50) == 1 * 2 * (64 + 2) * 4
    assert lib.attn_decode_workspace_size(1, 3, 2, 1, 100, 64, 1) == 0  # Hq % Hkv != 0
    assert lib.attn_decode_workspace_size(1, 2, 2, 1, 100, 96, 1) == 0  # bad d
    assert lib.attn_decode_num_splits(8, 32, 8, 4, 8192, 128) >= 1


def test_decode_rejects_bad_workspace_on_host(lib):
    args = dict(B=2, Hq=4, Hkv=2, Sq=1, Sk=256, d=128)
    need = lib.attn_decode_workspace_size(*args.values(), 0)
    call = lambda ws, nbytes, splits=0: lib.attn_decode_splitkv(
        P, P, P, P, None, *args.values(), 0.0, 2, splits, ws, nbytes, None)
    assert call(None, need) == 7
    assert call(P + 4, need) == 7
    assert call(P, need - 1) == 7
    assert lib.attn_decode_splitkv(P, P, P, P, None, 2, 4, 2, 1, 256, 128, 0.0, 2, -1, P, need, None) == 2
    assert lib.attn_decode_splitkv(P, P, P, P, None, 2, 4, 3, 1, 256, 128, 0.0, 2, 0, P, need, None) == 3


def test_varlen_decode_rejects_bad_lengths_pointer_on_host(lib):
    args = (2, 4, 2, 1, 256, 128)
    need = lib.attn_decode_workspace_size(*args, 0)
    call = lambda seqlens: lib.attn_decode_splitkv_varlen(P, P, P, seqlens, P, None, *args, 0.0, 2, 0, P, need, None)
    assert call(None) == 1      # ATTN_ERR_NULL
    assert call(P + 2) == 5     # ATTN_ERR_ALIGN (int32 array)
    # an empty problem needs no lengths
    assert lib.attn_decode_splitkv_varlen(None, None, None, None, None, None, 0, 4, 2, 1, 256, 128, 0.0, 2, 0,
                                          None, 0, None) == 0
    assert lib.attn_status_string(13)


def test_varlen_forward_rejects_bad_lengths_pointers_on_host(lib):
    call = lambda sq, sk: lib.attn_fwd_varlen(P, P, P, sq, sk, P, None, 2, 4, 2, 64, 64, 128, 0.0, 0, None)
    assert call(None, P) == 1
    assert call(P, None) == 1
    assert call(P + 2, P) == 5
    assert call(P, P + 1) == 5
    assert lib.attn_fwd_varlen(None, None, None, None, None, None, None, 0, 4, 2, 64, 64, 128, 0.0, 0, None) == 0


def test_extras_are_validated_on_host(lib):
    from scaled_dot_product_fa2_b200._lib import Extras
    ex = Extras()
    ex.bias = P
    ex.bias_b, ex.bias_h = 1, 1
    fwd = lambda Sk, e: lib.attn_fwd_ex(P, P, P, P, None, 2, 4, 2, 64, Sk, 128, 0.0, 0, ctypes.byref(e), None)
    assert fwd(12, ex) == 5          # forward bias rows must be 16-byte aligned: Sk % 8 == 0
    ex.bias_b = 3
    assert fwd(64, ex) == 2          # bias_b must be 1 or B
    ex.bias_b, ex.bias_h = 2, 2
    assert fwd(64, ex) == 2          # bias_h must be 1 or Hq
    ex.bias_h = 4
    ex.bias = P + 2
    assert fwd(64, ex) == 5          # 16-byte aligned bias base for the forward
    dec = lambda e: lib.attn_decode_splitkv_ex(P, P, P, P, None, 2, 4, 2, 1, 256, 128, 0.0, 2, 0, P,
                                               1 << 30, ctypes.byref(e), None)
    ex.bias = P + 1
    assert dec(ex) == 5              # 2-byte alignment for the decode's bias
    ex2 = Extras()
    ex2.seqlens_q = P
    assert dec(ex2) == 2             # the decode takes no query lengths
    ex3 = Extras()
    ex3.layout = 2
    assert dec(ex3) == 2             # unknown layout


def test_ptxas_report_checker():
    regs = build.PREFILL_LAUNCH_REGS
    ok = ("ptxas info    : Compiling entry function '_ZN4sdpa14prefill_kernelILi128ELi4EEEvNS_13PrefillParamsE'\n"
          "    0 bytes stack frame, 0 bytes spill stores, 0 bytes spill loads\n"
          f"ptxas info    : Used {regs} registers, used 16 barriers\n")
    build.check_ptxas_report(ok)
    with pytest.raises(RuntimeError):
        build.check_ptxas_report(ok.replace(f"Used {regs}", f"Used {regs - 8}"))
    with pytest.raises(RuntimeError):
        build.check_ptxas_report(ok.replace("0 bytes spill stores", "8 bytes spill stores"))
    # the bias instantiation may spill a few bytes, nothing more
    bias = ok.replace("Li4EEEv", "Li4ELb1EEEv")
    build.check_ptxas_report(bias.replace("0 bytes spill stores, 0 bytes spill loads",
                                          "4 bytes spill stores, 16 bytes spill loads"))
    with pytest.raises(RuntimeError):
        build.check_ptxas_report(bias.replace("0 bytes spill stores", "64 bytes spill stores"))


def test_decode_split_policy_fills_one_wave(lib):
    """The automatic split count keeps every decode CTA resident in one wave
    when the (batch, kv head, row group) pairs alone fit in one (148 SMs x 2
    CTAs without a device), and never makes more splits than 64-key tiles."""
    slots = 148 * 2
    for (B, Hq, Hkv, Sq, Sk) in [(8, 32, 8, 1, 8192), (8, 32, 8, 4, 8192), (1, 32, 8, 1, 8192),
                                 (2, 16, 16, 1, 4096), (4, 8, 2, 2, 30000)]:
        rg = -(-(Hq // Hkv) * Sq // 16)
        pairs = B * Hkv * rg
        ns = lib.attn_decode_num_splits(B, Hq, Hkv, Sq, Sk, 128)
        tiles = -(-Sk // 64)
        assert 1 <= ns <= tiles
        assert pairs * ns <= slots, (B, Hq, Hkv, Sq, Sk, ns)
    # the decode workload: 64 (batch, kv head) pairs -> 4 splits of 32 tiles, 256 CTAs
    assert lib.attn_decode_num_splits(8, 32, 8, 1, 8192, 128) == 4
    # more pairs than resident slots: no splitting
    assert lib.attn_decode_num_splits(64, 32, 8, 1, 8192, 128) == 1



def test_decode_split_policy_is_quick_for_any_cache_length(lib):
    """The automatic split search is bounded: a cache of 2^30 keys (16M tiles)
    with many (batch, kv head) pairs is sized in well under a second."""
    import time
    t0 = time.perf_counter()
    for B, Hkv in [(1, 1), (64, 8), (1024, 64)]:
        ns = lib.attn_decode_num_splits(B, Hkv * 4, Hkv, 1, 1 << 30, 128)
        assert ns >= 1
        assert lib.attn_decode_workspace_size(B, Hkv * 4, Hkv, 1, 1 << 30, 128, 0) > 0
    assert time.perf_counter() - t0 < 1.0


def test_decode_rejects_query_rows_per_kv_head_beyond_int(lib):
    # group * Sq = 65536 * 32768 = 2^31 query rows share one KV head
    assert lib.attn_decode_workspace_size(1, 1 << 16, 1, 1 << 15, 128, 128, 0) == 0
    assert lib.attn_decode_num_splits(1, 1 << 16, 1, 1 << 15, 128, 128) == 0


def test_selftest_timeout_entry_rejects_empty_problems_on_host(lib):
    P = ctypes.c_void_p(16)
    for B, Sq, Sk in [(0, 1, 1), (1, 0, 1), (1, 1, 0)]:
        assert lib.attn_selftest_decode_wait_timeout(P, P, P, P, None, B, 4, 1, Sq, Sk, 128, P, 1 << 20, None) == 2


def test_rope_append_rejects_bad_arguments_on_host(lib):
    def call(packed=P, cos=P, sin=P, max_pos=64, past=P, q=P, kc=P, vc=P, tot=P, B=2, S_new=3, Hq=4, Hkv=2,
             cap=64, d=128, layout=0):
        return lib.attn_rope_append(packed, cos, sin, max_pos, past, q, kc, vc, tot, B, S_new, Hq, Hkv, cap, d,
                                    layout, None)
    for kw, status in [
        (dict(packed=None), 1), (dict(cos=None), 1), (dict(sin=None), 1), (dict(past=None), 1),
        (dict(q=None), 1), (dict(kc=None), 1), (dict(vc=None), 1),
        (dict(B=-1), 2), (dict(S_new=-1), 2), (dict(Hq=0), 2), (dict(Hkv=0), 2), (dict(cap=0), 2),
        (dict(max_pos=0), 2), (dict(layout=2), 2), (dict(S_new=(1 << 30) + 1), 2),
        (dict(Hq=6, Hkv=4), 3),
        (dict(d=96), 4), (dict(d=32), 4),
        (dict(packed=P + 8), 5), (dict(cos=P + 4), 5), (dict(sin=P + 4), 5), (dict(q=P + 2), 5),
        (dict(kc=P + 8), 5), (dict(vc=P + 8), 5), (dict(past=P + 2), 5), (dict(tot=P + 1), 5),
    ]:
        assert call(**kw) == status, kw
    # nothing to do: no batch, or no new token and no total lengths wanted
    assert call(B=0, packed=None, cos=None, sin=None, past=None, q=None, kc=None, vc=None, tot=None) == 0
    assert call(S_new=0, packed=None, cos=None, sin=None, q=None, kc=None, vc=None, tot=None) == 0


def test_bwd_rejects_bad_arguments_on_host(lib):
    need = lib.attn_bwd_workspace_size(2, 4, 100)
    assert need == 2 * 2 * 4 * 128 * 4  # rows padded to whole 128-row tiles, two fp32 vectors
    assert lib.attn_bwd_workspace_size(-1, 4, 100) == 0

    def call(q=P, k=P, v=P, o=P, lse=P, do=P, dq=P, dk=P, dv=P, B=2, Hq=4, Hkv=2, Sq=100, Sk=90, d=128,
             scale=0.0, causal=0, ws=P, wsb=None):
        return lib.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Hq, Hkv, Sq, Sk, d, scale, causal, ws,
                            need if wsb is None else wsb, None)
    for kw, status in [
        (dict(q=None), 1), (dict(o=None), 1), (dict(dq=None), 1), (dict(do=None), 1), (dict(dk=None), 1),
        (dict(dv=None), 1), (dict(B=-1), 2), (dict(Hq=6, Hkv=4), 3), (dict(d=96), 4),
        (dict(dq=P + 8), 5), (dict(dk=P + 2), 5), (dict(do=P + 4), 5), (dict(causal=3), 6),
        (dict(scale=-1.0), 11),
    ]:
        assert call(**kw) == status, kw
    assert call(B=0, q=None, k=None, v=None, o=None, lse=None, do=None, dq=None, dk=None, dv=None, ws=None) == 0


def test_python_entry_points_refuse_host_tensors(lib):
    """The binding has no CPU path: host tensors are rejected before any call."""
    import torch
    import scaled_dot_product_fa2_b200 as sdpa
    assert sdpa.bwd_workspace_size(2, 4, 100) == lib.attn_bwd_workspace_size(2, 4, 100)
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="CUDA"):
        sdpa.attn_fwd(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        sdpa.attn_bwd(q, q, q, q, lse, q)
    packed = torch.zeros(1, 1, 4 * 64, dtype=torch.bfloat16)
    cos = torch.zeros(8, 32)
    with pytest.raises(ValueError, match="CUDA"):
        sdpa.attn_rope_append(packed, cos, cos, torch.zeros(1, dtype=torch.int32), q[:, :1], q[:, :1], 2, 1)


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-x", "c", "-std=c99"]), ("g++", ["-x", "c++", "-std=c++17"])])
def test_header_compiles_as_c_and_cpp(tmp_path, compiler, flags):
    """The boundary is a C ABI: the header must stand alone in a plain C99
    translation unit (no CUDA or torch headers needed) and in C++."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not found")
    src = tmp_path / "use_header.src"
    src.write_text('#include "sdpa_b200.h"\n'
                   'int main(void) { return sizeof(attn_extras_t) > 0 && attn_version() > 0 && '
                   'attn_status_string(ATTN_OK) != 0 ? 0 : 1; }\n')
    r = subprocess.run([compiler, *flags, "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

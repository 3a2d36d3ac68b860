"""The C-ABI library builds, loads and exports every entry point that include/saw.h declares;
host-side argument checks return their status codes before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

from bit_paged_kv_block_b200 import build, saw

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "saw.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(saw_[a-z0-9_]+)\s*\(", text)))


def test_library_is_built_in_tree():
    assert build.up_to_date()
    assert os.path.dirname(build.LIB) == os.path.dirname(saw.__file__)


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"saw_rotate_quantize_paged", "saw_paged_decode_attn", "saw_decode_step",
            "saw_paged_decode_workspace_bytes", "saw_paged_decode_workspace_init",
            "saw_status_string", "saw_version"} <= set(names)
    lib = ctypes.CDLL(build.LIB)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert saw.saw_version() == 100
    for code in range(5):
        assert saw.saw_status_string(code)
    assert saw.saw_status_string(99) == "unknown status"


def _desc(hkv=8, d=128, p=16, pages=64):
    return saw.saw_cache_desc(hkv, d, p, pages)


def _rq(desc, T=4, k=16, v=16, slots=16, pages=16, scales=16):
    P = ctypes.c_void_p
    return saw.lib.saw_rotate_quantize_paged(
        None if desc is None else ctypes.byref(desc), P(k), P(v), P(slots), T, P(pages),
        P(scales), None, None)


def test_append_argument_checks():
    assert _rq(None) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _rq(_desc(d=96)) == saw.SAW_ERR_UNSUPPORTED
    assert _rq(_desc(p=32)) == saw.SAW_ERR_UNSUPPORTED
    assert _rq(_desc(hkv=0)) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _rq(_desc(pages=1 << 30)) == saw.SAW_ERR_UNSUPPORTED
    assert _rq(_desc(), T=-1) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _rq(_desc(), k=0) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _rq(_desc(), k=8) == saw.SAW_ERR_INVALID_ARGUMENT          # not 16-byte aligned
    assert _rq(_desc(), slots=4) == saw.SAW_ERR_INVALID_ARGUMENT      # not 8-byte aligned
    assert _rq(_desc(), T=0, k=0, v=0, slots=0, pages=0, scales=0) == saw.SAW_OK  # no-op


def _dec(desc, hq=32, S=2, q=16, out=16, bt=16, lens=16, ws=256, ws_bytes=1 << 20,
         max_blocks=4, sm_scale=0.088):
    P = ctypes.c_void_p
    return saw.lib.saw_paged_decode_attn(
        ctypes.byref(desc), hq, P(q), P(16), P(16), P(bt), max_blocks, P(lens), S, sm_scale,
        P(out), P(ws), ws_bytes, None, None)


def test_decode_argument_checks():
    d = _desc()
    assert _dec(d, hq=12) == saw.SAW_ERR_INVALID_ARGUMENT             # Hq % Hkv
    assert _dec(d, hq=136) == saw.SAW_ERR_UNSUPPORTED                 # G = 17 (at most 16)
    assert _dec(d, S=-1) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, q=0) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, q=8) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, out=4) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, lens=2) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, max_blocks=0) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, sm_scale=float("nan")) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _dec(d, S=0) == saw.SAW_OK                                  # nothing to do
    assert _dec(_desc(pages=0)) == saw.SAW_ERR_INVALID_ARGUMENT


def test_workspace_init_checks():
    assert saw.lib.saw_paged_decode_workspace_init(None, 16, None) == saw.SAW_ERR_INVALID_ARGUMENT
    assert saw.lib.saw_paged_decode_workspace_init(None, 0, None) == saw.SAW_OK


def test_workspace_bytes_rejects_bad_shapes():
    f = saw.lib.saw_paged_decode_workspace_bytes
    assert f(ctypes.byref(_desc()), 12, 4) == 0
    assert f(ctypes.byref(_desc()), 72, 4) == 0
    assert f(ctypes.byref(_desc(d=96)), 32, 4) == 0


def test_python_binding_rejects_cpu_tensors():
    import torch
    k = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    kv = torch.zeros(4, 8, 2, 16, 64, dtype=torch.uint8)
    sc = torch.zeros(4, 8, 2, 16, 2, dtype=torch.float16)
    with pytest.raises(ValueError):
        saw.saw_rotate_quantize_paged(k, k, torch.zeros(2, dtype=torch.int64), kv, sc)
    with pytest.raises(TypeError):
        saw.saw_rotate_quantize_paged(k.float(), k, torch.zeros(2, dtype=torch.int64), kv, sc)


def test_strided_append_argument_checks():
    """Strides below a token's Hkv * 128 elements or not a multiple of 8 are invalid; Hkv that
    neither divides nor is a multiple of 8 is unsupported (checked before any launch)."""
    def call(hkv, ks, vs):
        desc = saw.saw_cache_desc(hkv, 128, 16, 4)
        return saw.lib.saw_rotate_quantize_paged_strided(
            ctypes.byref(desc), ctypes.c_void_p(16), ks, ctypes.c_void_p(16), vs,
            ctypes.c_void_p(16), 10, ctypes.c_void_p(16), ctypes.c_void_p(16), None, None)
    assert call(2, 0, 256) == saw.SAW_ERR_INVALID_ARGUMENT
    assert call(2, 200, 256) == saw.SAW_ERR_INVALID_ARGUMENT       # < Hkv * 128
    assert call(2, 260, 256) == saw.SAW_ERR_INVALID_ARGUMENT       # not a multiple of 8
    assert call(3, 384, 384) == saw.SAW_ERR_UNSUPPORTED
    assert call(12, 12 * 128, 12 * 128) == saw.SAW_ERR_UNSUPPORTED


def _win(sink=16, recent=112, kv=16, pages=8, table=16, blocks=8):
    return saw.saw_window_cache(sink, recent, kv, pages, table, blocks)


def _wapp(desc, win, S=2, k=16, v=16, lens=16, pages=16, scales=16, bt=16, max_blocks=4):
    P = ctypes.c_void_p
    return saw.lib.saw_window_append(
        ctypes.byref(desc), None if win is None else ctypes.byref(win), P(k), P(v), P(lens), S,
        P(pages), P(scales), P(bt), max_blocks, None, None)


def _wdec(desc, win, hq=32, S=2, q=16, out=16, ws=256, ws_bytes=1 << 30):
    P = ctypes.c_void_p
    return saw.lib.saw_paged_decode_attn_window(
        ctypes.byref(desc), None if win is None else ctypes.byref(win), hq, P(q), P(16), P(16),
        P(16), 4, P(16), S, 0.088, P(out), P(ws), ws_bytes, None, None)


def test_window_argument_checks():
    """The windowed entry points check the window description before any CUDA call."""
    d = _desc()
    assert _wapp(d, None) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wapp(d, _win(sink=-1)) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wapp(d, _win(recent=200, blocks=8)) == saw.SAW_ERR_INVALID_ARGUMENT   # W > 16 blocks
    assert _wapp(d, _win(kv=0)) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wapp(d, _win(table=2)) == saw.SAW_ERR_INVALID_ARGUMENT                # misaligned
    assert _wapp(d, _win(pages=1 << 30)) == saw.SAW_ERR_UNSUPPORTED               # 2^31 rows
    assert _wapp(_desc(d=256), _win()) == saw.SAW_ERR_UNSUPPORTED                 # bf16 window
    assert _wapp(d, _win(), k=8) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wapp(d, _win(), max_blocks=0) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wapp(d, _win(), S=0) == saw.SAW_OK                                    # nothing to do
    assert _wdec(d, None) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _wdec(d, _win(), hq=12) == saw.SAW_ERR_INVALID_ARGUMENT                # Hq % Hkv
    assert _wdec(d, _win(), hq=136) == saw.SAW_ERR_UNSUPPORTED                    # G = 17
    assert _wdec(_desc(d=64), _win()) == saw.SAW_ERR_UNSUPPORTED
    assert _wdec(d, _win(), S=0) == saw.SAW_OK
    f = saw.lib.saw_paged_decode_window_workspace_bytes
    assert f(ctypes.byref(_desc(d=256)), 32, 4) == 0
    assert f(ctypes.byref(d), 12, 4) == 0


def _pf(desc, hq=32, S=2, q=16, q_start=16, total_q=64, out=16, bt=16, lens=16, ws=256,
        ws_bytes=1 << 20, max_blocks=4, sm_scale=0.088):
    P = ctypes.c_void_p
    return saw.lib.saw_paged_prefill_attn(
        None if desc is None else ctypes.byref(desc), hq, P(q), P(q_start), total_q, P(16), P(16),
        P(bt), max_blocks, P(lens), S, sm_scale, P(out), P(ws), ws_bytes, None, None)


def test_prefill_argument_checks():
    """The chunked-prefill entry point rejects bad arguments on the host, before any CUDA call."""
    d = _desc()
    assert _pf(None) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _pf(_desc(d=96)) == saw.SAW_ERR_UNSUPPORTED
    assert _pf(d, total_q=-1) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _pf(d, total_q=1 << 31) == saw.SAW_ERR_INVALID_ARGUMENT     # more rows than int32
    assert _pf(d, q_start=0) == saw.SAW_ERR_INVALID_ARGUMENT           # no chunk starts
    assert _pf(d, q_start=2) == saw.SAW_ERR_INVALID_ARGUMENT           # not 4-byte aligned
    assert _pf(d, hq=12) == saw.SAW_ERR_INVALID_ARGUMENT               # Hq % Hkv
    assert _pf(d, hq=136) == saw.SAW_ERR_UNSUPPORTED                   # G = 17
    assert _pf(d, q=8) == saw.SAW_ERR_INVALID_ARGUMENT                 # q not 16-byte aligned
    assert _pf(d, out=0) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _pf(d, sm_scale=float("inf")) == saw.SAW_ERR_INVALID_ARGUMENT
    assert _pf(d, S=0, q_start=0) == saw.SAW_OK                          # nothing to do

"""CPU oracle for SAW-INT4 paged INT4 KV-cache compression.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never imports, links or executes anything here, and this package never
imports the product package: the two share no code.

The arithmetic lives in ``saw_oracle.c`` (plain C, ``-O2 -ffp-contract=off``, no fast-math);
this module compiles it on first use with gcc and exposes numpy-level wrappers.  The method
it restates is token-wise INT4 quantization with a block-diagonal Hadamard rotation, fused
into a paged KV cache, and decode attention over that cache ("SAW-INT4: System-Aware 4-Bit
KV-Cache Quantization for Real-World LLM Serving", Research Findings; restated on the idea
page "Memory compression method reducing KV-cache size...", Core Innovation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "saw_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-fopenmp",
             "-std=gnu11"]


def build(force: bool = False) -> str:
    """Compile saw_oracle.c into _build/liboracle.so (a no-op when it is up to date)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_f16_bits.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16_bits.restype = ctypes.c_uint16
        lib.oracle_f16_bits_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_bits_to_f64.restype = dbl
        lib.oracle_fwht_f32.argtypes = [P, i32]
        lib.oracle_fwht_f32.restype = None
        lib.oracle_rotate_f32.argtypes = [P, i32]
        lib.oracle_rotate_f32.restype = None
        lib.oracle_fwht_f64.argtypes = [P, i32]
        lib.oracle_fwht_f64.restype = None
        lib.oracle_rotate_f64.argtypes = [P, i32]
        lib.oracle_rotate_f64.restype = None
        lib.oracle_quantize_vec.argtypes = [P, i32, P, P, P, P, P]
        lib.oracle_quantize_vec.restype = None
        lib.oracle_rotate_quantize_paged.argtypes = [P, P, P, i64, i32, i32, i32, i64, P, P,
                                                     i32, i32]
        lib.oracle_rotate_quantize_paged.restype = i64
        lib.oracle_dequant_row_f64.argtypes = [P, P, i32, i32, i32, i64, i32, i32, i32, P]
        lib.oracle_dequant_row_f64.restype = None
        lib.oracle_decode_fp64.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, dbl,
                                           i32, P, i32]
        lib.oracle_decode_fp64.restype = None
        lib.oracle_prefill_fp64.argtypes = [P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, dbl,
                                            i32, P, i32]
        lib.oracle_prefill_fp64.restype = None
        lib.oracle_append_bf16.argtypes = [P, P, P, i64, i32, i32, i32, i64, P]
        lib.oracle_append_bf16.restype = i64
        lib.oracle_decode_bf16_fp64.argtypes = [P, P, P, i32, P, i32, i32, i32, i32, i32, dbl,
                                                P, i32]
        lib.oracle_decode_bf16_fp64.restype = None
        lib.oracle_decode_window_fp64.argtypes = [P, P, P, i32, P, P, P, i32, P, i32, i32, i32,
                                                  i32, i32, i32, i32, dbl, i32, P, i32]
        lib.oracle_decode_window_fp64.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _as(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


# ---- scalar helpers ------------------------------------------------------------------

def bf16_to_f32(bits: int) -> float:
    return float(_load().oracle_bf16_to_f32(int(bits)))


def f32_to_f16_bits(x: float) -> int:
    return int(_load().oracle_f32_to_f16_bits(float(np.float32(x))))


def f16_bits_to_f64(bits: int) -> float:
    return float(_load().oracle_f16_bits_to_f64(int(bits)))


# ---- rotation --------------------------------------------------------------------------

def fwht_f32(x: np.ndarray) -> np.ndarray:
    """Normalised Sylvester Hadamard transform of each length-n row (fp32 butterfly)."""
    y = np.array(x, dtype=np.float32, copy=True, order="C")
    n = y.shape[-1]
    flat = y.reshape(-1, n)
    lib = _load()
    for r in range(flat.shape[0]):
        row = flat[r]
        lib.oracle_fwht_f32(ctypes.c_void_p(row.ctypes.data), n)
    return y


def rotate_f32(x: np.ndarray) -> np.ndarray:
    """Block-diagonal normalised Hadamard rotation of each row, fp32: 128-wide blocks, or the
    whole row when it is 64 wide."""
    y = np.array(x, dtype=np.float32, copy=True, order="C")
    D = y.shape[-1]
    flat = y.reshape(-1, D)
    lib = _load()
    for r in range(flat.shape[0]):
        lib.oracle_rotate_f32(ctypes.c_void_p(flat[r].ctypes.data), D)
    return y


def rotate_f64(x: np.ndarray) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True, order="C")
    D = y.shape[-1]
    flat = y.reshape(-1, D)
    lib = _load()
    for r in range(flat.shape[0]):
        lib.oracle_rotate_f64(ctypes.c_void_p(flat[r].ctypes.data), D)
    return y


# ---- quantizer ---------------------------------------------------------------------------

def quantize_vec(y: np.ndarray):
    """Quantize one fp32 vector.  Returns (packed uint8[n/2], scale_f16_bits, zero_f16_bits,
    scale_f32, min_f32)."""
    y = _as(np.asarray(y, dtype=np.float32), np.float32)
    n = y.shape[0]
    assert y.ndim == 1 and n % 2 == 0
    packed = np.zeros(n // 2, dtype=np.uint8)
    sh = np.zeros(1, dtype=np.uint16)
    zh = np.zeros(1, dtype=np.uint16)
    sf = np.zeros(1, dtype=np.float32)
    mf = np.zeros(1, dtype=np.float32)
    _load().oracle_quantize_vec(_ptr(y), n, _ptr(packed), _ptr(sh), _ptr(zh), _ptr(sf), _ptr(mf))
    return packed, int(sh[0]), int(zh[0]), float(sf[0]), float(mf[0])


def rotate_quantize_paged(k_bits, v_bits, slot_mapping, kv_pages, scales, *, page_size=16,
                          rotate=True, nthreads=1) -> int:
    """Rotate, quantize and scatter tokens into the paged cache (in place).

    k_bits, v_bits: uint16 bf16 bits [T][Hkv][D].  slot_mapping: int64 [T].
    kv_pages: uint8 [num_pages][Hkv][2][page_size][D/2] (updated in place).
    scales: uint16 fp16 bits [num_pages][Hkv][2][page_size][2] (updated in place).
    Returns the number of out-of-range slots (skipped)."""
    k_bits = _as(k_bits, np.uint16)
    v_bits = _as(v_bits, np.uint16)
    slot_mapping = _as(slot_mapping, np.int64)
    assert kv_pages.dtype == np.uint8 and kv_pages.flags["C_CONTIGUOUS"]
    assert scales.dtype == np.uint16 and scales.flags["C_CONTIGUOUS"]
    T, Hkv, D = k_bits.shape
    assert v_bits.shape == k_bits.shape and slot_mapping.shape == (T,)
    num_pages = kv_pages.shape[0]
    assert kv_pages.shape == (num_pages, Hkv, 2, page_size, D // 2)
    assert scales.shape == (num_pages, Hkv, 2, page_size, 2)
    return int(_load().oracle_rotate_quantize_paged(
        _ptr(k_bits), _ptr(v_bits), _ptr(slot_mapping), T, Hkv, D, page_size, num_pages,
        _ptr(kv_pages), _ptr(scales), 1 if rotate else 0, int(nthreads)))


def dequant_row_f64(kv_pages, scales, page, h, sel, off) -> np.ndarray:
    num_pages, Hkv, _, page_size, half = kv_pages.shape
    D = 2 * half
    y = np.zeros(D, dtype=np.float64)
    _load().oracle_dequant_row_f64(_ptr(kv_pages), _ptr(scales), Hkv, D, page_size, int(page),
                                   int(h), int(sel), int(off), _ptr(y))
    return y


def decode_fp64(q_bits, kv_pages, scales, block_table, seq_lens, *, sm_scale=None,
                rotate=True, nthreads=1) -> np.ndarray:
    """fp64 decode attention over the INT4 paged cache.

    q_bits: uint16 bf16 bits [S][Hq][D]; block_table: int32 [S][max_blocks];
    seq_lens: int32 [S].  Returns fp64 [S][Hq][D]."""
    q_bits = _as(q_bits, np.uint16)
    block_table = _as(block_table, np.int32)
    seq_lens = _as(seq_lens, np.int32)
    S, Hq, D = q_bits.shape
    num_pages, Hkv, _, page_size, half = kv_pages.shape
    assert half * 2 == D and Hq % Hkv == 0
    assert block_table.ndim == 2 and block_table.shape[0] == S and seq_lens.shape == (S,)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    _load().oracle_decode_fp64(_ptr(q_bits), _ptr(kv_pages), _ptr(scales), _ptr(block_table),
                               block_table.shape[1], _ptr(seq_lens), S, Hq, Hkv, D, page_size,
                               float(sm_scale), 1 if rotate else 0, _ptr(out), int(nthreads))
    return out


def prefill_fp64(q_bits, q_start, kv_pages, scales, block_table, seq_lens, *, sm_scale=None,
                 rotate=True, nthreads=1) -> np.ndarray:
    """fp64 chunked-prefill attention over the INT4 paged cache: the C_s = q_start[s + 1] -
    q_start[s] queries of sequence s (rows q_start[s].. of q_bits [total][Hq][D]) are its last
    C_s cached tokens, query i attending causally to tokens 0 .. seq_lens[s] - C_s + i.
    Returns fp64 [total][Hq][D]."""
    q_bits = _as(q_bits, np.uint16)
    q_start = _as(q_start, np.int32)
    block_table = _as(block_table, np.int32)
    seq_lens = _as(seq_lens, np.int32)
    total, Hq, D = q_bits.shape
    S = seq_lens.shape[0]
    num_pages, Hkv, _, page_size, half = kv_pages.shape
    assert half * 2 == D and Hq % Hkv == 0 and q_start.shape == (S + 1,) and q_start[S] == total
    assert np.all(np.diff(q_start) >= 0) and np.all(np.diff(q_start) <= seq_lens)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((total, Hq, D), dtype=np.float64)
    _load().oracle_prefill_fp64(_ptr(q_bits), _ptr(q_start), _ptr(kv_pages), _ptr(scales),
                                _ptr(block_table), block_table.shape[1], _ptr(seq_lens), S, Hq,
                                Hkv, D, page_size, float(sm_scale), 1 if rotate else 0, _ptr(out),
                                int(nthreads))
    return out


def empty_cache_bf16(num_pages: int, Hkv: int, D: int = 128, page_size: int = 16) -> np.ndarray:
    """Zero-filled bf16 cache (uint16 bits) [num_pages][Hkv][2][page_size][D]."""
    return np.zeros((num_pages, Hkv, 2, page_size, D), dtype=np.uint16)


def append_bf16(k_bits, v_bits, slot_mapping, kv_bf16) -> int:
    """Scatter bf16 K, V [T][Hkv][D] into the bf16 pages in place (the uncompressed baseline
    cache).  Negative slots are skipped; slots past the cache are skipped and counted."""
    k_bits = _as(k_bits, np.uint16)
    v_bits = _as(v_bits, np.uint16)
    slot_mapping = _as(slot_mapping, np.int64)
    T, Hkv, D = k_bits.shape
    num_pages, hkv2, _, page_size, d2 = kv_bf16.shape
    assert hkv2 == Hkv and d2 == D and kv_bf16.dtype == np.uint16 and kv_bf16.flags.c_contiguous
    return int(_load().oracle_append_bf16(_ptr(k_bits), _ptr(v_bits), _ptr(slot_mapping), T, Hkv,
                                          D, page_size, num_pages, _ptr(kv_bf16)))


def decode_bf16_fp64(q_bits, kv_bf16, block_table, seq_lens, *, sm_scale=None,
                     nthreads=1) -> np.ndarray:
    """fp64 decode attention over the bf16 paged cache (no rotation, no quantization).
    Returns fp64 [S][Hq][D]."""
    q_bits = _as(q_bits, np.uint16)
    kv_bf16 = _as(kv_bf16, np.uint16)
    block_table = _as(block_table, np.int32)
    seq_lens = _as(seq_lens, np.int32)
    S, Hq, D = q_bits.shape
    num_pages, Hkv, _, page_size, d2 = kv_bf16.shape
    assert d2 == D and Hq % Hkv == 0
    assert block_table.ndim == 2 and block_table.shape[0] == S and seq_lens.shape == (S,)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    _load().oracle_decode_bf16_fp64(_ptr(q_bits), _ptr(kv_bf16), _ptr(block_table),
                                    block_table.shape[1], _ptr(seq_lens), S, Hq, Hkv, D, page_size,
                                    float(sm_scale), _ptr(out), int(nthreads))
    return out


def empty_cache(num_pages: int, Hkv: int, D: int = 128, page_size: int = 16):
    """Zero-filled cache arrays in the oracle's layout (pages, scales)."""
    return (np.zeros((num_pages, Hkv, 2, page_size, D // 2), dtype=np.uint8),
            np.zeros((num_pages, Hkv, 2, page_size, 2), dtype=np.uint16))


# ---- full-precision sink / recent window beside the INT4 cache ----------------------------
# "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language Models",
# Abstract and Figure 2.  The readings (which positions are sinks, recent or quantized, and
# where each lives) are stated above oracle_decode_window_fp64 in saw_oracle.c.

def window_slot(p: int, w_sink: int, w_recent: int) -> int:
    """Window slot of position p (a sink or a recent token)."""
    return p if p < w_sink else w_sink + (p - w_sink) % w_recent


def _win_page_off(win_table, s, slot):
    return int(win_table[s, slot // 16]), slot % 16


def _q_slot(block_table, s, j):
    return int(block_table[s, j // 16]) * 16 + j % 16


def window_fill(k_bits, v_bits, seq_lens, w_sink, w_recent, win_kv, win_table, kv_pages, scales,
                block_table, *, rotate=True):
    """Place every token of each sequence where the window layout puts it: sinks and the last
    w_recent positions (>= w_sink) into their window slots (bf16 bits), the others rotated and
    quantized into the INT4 pages at their quantized index.  k_bits, v_bits: uint16
    [S][Lmax][Hkv][D] (positions beyond seq_lens[s] ignored)."""
    k_bits = _as(k_bits, np.uint16)
    v_bits = _as(v_bits, np.uint16)
    S = len(seq_lens)
    for s in range(S):
        L = int(seq_lens[s])
        slots = []
        for p in range(L):
            if p < w_sink or p >= max(w_sink, L - w_recent):
                pg, off = _win_page_off(win_table, s, window_slot(p, w_sink, w_recent))
                win_kv[pg, :, 0, off] = k_bits[s, p]
                win_kv[pg, :, 1, off] = v_bits[s, p]
                slots.append(-1)
            else:
                slots.append(_q_slot(block_table, s, p - w_sink))
        if L:
            bad = rotate_quantize_paged(np.ascontiguousarray(k_bits[s, :L]),
                                        np.ascontiguousarray(v_bits[s, :L]),
                                        np.array(slots, dtype=np.int64), kv_pages, scales,
                                        rotate=rotate)
            assert bad == 0


def window_append(k_bits, v_bits, seq_lens, w_sink, w_recent, win_kv, win_table, kv_pages,
                  scales, block_table, *, rotate=True):
    """One serving step: the new token of each sequence (k_bits, v_bits: uint16 [S][Hkv][D]) sits
    at position p = seq_lens[s] - 1.  A sink goes to its window slot.  Otherwise the token that
    leaves the recent window (position p - w_recent, if it is not a sink) is rotated and
    quantized from its window slot into the INT4 pages at its quantized index, and the new
    token takes that slot; with w_recent = 0 the new token itself is quantized.  Sequences with
    seq_lens[s] <= 0 are skipped."""
    k_bits = _as(k_bits, np.uint16)
    v_bits = _as(v_bits, np.uint16)
    for s in range(len(seq_lens)):
        L = int(seq_lens[s])
        if L <= 0:
            continue
        p = L - 1
        if p < w_sink:
            pg, off = _win_page_off(win_table, s, p)
            win_kv[pg, :, 0, off] = k_bits[s]
            win_kv[pg, :, 1, off] = v_bits[s]
            continue
        if w_recent == 0:
            bad = rotate_quantize_paged(k_bits[s][None].copy(), v_bits[s][None].copy(),
                                        np.array([_q_slot(block_table, s, p - w_sink)], np.int64),
                                        kv_pages, scales, rotate=rotate)
            assert bad == 0
            continue
        pg, off = _win_page_off(win_table, s, window_slot(p, w_sink, w_recent))
        old = p - w_recent
        if old >= w_sink:
            bad = rotate_quantize_paged(win_kv[pg, :, 0, off][None].copy(),
                                        win_kv[pg, :, 1, off][None].copy(),
                                        np.array([_q_slot(block_table, s, old - w_sink)], np.int64),
                                        kv_pages, scales, rotate=rotate)
            assert bad == 0
        win_kv[pg, :, 0, off] = k_bits[s]
        win_kv[pg, :, 1, off] = v_bits[s]


def decode_window_fp64(q_bits, win_kv, win_table, kv_pages, scales, block_table, seq_lens,
                       w_sink, w_recent, *, sm_scale=None, rotate=True, nthreads=1) -> np.ndarray:
    """fp64 decode attention over the window (bf16 pages [P_w][Hkv][2][16][D] through win_table)
    and the quantized tokens (INT4 pages through block_table), one softmax over both, in the
    original domain.  Returns fp64 [S][Hq][D]."""
    q_bits = _as(q_bits, np.uint16)
    win_kv = _as(win_kv, np.uint16)
    win_table = _as(win_table, np.int32)
    block_table = _as(block_table, np.int32)
    seq_lens = _as(seq_lens, np.int32)
    S, Hq, D = q_bits.shape
    num_pages, Hkv, _, page_size, half = kv_pages.shape
    assert half * 2 == D and Hq % Hkv == 0 and win_kv.shape[1:] == (Hkv, 2, page_size, D)
    assert win_table.shape[0] == S and block_table.shape[0] == S and seq_lens.shape == (S,)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    _load().oracle_decode_window_fp64(_ptr(q_bits), _ptr(win_kv), _ptr(win_table),
                                      win_table.shape[1], _ptr(kv_pages), _ptr(scales),
                                      _ptr(block_table), block_table.shape[1], _ptr(seq_lens), S,
                                      Hq, Hkv, D, page_size, int(w_sink), int(w_recent),
                                      float(sm_scale), 1 if rotate else 0, _ptr(out), int(nthreads))
    return out

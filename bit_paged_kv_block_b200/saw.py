"""Python binding of libsaw (ctypes), with the C ABI's names.

Argument marshalling only: each function checks tensor devices, dtypes, shapes and contiguity,
then passes raw device pointers and the current CUDA stream to the C entry point.  Every step
of the path runs in the library's CUDA kernels; there is no CPU path.  Importing this module
loads libsaw.so from this package directory (building it with nvcc if it is missing) and raises
if that fails.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

HEAD_DIM = 128
PAGE_SIZE = 16

SAW_OK = 0
SAW_ERR_INVALID_ARGUMENT = 1
SAW_ERR_UNSUPPORTED = 2
SAW_ERR_CUDA = 3
SAW_ERR_WORKSPACE = 4
SAW_ERR_SCRATCH_LIMIT = 5

SAW_DEV_BAD_SLOT = 0x1
SAW_DEV_BAD_PAGE = 0x2
SAW_DEV_BAD_SEQ_LEN = 0x4
SAW_DEV_WAIT_TIMEOUT = 0x8
SAW_DEV_RANGE = 0x10


class SawError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status}: {saw_status_string(status)}")


class saw_cache_desc(ctypes.Structure):
    _fields_ = [("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int64)]


class saw_window_cache(ctypes.Structure):
    _fields_ = [("sink", ctypes.c_int32), ("recent", ctypes.c_int32), ("kv", ctypes.c_void_p),
                ("num_pages", ctypes.c_int64), ("table", ctypes.c_void_p),
                ("blocks", ctypes.c_int32)]


def _open_library() -> ctypes.CDLL:
    path = _build.LIB
    if not _build.up_to_date():
        try:
            _build.build()
        except Exception as exc:  # the CUDA library is required: fail loudly
            raise ImportError(f"libsaw.so is missing and could not be built: {exc}") from exc
    lib = ctypes.CDLL(path)
    P, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    D = ctypes.POINTER(saw_cache_desc)
    lib.saw_version.argtypes = []
    lib.saw_version.restype = ctypes.c_int
    lib.saw_status_string.argtypes = [ctypes.c_int]
    lib.saw_status_string.restype = ctypes.c_char_p
    lib.saw_rotate_quantize_paged.argtypes = [D, P, P, P, i64, P, P, P, P]
    lib.saw_rotate_quantize_paged.restype = ctypes.c_int
    lib.saw_paged_decode_workspace_bytes.argtypes = [D, i32, i32]
    lib.saw_paged_decode_workspace_bytes.restype = sz
    lib.saw_paged_decode_workspace_init.argtypes = [P, sz, P]
    lib.saw_paged_decode_workspace_init.restype = ctypes.c_int
    lib.saw_paged_decode_attn.argtypes = [D, i32, P, P, P, P, i32, P, i32, f32, P, P, sz, P, P]
    lib.saw_paged_decode_attn.restype = ctypes.c_int
    lib.saw_decode_step.argtypes = [D, i32, P, P, P, P, i64, P, P, P, i32, P, i32, f32, P, P,
                                    sz, P, P]
    lib.saw_decode_step.restype = ctypes.c_int
    lib.saw_quantize_paged_plain.argtypes = lib.saw_rotate_quantize_paged.argtypes
    lib.saw_quantize_paged_plain.restype = ctypes.c_int
    lib.saw_paged_decode_attn_plain.argtypes = lib.saw_paged_decode_attn.argtypes
    lib.saw_paged_decode_attn_plain.restype = ctypes.c_int
    lib.saw_decode_step_plain.argtypes = lib.saw_decode_step.argtypes
    lib.saw_decode_step_plain.restype = ctypes.c_int
    lib.saw_rotate_quantize_paged_strided.argtypes = [D, P, i64, P, i64, P, i64, P, P, P, P]
    lib.saw_rotate_quantize_paged_strided.restype = ctypes.c_int
    lib.saw_quantize_paged_plain_strided.argtypes = lib.saw_rotate_quantize_paged_strided.argtypes
    lib.saw_quantize_paged_plain_strided.restype = ctypes.c_int
    lib.saw_paged_prefill_workspace_bytes.argtypes = [D, i32, i32, i64]
    lib.saw_paged_prefill_workspace_bytes.restype = sz
    lib.saw_paged_prefill_attn.argtypes = [D, i32, P, P, i64, P, P, P, i32, P, i32, f32, P, P, sz,
                                           P, P]
    lib.saw_paged_prefill_attn.restype = ctypes.c_int
    lib.saw_paged_prefill_attn_plain.argtypes = lib.saw_paged_prefill_attn.argtypes
    lib.saw_paged_prefill_attn_plain.restype = ctypes.c_int
    lib.saw_append_bf16_paged.argtypes = [D, P, P, P, i64, P, P, P]
    lib.saw_append_bf16_paged.restype = ctypes.c_int
    lib.saw_paged_decode_bf16_workspace_bytes.argtypes = [D, i32, i32]
    lib.saw_paged_decode_bf16_workspace_bytes.restype = sz
    lib.saw_paged_decode_attn_bf16.argtypes = [D, i32, P, P, P, i32, P, i32, f32, P, P, sz, P, P]
    lib.saw_paged_decode_attn_bf16.restype = ctypes.c_int
    lib.saw_decode_step_bf16.argtypes = [D, i32, P, P, P, P, i64, P, P, i32, P, i32, f32, P, P,
                                         sz, P, P]
    lib.saw_decode_step_bf16.restype = ctypes.c_int
    Wc = ctypes.POINTER(saw_window_cache)
    lib.saw_paged_decode_window_workspace_bytes.argtypes = [D, i32, i32]
    lib.saw_paged_decode_window_workspace_bytes.restype = sz
    lib.saw_window_append.argtypes = [D, Wc, P, P, P, i32, P, P, P, i32, P, P]
    lib.saw_window_append.restype = ctypes.c_int
    lib.saw_paged_decode_attn_window.argtypes = [D, Wc, i32, P, P, P, P, i32, P, i32, f32, P, P,
                                                 sz, P, P]
    lib.saw_paged_decode_attn_window.restype = ctypes.c_int
    lib.saw_decode_step_window.argtypes = [D, Wc, i32, P, P, P, P, P, P, i32, P, i32, f32, P, P,
                                           sz, P, P]
    lib.saw_decode_step_window.restype = ctypes.c_int
    return lib


lib = _open_library()
lib.saw_paged_decode_attn_static.argtypes = [
    ctypes.POINTER(saw_cache_desc), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32,
    ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
lib.saw_paged_decode_attn_static.restype = ctypes.c_int


def saw_version() -> int:
    return int(lib.saw_version())


def saw_status_string(status: int) -> str:
    return lib.saw_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != SAW_OK:
        raise SawError(rc, where)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: torch.Tensor, name: str, dtype, ndim=None, cuda=True) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if cuda and t.device.type != "cuda":
        raise ValueError(f"{name} must be on a CUDA device")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def cache_desc(kv_pages: torch.Tensor) -> saw_cache_desc:
    """Descriptor of a cache tensor uint8 [num_pages][Hkv][2][16][D / 2] (D = 64, 128 or 256)."""
    _need(kv_pages, "kv_pages", torch.uint8, 5, cuda=False)
    num_pages, hkv, two, page, half = kv_pages.shape
    if two != 2 or half * 2 not in (64, 128, 256):
        raise ValueError(f"kv_pages must be [num_pages][Hkv][2][16][D / 2], got {tuple(kv_pages.shape)}")
    return saw_cache_desc(int(hkv), int(half * 2), int(page), int(num_pages))


def allocate_cache(num_pages: int, num_kv_heads: int, device="cuda", head_dim: int = HEAD_DIM):
    """Empty cache tensors: kv_pages uint8 [P][Hkv][2][16][D / 2], scales fp16 [P][Hkv][2][16][2]."""
    kv = torch.empty((num_pages, num_kv_heads, 2, PAGE_SIZE, head_dim // 2), dtype=torch.uint8,
                     device=device)
    sc = torch.empty((num_pages, num_kv_heads, 2, PAGE_SIZE, 2), dtype=torch.float16,
                     device=device)
    return kv, sc


def saw_rotate_quantize_paged(k, v, slot_mapping, kv_pages, scales, dev_status=None,
                              stream=None) -> None:
    """Rotate, quantize and scatter new tokens k, v (bf16 [T][Hkv][128]) into the cache."""
    _append(lib.saw_rotate_quantize_paged, "saw_rotate_quantize_paged", k, v, slot_mapping,
            kv_pages, scales, dev_status, stream)


def saw_quantize_paged_plain(k, v, slot_mapping, kv_pages, scales, dev_status=None,
                             stream=None) -> None:
    """Plain INT4 baseline: quantize and scatter without the Hadamard rotation."""
    _append(lib.saw_quantize_paged_plain, "saw_quantize_paged_plain", k, v, slot_mapping,
            kv_pages, scales, dev_status, stream)


def _append(fn, name, k, v, slot_mapping, kv_pages, scales, dev_status, stream) -> None:
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    desc = cache_desc(kv_pages)
    T = k.shape[0]
    if tuple(k.shape) != (T, desc.num_kv_heads, desc.head_dim) or v.shape != k.shape:
        raise ValueError("k and v must be [T][Hkv][D] matching the cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have one entry per token")
    if tuple(scales.shape) != (desc.num_pages, desc.num_kv_heads, 2, PAGE_SIZE, 2):
        raise ValueError("scales must be [num_pages][Hkv][2][16][2]")
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    rc = fn(ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(kv_pages),
            _ptr(scales), _ptr(dev_status), _stream(stream))
    _check(rc, name)


def saw_rotate_quantize_paged_strided(k, v, slot_mapping, kv_pages, scales, dev_status=None,
                                      stream=None, rotate=True) -> None:
    """saw_rotate_quantize_paged for k, v that are token-strided views (e.g. slices of a fused
    QKV output): [T][Hkv][128] with the heads of a token contiguous (strides (s, 128, 1)).
    rotate=False is the plain INT4 quantizer."""
    for t, name in ((k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.device.type != "cuda":
            raise TypeError(f"{name} must be a bf16 CUDA tensor")
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [T][Hkv][D] with contiguous heads within a token")
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    desc = cache_desc(kv_pages)
    T = k.shape[0]
    if tuple(k.shape) != (T, desc.num_kv_heads, desc.head_dim) or v.shape != k.shape:
        raise ValueError("k and v must be [T][Hkv][D] matching the cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have one entry per token")
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    fn = lib.saw_rotate_quantize_paged_strided if rotate else lib.saw_quantize_paged_plain_strided
    rc = fn(ctypes.byref(desc), _ptr(k), k.stride(0), _ptr(v), v.stride(0), _ptr(slot_mapping), T,
            _ptr(kv_pages), _ptr(scales), _ptr(dev_status), _stream(stream))
    _check(rc, "saw_rotate_quantize_paged_strided" if rotate else "saw_quantize_paged_plain_strided")


def saw_paged_decode_workspace_bytes(num_kv_heads: int, num_q_heads: int, num_seqs: int,
                                     num_pages: int = 1, head_dim: int = HEAD_DIM) -> int:
    desc = saw_cache_desc(int(num_kv_heads), int(head_dim), PAGE_SIZE, int(num_pages))
    return int(lib.saw_paged_decode_workspace_bytes(ctypes.byref(desc), int(num_q_heads),
                                                    int(num_seqs)))


def saw_paged_decode_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _need(workspace, "workspace", torch.uint8, 1)
    rc = lib.saw_paged_decode_workspace_init(_ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "saw_paged_decode_workspace_init")


def allocate_workspace(num_kv_heads: int, num_q_heads: int, num_seqs: int,
                       device="cuda", head_dim: int = HEAD_DIM) -> torch.Tensor:
    """A zero-initialised decode workspace for this shape on the current device."""
    n = saw_paged_decode_workspace_bytes(num_kv_heads, num_q_heads, num_seqs, head_dim=head_dim)
    if n == 0:
        raise SawError(SAW_ERR_CUDA, "saw_paged_decode_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    saw_paged_decode_workspace_init(ws)
    return ws


def _decode_checks(q, kv_pages, scales, block_table, seq_lens, out, workspace, dev_status):
    _need(q, "q", torch.bfloat16, 3)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(out, "out", torch.float32, 3)
    _need(workspace, "workspace", torch.uint8, 1)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    desc = cache_desc(kv_pages)
    S, hq, d = q.shape
    if d != desc.head_dim or tuple(out.shape) != (S, hq, desc.head_dim):
        raise ValueError(f"q and out must be [S][Hq][{desc.head_dim}] matching the cache")
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_table and seq_lens need one row per sequence")
    return desc, S, hq


def saw_paged_decode_attn(q, kv_pages, scales, block_table, seq_lens, out, workspace,
                          sm_scale=None, dev_status=None, stream=None) -> None:
    """Decode attention of q (bf16 [S][Hq][D], D = 128 or 256 as the cache) over the INT4 paged
    cache into out (fp32 [S][Hq][D])."""
    _decode(lib.saw_paged_decode_attn, "saw_paged_decode_attn", q, kv_pages, scales, block_table,
            seq_lens, out, workspace, sm_scale, dev_status, stream)


def saw_paged_decode_attn_plain(q, kv_pages, scales, block_table, seq_lens, out, workspace,
                                sm_scale=None, dev_status=None, stream=None) -> None:
    """Decode over a plain INT4 cache (written by saw_quantize_paged_plain)."""
    _decode(lib.saw_paged_decode_attn_plain, "saw_paged_decode_attn_plain", q, kv_pages, scales,
            block_table, seq_lens, out, workspace, sm_scale, dev_status, stream)


def _decode(fn, name, q, kv_pages, scales, block_table, seq_lens, out, workspace, sm_scale,
            dev_status, stream) -> None:
    desc, S, hq = _decode_checks(q, kv_pages, scales, block_table, seq_lens, out, workspace,
                                 dev_status)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(desc.head_dim)
    rc = fn(ctypes.byref(desc), hq, _ptr(q), _ptr(kv_pages), _ptr(scales), _ptr(block_table),
            block_table.shape[1], _ptr(seq_lens), S, float(sm_scale), _ptr(out), _ptr(workspace),
            workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(rc, name)


def saw_decode_step(q, k_new, v_new, slot_mapping, kv_pages, scales, block_table, seq_lens, out,
                    workspace, sm_scale=None, dev_status=None, stream=None) -> None:
    """Append k_new / v_new (bf16 [T][Hkv][128]) at slot_mapping, then decode q."""
    _step(lib.saw_decode_step, "saw_decode_step", q, k_new, v_new, slot_mapping, kv_pages, scales,
          block_table, seq_lens, out, workspace, sm_scale, dev_status, stream)


def saw_decode_step_plain(q, k_new, v_new, slot_mapping, kv_pages, scales, block_table, seq_lens,
                          out, workspace, sm_scale=None, dev_status=None, stream=None) -> None:
    """The serving step on a plain INT4 cache (no rotation)."""
    _step(lib.saw_decode_step_plain, "saw_decode_step_plain", q, k_new, v_new, slot_mapping,
          kv_pages, scales, block_table, seq_lens, out, workspace, sm_scale, dev_status, stream)


def _step(fn, name, q, k_new, v_new, slot_mapping, kv_pages, scales, block_table, seq_lens, out,
          workspace, sm_scale, dev_status, stream) -> None:
    desc, S, hq = _decode_checks(q, kv_pages, scales, block_table, seq_lens, out, workspace,
                                 dev_status)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    T = k_new.shape[0]
    if tuple(k_new.shape) != (T, desc.num_kv_heads, desc.head_dim) or v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must be [T][Hkv][D] matching the cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have one entry per new token")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(desc.head_dim)
    rc = fn(ctypes.byref(desc), hq, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T,
            _ptr(kv_pages), _ptr(scales), _ptr(block_table), block_table.shape[1], _ptr(seq_lens),
            S, float(sm_scale), _ptr(out), _ptr(workspace), workspace.numel(), _ptr(dev_status),
            _stream(stream))
    _check(rc, name)


def saw_paged_decode_attn_static(q, kv_pages, scales, block_table, seq_lens, out, sm_scale=None,
                                 dev_status=None, stream=None) -> None:
    """saw_paged_decode_attn without a workspace, for callers that cannot allocate device memory:
    the scratch is a fixed array inside the library (num_seqs * num_kv_heads * ceil(G / 8)
    <= 2048).  Calls
    share that array, so calls that can overlap on the GPU must be serialised by the caller."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(out, "out", torch.float32, 3)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    desc = cache_desc(kv_pages)
    S, hq, _ = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(desc.head_dim)
    rc = lib.saw_paged_decode_attn_static(ctypes.byref(desc), hq, _ptr(q), _ptr(kv_pages),
                                          _ptr(scales), _ptr(block_table), block_table.shape[1],
                                          _ptr(seq_lens), S, float(sm_scale), _ptr(out),
                                          _ptr(dev_status), _stream(stream))
    _check(rc, "saw_paged_decode_attn_static")


# ---- the uncompressed BF16 paged cache (baseline) --------------------------------------------

def cache_desc_bf16(kv_bf16: torch.Tensor) -> saw_cache_desc:
    """Descriptor of a bf16 cache tensor [num_pages][Hkv][2][16][128]."""
    _need(kv_bf16, "kv_bf16", torch.bfloat16, 5, cuda=False)
    num_pages, hkv, two, page, d = kv_bf16.shape
    if two != 2 or d != HEAD_DIM:
        raise ValueError(f"kv_bf16 must be [num_pages][Hkv][2][16][128], got {tuple(kv_bf16.shape)}")
    return saw_cache_desc(int(hkv), HEAD_DIM, int(page), int(num_pages))


def allocate_cache_bf16(num_pages: int, num_kv_heads: int, device="cuda") -> torch.Tensor:
    """Empty bf16 cache [P][Hkv][2][16][128]."""
    return torch.empty((num_pages, num_kv_heads, 2, PAGE_SIZE, HEAD_DIM), dtype=torch.bfloat16,
                       device=device)


def saw_append_bf16_paged(k, v, slot_mapping, kv_bf16, dev_status=None, stream=None) -> None:
    """Scatter new tokens k, v (bf16 [T][Hkv][128]) into the bf16 cache."""
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    desc = cache_desc_bf16(kv_bf16)
    _need(kv_bf16, "kv_bf16", torch.bfloat16, 5)
    T = k.shape[0]
    if tuple(k.shape) != (T, desc.num_kv_heads, HEAD_DIM) or v.shape != k.shape:
        raise ValueError("k and v must be [T][Hkv][128] matching the cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have one entry per token")
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    rc = lib.saw_append_bf16_paged(ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(slot_mapping), T,
                                   _ptr(kv_bf16), _ptr(dev_status), _stream(stream))
    _check(rc, "saw_append_bf16_paged")


def saw_paged_decode_bf16_workspace_bytes(num_kv_heads: int, num_q_heads: int,
                                          num_seqs: int) -> int:
    desc = saw_cache_desc(int(num_kv_heads), HEAD_DIM, PAGE_SIZE, 1)
    return int(lib.saw_paged_decode_bf16_workspace_bytes(ctypes.byref(desc), int(num_q_heads),
                                                         int(num_seqs)))


def allocate_workspace_bf16(num_kv_heads: int, num_q_heads: int, num_seqs: int,
                            device="cuda") -> torch.Tensor:
    n = saw_paged_decode_bf16_workspace_bytes(num_kv_heads, num_q_heads, num_seqs)
    if n == 0:
        raise SawError(SAW_ERR_CUDA, "saw_paged_decode_bf16_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _decode_checks_bf16(q, kv_bf16, block_table, seq_lens, out, workspace, dev_status):
    _need(q, "q", torch.bfloat16, 3)
    _need(kv_bf16, "kv_bf16", torch.bfloat16, 5)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(out, "out", torch.float32, 3)
    _need(workspace, "workspace", torch.uint8, 1)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    desc = cache_desc_bf16(kv_bf16)
    S, hq, d = q.shape
    if d != HEAD_DIM or tuple(out.shape) != (S, hq, HEAD_DIM):
        raise ValueError("q and out must be [S][Hq][128]")
    if block_table.shape[0] != S or seq_lens.shape[0] != S:
        raise ValueError("block_table and seq_lens need one row per sequence")
    return desc, S, hq


def saw_paged_decode_attn_bf16(q, kv_bf16, block_table, seq_lens, out, workspace, sm_scale=None,
                               dev_status=None, stream=None) -> None:
    """Decode attention of q (bf16 [S][Hq][128]) over the bf16 paged cache into out (fp32)."""
    desc, S, hq = _decode_checks_bf16(q, kv_bf16, block_table, seq_lens, out, workspace,
                                      dev_status)
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(HEAD_DIM)
    rc = lib.saw_paged_decode_attn_bf16(ctypes.byref(desc), hq, _ptr(q), _ptr(kv_bf16),
                                        _ptr(block_table), block_table.shape[1], _ptr(seq_lens),
                                        S, float(sm_scale), _ptr(out), _ptr(workspace),
                                        workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(rc, "saw_paged_decode_attn_bf16")


def saw_decode_step_bf16(q, k_new, v_new, slot_mapping, kv_bf16, block_table, seq_lens, out,
                         workspace, sm_scale=None, dev_status=None, stream=None) -> None:
    """The serving step on the bf16 cache: append k_new / v_new, then decode q."""
    desc, S, hq = _decode_checks_bf16(q, kv_bf16, block_table, seq_lens, out, workspace,
                                      dev_status)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int64, 1)
    T = k_new.shape[0]
    if tuple(k_new.shape) != (T, desc.num_kv_heads, desc.head_dim) or v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must be [T][Hkv][D] matching the cache")
    if slot_mapping.shape[0] != T:
        raise ValueError("slot_mapping must have one entry per new token")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(desc.head_dim)
    rc = lib.saw_decode_step_bf16(ctypes.byref(desc), hq, _ptr(q), _ptr(k_new), _ptr(v_new),
                                  _ptr(slot_mapping), T, _ptr(kv_bf16), _ptr(block_table),
                                  block_table.shape[1], _ptr(seq_lens), S, float(sm_scale),
                                  _ptr(out), _ptr(workspace), workspace.numel(), _ptr(dev_status),
                                  _stream(stream))
    _check(rc, "saw_decode_step_bf16")


# ---- chunked-prefill attention over the INT4 cache -------------------------------------------

def saw_paged_prefill_workspace_bytes(num_kv_heads: int, num_q_heads: int, num_seqs: int,
                                      total_q: int, head_dim: int = HEAD_DIM) -> int:
    desc = saw_cache_desc(int(num_kv_heads), int(head_dim), PAGE_SIZE, 1)
    return int(lib.saw_paged_prefill_workspace_bytes(ctypes.byref(desc), int(num_q_heads),
                                                     int(num_seqs), int(total_q)))


def allocate_prefill_workspace(num_kv_heads: int, num_q_heads: int, num_seqs: int, total_q: int,
                               device="cuda", head_dim: int = HEAD_DIM) -> torch.Tensor:
    n = saw_paged_prefill_workspace_bytes(num_kv_heads, num_q_heads, num_seqs, total_q,
                                          head_dim=head_dim)
    if n == 0:
        raise SawError(SAW_ERR_CUDA, "saw_paged_prefill_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def saw_paged_prefill_attn(q, q_start, kv_pages, scales, block_table, seq_lens, out, workspace,
                           sm_scale=None, dev_status=None, stream=None, rotate=True) -> None:
    """Causal attention of a chunk of query tokens (bf16 [total_q][Hq][D], sequence s owning
    rows q_start[s] .. q_start[s + 1] - 1, the last tokens of its cached seq_lens[s]) over the
    INT4 paged cache into out (fp32 [total_q][Hq][D]).  rotate=False reads a plain INT4
    cache."""
    _need(q_start, "q_start", torch.int32, 1)
    _need(q, "q", torch.bfloat16, 3)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    _need(out, "out", torch.float32, 3)
    _need(workspace, "workspace", torch.uint8, 1)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    desc = cache_desc(kv_pages)
    total_q, hq, d = q.shape
    S = seq_lens.shape[0]
    if d != desc.head_dim or tuple(out.shape) != (total_q, hq, desc.head_dim):
        raise ValueError(f"q and out must be [total_q][Hq][{desc.head_dim}] matching the cache")
    if q_start.shape[0] != S + 1 or block_table.shape[0] != S:
        raise ValueError("q_start needs num_seqs + 1 entries and block_table one row per sequence")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(desc.head_dim)
    fn = lib.saw_paged_prefill_attn if rotate else lib.saw_paged_prefill_attn_plain
    rc = fn(ctypes.byref(desc), hq, _ptr(q), _ptr(q_start), total_q, _ptr(kv_pages), _ptr(scales),
            _ptr(block_table), block_table.shape[1], _ptr(seq_lens), S, float(sm_scale), _ptr(out),
            _ptr(workspace), workspace.numel(), _ptr(dev_status), _stream(stream))
    _check(rc, "saw_paged_prefill_attn" if rotate else "saw_paged_prefill_attn_plain")


# ---- full-precision sink / recent window beside the INT4 cache --------------------------------

def allocate_window(num_seqs: int, num_kv_heads: int, sink: int, recent: int, device="cuda"):
    """Window pages for num_seqs sequences: kv bf16 [num_seqs * blocks][Hkv][2][16][128] and the
    table int32 [num_seqs][blocks] giving sequence s the pages s * blocks .. (blocks = the
    16-token pages sink + recent tokens need, at least 1)."""
    blocks = max(1, (sink + recent + PAGE_SIZE - 1) // PAGE_SIZE)
    kv = torch.zeros((num_seqs * blocks, num_kv_heads, 2, PAGE_SIZE, HEAD_DIM), dtype=torch.bfloat16,
                     device=device)
    table = torch.arange(num_seqs * blocks, dtype=torch.int32, device=device).view(num_seqs, blocks)
    return kv, table


def window_desc(sink: int, recent: int, win_kv: torch.Tensor, win_table: torch.Tensor):
    """The saw_window_cache of window pages win_kv (bf16 [P][Hkv][2][16][128]) and their table
    (int32 [num_seqs][blocks])."""
    _need(win_kv, "win_kv", torch.bfloat16, 5)
    _need(win_table, "win_table", torch.int32, 2)
    if tuple(win_kv.shape[2:]) != (2, PAGE_SIZE, HEAD_DIM):
        raise ValueError(f"win_kv must be [P][Hkv][2][16][128], got {tuple(win_kv.shape)}")
    return saw_window_cache(int(sink), int(recent), _ptr(win_kv), int(win_kv.shape[0]),
                            _ptr(win_table), int(win_table.shape[1]))


def saw_paged_decode_window_workspace_bytes(num_kv_heads: int, num_q_heads: int,
                                            num_seqs: int) -> int:
    desc = saw_cache_desc(int(num_kv_heads), HEAD_DIM, PAGE_SIZE, 1)
    return int(lib.saw_paged_decode_window_workspace_bytes(ctypes.byref(desc), int(num_q_heads),
                                                           int(num_seqs)))


def allocate_window_workspace(num_kv_heads: int, num_q_heads: int, num_seqs: int,
                              device="cuda") -> torch.Tensor:
    n = saw_paged_decode_window_workspace_bytes(num_kv_heads, num_q_heads, num_seqs)
    if n == 0:
        raise SawError(SAW_ERR_CUDA, "saw_paged_decode_window_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _window_checks(win, kv_pages, scales, block_table, seq_lens, dev_status):
    sink, recent, win_kv, win_table = win
    wd = window_desc(sink, recent, win_kv, win_table)
    _need(kv_pages, "kv_pages", torch.uint8, 5)
    _need(scales, "scales", torch.float16, 5)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    if dev_status is not None:
        _need(dev_status, "dev_status", torch.int32, 1)
    desc = cache_desc(kv_pages)
    S = seq_lens.shape[0]
    if block_table.shape[0] != S or win_table.shape[0] != S:
        raise ValueError("block_table and the window table need one row per sequence")
    return wd, desc, S


def saw_window_append(k, v, seq_lens, win, kv_pages, scales, block_table, dev_status=None,
                      stream=None) -> None:
    """One step's write into a windowed cache: k, v (bf16 [S][Hkv][128]) are the new tokens at
    positions seq_lens - 1; win = (sink, recent, win_kv, win_table).  The token each one displaces
    from the recent window is rotated, quantized and scattered into the INT4 pages."""
    wd, desc, S = _window_checks(win, kv_pages, scales, block_table, seq_lens, dev_status)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    if tuple(k.shape) != (S, desc.num_kv_heads, HEAD_DIM) or v.shape != k.shape:
        raise ValueError("k and v must be [S][Hkv][128] matching the cache")
    rc = lib.saw_window_append(ctypes.byref(desc), ctypes.byref(wd), _ptr(k), _ptr(v),
                               _ptr(seq_lens), S, _ptr(kv_pages), _ptr(scales), _ptr(block_table),
                               block_table.shape[1], _ptr(dev_status), _stream(stream))
    _check(rc, "saw_window_append")


def saw_paged_decode_attn_window(q, win, kv_pages, scales, block_table, seq_lens, out, workspace,
                                 sm_scale=None, dev_status=None, stream=None) -> None:
    """Decode attention of q (bf16 [S][Hq][128]) over each sequence's bf16 window and its
    quantized tokens, one softmax over both, into out (fp32 [S][Hq][128])."""
    wd, desc, S = _window_checks(win, kv_pages, scales, block_table, seq_lens, dev_status)
    _need(q, "q", torch.bfloat16, 3)
    _need(out, "out", torch.float32, 3)
    _need(workspace, "workspace", torch.uint8, 1)
    hq = q.shape[1]
    if tuple(q.shape) != (S, hq, HEAD_DIM) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [S][Hq][128]")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(HEAD_DIM)
    rc = lib.saw_paged_decode_attn_window(ctypes.byref(desc), ctypes.byref(wd), hq, _ptr(q),
                                          _ptr(kv_pages), _ptr(scales), _ptr(block_table),
                                          block_table.shape[1], _ptr(seq_lens), S, float(sm_scale),
                                          _ptr(out), _ptr(workspace), workspace.numel(),
                                          _ptr(dev_status), _stream(stream))
    _check(rc, "saw_paged_decode_attn_window")


def saw_decode_step_window(q, k_new, v_new, win, kv_pages, scales, block_table, seq_lens, out,
                           workspace, sm_scale=None, dev_status=None, stream=None) -> None:
    """saw_window_append then saw_paged_decode_attn_window on one stream."""
    wd, desc, S = _window_checks(win, kv_pages, scales, block_table, seq_lens, dev_status)
    for t, name in ((q, "q"), (k_new, "k_new"), (v_new, "v_new")):
        _need(t, name, torch.bfloat16, 3)
    _need(out, "out", torch.float32, 3)
    _need(workspace, "workspace", torch.uint8, 1)
    hq = q.shape[1]
    if tuple(k_new.shape) != (S, desc.num_kv_heads, HEAD_DIM) or v_new.shape != k_new.shape:
        raise ValueError("k_new and v_new must be [S][Hkv][128] matching the cache")
    if tuple(q.shape) != (S, hq, HEAD_DIM) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q and out must be [S][Hq][128]")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(HEAD_DIM)
    rc = lib.saw_decode_step_window(ctypes.byref(desc), ctypes.byref(wd), hq, _ptr(q),
                                    _ptr(k_new), _ptr(v_new), _ptr(kv_pages), _ptr(scales),
                                    _ptr(block_table), block_table.shape[1], _ptr(seq_lens), S,
                                    float(sm_scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                    _ptr(dev_status), _stream(stream))
    _check(rc, "saw_decode_step_window")

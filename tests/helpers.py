"""Shared helpers for the parity tests: the same seeded inputs go to the CUDA path (through
the C ABI) and to the CPU oracle.  No expected value here comes from the CUDA path."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from bit_paged_kv_block_b200 import synth

NTHREADS = max(1, os.cpu_count() or 1)
# Never-written cache rows: codes 0xA5 and fp16 NaN (0x7E00) in every scale and zero slot.  A
# cache a caller allocates with torch.empty may hold NaN bits in the rows past a sequence's end;
# the read kernels must keep them out of the result (a masked token's weight is 0, and 0 * NaN
# is NaN), so every parity test runs on such a cache.  The oracle reads only the valid tokens,
# and the cache comparisons are bitwise, so the NaN bits compare like any other canary.
CANARY_CODE = 0xA5
CANARY_SCALE = 0x7E00

# attention tolerance against the fp64 oracle
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_cache(wl, tokens="all", k=None, v=None, rotate=True):
    """Oracle cache (numpy) holding the selected tokens of the workload, canary elsewhere."""
    if k is None:
        k = synth.kv_values(wl, "K", tokens=tokens)
    if v is None:
        v = synth.kv_values(wl, "V", tokens=tokens)
    seq, pos = synth.token_index(wl, tokens)
    slots = synth.slot_mapping(wl, seq, pos)
    pages, scales = oracle.empty_cache(wl.num_pages, wl.num_kv_heads, wl.head_dim)
    pages[:] = CANARY_CODE
    scales[:] = CANARY_SCALE
    bad = oracle.rotate_quantize_paged(u16(k), u16(v), slots, pages, scales, rotate=rotate,
                                       nthreads=NTHREADS)
    assert bad == 0
    return pages, scales


def device_cache_from(pages: np.ndarray, scales: np.ndarray, device):
    kv = torch.from_numpy(pages).to(device)
    sc = torch.from_numpy(scales.view(np.int16)).view(torch.float16).to(device)
    return kv, sc


def canary_device_cache(wl, device):
    from bit_paged_kv_block_b200 import saw
    kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, device, head_dim=wl.head_dim)
    kv.fill_(CANARY_CODE)
    sc.view(torch.int16).fill_(CANARY_SCALE)
    return kv, sc


def attention_errors(got: np.ndarray, want: np.ndarray):
    d = np.abs(got.astype(np.float64) - want)
    return float(d.max()), float(d.mean())


def assert_attention_close(got, want, what=""):
    mx, mean = attention_errors(got, want)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def subset(wl, seqs):
    """The workload restricted to the given sequences (same pages and page ids)."""
    seqs = np.asarray(seqs)
    sub = synth.Workload(**{**wl.__dict__})
    sub.num_seqs = len(seqs)
    sub.seq_lens = wl.seq_lens[seqs].copy()
    sub.new_tokens = wl.new_tokens[seqs].copy()
    sub.block_table = np.ascontiguousarray(wl.block_table[seqs])
    return sub


EDGE_KINDS = ["small_ints", "zeros_and_constants", "tiny_magnitudes", "huge_range",
              "signed_zero", "single_spike", "scale_above_2m100", "scale_below_2m100"]


def edge_kv(kind: str, T: int, Hkv: int, D: int = 128):
    """bf16 K, V [T][Hkv][D] whose quantization hits a corner of the code computation:
    exact half-way quotients (small integers, before or after rotation), degenerate and
    constant vectors, subnormal scales, scales just above and just below 2^-100 (the smallest
    scale the kernel settles ties without a divide), huge dynamic range, signed zeros and one
    large spike per vector."""
    g = torch.Generator().manual_seed(7)
    if kind == "small_ints":
        x = torch.randint(-3, 4, (T, Hkv, D), generator=g).float()
    elif kind == "zeros_and_constants":
        x = torch.zeros(T, Hkv, D)
        x[1::3] = torch.randn(T, Hkv, 1, generator=g)[1::3]
        x[2::5, :, 7] = 1.0
    elif kind == "tiny_magnitudes":
        x = torch.randn(T, Hkv, D, generator=g) * 1e-37
        x[::2] *= 1e-2
    elif kind == "huge_range":
        x = torch.randn(T, Hkv, D, generator=g) * (10.0 ** torch.randint(-3, 4, (T, Hkv, 1), generator=g))
    elif kind == "signed_zero":
        x = torch.zeros(T, Hkv, D)
        x[::2, :, 3] = -0.0
        x[1::2, :, 5] = 1.0
        x[::4] = -x[::4]
    elif kind in ("scale_above_2m100", "scale_below_2m100"):
        # small integers times 2^-96 or 2^-103: scales just above and below 2^-100
        e = -96 if kind == "scale_above_2m100" else -103
        x = torch.randint(-3, 4, (T, Hkv, D), generator=g).float() * 2.0 ** e
    elif kind == "single_spike":
        x = torch.zeros(T, Hkv, D)
        x[torch.arange(T), :, torch.arange(T) % D] = 50.0
    else:
        raise ValueError(kind)
    return x.to(torch.bfloat16), (x.flip(-1) * 0.5).to(torch.bfloat16)

"""saw_paged_decode_attn_static: decode for callers that cannot allocate device memory.

Some callers of this library can't call cudaMalloc: a plug-in inside a serving framework whose
memory pool already owns the GPU, a request path that must not allocate (cudaMalloc
synchronises the device), or a host library that only receives input and output pointers.
For them the library has an entry point whose scratch is a fixed array in its own device code.
This test calls it through the C ABI and checks it against the workspace-based entry point on
the same inputs, twice in a row, after a call on a larger, different shape has left other data
in the array (the array keeps the previous call's contents).  Both entry points run the same
kernels and fold split results in a fixed order, so the outputs must be bit-identical.  It also
checks that shapes beyond the array's limit are refused with their own status.  The file sorts last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from bit_paged_kv_block_b200 import synth
from helpers import device_cache_from, oracle_cache

pytestmark = pytest.mark.gpu


def _static_call(saw, desc, q, kv, sc, table, lens, out, status):
    P = ctypes.c_void_p
    return saw.lib.saw_paged_decode_attn_static(
        ctypes.byref(desc), q.shape[1], P(q.data_ptr()), P(kv.data_ptr()), P(sc.data_ptr()),
        P(table.data_ptr()), table.shape[1], P(lens.data_ptr()), q.shape[0],
        1.0 / math.sqrt(128.0), P(out.data_ptr()), P(status.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))


def _dirty_scratch(saw, dev):
    """Run the fixed-scratch decode once on a larger shape than the checked ones (200 sequences
    of up to 8192 tokens, 1600 segments, random cache contents), so that the array holds other
    data when the checked calls start."""
    rng = np.random.default_rng(99)
    lens = rng.integers(1, 8193, size=200)
    wl = synth.custom("dirty", lens, num_q_heads=32, num_kv_heads=8, seed=99)
    g = torch.Generator(device=dev).manual_seed(99)
    kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
    kv.copy_(torch.randint(0, 256, kv.shape, dtype=torch.uint8, device=dev, generator=g))
    sc.copy_((torch.rand(sc.shape, device=dev, generator=g) * 0.1).to(torch.float16))
    q = torch.randn((wl.num_seqs, 32, 128), device=dev, generator=g).to(torch.bfloat16)
    out = torch.empty((wl.num_seqs, 32, 128), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = _static_call(saw, saw.cache_desc(kv), q, kv, sc, torch.from_numpy(wl.block_table).to(dev),
                      torch.from_numpy(wl.seq_lens).to(dev), out, status)
    assert rc == saw.SAW_OK, saw.saw_status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


@pytest.mark.parametrize("name", ["decode", "mixed"])
def test_static_scratch_matches_workspace_entry_point(cuda_device, name):
    from bit_paged_kv_block_b200 import saw
    dev = cuda_device
    if name == "decode":
        wl = synth.make_workload("decode")
    else:   # short and long sequences, one empty: several CTAs per sequence and many per CTA
        lens = [1, 17, 3000, 0, 64, 9000, 250, 16]
        wl = synth.custom("mixed", lens, num_q_heads=32, num_kv_heads=8, seed=3)
    pages, scales = oracle_cache(wl)
    kv, sc = device_cache_from(pages, scales, dev)
    q = synth.q_values(wl).to(dev)
    table = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    ref = torch.empty((wl.num_seqs, wl.num_q_heads, 128), dtype=torch.float32, device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    saw.saw_paged_decode_attn(q, kv, sc, table, lens, ref, ws, dev_status=status)
    torch.cuda.synchronize()
    ref = ref.cpu()
    assert torch.isfinite(ref).all()

    _dirty_scratch(saw, dev)
    desc = saw.cache_desc(kv)
    for call in range(2):
        out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=dev)
        rc = _static_call(saw, desc, q, kv, sc, table, lens, out, status)
        assert rc == saw.SAW_OK, saw.saw_status_string(rc)
        torch.cuda.synchronize()
        got = out.cpu()
        assert torch.equal(got, ref), \
            f"call {call}: max difference {float((got - ref).abs().max()):.3e}"
    assert int(status.item()) == 0


def test_static_scratch_rejects_shapes_beyond_its_limit(cuda_device):
    from bit_paged_kv_block_b200 import saw
    dev = cuda_device
    S, hkv = 257, 8                       # 2056 (sequence, kv head) pairs > 2048
    kv, sc = saw.allocate_cache(1, hkv, dev)
    q = torch.zeros((S, 32, 128), dtype=torch.bfloat16, device=dev)
    out = torch.zeros((S, 32, 128), dtype=torch.float32, device=dev)
    table = torch.zeros((S, 1), dtype=torch.int32, device=dev)
    lens = torch.ones(S, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rc = _static_call(saw, saw.cache_desc(kv), q, kv, sc, table, lens, out, status)
    assert rc == saw.SAW_ERR_SCRATCH_LIMIT
    assert "2048" in saw.saw_status_string(rc)
    torch.cuda.synchronize()
    assert not bool(out.any())            # nothing was queued

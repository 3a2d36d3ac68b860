"""The plain INT4 baseline (H = I) on the GPU: bit-exact codes and scales against the oracle with
its rotation switched off, decode within tolerance of the oracle's fp64 decode of the same cache,
and the method-level comparison run through the CUDA path: on keys with outlier channels the
rotated cache gives lower attention error than the plain one ("SAW-INT4", Concerns Raised:
naive INT4 degrades accuracy; Research Findings: the rotation recovers nearly all of it)."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import (EDGE_KINDS, NTHREADS, assert_attention_close, canary_device_cache,
                     device_cache_from, edge_kv, oracle_cache, subset, u16)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_plain_quantize_bit_exact(cuda_device, name):
    from bit_paged_kv_block_b200 import saw
    wl = synth.make_workload(name)
    k, v = synth.kv_values(wl, "K"), synth.kv_values(wl, "V")
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
    kv, sc = canary_device_cache(wl, cuda_device)
    saw.saw_quantize_paged_plain(k.to(cuda_device), v.to(cuda_device), slots, kv, sc)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k, v=v, rotate=False)
    assert np.array_equal(kv.cpu().numpy(), pages)
    assert np.array_equal(u16(sc), scales)


@pytest.mark.parametrize("kind", EDGE_KINDS)
def test_plain_quantize_edge_values(cuda_device, kind):
    """Unrotated bf16 values land on exact half-way quotients all the time; these inputs add
    degenerate vectors, subnormal scales and scales around 2^-100."""
    from bit_paged_kv_block_b200 import saw
    T, hkv = 137, 3
    k, v = edge_kv(kind, T, hkv)
    wl = synth.custom(kind, [T], num_q_heads=hkv, num_kv_heads=hkv, new_tokens=[T])
    seq, pos = synth.token_index(wl)
    kv, sc = canary_device_cache(wl, cuda_device)
    saw.saw_quantize_paged_plain(k.to(cuda_device), v.to(cuda_device),
                                 torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device),
                                 kv, sc)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k, v=v, rotate=False)
    assert np.array_equal(kv.cpu().numpy(), pages)
    assert np.array_equal(u16(sc), scales)


def _decode_plain(wl, pages, scales, dev, q):
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, dev)
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    saw.saw_paged_decode_attn_plain(q.to(dev), kv, sc, torch.from_numpy(wl.block_table).to(dev),
                                    torch.from_numpy(wl.seq_lens).to(dev), out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("G,lens", [(1, [1, 17]), (4, [15, 16, 33, 300]), (8, [1000, 5])])
def test_plain_decode_matches_oracle(cuda_device, G, lens):
    hkv = 2
    wl = synth.custom(f"plain{G}", lens, num_q_heads=G * hkv, num_kv_heads=hkv, seed=G,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl, rotate=False)
    q = synth.q_values(wl)
    got = _decode_plain(wl, pages, scales, cuda_device, q)
    want = oracle.decode_fp64(u16(q), pages, scales, wl.block_table, wl.seq_lens, rotate=False,
                              nthreads=NTHREADS)
    assert_attention_close(got, want, "plain")


def test_plain_step_full_size(cuda_device):
    from bit_paged_kv_block_b200 import saw
    wl = synth.make_workload("decode")
    dev = cuda_device
    hist_pages, hist_scales = oracle_cache(wl, tokens="history", rotate=False)
    kv, sc = device_cache_from(hist_pages, hist_scales, dev)
    k_new = synth.kv_values(wl, "K", tokens="new")
    v_new = synth.kv_values(wl, "V", tokens="new")
    seq, pos = synth.token_index(wl, "new")
    slots = synth.slot_mapping(wl, seq, pos)
    q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    saw.saw_decode_step_plain(q.to(dev), k_new.to(dev), v_new.to(dev),
                              torch.from_numpy(slots).to(dev), kv, sc,
                              torch.from_numpy(wl.block_table).to(dev),
                              torch.from_numpy(wl.seq_lens).to(dev), out, ws)
    torch.cuda.synchronize()
    full_pages, full_scales = hist_pages.copy(), hist_scales.copy()
    oracle.rotate_quantize_paged(u16(k_new), u16(v_new), slots, full_pages, full_scales,
                                 rotate=False)
    assert np.array_equal(kv.cpu().numpy(), full_pages)
    assert np.array_equal(u16(sc), full_scales)
    sample = [0, 31, 63]
    want = oracle.decode_fp64(u16(q[sample]), full_pages, full_scales,
                              subset(wl, sample).block_table, wl.seq_lens[sample], rotate=False,
                              nthreads=NTHREADS)
    assert_attention_close(out.cpu().numpy()[sample], want, "plain step")


def test_rotation_lowers_gpu_attention_error_on_outlier_keys(cuda_device):
    """Both caches built and decoded on the GPU; errors against unquantized fp64 attention."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("method", [2048, 700], num_q_heads=8, num_kv_heads=2, seed=4,
                      outlier_scale=20.0)
    dev = cuda_device
    k, v, q = synth.kv_values(wl, "K"), synth.kv_values(wl, "V"), synth.q_values(wl)
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(dev)
    table = torch.from_numpy(wl.block_table).to(dev)
    lens = torch.from_numpy(wl.seq_lens).to(dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    outs = {}
    for rotate in (True, False):
        kv, sc = saw.allocate_cache(wl.num_pages, wl.num_kv_heads, dev)
        out = torch.empty((wl.num_seqs, wl.num_q_heads, 128), device=dev)
        if rotate:
            saw.saw_rotate_quantize_paged(k.to(dev), v.to(dev), slots, kv, sc)
            saw.saw_paged_decode_attn(q.to(dev), kv, sc, table, lens, out, ws)
        else:
            saw.saw_quantize_paged_plain(k.to(dev), v.to(dev), slots, kv, sc)
            saw.saw_paged_decode_attn_plain(q.to(dev), kv, sc, table, lens, out, ws)
        torch.cuda.synchronize()
        outs[rotate] = out.cpu().double()
    kd, vd, qd = k.double(), v.double(), q.double()
    err = {True: [], False: []}
    start = 0
    for s_, L in enumerate(wl.seq_lens.tolist()):
        for hq in range(wl.num_q_heads):
            h = hq // wl.group
            ref = torch.nn.functional.scaled_dot_product_attention(
                qd[s_, hq][None, None, None], kd[start:start + L, h][None, None],
                vd[start:start + L, h][None, None])[0, 0, 0]
            for rot in (True, False):
                err[rot].append((outs[rot][s_, hq] - ref).abs().mean().item())
        start += L
    assert np.mean(err[True]) < np.mean(err[False])

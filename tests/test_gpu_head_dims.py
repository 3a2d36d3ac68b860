"""Head dimensions 64 and 256 on the GPU against the fp64 oracle: decode, chunked prefill and
the fused serving step over an INT4 cache whose vectors carry one (scale, zero) pair each; a
256-element vector is rotated as two independent 128-point blocks, a 64-element vector by the
64-point transform (it holds no 128-point block) ("SAW-INT4", Research Findings: block-diagonal
Hadamard rotation and token-wise INT4).  Tolerance as for D = 128: max abs 1e-2, mean abs 1e-3;
appended codes bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import (NTHREADS, assert_attention_close, device_cache_from, oracle_cache, subset,
                     u16)

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[64, 256], ids=lambda d: f"D{d}")
def D(request):
    return request.param


def _wl(name, lens, G, hkv, seed, D):
    return synth.custom(f"{name}_{D}", lens, num_q_heads=G * hkv, num_kv_heads=hkv, seed=seed,
                        outlier_range=(10.0, 30.0), head_dim=D)


def _decode(wl, pages, scales, device, rotate=True, q=None, ws=None):
    D = wl.head_dim
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, device)
    if q is None:
        q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, D), float("nan"), device=device)
    if ws is None:
        ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, device,
                                    head_dim=D)
    fn = saw.saw_paged_decode_attn if rotate else saw.saw_paged_decode_attn_plain
    fn(q.to(device), kv, sc, torch.from_numpy(wl.block_table).to(device),
       torch.from_numpy(wl.seq_lens).to(device), out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _oracle(wl, pages, scales, rotate=True, q=None):
    if q is None:
        q = synth.q_values(wl)
    return oracle.decode_fp64(u16(q), pages, scales, wl.block_table, wl.seq_lens, rotate=rotate,
                              nthreads=NTHREADS)


@pytest.mark.parametrize("G", [1, 4, 8, 16])
@pytest.mark.parametrize("lens", [[1], [15, 16, 17], [1000, 3, 257, 48, 16 * 37 + 5]])
def test_hd_decode_shapes(cuda_device, D, G, lens):
    """Page boundaries, single tokens, ragged lengths and group sizes up to 16."""
    hkv = 2 if G < 8 else 1
    wl = _wl(f"hd_{G}_{len(lens)}", lens, G, hkv, seed=len(lens) * 10 + G, D=D)
    pages, scales = oracle_cache(wl)
    assert_attention_close(_decode(wl, pages, scales, cuda_device), _oracle(wl, pages, scales),
                           wl.name)


def test_hd_decode_split_segments(cuda_device, D):
    """Long and short sequences mixed: long segments are split over several warps and combined
    by the merge kernel (16 output tiles per slot); two calls on the same dirty workspace are
    bit-identical."""
    from bit_paged_kv_block_b200 import saw
    wl = _wl("hd_split", [5000, 3000, 20, 1, 700], 4, 8, seed=31, D=D)
    pages, scales = oracle_cache(wl)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, cuda_device,
                                head_dim=D)
    got = _decode(wl, pages, scales, cuda_device, ws=ws)
    again = _decode(wl, pages, scales, cuda_device, ws=ws)
    assert np.array_equal(got, again)
    assert_attention_close(got, _oracle(wl, pages, scales), f"D={D} split")


def test_hd_plain_cache(cuda_device, D):
    wl = _wl("hd_plain", [70, 33, 300], 4, 2, seed=32, D=D)
    pages, scales = oracle_cache(wl, rotate=False)
    got = _decode(wl, pages, scales, cuda_device, rotate=False)
    assert_attention_close(got, _oracle(wl, pages, scales, rotate=False), f"D={D} plain")


def test_hd_prefill(cuda_device, D):
    """Chunks of 7, 17 (a whole sequence), 1 and 64 tokens and an empty one, causal limits
    inside pages."""
    from bit_paged_kv_block_b200 import saw
    lens, chunks = [40, 17, 33, 300, 20], [7, 17, 1, 64, 0]
    wl = _wl("hd_pf", lens, 4, 2, seed=33, D=D)
    pages, scales = oracle_cache(wl)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    total = int(q_start[-1])
    g = torch.Generator().manual_seed(33)
    q = torch.randn(total, wl.num_q_heads, D, generator=g).to(torch.bfloat16)
    dev = cuda_device
    kv, sc = device_cache_from(pages, scales, dev)
    out = torch.full((total, wl.num_q_heads, D), float("nan"), device=dev)
    ws = saw.allocate_prefill_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, total, dev,
                                        head_dim=D)
    saw.saw_paged_prefill_attn(q.to(dev), torch.from_numpy(q_start).to(dev), kv, sc,
                               torch.from_numpy(wl.block_table).to(dev),
                               torch.from_numpy(wl.seq_lens).to(dev), out, ws)
    torch.cuda.synchronize()
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               nthreads=NTHREADS)
    assert_attention_close(out.cpu().numpy(), want, f"D={D} prefill")


def test_hd_decode_step(cuda_device, D):
    """The fused serving step: one new token per sequence is rotated, quantised and
    appended (codes and scales bit-exact against the oracle), then every sequence is decoded."""
    from bit_paged_kv_block_b200 import saw
    wl = _wl("hd_step", [100, 16, 1, 513, 64, 2000], 4, 4, seed=34, D=D)
    dev = cuda_device
    hist_pages, hist_scales = oracle_cache(wl, tokens="history")
    kv, sc = device_cache_from(hist_pages, hist_scales, dev)
    k_new = synth.kv_values(wl, "K", tokens="new")
    v_new = synth.kv_values(wl, "V", tokens="new")
    seq, pos = synth.token_index(wl, "new")
    slots = synth.slot_mapping(wl, seq, pos)
    q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, D), float("nan"), device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev, head_dim=D)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    saw.saw_decode_step(q.to(dev), k_new.to(dev), v_new.to(dev), torch.from_numpy(slots).to(dev),
                        kv, sc, torch.from_numpy(wl.block_table).to(dev),
                        torch.from_numpy(wl.seq_lens).to(dev), out, ws, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    full_pages, full_scales = hist_pages.copy(), hist_scales.copy()
    oracle.rotate_quantize_paged(u16(k_new), u16(v_new), slots, full_pages, full_scales)
    assert np.array_equal(kv.cpu().numpy(), full_pages)
    assert np.array_equal(u16(sc), full_scales)
    want = oracle.decode_fp64(u16(q), full_pages, full_scales, wl.block_table, wl.seq_lens,
                              nthreads=NTHREADS)
    assert_attention_close(out.cpu().numpy(), want, f"D={D} step")


def test_hd_static_entry_matches_workspace_entry(cuda_device, D):
    """The fixed-scratch entry point serves shapes that fit its scratch, bit-identical
    to the workspace entry point."""
    from bit_paged_kv_block_b200 import saw
    wl = _wl("hd_static", [300, 17, 1, 64], 8, 2, seed=35, D=D)
    pages, scales = oracle_cache(wl)
    got = _decode(wl, pages, scales, cuda_device)
    kv, sc = device_cache_from(pages, scales, cuda_device)
    out = torch.empty((wl.num_seqs, wl.num_q_heads, D), device=cuda_device)
    saw.saw_paged_decode_attn_static(synth.q_values(wl).to(cuda_device), kv, sc,
                                     torch.from_numpy(wl.block_table).to(cuda_device),
                                     torch.from_numpy(wl.seq_lens).to(cuda_device), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), got)


@pytest.mark.parametrize("sample", [[0, 3, 7]])
def test_hd_full_size_sampled(cuda_device, D, sample):
    """A serving-sized batch (8 sequences of 4096 tokens, 32 q / 8 kv heads), sampled sequences
    against the oracle."""
    wl = _wl("hd_full", [4096] * 8, 4, 8, seed=36, D=D)
    pages, scales = oracle_cache(wl)
    q = synth.q_values(wl)
    got = _decode(wl, pages, scales, cuda_device, q=q)
    assert np.isfinite(got).all()
    want = _oracle(subset(wl, sample), pages, scales, q=q[sample])
    assert_attention_close(got[sample], want, f"D={D} full")

"""GPU parity of the INT4 paged decode kernel and of the fused serving step against the fp64
oracle over the same cache: max abs error <= 1e-2 and mean abs error <= 1e-3
("SAW-INT4", Research Findings: fused attention execution over the paged INT4 cache;
"BitDecoding-FP4", abstract: stacked query heads over paged KV)."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import (NTHREADS, assert_attention_close, device_cache_from, oracle_cache, subset,
                     u16)

pytestmark = pytest.mark.gpu


def run_decode(wl, pages, scales, device, q=None, sm_scale=None, status=None, ws=None):
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, device)
    if q is None:
        q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, wl.head_dim), float("nan"), device=device)
    if ws is None:
        ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, device,
                                    head_dim=wl.head_dim)
    saw.saw_paged_decode_attn(q.to(device), kv, sc,
                              torch.from_numpy(wl.block_table).to(device),
                              torch.from_numpy(wl.seq_lens).to(device), out, ws,
                              sm_scale=sm_scale, dev_status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), ws


def oracle_decode(wl, pages, scales, q=None, sm_scale=None):
    if q is None:
        q = synth.q_values(wl)
    return oracle.decode_fp64(u16(q), pages, scales, wl.block_table, wl.seq_lens,
                              sm_scale=sm_scale, nthreads=NTHREADS)


def check(wl, device, what=None, sm_scale=None):
    pages, scales = oracle_cache(wl)
    got, _ = run_decode(wl, pages, scales, device, sm_scale=sm_scale)
    want = oracle_decode(wl, pages, scales, sm_scale=sm_scale)
    return assert_attention_close(got, want, what or wl.name)


def test_decode_tiny(cuda_device):
    check(synth.make_workload("tiny"), cuda_device)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 9, 12, 16])
@pytest.mark.parametrize("lens", [[1], [15, 16, 17], [2, 31, 32, 33, 64, 100],
                                  [1000, 3, 257, 48, 16 * 37 + 5]])
def test_decode_shapes(cuda_device, G, lens):
    """Page boundaries (15/16/17, 31/32/33), single tokens, ragged lengths, group sizes up to 16
    (above 8 the query heads of a kv head run as ceil(G / 8) sub-groups, uneven for G = 9)."""
    hkv = 2 if G < 8 else 1
    wl = synth.custom(f"shape{G}_{len(lens)}", lens, num_q_heads=G * hkv, num_kv_heads=hkv,
                      seed=len(lens) * 10 + G, outlier_range=(10.0, 30.0))
    check(wl, cuda_device)


def test_decode_many_short_sequences(cuda_device):
    """Hundreds of segments, several per CTA slice, with empty sequences mixed in."""
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 70, size=300)
    lens[::17] = 0
    wl = synth.custom("many", lens, num_q_heads=32, num_kv_heads=8, seed=5)
    check(wl, cuda_device)


def test_decode_sm_scale(cuda_device):
    wl = synth.custom("smscale", [200, 77], num_q_heads=8, num_kv_heads=2, seed=9)
    check(wl, cuda_device, sm_scale=0.25)
    check(wl, cuda_device, sm_scale=0.0)


def test_decode_workspace_reuse_is_deterministic(cuda_device):
    """A second call on the same (dirty) workspace gives bit-identical results."""
    wl = synth.custom("reuse", [5000, 3000, 20], num_q_heads=32, num_kv_heads=8, seed=11)
    pages, scales = oracle_cache(wl)
    a, ws = run_decode(wl, pages, scales, cuda_device)
    b, _ = run_decode(wl, pages, scales, cuda_device, ws=ws)
    assert np.array_equal(a, b)
    want = oracle_decode(wl, pages, scales)
    assert_attention_close(a, want, "reuse")


def test_decode_bad_page_and_seq_len_flags(cuda_device):
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("bad", [40, 20, 33], num_q_heads=4, num_kv_heads=1, seed=12)
    pages, scales = oracle_cache(wl)
    wl_bad = subset(wl, [0, 1, 2])
    wl_bad.block_table = wl.block_table.copy()
    wl_bad.block_table[1, 0] = wl.num_pages + 7        # out of range page id
    wl_bad.seq_lens = wl.seq_lens.copy()
    wl_bad.seq_lens[2] = 16 * wl.max_blocks + 1        # longer than its block table
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got, _ = run_decode(wl_bad, pages, scales, cuda_device, status=status)
    st = int(status.item())
    assert st & saw.SAW_DEV_BAD_PAGE and st & saw.SAW_DEV_BAD_SEQ_LEN
    assert np.all(got[2] == 0)                          # invalid length: zero output
    want = oracle_decode(subset(wl, [0]), pages, scales, q=synth.q_values(wl)[:1])
    assert_attention_close(got[:1], want, "unaffected sequence")


@pytest.mark.parametrize("name,sample", [("decode", [0, 17, 40, 63]), ("long", [2, 5]),
                                         ("serving", [0, 1, 100, 200, 255])])
def test_decode_full_size_sampled(cuda_device, name, sample):
    """Full-size workloads in the launch configuration the benchmark uses; the oracle checks a
    sample of sequences one by one."""
    wl = synth.make_workload(name)
    pages, scales = oracle_cache(wl)
    q = synth.q_values(wl)
    got, _ = run_decode(wl, pages, scales, cuda_device, q=q)
    assert np.isfinite(got).all()
    sub = subset(wl, sample)
    want = oracle_decode(sub, pages, scales, q=q[sample])
    assert_attention_close(got[sample], want, name)


@pytest.mark.parametrize("name", ["decode", "serving"])
def test_decode_step_full_size(cuda_device, name):
    """The fused serving step: append one token per sequence on the GPU, then decode.  The
    appended codes must be bit-exact and the outputs within tolerance (sampled)."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.make_workload(name)
    dev = cuda_device
    hist_pages, hist_scales = oracle_cache(wl, tokens="history")
    kv, sc = device_cache_from(hist_pages, hist_scales, dev)
    k_new = synth.kv_values(wl, "K", tokens="new")
    v_new = synth.kv_values(wl, "V", tokens="new")
    seq, pos = synth.token_index(wl, "new")
    slots = synth.slot_mapping(wl, seq, pos)
    q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=dev)
    ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
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
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    sample = [0, 1, wl.num_seqs // 2, wl.num_seqs - 1]
    want = oracle_decode(subset(wl, sample), full_pages, full_scales, q=q[sample])
    assert_attention_close(got[sample], want, name + " step")


def test_decode_g16_several_kv_heads_and_static_entry(cuda_device):
    """G = 16 with 4 kv heads (8 segments per sequence), through both the workspace entry point
    and the fixed-scratch one; the two results are bit-identical."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("g16", [300, 17, 1, 64], num_q_heads=64, num_kv_heads=4, seed=16,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl)
    got, _ = run_decode(wl, pages, scales, cuda_device)
    assert_attention_close(got, oracle_decode(wl, pages, scales), "g16")
    kv, sc = device_cache_from(pages, scales, cuda_device)
    out = torch.empty((wl.num_seqs, wl.num_q_heads, 128), device=cuda_device)
    saw.saw_paged_decode_attn_static(synth.q_values(wl).to(cuda_device), kv, sc,
                                     torch.from_numpy(wl.block_table).to(cuda_device),
                                     torch.from_numpy(wl.seq_lens).to(cuda_device), out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), got)

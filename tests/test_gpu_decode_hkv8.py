"""GPU parity of the INT4 decode at the benchmark workloads' head layout (8 kv heads, 1 to 8
query heads each, head_dim 128): ragged lengths and empty sequences, hundreds of sequences,
the plain cache, bad ids, and long sequences split over many warps whose partials the merge kernel
folds.  Checked against the fp64 oracle over the same cache: max abs error <= 1e-2, mean abs
error <= 1e-3 ("SAW-INT4", Research Findings: fused attention execution over the paged INT4
cache; "BitDecoding-FP4", abstract: stacked query heads over paged KV)."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import (NTHREADS, assert_attention_close, device_cache_from, oracle_cache, subset,
                     u16)

pytestmark = pytest.mark.gpu


def run_decode(wl, pages, scales, device, q=None, status=None, ws=None, plain=False):
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, device)
    if q is None:
        q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=device)
    if ws is None:
        ws = saw.allocate_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, device)
    fn = saw.saw_paged_decode_attn_plain if plain else saw.saw_paged_decode_attn
    fn(q.to(device), kv, sc, torch.from_numpy(wl.block_table).to(device),
       torch.from_numpy(wl.seq_lens).to(device), out, ws, dev_status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy(), ws


def oracle_decode(wl, pages, scales, q=None, plain=False):
    if q is None:
        q = synth.q_values(wl)
    return oracle.decode_fp64(u16(q), pages, scales, wl.block_table, wl.seq_lens,
                              rotate=not plain, nthreads=NTHREADS)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_hkv8_decode_ragged_lengths(cuda_device, G):
    """Page boundaries (15/16/17, 31/32/33), single tokens, empty sequences and one long sequence
    that several warps share."""
    lens = [1, 15, 16, 17, 0, 31, 32, 33, 100, 3000, 7, 0, 257]
    wl = synth.custom(f"hkv8_{G}", lens, num_q_heads=8 * G, num_kv_heads=8, seed=60 + G,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl)
    got, _ = run_decode(wl, pages, scales, cuda_device)
    want = oracle_decode(wl, pages, scales)
    assert_attention_close(got, want, f"hkv8 G={G}")
    assert np.all(got[[4, 11]] == 0)


def test_hkv8_decode_many_sequences(cuda_device):
    """700 short sequences (some empty): most warps hold several whole segments, a few split
    one."""
    rng = np.random.default_rng(61)
    lens = rng.integers(1, 400, size=700)
    lens[::37] = 0
    wl = synth.custom("hkv8_many", lens, num_q_heads=32, num_kv_heads=8, seed=61)
    pages, scales = oracle_cache(wl)
    got, _ = run_decode(wl, pages, scales, cuda_device)
    assert_attention_close(got, oracle_decode(wl, pages, scales), "hkv8 many")


def test_hkv8_decode_plain_cache(cuda_device):
    wl = synth.custom("hkv8_plain", [900, 17, 4000, 1], num_q_heads=32, num_kv_heads=8, seed=62,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl, rotate=False)
    got, _ = run_decode(wl, pages, scales, cuda_device, plain=True)
    assert_attention_close(got, oracle_decode(wl, pages, scales, plain=True), "hkv8 plain")


def test_hkv8_decode_workspace_reuse_is_deterministic(cuda_device):
    """Two calls on the same (dirty) workspace give bit-identical results: split segments are
    folded in a fixed order."""
    wl = synth.custom("hkv8_reuse", [9000, 5000, 20, 7777], num_q_heads=64, num_kv_heads=8, seed=63)
    pages, scales = oracle_cache(wl)
    a, ws = run_decode(wl, pages, scales, cuda_device)
    b, _ = run_decode(wl, pages, scales, cuda_device, ws=ws)
    assert np.array_equal(a, b)
    assert_attention_close(a, oracle_decode(wl, pages, scales), "hkv8 reuse")


def test_hkv8_decode_bad_page_and_seq_len_flags(cuda_device):
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("hkv8_bad", [40, 20, 33, 500], num_q_heads=32, num_kv_heads=8, seed=64)
    pages, scales = oracle_cache(wl)
    bad = subset(wl, [0, 1, 2, 3])
    bad.block_table = wl.block_table.copy()
    bad.block_table[1, 0] = wl.num_pages + 7           # out of range page id
    bad.seq_lens = wl.seq_lens.copy()
    bad.seq_lens[2] = 16 * wl.max_blocks + 1           # longer than its block table
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got, _ = run_decode(bad, pages, scales, cuda_device, status=status)
    st = int(status.item())
    assert st & saw.SAW_DEV_BAD_PAGE and st & saw.SAW_DEV_BAD_SEQ_LEN
    assert np.all(got[2] == 0)
    keep = [0, 3]
    want = oracle_decode(subset(wl, keep), pages, scales, q=synth.q_values(wl)[keep])
    assert_attention_close(got[keep], want, "unaffected sequences")


def test_hkv8_decode_long_sequences_split_across_warps(cuda_device):
    """Two long sequences at G = 8: each spreads over many warps, so every output row comes from
    the merge kernel's fold of many partials."""
    wl = synth.custom("hkv8_long", [32768, 16000], num_q_heads=64, num_kv_heads=8, seed=65,
                      outlier_scale=20.0)
    pages, scales = oracle_cache(wl)
    got, _ = run_decode(wl, pages, scales, cuda_device)
    assert_attention_close(got, oracle_decode(wl, pages, scales), "hkv8 long")

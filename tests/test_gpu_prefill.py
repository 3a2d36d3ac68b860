"""Chunked-prefill attention over the INT4 paged cache on the GPU against the fp64 oracle: the
C_s newest cached tokens of each sequence are queries, query i attending causally to tokens
0 .. L_s - C_s + i ("SAW-INT4", Research Findings: the quantized cache must serve fused
attention over paged memory).  Tolerance as for decode: max abs 1e-2, mean abs 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import NTHREADS, assert_attention_close, device_cache_from, oracle_cache, u16

pytestmark = pytest.mark.gpu


def _queries(total, hq, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(total, hq, 128, generator=g).to(torch.bfloat16)


def _prefill(wl, pages, scales, q, q_start, device, rotate=True, status=None):
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, device)
    total = int(q_start[-1])
    out = torch.full((total, wl.num_q_heads, 128), float("nan"), device=device)
    ws = saw.allocate_prefill_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, total, device)
    ws.fill_(0x5A)
    saw.saw_paged_prefill_attn(q.to(device), torch.from_numpy(q_start).to(device), kv, sc,
                               torch.from_numpy(wl.block_table).to(device),
                               torch.from_numpy(wl.seq_lens).to(device), out, ws,
                               dev_status=status, rotate=rotate)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _case(lens, chunks, G, hkv, seed, rotate=True):
    wl = synth.custom(f"pf{seed}", lens, num_q_heads=G * hkv, num_kv_heads=hkv, seed=seed,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl, rotate=rotate)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = _queries(int(q_start[-1]), G * hkv, seed)
    return wl, pages, scales, q, q_start


@pytest.mark.parametrize("G,hkv", [(1, 2), (4, 2), (8, 1), (16, 1)])
def test_prefill_chunks_match_oracle(cuda_device, G, hkv):
    """Chunks of 7, 17 (the whole sequence), 1 and 64 tokens, 0 tokens, over lengths around page
    boundaries: causal limits inside pages, blocks of 8 rows spanning several tokens (G < 8) or
    one token's heads (G >= 8)."""
    lens, chunks = [40, 17, 33, 300, 20], [7, 17, 1, 64, 0]
    wl, pages, scales, q, q_start = _case(lens, chunks, G, hkv, seed=G + hkv)
    got = _prefill(wl, pages, scales, q, q_start, cuda_device)
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               nthreads=NTHREADS)
    assert_attention_close(got, want, f"prefill G={G}")


def test_prefill_plain_cache(cuda_device):
    lens, chunks = [70, 33], [20, 33]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 2, seed=9, rotate=False)
    got = _prefill(wl, pages, scales, q, q_start, cuda_device, rotate=False)
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               rotate=False, nthreads=NTHREADS)
    assert_attention_close(got, want, "prefill plain")


@pytest.mark.parametrize("lens,hq", [
    ([300, 17, 1, 64, 1000], 8),
    # 70 sequences x 2 kv heads at G = 1: 140 decode segments, at most one per SM of a B200, while
    # the prefill's segment bound is larger; both must still pick the same split-K merge
    ([2000 + 37 * i for i in range(70)], 2),
])
def test_prefill_of_one_token_is_the_decode(cuda_device, lens, hq):
    """C_s = 1 for every sequence is a decode: the same segments, split and merge, so the outputs
    are bit-identical to saw_paged_decode_attn."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("pf1", lens, num_q_heads=hq, num_kv_heads=2, seed=12)
    pages, scales = oracle_cache(wl)
    q = synth.q_values(wl)
    q_start = np.arange(wl.num_seqs + 1, dtype=np.int32)
    got = _prefill(wl, pages, scales, q, q_start, cuda_device)
    kv, sc = device_cache_from(pages, scales, cuda_device)
    out = torch.empty((wl.num_seqs, hq, 128), device=cuda_device)
    ws = saw.allocate_workspace(2, hq, wl.num_seqs, cuda_device)
    saw.saw_paged_decode_attn(q.to(cuda_device), kv, sc,
                              torch.from_numpy(wl.block_table).to(cuda_device),
                              torch.from_numpy(wl.seq_lens).to(cuda_device), out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(got, out.cpu().numpy())


def test_prefill_invalid_chunk_is_flagged_and_skipped(cuda_device):
    """A chunk longer than its sequence is flagged; the other sequences are unaffected."""
    lens, chunks = [40, 10, 33], [5, 12, 3]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 2, seed=13)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = _prefill(wl, pages, scales, q, q_start, cuda_device, status=status)
    assert int(status.item()) & 4                       # SAW_DEV_BAD_SEQ_LEN
    keep = np.r_[0:5, 17:20]
    ok_starts = np.array([0, 5, 5, 8], dtype=np.int32)  # sequence 1 without queries
    qk = q[torch.from_numpy(keep)]
    want = oracle.prefill_fp64(u16(qk), ok_starts, pages, scales, wl.block_table,
                               np.array([40, 10, 33], dtype=np.int32), nthreads=NTHREADS)
    assert_attention_close(got[keep], want, "prefill valid rows")


def test_prefill_long_chunk_sampled(cuda_device):
    """A 256-token chunk at the end of two 4096-token sequences (32 q / 8 kv heads), sampled rows
    against the oracle."""
    lens, chunks = [4096, 4096], [256, 256]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 8, seed=14)
    got = _prefill(wl, pages, scales, q, q_start, cuda_device)
    rows = np.array([0, 1, 100, 255, 256, 300, 511])
    for r in rows:
        s = int(np.searchsorted(q_start, r, side="right") - 1)
        i = r - q_start[s]
        sub_start = np.array([0, 1], dtype=np.int32)
        want = oracle.decode_fp64(u16(q[r:r + 1]), pages, scales, wl.block_table[s:s + 1],
                                  np.array([lens[s] - chunks[s] + i + 1], dtype=np.int32),
                                  nthreads=NTHREADS)
        assert_attention_close(got[r:r + 1], want, f"row {r}")

"""Chunked-prefill attention on the tensor cores (tcgen05: 128-row query tiles, the INT4 pages
unpacked once per tile into fp16 operand tiles, accumulators in tensor memory) against the fp64
oracle ("SAW-INT4", Research Findings: the quantized cache must serve fused attention over paged
memory).  These shapes average at least half a tile (64 query rows) per sequence, so the library
takes the tensor-core path.  Tolerance as for decode: max abs 1e-2, mean abs 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import NTHREADS, assert_attention_close, device_cache_from, oracle_cache, u16

pytestmark = pytest.mark.gpu


def _run(wl, pages, scales, q, q_start, device, rotate=True, status=None):
    from bit_paged_kv_block_b200 import saw
    kv, sc = device_cache_from(pages, scales, device)
    total = int(q_start[-1])
    out = torch.full((total, wl.num_q_heads, 128), float("nan"), device=device)
    ws = saw.allocate_prefill_workspace(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, total, device)
    saw.saw_paged_prefill_attn(q.to(device), torch.from_numpy(q_start).to(device), kv, sc,
                               torch.from_numpy(wl.block_table).to(device),
                               torch.from_numpy(wl.seq_lens).to(device), out, ws,
                               dev_status=status, rotate=rotate)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _case(lens, chunks, G, hkv, seed, rotate=True):
    wl = synth.custom(f"tc{seed}", lens, num_q_heads=G * hkv, num_kv_heads=hkv, seed=seed,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl, rotate=rotate)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(int(q_start[-1]), G * hkv, 128, generator=g).to(torch.bfloat16)
    assert int(q_start[-1]) * G >= 64 * len(lens)    # the tensor-core path
    return wl, pages, scales, q, q_start


@pytest.mark.parametrize("G,hkv", [(1, 2), (2, 2), (3, 2), (4, 2), (8, 1), (16, 1)])
def test_prefill_tc_matches_oracle(cuda_device, G, hkv):
    """Tiles of 128 / G query tokens (ragged last tiles, G = 3 leaving two rows idle), causal
    limits inside blocks of 64 cache tokens, ragged last blocks and pages, a chunk that is a whole
    sequence and one shorter than a tile."""
    lens, chunks = [300, 700, 64, 1000, 129], [300, 150, 64, 100, 29]
    wl, pages, scales, q, q_start = _case(lens, chunks, G, hkv, seed=20 + G)
    got = _run(wl, pages, scales, q, q_start, cuda_device)
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               nthreads=NTHREADS)
    assert_attention_close(got, want, f"tensor-core prefill G={G}")


def test_prefill_tc_plain_cache(cuda_device):
    lens, chunks = [500, 90], [200, 90]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 2, seed=31, rotate=False)
    got = _run(wl, pages, scales, q, q_start, cuda_device, rotate=False)
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               rotate=False, nthreads=NTHREADS)
    assert_attention_close(got, want, "tensor-core prefill, plain cache")


def test_prefill_tc_invalid_chunk_is_flagged_and_skipped(cuda_device):
    """A chunk longer than its sequence is flagged; the other sequences are unaffected."""
    lens, chunks = [100, 50, 300], [64, 60, 100]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 2, seed=32)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = _run(wl, pages, scales, q, q_start, cuda_device, status=status)
    assert int(status.item()) & 4                          # SAW_DEV_BAD_SEQ_LEN
    keep = np.r_[0:64, 124:224]
    ok_starts = np.array([0, 64, 64, 164], dtype=np.int32)  # sequence 1 without queries
    want = oracle.prefill_fp64(u16(q[torch.from_numpy(keep)]), ok_starts, pages, scales,
                               wl.block_table, np.array(lens, dtype=np.int32), nthreads=NTHREADS)
    assert_attention_close(got[keep], want, "valid rows")


def test_prefill_tc_rows_match_decode(cuda_device):
    """Each query row equals a decode over its causal prefix (sampled rows of a long chunk)."""
    lens, chunks = [2000, 1500], [512, 300]
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 4, seed=33)
    got = _run(wl, pages, scales, q, q_start, cuda_device)
    for r in [0, 1, 31, 32, 33, 255, 511, 512, 700, 811]:
        s = int(np.searchsorted(q_start, r, side="right") - 1)
        i = r - q_start[s]
        want = oracle.decode_fp64(u16(q[r:r + 1]), pages, scales, wl.block_table[s:s + 1],
                                  np.array([lens[s] - chunks[s] + i + 1], dtype=np.int32),
                                  nthreads=NTHREADS)
        assert_attention_close(got[r:r + 1], want, f"row {r}")


def test_prefill_tc_bench_workload_sampled(cuda_device):
    """The bench's chunked-prefill workload itself (8 sequences of 4096 cached tokens, the last
    512 of each as queries, 32 q / 8 kv heads, the bench's seeds), in the launch configuration the
    bench times; sampled rows at tile boundaries against the oracle's decode of their prefix."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("chunked_prefill", [4096] * 8, num_q_heads=32, num_kv_heads=8, seed=40,
                      outlier_range=(10.0, 30.0))
    pages, scales = oracle_cache(wl)
    chunk = 512
    q_start = np.arange(0, 9 * chunk, chunk, dtype=np.int32)
    q = torch.randn(8 * chunk, 32, 128, generator=torch.Generator(device="cpu").manual_seed(41)).to(torch.bfloat16)
    got = _run(wl, pages, scales, q, q_start, cuda_device)
    for s in (0, 3, 7):
        for i in (0, 31, 32, 255, 480, 511):   # tiles are 32 query tokens at G = 4
            r = s * chunk + i
            want = oracle.decode_fp64(u16(q[r:r + 1]), pages, scales, wl.block_table[s:s + 1],
                                      np.array([4096 - chunk + i + 1], dtype=np.int32),
                                      nthreads=NTHREADS)
            assert_attention_close(got[r:r + 1], want, f"sequence {s} query {i}")


def test_prefill_tc_many_sequences(cuda_device):
    """300 sequences (the tile search scans the sequences 256 at a time, so a second pass finds
    the tiles of the last 44), short ragged lengths and 16-token chunks: at G = 4 that is 64 rows
    per sequence, the tensor-core path."""
    rng = np.random.default_rng(77)
    lens = [int(x) for x in rng.integers(16, 200, size=300)]
    chunks = [16] * 300
    wl, pages, scales, q, q_start = _case(lens, chunks, 4, 2, seed=34)
    got = _run(wl, pages, scales, q, q_start, cuda_device)
    want = oracle.prefill_fp64(u16(q), q_start, pages, scales, wl.block_table, wl.seq_lens,
                               nthreads=NTHREADS)
    assert_attention_close(got, want, "tensor-core prefill, 300 sequences")

"""The full-precision sink / recent window beside the INT4 cache on the GPU against the oracle
("InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language Models",
Abstract and Figure 2: a bf16 window of attention-sink and recent tokens beside the quantized
cache, the two attention results merged).  The append (window slots, and the codes and scales of
each token leaving the window) is bit-exact; the decode is within max abs 1e-2 / mean abs 1e-3 of
the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import NTHREADS, assert_attention_close, u16

pytestmark = pytest.mark.gpu

D = 128


def _tokens(S, Lmax, hkv, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(S, max(Lmax, 1), hkv, D, generator=g)
    k[..., 5] *= 25.0                                    # an outlier key channel
    v = torch.randn(S, max(Lmax, 1), hkv, D, generator=g)
    return synth.bf16_bits(k.to(torch.bfloat16)), synth.bf16_bits(v.to(torch.bfloat16))


def _state(lens_max, S, hkv, sink, recent, seed):
    """Empty oracle state (window pages with a scattered table, INT4 pages with a shuffled block
    table) able to hold lens_max tokens per sequence."""
    rng = np.random.default_rng(seed)
    pw = max(1, (sink + recent + 15) // 16)
    win_table = rng.permutation(S * pw).astype(np.int32).reshape(S, pw)
    win_kv = np.full((S * pw, hkv, 2, 16, D), 0x7FC1, np.uint16)     # NaN bits: never read
    nq = max(1, (lens_max + 15) // 16)
    block_table = rng.permutation(S * nq + 3).astype(np.int32)[:S * nq].reshape(S, nq)
    pages, scales = oracle.empty_cache(S * nq + 3, hkv, D)
    pages[:] = 0xA5
    scales[:] = 0x5A5A
    return win_kv, win_table, pages, scales, block_table


def _dev(state, device):
    win_kv, win_table, pages, scales, block_table = state
    bf = torch.from_numpy(win_kv.view(np.int16)).view(torch.bfloat16).to(device)
    return (bf, torch.from_numpy(win_table).to(device), torch.from_numpy(pages).to(device),
            torch.from_numpy(scales.view(np.int16)).view(torch.float16).to(device),
            torch.from_numpy(block_table).to(device))


def _assert_state(dstate, state):
    win_kv, _, pages, scales, _ = state
    assert np.array_equal(u16(dstate[0]), win_kv), "window pages differ"
    assert np.array_equal(dstate[2].cpu().numpy(), pages), "INT4 codes differ"
    assert np.array_equal(u16(dstate[3]), scales), "scales differ"


WINDOWS = [(4, 12), (16, 112), (0, 32), (8, 0), (16, 16), (3, 61)]


@pytest.mark.parametrize("sink,recent", WINDOWS)
def test_window_append_steps_bit_exact(cuda_device, sink, recent):
    """From a filled state, 40 GPU steps (sequences crossing the sink boundary, filling the ring,
    evicting into the INT4 pages) leave window bits, codes and scales equal to the oracle's.
    15 (sequence, kv head) pairs: a ragged last warp."""
    from bit_paged_kv_block_b200 import saw
    L0, steps, hkv = [0, 2, 20, 140, 700], 40, 3
    S, L1 = len(L0), [x + steps for x in L0]
    k, v = _tokens(S, max(L1), hkv, seed=sink + recent)
    state = _state(max(L1), S, hkv, sink, recent, seed=1)
    win_kv, win_table, pages, scales, bt = state
    oracle.window_fill(k, v, np.array(L0), sink, recent, win_kv, win_table, pages, scales, bt)
    dstate = _dev(state, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for i in range(1, steps + 1):
        lens = np.array([x + i for x in L0], dtype=np.int32)
        kn = np.stack([k[s, lens[s] - 1] for s in range(S)])
        vn = np.stack([v[s, lens[s] - 1] for s in range(S)])
        oracle.window_append(kn, vn, lens, sink, recent, win_kv, win_table, pages, scales, bt)
        to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(cuda_device)
        saw.saw_window_append(to(kn), to(vn), torch.from_numpy(lens).to(cuda_device),
                              (sink, recent, dstate[0], dstate[1]), dstate[2], dstate[3],
                              dstate[4], dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _assert_state(dstate, state)


def _decode_case(device, lens, G, hkv, sink, recent, seed):
    from bit_paged_kv_block_b200 import saw
    S = len(lens)
    k, v = _tokens(S, max(lens), hkv, seed)
    state = _state(max(lens), S, hkv, sink, recent, seed)
    win_kv, win_table, pages, scales, bt = state
    oracle.window_fill(k, v, np.array(lens), sink, recent, win_kv, win_table, pages, scales, bt)
    q = torch.randn(S, G * hkv, D, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    dstate = _dev(state, device)
    out = torch.full((S, G * hkv, D), float("nan"), device=device)
    ws = saw.allocate_window_workspace(hkv, G * hkv, S, device)
    ws.fill_(0x5A)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=device)
    saw.saw_paged_decode_attn_window(q.to(device), (sink, recent, dstate[0], dstate[1]),
                                     dstate[2], dstate[3], dstate[4], seq_lens, out, ws)
    torch.cuda.synchronize()
    want = oracle.decode_window_fp64(u16(q), win_kv, win_table, pages, scales, bt,
                                     np.array(lens, np.int32), sink, recent, nthreads=NTHREADS)
    return out.cpu().numpy(), want


@pytest.mark.parametrize("sink,recent", WINDOWS + [(0, 0)])
@pytest.mark.parametrize("G", [1, 4, 16])
def test_window_decode_matches_oracle(cuda_device, sink, recent, G):
    """Lengths 0, 1, inside the sinks, filling the ring, and long ones whose quantized part is
    split over several warps; the two parts merged by their softmax denominators."""
    hkv = 2 if G < 16 else 1
    lens = [0, 1, 3, 17, sink + recent, sink + recent + 1, 300, 2500]
    got, want = _decode_case(cuda_device, lens, G, hkv, sink, recent, seed=G + sink)
    assert_attention_close(got, want, f"window ({sink}, {recent}) G={G}")


def test_window_step_matches_oracle(cuda_device):
    """The fused step: append with eviction, then the windowed decode; state bit-exact, output
    within tolerance."""
    from bit_paged_kv_block_b200 import saw
    sink, recent, hkv, G = 4, 60, 2, 4
    L0 = [0, 5, 63, 64, 1000]
    S = len(L0)
    lens = np.array([x + 1 for x in L0], dtype=np.int32)
    k, v = _tokens(S, int(lens.max()), hkv, seed=9)
    state = _state(int(lens.max()), S, hkv, sink, recent, seed=9)
    win_kv, win_table, pages, scales, bt = state
    oracle.window_fill(k, v, np.array(L0), sink, recent, win_kv, win_table, pages, scales, bt)
    dstate = _dev(state, cuda_device)
    kn = np.stack([k[s, lens[s] - 1] for s in range(S)])
    vn = np.stack([v[s, lens[s] - 1] for s in range(S)])
    oracle.window_append(kn, vn, lens, sink, recent, win_kv, win_table, pages, scales, bt)
    q = torch.randn(S, G * hkv, D, generator=torch.Generator().manual_seed(10)).to(torch.bfloat16)
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    out = torch.full((S, G * hkv, D), float("nan"), device=cuda_device)
    ws = saw.allocate_window_workspace(hkv, G * hkv, S, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    saw.saw_decode_step_window(q.to(cuda_device), to(kn), to(vn),
                               (sink, recent, dstate[0], dstate[1]), dstate[2], dstate[3],
                               dstate[4], torch.from_numpy(lens).to(cuda_device), out, ws,
                               dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _assert_state(dstate, state)
    want = oracle.decode_window_fp64(u16(q), win_kv, win_table, pages, scales, bt, lens, sink,
                                     recent, nthreads=NTHREADS)
    assert_attention_close(out.cpu().numpy(), want, "window step")


def test_window_append_flags_bad_pages(cuda_device):
    """A window page id out of range, or a quantized index past the block table, leaves the
    pair untouched and sets the status bits; the other sequences are written."""
    from bit_paged_kv_block_b200 import saw
    sink, recent, hkv = 4, 12, 2
    L0 = [20, 20, 20]
    S = len(L0)
    k, v = _tokens(S, 64, hkv, seed=11)
    state = _state(21, S, hkv, sink, recent, seed=11)
    win_kv, win_table, pages, scales, bt = state
    oracle.window_fill(k, v, np.array(L0), sink, recent, win_kv, win_table, pages, scales, bt)
    win_table[1, :] = 10 ** 6                          # sequence 1: bad window page
    dstate = _dev(state, cuda_device)
    lens = np.array([21, 21, 64], dtype=np.int32)      # sequence 2: index past its two blocks
    kn = np.stack([k[s, lens[s] - 1] for s in range(S)])
    vn = np.stack([v[s, lens[s] - 1] for s in range(S)])
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    to = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(cuda_device)
    saw.saw_window_append(to(kn), to(vn), torch.from_numpy(lens).to(cuda_device),
                          (sink, recent, dstate[0], dstate[1]), dstate[2], dstate[3], dstate[4],
                          dev_status=status)
    torch.cuda.synchronize()
    st = int(status.item())
    assert st & saw.SAW_DEV_BAD_PAGE and st & saw.SAW_DEV_BAD_SEQ_LEN
    # only sequence 0 changed: apply its step to the oracle state
    oracle.window_append(kn[:1], vn[:1], lens[:1], sink, recent, win_kv, win_table[:1], pages,
                         scales, bt[:1])
    _assert_state(dstate, state)

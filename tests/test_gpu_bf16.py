"""The uncompressed BF16 paged cache on the GPU (the baseline the INT4 format is measured
against: "SAW-INT4", Research Findings; "BitDecoding-FP4", abstract): the scatter is
bit-exact against the oracle's, and decode attention is within tolerance of the oracle's fp64
attention over the same cache."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import NTHREADS, assert_attention_close, subset

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0   # fill for never-written cache rows: a masked tail must never reach the output


def _device_bf16(kv_bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(kv_bits.copy()).view(torch.bfloat16).to(device)


def _oracle_bf16_cache(wl, tokens="all", fill=NAN_BF16):
    k, v = synth.kv_values(wl, "K", tokens=tokens), synth.kv_values(wl, "V", tokens=tokens)
    seq, pos = synth.token_index(wl, tokens)
    kv = np.full((wl.num_pages, wl.num_kv_heads, 2, 16, 128), fill, dtype=np.uint16)
    oracle.append_bf16(synth.bf16_bits(k), synth.bf16_bits(v), synth.slot_mapping(wl, seq, pos), kv)
    return kv


def _gpu_append(wl, device, tokens="all", fill=NAN_BF16, status=None):
    from bit_paged_kv_block_b200 import saw
    k, v = synth.kv_values(wl, "K", tokens=tokens), synth.kv_values(wl, "V", tokens=tokens)
    seq, pos = synth.token_index(wl, tokens)
    kv = _device_bf16(np.full((wl.num_pages, wl.num_kv_heads, 2, 16, 128), fill, dtype=np.uint16),
                      device)
    saw.saw_append_bf16_paged(k.to(device), v.to(device),
                              torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(device), kv,
                              dev_status=status)
    torch.cuda.synchronize()
    return kv


def _bits(kv: torch.Tensor) -> np.ndarray:
    return kv.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["tiny", "prefill"])
def test_bf16_append_bit_exact(cuda_device, name):
    wl = synth.make_workload(name)
    assert np.array_equal(_bits(_gpu_append(wl, cuda_device)), _oracle_bf16_cache(wl))


def test_bf16_append_skips_and_flags_bad_slots(cuda_device):
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("bf16slots", [50], num_q_heads=2, num_kv_heads=2, new_tokens=[50])
    k, v = synth.kv_values(wl, "K"), synth.kv_values(wl, "V")
    seq, pos = synth.token_index(wl)
    slots = synth.slot_mapping(wl, seq, pos)
    slots[4] = -1
    slots[9] = wl.num_pages * 16 + 3
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    kv = _device_bf16(np.full((wl.num_pages, 2, 2, 16, 128), NAN_BF16, dtype=np.uint16), cuda_device)
    saw.saw_append_bf16_paged(k.to(cuda_device), v.to(cuda_device),
                              torch.from_numpy(slots).to(cuda_device), kv, dev_status=status)
    torch.cuda.synchronize()
    want = np.full((wl.num_pages, 2, 2, 16, 128), NAN_BF16, dtype=np.uint16)
    assert oracle.append_bf16(synth.bf16_bits(k), synth.bf16_bits(v), slots, want) == 1
    assert np.array_equal(_bits(kv), want)
    assert int(status.item()) & 1          # SAW_DEV_BAD_SLOT


def _decode_bf16(wl, kv, device, q, sm_scale=None):
    from bit_paged_kv_block_b200 import saw
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=device)
    ws = saw.allocate_workspace_bf16(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, device)
    ws.fill_(0xA5)                          # any workspace contents are fine
    saw.saw_paged_decode_attn_bf16(q.to(device), kv, torch.from_numpy(wl.block_table).to(device),
                                   torch.from_numpy(wl.seq_lens).to(device), out, ws,
                                   sm_scale=sm_scale)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("G,lens", [(1, [1, 16, 17]), (2, [15, 31, 33, 64]), (4, [5, 300, 0, 129]),
                                    (8, [1000, 1, 48]), (12, [70, 1, 33]), (16, [257, 16])])
def test_bf16_decode_matches_oracle(cuda_device, G, lens):
    hkv = 2
    wl = synth.custom(f"bf16dec{G}", lens, num_q_heads=G * hkv, num_kv_heads=hkv, seed=G + 20,
                      outlier_range=(10.0, 30.0))
    kv = _oracle_bf16_cache(wl)
    q = synth.q_values(wl)
    got = _decode_bf16(wl, _device_bf16(kv, cuda_device), cuda_device, q)
    want = oracle.decode_bf16_fp64(synth.bf16_bits(q), kv, wl.block_table, wl.seq_lens,
                                   nthreads=NTHREADS)
    assert_attention_close(got, want, f"bf16 G={G}")


def test_bf16_decode_many_short_sequences_and_sm_scale(cuda_device):
    rng = np.random.default_rng(4)
    lens = rng.integers(0, 70, 300).tolist()
    wl = synth.custom("bf16many", lens, num_q_heads=8, num_kv_heads=2, seed=31)
    kv = _oracle_bf16_cache(wl)
    q = synth.q_values(wl)
    got = _decode_bf16(wl, _device_bf16(kv, cuda_device), cuda_device, q, sm_scale=0.25)
    want = oracle.decode_bf16_fp64(synth.bf16_bits(q), kv, wl.block_table, wl.seq_lens,
                                   sm_scale=0.25, nthreads=NTHREADS)
    assert_attention_close(got, want, "bf16 many")


def test_bf16_step_full_size(cuda_device):
    """The decode workload at full size through saw_decode_step_bf16 (the bench's launch
    configuration): appended rows bit-exact, outputs of sampled sequences within tolerance."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.make_workload("decode")
    dev = cuda_device
    hist = _oracle_bf16_cache(wl, tokens="history")
    kv = _device_bf16(hist, dev)
    k_new, v_new = synth.kv_values(wl, "K", tokens="new"), synth.kv_values(wl, "V", tokens="new")
    seq, pos = synth.token_index(wl, "new")
    slots = synth.slot_mapping(wl, seq, pos)
    q = synth.q_values(wl)
    out = torch.full((wl.num_seqs, wl.num_q_heads, 128), float("nan"), device=dev)
    ws = saw.allocate_workspace_bf16(wl.num_kv_heads, wl.num_q_heads, wl.num_seqs, dev)
    saw.saw_decode_step_bf16(q.to(dev), k_new.to(dev), v_new.to(dev), torch.from_numpy(slots).to(dev),
                             kv, torch.from_numpy(wl.block_table).to(dev),
                             torch.from_numpy(wl.seq_lens).to(dev), out, ws)
    torch.cuda.synchronize()
    full = hist.copy()
    oracle.append_bf16(synth.bf16_bits(k_new), synth.bf16_bits(v_new), slots, full)
    assert np.array_equal(_bits(kv), full)
    sample = [0, 17, 63]
    want = oracle.decode_bf16_fp64(synth.bf16_bits(q[sample]), full, subset(wl, sample).block_table,
                                   wl.seq_lens[sample], nthreads=NTHREADS)
    assert_attention_close(out.cpu().numpy()[sample], want, "bf16 step")

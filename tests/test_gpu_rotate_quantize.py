"""GPU parity of the rotate + quantize + scatter kernel against the CPU oracle: packed codes and
fp16 scale / zero must be bit-identical ("SAW-INT4", Research Findings: the fused
rotation-quantization kernel writing token-wise INT4 into the paged cache)."""
import numpy as np
import pytest
import torch

import oracle
from bit_paged_kv_block_b200 import synth
from helpers import (CANARY_CODE, CANARY_SCALE, EDGE_KINDS, NTHREADS, canary_device_cache,
                     edge_kv, oracle_cache, u16)

pytestmark = pytest.mark.gpu


def gpu_append(wl, device, tokens="all", k=None, v=None, status=None):
    from bit_paged_kv_block_b200 import saw
    if k is None:
        k = synth.kv_values(wl, "K", tokens=tokens)
    if v is None:
        v = synth.kv_values(wl, "V", tokens=tokens)
    seq, pos = synth.token_index(wl, tokens)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(device)
    kv, sc = canary_device_cache(wl, device)
    saw.saw_rotate_quantize_paged(k.to(device), v.to(device), slots, kv, sc, dev_status=status)
    torch.cuda.synchronize()
    return kv, sc


def assert_cache_equal(kv, sc, pages, scales):
    got_p = kv.cpu().numpy()
    got_s = u16(sc)
    if not np.array_equal(got_p, pages):
        bad = np.argwhere(got_p != pages)
        raise AssertionError(f"{len(bad)} code bytes differ, first at {bad[0].tolist()}: "
                             f"{got_p[tuple(bad[0])]:#x} vs {pages[tuple(bad[0])]:#x}")
    if not np.array_equal(got_s, scales):
        bad = np.argwhere(got_s != scales)
        raise AssertionError(f"{len(bad)} scale words differ, first at {bad[0].tolist()}: "
                             f"{got_s[tuple(bad[0])]:#x} vs {scales[tuple(bad[0])]:#x}")


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode", "long", "serving"])
def test_rotate_quantize_bit_exact_workloads(cuda_device, name):
    wl = synth.make_workload(name)
    k = synth.kv_values(wl, "K")
    v = synth.kv_values(wl, "V")
    kv, sc = gpu_append(wl, cuda_device, k=k, v=v)
    pages, scales = oracle_cache(wl, k=k, v=v)
    assert_cache_equal(kv, sc, pages, scales)


def _custom_tokens(T, Hkv, maker, seed=0):
    g = torch.Generator().manual_seed(seed)
    return maker(g, (T, Hkv, 128)).to(torch.bfloat16)


@pytest.mark.parametrize("kind", EDGE_KINDS)
def test_rotate_quantize_edge_values(cuda_device, kind):
    """Inputs chosen to hit exact ties, degenerate vectors, subnormal scales and both sides of
    the smallest scale the remainder test handles; every code must still equal the
    IEEE-divide definition."""
    T, Hkv = 203, 3                  # ragged: 609 vectors, not a multiple of 16 per warp
    k, v = edge_kv(kind, T, Hkv)
    wl = synth.custom(kind, [T], num_q_heads=Hkv, num_kv_heads=Hkv, new_tokens=[T],
                      num_pages=(T + 15) // 16 + 3)
    kv, sc = gpu_append(wl, cuda_device, k=k, v=v)
    pages, scales = oracle_cache(wl, k=k, v=v)
    assert_cache_equal(kv, sc, pages, scales)


def test_slots_skip_and_out_of_range(cuda_device):
    """slot < 0 skips the token, slot >= num_pages * 16 skips it and sets SAW_DEV_BAD_SLOT;
    everything not written keeps its canary."""
    from bit_paged_kv_block_b200 import saw
    T, Hkv, num_pages = 57, 2, 6
    k = torch.randn(T, Hkv, 128).to(torch.bfloat16)
    v = torch.randn(T, Hkv, 128).to(torch.bfloat16)
    rng = np.random.default_rng(3)
    slots = rng.permutation(num_pages * 16)[:T].astype(np.int64)
    slots[::7] = -1
    slots[5] = num_pages * 16 + 3
    wl = synth.custom("slots", [T], num_q_heads=Hkv, num_kv_heads=Hkv, new_tokens=[T],
                      num_pages=num_pages)
    kv, sc = canary_device_cache(wl, cuda_device)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    saw.saw_rotate_quantize_paged(k.to(cuda_device), v.to(cuda_device),
                                  torch.from_numpy(slots).to(cuda_device), kv, sc,
                                  dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == saw.SAW_DEV_BAD_SLOT
    pages, scales = oracle.empty_cache(num_pages, Hkv)
    pages[:] = CANARY_CODE
    scales[:] = CANARY_SCALE
    assert oracle.rotate_quantize_paged(u16(k), u16(v), slots, pages, scales) == 1
    assert_cache_equal(kv, sc, pages, scales)


def test_overwrite_in_place_and_repeat(cuda_device):
    """Writing the same tokens twice gives the same bytes (the kernel is deterministic and
    overwrites whole rows)."""
    wl = synth.make_workload("tiny")
    kv1, sc1 = gpu_append(wl, cuda_device)
    kv2, sc2 = gpu_append(wl, cuda_device)
    assert torch.equal(kv1, kv2) and torch.equal(sc1.view(torch.int16), sc2.view(torch.int16))


def test_empty_append_is_noop(cuda_device):
    from bit_paged_kv_block_b200 import saw
    wl = synth.make_workload("tiny")
    kv, sc = canary_device_cache(wl, cuda_device)
    e = torch.empty(0, wl.num_kv_heads, 128, dtype=torch.bfloat16, device=cuda_device)
    saw.saw_rotate_quantize_paged(e, e, torch.empty(0, dtype=torch.int64, device=cuda_device),
                                  kv, sc)
    torch.cuda.synchronize()
    assert bool((kv == CANARY_CODE).all())


@pytest.mark.parametrize("hkv", [1, 2, 8, 16])
@pytest.mark.parametrize("rotate", [True, False])
def test_strided_kv_from_fused_qkv(cuda_device, hkv, rotate):
    """k and v as slices of a fused QKV projection output [T][(Hq + 2 Hkv) * 128] (token
    stride (Hq + 2 Hkv) * 128): codes and scales bit-identical to the oracle on the same
    values, for Hkv dividing 8 (one tile spans several tokens) and multiples of 8."""
    from bit_paged_kv_block_b200 import saw
    T, hq = 203, 4 * hkv
    g = torch.Generator().manual_seed(hkv + 10 * rotate)
    qkv = (torch.randn(T, (hq + 2 * hkv) * 128, generator=g) * 3.0).to(torch.bfloat16)
    k = qkv[:, hq * 128:(hq + hkv) * 128].view(T, hkv, 128)
    v = qkv[:, (hq + hkv) * 128:].view(T, hkv, 128)
    wl = synth.custom(f"qkv{hkv}", [T], num_q_heads=hq, num_kv_heads=hkv, new_tokens=[T],
                      num_pages=(T + 15) // 16 + 2)
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
    kv, sc = canary_device_cache(wl, cuda_device)
    qkv_d = qkv.to(cuda_device)
    saw.saw_rotate_quantize_paged_strided(qkv_d[:, hq * 128:(hq + hkv) * 128].view(T, hkv, 128),
                                          qkv_d[:, (hq + hkv) * 128:].view(T, hkv, 128), slots,
                                          kv, sc, rotate=rotate)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k.contiguous(), v=v.contiguous(), rotate=rotate)
    assert_cache_equal(kv, sc, pages, scales)


@pytest.mark.parametrize("hkv", [2, 4, 8])
@pytest.mark.parametrize("rotate", [True, False])
def test_head_dim_256_block_diagonal(cuda_device, hkv, rotate):
    """D = 256: two independent 128-point rotation blocks per vector, one scale and zero over
    all 256 elements, 128 code bytes per row; bit-exact against the oracle on outlier data and
    on small integers (exact ties), ragged token counts."""
    from bit_paged_kv_block_b200 import saw
    for kind, T in (("randn", 137), ("small_ints", 61)):
        wl = synth.custom(f"d256{kind}{hkv}", [T], num_q_heads=hkv, num_kv_heads=hkv,
                          new_tokens=[T], head_dim=256, seed=hkv, outlier_range=(10.0, 30.0))
        if kind == "randn":
            k, v = synth.kv_values(wl, "K"), synth.kv_values(wl, "V")
        else:
            g = torch.Generator().manual_seed(hkv)
            k = torch.randint(-3, 4, (T, hkv, 256), generator=g).to(torch.bfloat16)
            v = torch.randint(0, 5, (T, hkv, 256), generator=g).to(torch.bfloat16)
        seq, pos = synth.token_index(wl)
        slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
        kv, sc = canary_device_cache(wl, cuda_device)
        if rotate:
            saw.saw_rotate_quantize_paged(k.to(cuda_device), v.to(cuda_device), slots, kv, sc)
        else:
            saw.saw_quantize_paged_plain(k.to(cuda_device), v.to(cuda_device), slots, kv, sc)
        torch.cuda.synchronize()
        pages, scales = oracle_cache(wl, k=k, v=v, rotate=rotate)
        assert_cache_equal(kv, sc, pages, scales)


def test_head_dim_256_strided(cuda_device):
    """D = 256 k / v sliced from a fused QKV output (Hkv = 4: one tile of 4 vectors per token)."""
    from bit_paged_kv_block_b200 import saw
    T, hkv, hq = 90, 4, 16
    g = torch.Generator().manual_seed(5)
    qkv = (torch.randn(T, (hq + 2 * hkv) * 256, generator=g) * 2.0).to(torch.bfloat16)
    k = qkv[:, hq * 256:(hq + hkv) * 256].view(T, hkv, 256)
    v = qkv[:, (hq + hkv) * 256:].view(T, hkv, 256)
    wl = synth.custom("d256qkv", [T], num_q_heads=hkv, num_kv_heads=hkv, new_tokens=[T],
                      head_dim=256)
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
    kv, sc = canary_device_cache(wl, cuda_device)
    qd = qkv.to(cuda_device)
    saw.saw_rotate_quantize_paged_strided(qd[:, hq * 256:(hq + hkv) * 256].view(T, hkv, 256),
                                          qd[:, (hq + hkv) * 256:].view(T, hkv, 256), slots, kv, sc)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k.contiguous(), v=v.contiguous())
    assert_cache_equal(kv, sc, pages, scales)


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("kind", ["randn"] + EDGE_KINDS)
def test_head_dim_64(cuda_device, kind, rotate):
    """D = 64: the whole vector is one 64-point rotation block (1/8), one thread per vector,
    16 vectors of K and 16 of V per tile, 32 code bytes per row; bit-exact against the oracle on
    outlier data and on every edge input, ragged token counts."""
    from bit_paged_kv_block_b200 import saw
    T, hkv = 203, 3
    wl = synth.custom(f"d64{kind}", [T], num_q_heads=hkv, num_kv_heads=hkv, new_tokens=[T],
                      head_dim=64, seed=3, outlier_range=(10.0, 30.0),
                      num_pages=(T + 15) // 16 + 3)
    if kind == "randn":
        k, v = synth.kv_values(wl, "K"), synth.kv_values(wl, "V")
    else:
        k, v = edge_kv(kind, T, hkv, D=64)
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
    kv, sc = canary_device_cache(wl, cuda_device)
    fn = saw.saw_rotate_quantize_paged if rotate else saw.saw_quantize_paged_plain
    fn(k.to(cuda_device), v.to(cuda_device), slots, kv, sc)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k, v=v, rotate=rotate)
    assert_cache_equal(kv, sc, pages, scales)


@pytest.mark.parametrize("hkv", [2, 8, 16])
def test_head_dim_64_strided(cuda_device, hkv):
    """D = 64 k / v sliced from a fused QKV output (tiles of 16 vectors: Hkv dividing or a
    multiple of 16)."""
    from bit_paged_kv_block_b200 import saw
    T, hq = 77, 2 * hkv
    g = torch.Generator().manual_seed(hkv)
    qkv = (torch.randn(T, (hq + 2 * hkv) * 64, generator=g) * 2.0).to(torch.bfloat16)
    k = qkv[:, hq * 64:(hq + hkv) * 64].view(T, hkv, 64)
    v = qkv[:, (hq + hkv) * 64:].view(T, hkv, 64)
    wl = synth.custom(f"d64qkv{hkv}", [T], num_q_heads=hkv, num_kv_heads=hkv, new_tokens=[T],
                      head_dim=64)
    seq, pos = synth.token_index(wl)
    slots = torch.from_numpy(synth.slot_mapping(wl, seq, pos)).to(cuda_device)
    kv, sc = canary_device_cache(wl, cuda_device)
    qd = qkv.to(cuda_device)
    saw.saw_rotate_quantize_paged_strided(qd[:, hq * 64:(hq + hkv) * 64].view(T, hkv, 64),
                                          qd[:, (hq + hkv) * 64:].view(T, hkv, 64), slots, kv, sc)
    torch.cuda.synchronize()
    pages, scales = oracle_cache(wl, k=k.contiguous(), v=v.contiguous())
    assert_cache_equal(kv, sc, pages, scales)


def test_rotate_quantize_out_of_fp16_range_sets_status(cuda_device):
    """A constant vector of -6000 rotates to (-6000 sqrt(128), 0, ..., 0): its minimum -67882 lies
    beyond fp16's range, so the stored zero point is -inf (the round-to-nearest conversion of the
    definition, bit-identical to the oracle) and the kernel reports SAW_DEV_RANGE.  Vectors in
    range in the same call are stored as usual and leave the bit alone when they are alone."""
    from bit_paged_kv_block_b200 import saw
    wl = synth.custom("range", [32], num_q_heads=8, num_kv_heads=2, seed=3, new_tokens=[32])
    k = torch.randn(32, 2, 128, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    v = k.flip(-1).clone()
    k[5, 1] = -6000.0                                  # out of range: K of token 5, head 1
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    kv, sc = gpu_append(wl, cuda_device, k=k, v=v, status=status)
    assert int(status.item()) & saw.SAW_DEV_RANGE
    pages, scales = oracle_cache(wl, k=k, v=v)
    assert_cache_equal(kv, sc, pages, scales)
    k_ok = k.clone()
    k_ok[5, 1] = -100.0
    status.zero_()
    gpu_append(wl, cuda_device, k=k_ok, v=v, status=status)
    assert int(status.item()) == 0

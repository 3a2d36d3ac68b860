"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a closed form, an invariant, a library routine, a
hand-derived worked case (tests/golden/quant_cases.json) or brute force, so that a dropped
term, a wrong sign or index, a swapped nibble or a transposed operand fails somewhere.
The method is SAW-INT4 ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
LLM Serving", Research Findings): token-wise INT4 quantization with a block-diagonal Hadamard
rotation, written into a paged KV cache that fused attention reads.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.linalg import hadamard

import oracle
from bit_paged_kv_block_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_cases.json")
C32 = np.float32(1.0 / np.sqrt(128.0))
H128 = hadamard(128).astype(np.float64)          # library Sylvester matrix, entries +-1


def popcount_sign(i, j):
    return -1.0 if bin(i & j).count("1") % 2 else 1.0


# ---------------------------------------------------------------------------------------
# Hadamard rotation
# ---------------------------------------------------------------------------------------

def test_normalisation_constant_bits():
    assert np.array(C32).view(np.uint32) == 0x3DB504F3


def test_fwht_unit_vectors_are_signed_columns_exactly():
    """e_j maps to column j of H, times c, bit-exactly: H[i][j] = (-1)^popcount(i & j)."""
    cols = []
    for j in range(128):
        e = np.zeros(128, np.float32)
        e[j] = 1.0
        y = oracle.fwht_f32(e)
        want = np.array([popcount_sign(i, j) for i in range(128)], np.float32) * C32
        assert np.array_equal(y.view(np.uint32), want.view(np.uint32)), j
        cols.append(np.sign(y))
    S = np.stack(cols, axis=1).astype(np.int64)
    assert np.array_equal(S, H128.astype(np.int64))                 # scipy's Sylvester order
    assert np.array_equal(S @ S.T, 128 * np.eye(128, dtype=np.int64))  # H H^T = B I


@pytest.mark.parametrize("scale", [1.0, 30.0, 1e-3])
def test_fwht_matches_matrix_product(scale):
    rng = np.random.default_rng(7)
    H = H128 / np.sqrt(128.0)
    for _ in range(200):
        x = (rng.standard_normal(128) * scale).astype(np.float32)
        x[rng.choice(128, 4, replace=False)] *= 20
        y = oracle.fwht_f32(x)
        exact = H @ x.astype(np.float64)
        assert np.abs(y - exact).max() <= 2.5e-7 * np.linalg.norm(x.astype(np.float64))


def test_fwht_constant_vector():
    """a * 1 -> (fl(128 a * c), +0, ..., +0): every entry but the first is exactly +0."""
    for a in [1.0, -3.5, 0.015625, 1000.0]:
        y = oracle.fwht_f32(np.full(128, a, np.float32))
        assert y[0] == np.float32(np.float32(128 * a) * C32)
        assert np.all(y[1:].view(np.uint32) == 0)


def test_fwht_round_trip_normwise():
    """H_norm is symmetric and orthogonal, so it is its own inverse: within 1e-6 normwise."""
    rng = np.random.default_rng(3)
    for _ in range(200):
        x = rng.standard_normal(128).astype(np.float32)
        x[rng.choice(128, 4, replace=False)] *= 25
        z = oracle.fwht_f32(oracle.fwht_f32(x))
        assert np.abs(z - x).max() <= 1e-6 * np.abs(x).max()


def test_fwht_f64_round_trip_absolute():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((50, 128))
    z = oracle.rotate_f64(oracle.rotate_f64(x))
    assert np.abs(z - x).max() <= 1e-6
    assert np.abs(oracle.rotate_f64(x) - x @ (H128 / np.sqrt(128.0)).T).max() <= 1e-12


def test_rotation_is_block_diagonal():
    """D = 256 rotates each 128 block on its own, which is not the 256-point transform."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 256)).astype(np.float32)
    y = oracle.rotate_f32(x)
    assert np.array_equal(y[:, :128], oracle.fwht_f32(x[:, :128]))
    assert np.array_equal(y[:, 128:], oracle.fwht_f32(x[:, 128:]))
    full = x.astype(np.float64) @ (hadamard(256) / 16.0).T
    assert np.abs(y - full).max() > 1e-2


def test_rotation_d64_is_the_64_point_transform():
    """A 64-wide head vector holds no 128-point block: it is rotated by the normalised 64-point
    Sylvester transform (c = 1/8, exact in fp32)."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal((6, 64)).astype(np.float32)
    y = oracle.rotate_f32(x)
    assert np.array_equal(y, oracle.fwht_f32(x))
    H64 = hadamard(64).astype(np.float64)
    ref = x.astype(np.float64) @ (H64 / 8.0).T
    assert np.abs(y - ref).max() <= 2.5e-7 * np.abs(x).sum(axis=1).max()
    for j in (0, 1, 37, 63):                       # unit vectors: column j times 1/8, exactly
        e = np.zeros(64, np.float32)
        e[j] = 1.0
        assert np.array_equal(oracle.rotate_f32(e), (H64[:, j] / 8.0).astype(np.float32))
    c = oracle.rotate_f32(np.full(64, 0.75, np.float32))
    assert c[0] == np.float32(6.0) and np.all(c[1:] == 0)
    xd = rng.standard_normal((5, 64))
    assert np.abs(oracle.rotate_f64(xd) - xd @ (H64 / 8.0).T).max() <= 1e-12


# ---------------------------------------------------------------------------------------
# scalar conversions
# ---------------------------------------------------------------------------------------

def test_f32_to_f16_matches_numpy_rne():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(
            -9, 6, 20000).astype(np.float32),
        np.array([0.0, -0.0, 65504.0, 65520.0, 65519.99, 1e9, -1e9, 6.1e-5, 5.96e-8,
                  2.98e-8, 2.99e-8, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11], np.float32),
    ]).astype(np.float32)
    # exact halfway points between adjacent fp16 values exercise ties-to-even
    h = np.arange(0x0400, 0x7BFF, 37, dtype=np.uint16).view(np.float16).astype(np.float32)
    h_next = (np.arange(0x0400, 0x7BFF, 37, dtype=np.uint16) + 1).view(np.float16).astype(
        np.float32)
    vals = np.concatenate([vals, (h + h_next) / 2]).astype(np.float32)
    got = np.array([oracle.f32_to_f16_bits(v) for v in vals], np.uint16)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_f16_to_f64_all_patterns():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    sel = ~np.isnan(want)
    got = np.array([oracle.f16_bits_to_f64(b) for b in bits[sel][::7]])
    assert np.array_equal(got, want[sel][::7])


def test_bf16_to_f32_matches_torch():
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 1 << 16, 5000).astype(np.uint16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([oracle.bf16_to_f32(b) for b in bits], np.float32)
    fin = np.isfinite(want)
    assert np.array_equal(got[fin].view(np.uint32), want[fin].view(np.uint32))


# ---------------------------------------------------------------------------------------
# quantizer
# ---------------------------------------------------------------------------------------

def _golden_input(spec):
    x = np.zeros(128, np.float32)
    if spec["kind"] == "sparse":
        for k, v in spec["entries"].items():
            x[int(k)] = v
    elif spec["kind"] == "constant":
        x[:] = spec["value"]
    elif spec["kind"] == "list_then_fill":
        x[:] = spec["fill"]
        x[:len(spec["values"])] = spec["values"]
    return x


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_quantizer_golden(case):
    x = _golden_input(case["input"])
    y = oracle.fwht_f32(x) if case["rotate"] else x
    packed, sh, zh, _, _ = oracle.quantize_vec(y)
    if "packed_hex_all" in case:
        want = bytes.fromhex(case["packed_hex_all"]) * 64
    else:
        pre = bytes.fromhex(case["packed_hex_prefix"])
        want = pre + bytes.fromhex(case["packed_rest"]) * (64 - len(pre))
    assert packed.tobytes() == want
    assert sh == int(case["scale_f16"], 16)
    assert zh == int(case["zero_f16"], 16)


def _unpack(packed):
    codes = np.empty(packed.size * 2, np.int64)
    codes[0::2] = packed & 0xF
    codes[1::2] = packed >> 4
    return codes


def _random_vectors(n, rng):
    out = []
    for i in range(n):
        kind = i % 4
        x = rng.standard_normal(128).astype(np.float32)
        if kind == 1:
            x[rng.choice(128, 4, replace=False)] *= np.float32(rng.uniform(10, 30))
        if kind == 2:
            x = (x * np.float32(10.0) ** rng.integers(-20, 20)).astype(np.float32)
        if kind == 3:
            x = np.round(x * 4) / 4            # many exact ties
        out.append(oracle.fwht_f32(x) if i % 2 == 0 else x)
    return out


def test_quantizer_invariants_and_bound():
    """min -> 0, max -> 15, monotone codes, |y - (min + code scale)| <= scale/2 (fp32 values),
    and with the stored fp16 values the reading's widened bound holds."""
    rng = np.random.default_rng(21)
    for y in _random_vectors(400, rng):
        packed, sh, zh, sf, mf = oracle.quantize_vec(y)
        codes = _unpack(packed)
        assert sf > 0
        assert codes[np.argmin(y)] == 0 and codes[np.argmax(y)] == 15
        order = np.argsort(y, kind="stable")
        assert np.all(np.diff(codes[order]) >= 0)
        yd = y.astype(np.float64)
        err = np.abs(yd - (np.float64(mf) + codes * np.float64(sf)))
        ulp = np.spacing(np.float32(np.abs(y).max())).astype(np.float64)
        assert err.max() <= np.float64(sf) / 2 + 16 * ulp
        s16, z16 = oracle.f16_bits_to_f64(sh), oracle.f16_bits_to_f64(zh)
        if not (6.2e-5 < sf < 6e4 and abs(mf) < 6e4 and (mf == 0 or abs(mf) > 6.2e-5)):
            continue                 # fp16 storage range: overflow/underflow is unsupported
        err16 = np.abs(yd - (z16 + codes * s16))
        bound16 = s16 / 2 + 15 * abs(sf - s16) + abs(mf - z16) + 16 * ulp + abs(sf - s16) / 2
        assert err16.max() <= bound16


def test_quantizer_brute_force_nearest_level():
    """Each code is the level k in 0..15 nearest (exact rationals) to (y - min)/scale as the
    fp32 values give it; within a hair of a half-integer either neighbour is allowed and an
    exact half goes to the even level."""
    rng = np.random.default_rng(22)
    for y in _random_vectors(120, rng):
        packed, _, _, sf, mf = oracle.quantize_vec(y)
        codes = _unpack(packed)
        S, M = Fraction(float(sf)), Fraction(float(mf))
        for i in range(128):
            d = Fraction(float(np.float32(y[i] - np.float32(mf))))   # the fp32 difference
            q = d / S
            lo = int(q)                                               # q >= 0
            frac = q - lo
            half = Fraction(1, 2)
            if abs(frac - half) <= Fraction(1, 1 << 18):
                assert codes[i] in (lo, min(lo + 1, 15))
                if frac == half:
                    assert codes[i] % 2 == 0 or codes[i] == 15
            else:
                want = lo + (1 if frac > half else 0)
                assert codes[i] == min(max(want, 0), 15)
        del M


def test_quantizer_degenerate_and_signed_zero():
    packed, sh, zh, sf, _ = oracle.quantize_vec(np.full(128, -2.5, np.float32))
    assert sf == 0.0 and sh == 0 and zh == np.array(np.float16(-2.5)).view(np.uint16)
    assert not packed.any()
    y = np.zeros(128, np.float32)
    y[5] = -0.0
    y[9] = 1.0
    packed, sh, zh, _, _ = oracle.quantize_vec(y)
    assert zh == 0x0000                        # a zero minimum is stored as +0
    assert _unpack(packed)[9] == 15 and _unpack(packed)[5] == 0


def test_quantizer_subnormal_scale():
    """Tiny vectors whose scale is subnormal still satisfy min -> 0 and max -> 15."""
    y = np.zeros(128, np.float32)
    y[3] = np.float32(1e-39)
    y[7] = np.float32(-2e-39)
    packed, _, _, sf, _ = oracle.quantize_vec(y)
    codes = _unpack(packed)
    assert 0 < sf < np.finfo(np.float32).tiny
    assert codes[7] == 0 and codes[3] == 15


# ---------------------------------------------------------------------------------------
# scatter into the paged layout
# ---------------------------------------------------------------------------------------

@pytest.mark.parametrize("D", [64, 128])
def test_scatter_layout_and_skips(D):
    rng = np.random.default_rng(31)
    T, Hkv, P, num_pages = 40, 3, 16, 6
    k = synth.bf16_bits(torch.randn(T, Hkv, D).to(torch.bfloat16))
    v = synth.bf16_bits(torch.randn(T, Hkv, D).to(torch.bfloat16))
    slots = rng.permutation(num_pages * P)[:T].astype(np.int64)
    slots[3] = -1
    slots[11] = num_pages * P + 5          # out of range: skipped and counted
    pages, scales = oracle.empty_cache(num_pages, Hkv, D, P)
    pages[:] = 0xA5
    scales[:] = 0x5A5A
    bad = oracle.rotate_quantize_paged(k, v, slots, pages, scales, page_size=P)
    assert bad == 1
    touched = np.zeros((num_pages, P), bool)
    for t in range(T):
        s = slots[t]
        if s < 0 or s >= num_pages * P:
            continue
        pg, off = divmod(int(s), P)
        touched[pg, off] = True
        for h in range(Hkv):
            for sel, src in enumerate((k, v)):
                x = src[t, h].view(np.int16).astype(np.int32) << 16
                y = oracle.fwht_f32(x.astype(np.uint32).view(np.float32))
                pk, sh, zh, _, _ = oracle.quantize_vec(y)
                assert np.array_equal(pages[pg, h, sel, off], pk)
                assert scales[pg, h, sel, off, 0] == sh and scales[pg, h, sel, off, 1] == zh
    for pg in range(num_pages):
        for off in range(P):
            if not touched[pg, off]:
                assert np.all(pages[pg, :, :, off] == 0xA5)
                assert np.all(scales[pg, :, :, off] == 0x5A5A)


def test_scatter_unrotated_variant():
    T, Hkv, D = 4, 1, 128
    k = synth.bf16_bits(torch.randn(T, Hkv, D).to(torch.bfloat16))
    pages, scales = oracle.empty_cache(1, Hkv, D)
    oracle.rotate_quantize_paged(k, k, np.arange(T, dtype=np.int64), pages, scales,
                                 rotate=False)
    x = (k[2, 0].view(np.int16).astype(np.int32) << 16).astype(np.uint32).view(np.float32)
    pk, _, _, _, _ = oracle.quantize_vec(x)
    assert np.array_equal(pages[0, 0, 0, 2], pk)


def test_dequant_round_trip_bound():
    """Dequantising the stored codes lands within the quantizer's error bound of y."""
    rng = np.random.default_rng(41)
    wl = synth.make_workload("tiny")
    k = synth.bf16_bits(synth.kv_values(wl, "K"))
    v = synth.bf16_bits(synth.kv_values(wl, "V"))
    seq, pos = synth.token_index(wl)
    slots = synth.slot_mapping(wl, seq, pos)
    pages, scales = oracle.empty_cache(wl.num_pages, wl.num_kv_heads)
    oracle.rotate_quantize_paged(k, v, slots, pages, scales)
    for t in rng.choice(len(slots), 20, replace=False):
        pg, off = divmod(int(slots[t]), 16)
        for h in range(wl.num_kv_heads):
            x = (k[t, h].view(np.int16).astype(np.int32) << 16).astype(np.uint32).view(
                np.float32)
            y = oracle.fwht_f32(x).astype(np.float64)
            yhat = oracle.dequant_row_f64(pages, scales, pg, h, 0, off)
            s16 = oracle.f16_bits_to_f64(scales[pg, h, 0, off, 0])
            assert np.abs(yhat - y).max() <= 0.5 * s16 * 1.01 + 15 * s16 * 2 ** -11 + \
                abs(y.min()) * 2 ** -11


# ---------------------------------------------------------------------------------------
# decode attention
# ---------------------------------------------------------------------------------------

def _cache_for(wl, rotate=True):
    k = synth.bf16_bits(synth.kv_values(wl, "K"))
    v = synth.bf16_bits(synth.kv_values(wl, "V"))
    seq, pos = synth.token_index(wl)
    slots = synth.slot_mapping(wl, seq, pos)
    pages, scales = oracle.empty_cache(wl.num_pages, wl.num_kv_heads, wl.head_dim,
                                       wl.page_size)
    oracle.rotate_quantize_paged(k, v, slots, pages, scales, page_size=wl.page_size,
                                 rotate=rotate)
    return k, v, pages, scales


def _dequant_seq(wl, pages, scales, s, h, sel):
    L = int(wl.seq_lens[s])
    rows = []
    for t in range(L):
        pg = wl.block_table[s, t // 16]
        rows.append(oracle.dequant_row_f64(pages, scales, pg, h, sel, t % 16))
    return np.stack(rows)


def test_decode_single_token_is_rotated_value():
    wl = synth.custom("one", [1], num_q_heads=4, num_kv_heads=2, seed=1)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens)
    Hn = H128 / np.sqrt(128.0)
    for hq in range(4):
        vhat = _dequant_seq(wl, pages, scales, 0, hq // 2, 1)[0]
        assert np.abs(out[0, hq] - Hn @ vhat).max() <= 1e-12


def test_decode_matches_torch_sdpa_fp64():
    """G = 1: the oracle equals torch's fp64 scaled-dot-product attention run on the rotated
    query and the dequantised cache, rotated back."""
    wl = synth.custom("sdpa", [37, 16, 17, 1, 64], num_q_heads=2, num_kv_heads=2, seed=2)
    _, _, pages, scales = _cache_for(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(qb, pages, scales, wl.block_table, wl.seq_lens)
    Hn = torch.tensor(H128 / np.sqrt(128.0))
    qf = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double()
    for s in range(wl.num_seqs):
        for h in range(2):
            K = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 0))
            V = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 1))
            qr = Hn @ qf[s, h]
            o = torch.nn.functional.scaled_dot_product_attention(
                qr[None, None, None], K[None, None], V[None, None])[0, 0, 0]
            assert torch.allclose(torch.from_numpy(out[s, h]), Hn @ o, atol=1e-12, rtol=0)


def test_decode_d256_matches_torch_sdpa_fp64():
    """D = 256: one (scale, zero) per 256-element vector, each 128-element half rotated on its
    own, sm_scale 1/16.  The oracle equals torch's fp64 SDPA on the block-diagonally rotated
    query and the dequantised cache, rotated back block by block."""
    wl = synth.custom("sdpa256", [37, 16, 1, 50], num_q_heads=4, num_kv_heads=2, seed=21,
                      head_dim=256)
    _, _, pages, scales = _cache_for(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(qb, pages, scales, wl.block_table, wl.seq_lens)
    Hn = H128 / np.sqrt(128.0)
    R = torch.tensor(np.block([[Hn, np.zeros((128, 128))], [np.zeros((128, 128)), Hn]]))
    qf = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double()
    for s in range(wl.num_seqs):
        for hq in range(4):
            h = hq // 2
            K = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 0))
            V = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 1))
            o = torch.nn.functional.scaled_dot_product_attention(
                (R @ qf[s, hq])[None, None, None], K[None, None], V[None, None])[0, 0, 0]
            assert torch.allclose(torch.from_numpy(out[s, hq]), R @ o, atol=1e-12, rtol=0)


def test_decode_d64_matches_torch_sdpa_fp64():
    """D = 64: the 64-point rotation (1/8) and sm_scale 1/8; the oracle equals torch's fp64 SDPA
    on the rotated query and the dequantised cache, rotated back."""
    wl = synth.custom("sdpa64", [37, 16, 1, 50], num_q_heads=4, num_kv_heads=2, seed=22,
                      head_dim=64)
    _, _, pages, scales = _cache_for(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(qb, pages, scales, wl.block_table, wl.seq_lens)
    R = torch.tensor(hadamard(64).astype(np.float64) / 8.0)
    qf = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).double()
    for s in range(wl.num_seqs):
        for hq in range(4):
            h = hq // 2
            K = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 0))
            V = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 1))
            o = torch.nn.functional.scaled_dot_product_attention(
                (R @ qf[s, hq])[None, None, None], K[None, None], V[None, None])[0, 0, 0]
            assert torch.allclose(torch.from_numpy(out[s, hq]), R @ o, atol=1e-12, rtol=0)


def test_decode_identical_keys_and_zero_scale_give_mean():
    """If every key is the same, or sm_scale is 0, the weights are uniform: the output is the
    rotated mean of the dequantised values."""
    wl = synth.custom("flat", [50], num_q_heads=2, num_kv_heads=1, seed=3)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    Hn = H128 / np.sqrt(128.0)
    V = _dequant_seq(wl, pages, scales, 0, 0, 1)
    out0 = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens, sm_scale=0.0)
    assert np.abs(out0[0, 0] - Hn @ V.mean(0)).max() <= 1e-12
    pages2, scales2 = pages.copy(), scales.copy()
    first = wl.block_table[0, 0]
    for t in range(50):
        pg = wl.block_table[0, t // 16]
        pages2[pg, 0, 0, t % 16] = pages[first, 0, 0, 0]
        scales2[pg, 0, 0, t % 16] = scales[first, 0, 0, 0]
    out = oracle.decode_fp64(q, pages2, scales2, wl.block_table, wl.seq_lens)
    assert np.abs(out[0, 1] - Hn @ V.mean(0)).max() <= 1e-12


def test_decode_dominant_key_selects_its_value():
    wl = synth.custom("dom", [40], num_q_heads=1, num_kv_heads=1, seed=4)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    V = _dequant_seq(wl, pages, scales, 0, 0, 1)
    K = _dequant_seq(wl, pages, scales, 0, 0, 0)
    qf = (q[0, 0].view(np.int16).astype(np.int32) << 16).astype(np.uint32).view(np.float32)
    qr = (H128 / np.sqrt(128.0)) @ qf.astype(np.float64)
    t = int(np.argmax(K @ qr))
    out = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens, sm_scale=1e4)
    assert np.abs(out[0, 0] - (H128 / np.sqrt(128.0)) @ V[t]).max() <= 1e-9


def test_decode_gqa_head_mapping():
    """Query head hq reads kv head hq // G: the same as a G = 1 run on that head alone."""
    wl = synth.custom("gqa", [33, 70], num_q_heads=8, num_kv_heads=2, seed=5)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens)
    for hq in range(8):
        h = hq // 4
        p1 = np.ascontiguousarray(pages[:, h:h + 1])
        s1 = np.ascontiguousarray(scales[:, h:h + 1])
        o1 = oracle.decode_fp64(np.ascontiguousarray(q[:, hq:hq + 1]), p1, s1,
                                wl.block_table, wl.seq_lens)
        assert np.array_equal(o1[:, 0], out[:, hq])
    assert np.abs(out[:, 0] - out[:, 4]).max() > 1e-3     # the two kv heads differ


def test_decode_page_permutation_invariance():
    wl = synth.custom("perm", [45, 16, 17], num_q_heads=4, num_kv_heads=1, seed=6)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens)
    perm = np.random.default_rng(0).permutation(wl.num_pages)
    inv = np.argsort(perm)
    table2 = np.where(wl.block_table >= 0, inv[np.maximum(wl.block_table, 0)], -1).astype(
        np.int32)
    out2 = oracle.decode_fp64(q, np.ascontiguousarray(pages[perm]),
                              np.ascontiguousarray(scales[perm]), table2, wl.seq_lens)
    assert np.array_equal(out, out2)


def test_decode_empty_sequence_is_zero():
    wl = synth.custom("empty", [0, 5], num_q_heads=2, num_kv_heads=1, seed=7)
    _, _, pages, scales = _cache_for(wl)
    q = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_fp64(q, pages, scales, wl.block_table, wl.seq_lens)
    assert not out[0].any() and np.abs(out[1]).max() > 0


# ---------------------------------------------------------------------------------------
# method-level check: rotation helps on outlier keys
# ---------------------------------------------------------------------------------------

def test_rotation_lowers_quantized_attention_error():
    """On keys with outlier channels, rotating before the INT4 quantizer gives lower logit and
    output error against unquantized fp64 attention than the plain INT4 quantizer does
    ("SAW-INT4", Research Findings: naive INT4 degrades accuracy; the rotation recovers most
    of it).  The size of the gain is not given on the pages (parity unpinned)."""
    wl = synth.make_workload("tiny")
    kb = synth.bf16_bits(synth.kv_values(wl, "K"))
    vb = synth.bf16_bits(synth.kv_values(wl, "V"))
    qb = synth.bf16_bits(synth.q_values(wl))
    tof = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double()
    K, V, Q = tof(kb), tof(vb), tof(qb)                 # [T][Hkv][D], [S][Hq][D]
    G = wl.group
    errs = {}
    for rotate in (True, False):
        seq, pos = synth.token_index(wl)
        slots = synth.slot_mapping(wl, seq, pos)
        pages, scales = oracle.empty_cache(wl.num_pages, wl.num_kv_heads)
        oracle.rotate_quantize_paged(kb, vb, slots, pages, scales, rotate=rotate)
        out = oracle.decode_fp64(qb, pages, scales, wl.block_table, wl.seq_lens,
                                 rotate=rotate)
        o_err, l_err = [], []
        for hq in range(wl.num_q_heads):
            h = hq // G
            ref = torch.nn.functional.scaled_dot_product_attention(
                Q[0, hq][None, None, None], K[:, h][None, None], V[:, h][None, None])[0, 0, 0]
            o_err.append(np.abs(out[0, hq] - ref.numpy()).mean())
            Kq = torch.from_numpy(_dequant_seq(wl, pages, scales, 0, h, 0))
            Hn = torch.tensor(H128 / np.sqrt(128.0))
            qr = Hn @ Q[0, hq] if rotate else Q[0, hq]
            l_err.append((Kq @ qr - K[:, h] @ Q[0, hq]).abs().mean().item())
        errs[rotate] = (np.mean(o_err), np.mean(l_err))
    assert errs[True][0] < errs[False][0]
    assert errs[True][1] < errs[False][1]


# ---- the BF16 paged-cache baseline (uncompressed; no rotation, no quantization) ---------------

def _bf16_cache(wl):
    """Oracle bf16 cache of every token of the workload, and the bf16 bits of K and V."""
    k, v = synth.kv_values(wl, "K"), synth.kv_values(wl, "V")
    seq, pos = synth.token_index(wl)
    kv = oracle.empty_cache_bf16(wl.num_pages, wl.num_kv_heads)
    assert oracle.append_bf16(synth.bf16_bits(k), synth.bf16_bits(v),
                              synth.slot_mapping(wl, seq, pos), kv) == 0
    return kv, synth.bf16_bits(k), synth.bf16_bits(v)


def test_bf16_append_scatter_and_skips():
    """Every row lands at page = slot / 16, offset slot % 16, (kv head, K|V) untouched otherwise;
    negative slots are skipped, slots past the cache are skipped and counted."""
    rng = np.random.default_rng(11)
    T, Hkv, P = 40, 3, 4
    k = rng.integers(0, 1 << 16, (T, Hkv, 128), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, (T, Hkv, 128), dtype=np.uint16)
    slots = rng.permutation(P * 16)[:T].astype(np.int64)
    slots[3] = -1
    slots[7] = P * 16 + 5
    kv = np.full((P, Hkv, 2, 16, 128), 0xABCD, dtype=np.uint16)
    assert oracle.append_bf16(k, v, slots, kv) == 1
    written = np.zeros((P, 16), dtype=bool)
    for t, slot in enumerate(slots):
        if 0 <= slot < P * 16:
            page, off = divmod(int(slot), 16)
            written[page, off] = True
            assert np.array_equal(kv[page, :, 0, off], k[t]) and np.array_equal(kv[page, :, 1, off], v[t])
    assert np.all(kv.transpose(0, 3, 1, 2, 4)[~written] == 0xABCD)


def test_bf16_decode_matches_torch_sdpa_fp64():
    wl = synth.custom("bf16sdpa", [1, 16, 17, 40], num_q_heads=4, num_kv_heads=4, seed=5)
    kv, kb, vb = _bf16_cache(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    got = oracle.decode_bf16_fp64(qb, kv, wl.block_table, wl.seq_lens)
    q = torch.from_numpy(qb.astype(np.uint32) << 16).view(torch.float32).double()
    k = torch.from_numpy(kb.astype(np.uint32) << 16).view(torch.float32).double()
    v = torch.from_numpy(vb.astype(np.uint32) << 16).view(torch.float32).double()
    start = 0
    for s, L in enumerate(wl.seq_lens.tolist()):
        for hq in range(wl.num_q_heads):
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[s, hq][None, None, None], k[start:start + L, hq][None, None],
                v[start:start + L, hq][None, None])[0, 0, 0]
            assert np.allclose(got[s, hq], ref.numpy(), atol=1e-12, rtol=1e-12)
        start += L


def test_bf16_decode_single_token_gqa_and_empty():
    """seq_len 1 gives that token's value exactly; query head hq reads kv head hq / G; an empty
    sequence gives zeros."""
    wl = synth.custom("bf16g", [1, 0, 33], num_q_heads=8, num_kv_heads=2, seed=6)
    kv, kb, vb = _bf16_cache(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    out = oracle.decode_bf16_fp64(qb, kv, wl.block_table, wl.seq_lens)
    vf = (vb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for hq in range(8):
        assert np.array_equal(out[0, hq], vf[0, hq // 4])
    assert np.all(out[1] == 0.0)
    for hq in range(8):   # the same output as a single-head cache holding only kv head hq / G
        sub = kv[:, hq // 4: hq // 4 + 1].copy()
        one = oracle.decode_bf16_fp64(qb[2:3, hq:hq + 1], sub, wl.block_table[2:3], wl.seq_lens[2:3])
        assert np.array_equal(one[0, 0], out[2, hq])


def test_bf16_decode_page_permutation_invariance():
    wl = synth.custom("bf16perm", [70], num_q_heads=2, num_kv_heads=2, seed=8)
    kv, _, _ = _bf16_cache(wl)
    qb = synth.bf16_bits(synth.q_values(wl))
    base = oracle.decode_bf16_fp64(qb, kv, wl.block_table, wl.seq_lens)
    perm = np.random.default_rng(3).permutation(wl.num_pages)
    kv2 = np.empty_like(kv)
    kv2[perm] = kv
    table2 = np.where(wl.block_table >= 0, perm[np.maximum(wl.block_table, 0)], -1).astype(np.int32)
    assert np.array_equal(oracle.decode_bf16_fp64(qb, kv2, table2, wl.seq_lens), base)


# ---- chunked prefill over the INT4 cache ------------------------------------------------------

def _prefill_case(lens, chunks, hq, hkv, seed):
    wl = synth.custom(f"pf{seed}", lens, num_q_heads=hq, num_kv_heads=hkv, seed=seed,
                      outlier_range=(10.0, 30.0))
    _, _, pages, scales = _cache_for(wl)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    qb = synth.bf16_bits(torch.randn(int(q_start[-1]), hq, 128, generator=g).to(torch.bfloat16))
    return wl, pages, scales, q_start, qb


def test_prefill_matches_torch_causal_sdpa_fp64():
    """Each chunk query against torch fp64 SDPA with an explicit causal mask, on the rotated
    query (Sylvester matrix from scipy) and the dequantized (rotated-domain) cache, rotated
    back."""
    lens, chunks = [40, 17, 33], [7, 17, 1]
    wl, pages, scales, q_start, qb = _prefill_case(lens, chunks, hq=4, hkv=2, seed=3)
    got = oracle.prefill_fp64(qb, q_start, pages, scales, wl.block_table, wl.seq_lens)
    H = torch.from_numpy(hadamard(128).astype(np.float64)) / np.sqrt(128.0)
    q = torch.from_numpy(qb.astype(np.uint32) << 16).view(torch.float32).double()
    for s, (L, C) in enumerate(zip(lens, chunks)):
        for hq in range(4):
            h = hq // 2
            k = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 0))[:L]
            v = torch.from_numpy(_dequant_seq(wl, pages, scales, s, h, 1))[:L]
            qr = q[q_start[s]:q_start[s + 1], hq] @ H
            mask = torch.arange(L)[None, :] <= (L - C + torch.arange(C))[:, None]
            o = torch.nn.functional.scaled_dot_product_attention(
                qr[None, None], k[None, None], v[None, None], attn_mask=mask[None, None])[0, 0]
            assert np.allclose(got[q_start[s]:q_start[s + 1], hq], (o @ H).numpy(), atol=1e-10)


def test_prefill_rows_equal_decode_on_their_prefix():
    """Query i of a chunk is a decode over the first L - C + i + 1 tokens."""
    lens, chunks = [50, 20], [9, 20]
    wl, pages, scales, q_start, qb = _prefill_case(lens, chunks, hq=8, hkv=2, seed=4)
    got = oracle.prefill_fp64(qb, q_start, pages, scales, wl.block_table, wl.seq_lens)
    for s, (L, C) in enumerate(zip(lens, chunks)):
        for i in range(C):
            row = q_start[s] + i
            dec = oracle.decode_fp64(qb[row:row + 1], pages, scales, wl.block_table[s:s + 1],
                                     np.array([L - C + i + 1], dtype=np.int32))
            assert np.allclose(got[row], dec[0], atol=1e-12, rtol=1e-12)


# ---------------------------------------------------------------------------------------
# full-precision sink / recent window ("InnerQ", Abstract and Figure 2)
# ---------------------------------------------------------------------------------------

def _window_state(lens, w_sink, w_recent, Hkv=2, D=128, seed=0, rotate=True):
    """Token values for every position and the oracle window state after filling them."""
    S, Lmax = len(lens), max(max(lens), 1)
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(S, Lmax, Hkv, D, generator=g)
    k[..., 3] *= 20.0                                   # an outlier key channel
    k = synth.bf16_bits(k.to(torch.bfloat16))
    v = synth.bf16_bits(torch.randn(S, Lmax, Hkv, D, generator=g).to(torch.bfloat16))
    W = w_sink + w_recent
    pw = max(1, (W + 15) // 16)
    win_table = (np.arange(S * pw, dtype=np.int32).reshape(S, pw) * 7 + 3) % (S * pw)
    win_kv = np.zeros((S * pw, Hkv, 2, 16, D), np.uint16)
    nq = max(1, (Lmax + 15) // 16)
    block_table = np.random.default_rng(seed).permutation(S * nq).astype(np.int32).reshape(S, nq)
    pages, scales = oracle.empty_cache(S * nq, Hkv, D)
    oracle.window_fill(k, v, np.array(lens), w_sink, w_recent, win_kv, win_table, pages, scales,
                       block_table, rotate=rotate)
    return k, v, win_kv, win_table, pages, scales, block_table


def test_window_of_width_zero_is_the_int4_decode():
    """w_sink = w_recent = 0: every token is quantized; the window decode (which rotates keys and
    values back) equals the INT4 decode (which rotates the query and the output)."""
    lens = [37, 1, 16, 70]
    k, v, win_kv, win_table, pages, scales, bt = _window_state(lens, 0, 0, seed=1)
    q = synth.bf16_bits(torch.randn(len(lens), 4, 128).to(torch.bfloat16))
    a = oracle.decode_window_fp64(q, win_kv, win_table, pages, scales, bt,
                                  np.array(lens, np.int32), 0, 0)
    b = oracle.decode_fp64(q, pages, scales, bt, np.array(lens, np.int32))
    assert np.abs(a - b).max() <= 1e-12


@pytest.mark.parametrize("w_sink,w_recent", [(4, 60), (16, 112), (0, 40)])
def test_window_covering_the_sequence_is_bf16_attention(w_sink, w_recent):
    """L <= W: nothing is quantized; the output is fp64 SDPA over the bf16 keys and values."""
    lens = [1, 5, w_sink + w_recent, 17]
    k, v, win_kv, win_table, pages, scales, bt = _window_state(lens, w_sink, w_recent, seed=2)
    q = synth.bf16_bits(torch.randn(len(lens), 2, 128).to(torch.bfloat16))
    out = oracle.decode_window_fp64(q, win_kv, win_table, pages, scales, bt,
                                    np.array(lens, np.int32), w_sink, w_recent)
    tq = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()
    tk = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).double()
    tv = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).double()
    for s, L in enumerate(lens):
        for hq in range(2):
            o = torch.nn.functional.scaled_dot_product_attention(
                tq[s, hq][None, None, None], tk[s, :L, hq][None, None], tv[s, :L, hq][None, None])
            assert torch.allclose(torch.from_numpy(out[s, hq]), o[0, 0, 0], atol=1e-12, rtol=0)


@pytest.mark.parametrize("w_sink,w_recent", [(4, 12), (16, 112), (0, 32), (8, 0)])
def test_window_matches_sdpa_over_bf16_window_and_dequantized_middle(w_sink, w_recent):
    """Every position once: sinks and recent tokens with their bf16 values, the middle tokens
    dequantized and rotated back; fp64 SDPA over that set equals the oracle."""
    lens = [300, 3, 150, 128]
    k, v, win_kv, win_table, pages, scales, bt = _window_state(lens, w_sink, w_recent, seed=3)
    q = synth.bf16_bits(torch.randn(len(lens), 4, 128).to(torch.bfloat16))
    out = oracle.decode_window_fp64(q, win_kv, win_table, pages, scales, bt,
                                    np.array(lens, np.int32), w_sink, w_recent)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    tq, tk, tv = bf(q), bf(k), bf(v)
    for s, L in enumerate(lens):
        for hq in range(4):
            h = hq // 2
            keys, vals = [], []
            for p in range(L):
                if p < w_sink or p >= max(w_sink, L - w_recent):
                    keys.append(tk[s, p, h])
                    vals.append(tv[s, p, h])
                else:
                    j = p - w_sink
                    pg, off = int(bt[s, j // 16]), j % 16
                    keys.append(torch.from_numpy(oracle.rotate_f64(
                        oracle.dequant_row_f64(pages, scales, pg, h, 0, off))))
                    vals.append(torch.from_numpy(oracle.rotate_f64(
                        oracle.dequant_row_f64(pages, scales, pg, h, 1, off))))
            o = torch.nn.functional.scaled_dot_product_attention(
                tq[s, hq][None, None, None], torch.stack(keys)[None, None],
                torch.stack(vals)[None, None])[0, 0, 0]
            assert torch.allclose(torch.from_numpy(out[s, hq]), o, atol=1e-12, rtol=0)


@pytest.mark.parametrize("w_sink,w_recent", [(4, 12), (16, 112), (0, 32), (8, 0), (16, 16)])
def test_window_append_steps_equal_fill(w_sink, w_recent):
    """Appending tokens one step at a time (the quantized token is the one leaving the recent
    window) reaches exactly the state that placing every token directly gives: window bits and
    INT4 codes / scales bit-identical.  The window then holds the sinks and the last w_recent
    tokens at their slots."""
    L0, steps = [0, 3, 20, 140], 37
    L1 = [x + steps for x in L0]
    k, v, win_kv, win_table, pages, scales, bt = _window_state(L1, w_sink, w_recent, seed=4)
    win2 = np.zeros_like(win_kv)
    pages2, scales2 = oracle.empty_cache(*pages.shape[:2], 128)
    oracle.window_fill(k, v, np.array(L0), w_sink, w_recent, win2, win_table, pages2, scales2, bt)
    for i in range(1, steps + 1):
        lens = np.array([x + i for x in L0])
        kn = np.stack([k[s, lens[s] - 1] for s in range(len(L0))])
        vn = np.stack([v[s, lens[s] - 1] for s in range(len(L0))])
        oracle.window_append(kn, vn, lens, w_sink, w_recent, win2, win_table, pages2, scales2, bt)
    assert np.array_equal(win2, win_kv)
    assert np.array_equal(pages2, pages) and np.array_equal(scales2, scales)
    s, L = 3, L1[3]                                   # direct check of the window contents
    for p in list(range(min(L, w_sink))) + list(range(max(w_sink, L - w_recent), L)):
        slot = oracle.window_slot(p, w_sink, w_recent)
        pg = win_table[s, slot // 16]
        assert np.array_equal(win_kv[pg, :, 0, slot % 16], k[s, p])
        assert np.array_equal(win_kv[pg, :, 1, slot % 16], v[s, p])


def test_window_decode_ignores_the_order_of_window_slots():
    """The window is a set: moving its tokens to other slots (and pages) leaves the output."""
    lens = [200, 90]
    k, v, win_kv, win_table, pages, scales, bt = _window_state(lens, 16, 48, seed=5)
    q = synth.bf16_bits(torch.randn(2, 4, 128).to(torch.bfloat16))
    a = oracle.decode_window_fp64(q, win_kv, win_table, pages, scales, bt,
                                  np.array(lens, np.int32), 16, 48)
    perm = np.random.default_rng(0).permutation(64)
    win_b = win_kv.copy()
    for s in range(2):
        for i in range(64):
            j = perm[i]
            win_b[win_table[s, j // 16], :, :, j % 16] = win_kv[win_table[s, i // 16], :, :, i % 16]
    b = oracle.decode_window_fp64(q, win_b, win_table, pages, scales, bt,
                                  np.array(lens, np.int32), 16, 48)
    assert np.abs(a - b).max() <= 1e-12

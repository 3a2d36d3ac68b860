"""Seeded synthetic inputs for the SAW-INT4 paged KV-cache path.

This module only draws inputs: sequence lengths, page assignments, slot mappings and bf16
query/key/value tensors.  It contains none of the method's arithmetic (no rotation, no
quantization, no attention), so both the CUDA path and the CPU oracle can take their inputs
from it.

Value distribution (the pages describe LLM KV caches whose keys carry a few outlier channels,
which is what the Hadamard rotation is for -- "SAW-INT4", Research Findings; "BitDecoding-FP4",
abstract: "suppress key outliers under token-wise scaling"): q, K and V are i.i.d. N(0, 1)
rounded to bf16; in K, four fixed channels per kv head are multiplied by a per-(head, channel)
factor before the rounding.  V and q carry no outliers.

Workloads (all head_dim 128, 16-token pages):
  tiny     1 seq x 256 tokens, 2 kv / 8 q heads, key outliers x20, block table shuffled
  prefill  32 seqs x 2048 tokens appended, 8 kv heads, outliers x U[10, 30], pages by a seeded
           random permutation of 4096 pages assigned to (seq, block) in order
  decode   64 seqs, lengths uniform on {512..8192}, 32 q / 8 kv heads, one new token per seq
           appended then decoded, outliers x U[10, 30], pages from a shuffled pool
  long     8 seqs x 32768 tokens, 64 q / 8 kv heads, outliers x20, block table a shuffled
           permutation of 16384 pages, decode only
  serving  256 seqs, lengths round(lognormal(ln 1024, sigma 1.0)) clipped to [64, 16384],
           32 q / 8 kv heads, one new token per seq appended then decoded, outliers x U[10, 30]
"""
from __future__ import annotations

import dataclasses
import hashlib

import numpy as np
import torch

PAGE_SIZE = 16
HEAD_DIM = 128
N_OUTLIER_CHANNELS = 4


@dataclasses.dataclass
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    seq_lens: np.ndarray          # int32 [S]: tokens in the cache once this step's tokens are in
    new_tokens: np.ndarray        # int32 [S]: tokens of each seq appended in this step
    num_pages: int
    block_table: np.ndarray       # int32 [S][max_blocks]; -1 marks an unused entry
    outlier_channels: np.ndarray  # int64 [Hkv][4]
    outlier_scale: np.ndarray     # float32 [Hkv][4]
    seed: int
    decode: bool = True           # whether the step runs decode attention after the append

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.astype(np.int64).sum())

    @property
    def history_lens(self) -> np.ndarray:
        return (self.seq_lens - self.new_tokens).astype(np.int32)


def _seed_for(seed: int, *names) -> int:
    """A stable 63-bit seed for one named tensor of one workload."""
    h = hashlib.sha256(("%d|" % seed + "|".join(str(n) for n in names)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _rng(seed: int, *names) -> np.random.Generator:
    return np.random.default_rng(_seed_for(seed, *names))


def _assign_pages(seq_lens: np.ndarray, num_pages: int, page_size: int, rng) -> np.ndarray:
    blocks = (seq_lens.astype(np.int64) + page_size - 1) // page_size
    need = int(blocks.sum())
    if need > num_pages:
        raise ValueError(f"{need} pages needed, pool has {num_pages}")
    perm = rng.permutation(num_pages).astype(np.int32)
    max_blocks = max(1, int(blocks.max()) if len(blocks) else 1)
    table = np.full((len(seq_lens), max_blocks), -1, dtype=np.int32)
    k = 0
    for s, nb in enumerate(blocks):
        table[s, :nb] = perm[k:k + nb]
        k += nb
    return table


def custom(name: str, seq_lens, *, num_q_heads: int, num_kv_heads: int, seed: int = 0,
           new_tokens=None, num_pages: int | None = None, outlier_scale=20.0,
           outlier_range=None, head_dim: int = HEAD_DIM, page_size: int = PAGE_SIZE,
           shuffle_pages: bool = True, decode: bool = True) -> Workload:
    """Build a workload from explicit sequence lengths.

    new_tokens: per-seq tokens appended in the step (default: 1 per seq).
    outlier_scale: constant factor for the outlier key channels, or None for no outliers;
    outlier_range=(lo, hi) draws the factor per (head, channel) uniformly instead."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32).reshape(-1)
    S = len(seq_lens)
    if new_tokens is None:
        new_tokens = np.minimum(seq_lens, 1)
    new_tokens = np.broadcast_to(np.asarray(new_tokens, dtype=np.int32), (S,)).copy()
    need = int(((seq_lens.astype(np.int64) + page_size - 1) // page_size).sum())
    if num_pages is None:
        num_pages = max(need, 1)
    rng_pages = _rng(seed, name, "pages")
    if shuffle_pages:
        table = _assign_pages(seq_lens, num_pages, page_size, rng_pages)
    else:
        blocks = (seq_lens.astype(np.int64) + page_size - 1) // page_size
        table = np.full((S, max(1, int(blocks.max()) if S else 1)), -1, dtype=np.int32)
        k = 0
        for s, nb in enumerate(blocks):
            table[s, :nb] = np.arange(k, k + nb, dtype=np.int32)
            k += nb
    rng_o = _rng(seed, name, "outliers")
    chans = np.stack([rng_o.choice(head_dim, N_OUTLIER_CHANNELS, replace=False)
                      for _ in range(num_kv_heads)]).astype(np.int64)
    if outlier_range is not None:
        lo, hi = outlier_range
        fac = rng_o.uniform(lo, hi, size=(num_kv_heads, N_OUTLIER_CHANNELS)).astype(np.float32)
    elif outlier_scale is None:
        fac = np.ones((num_kv_heads, N_OUTLIER_CHANNELS), dtype=np.float32)
    else:
        fac = np.full((num_kv_heads, N_OUTLIER_CHANNELS), outlier_scale, dtype=np.float32)
    return Workload(name=name, num_seqs=S, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
                    head_dim=head_dim, page_size=page_size, seq_lens=seq_lens,
                    new_tokens=new_tokens, num_pages=int(num_pages), block_table=table,
                    outlier_channels=chans, outlier_scale=fac, seed=seed, decode=decode)


def make_workload(config, seed: int = 0) -> Workload:
    """One of the five named workloads ('tiny', 'prefill', 'decode', 'long', 'serving')."""
    name = {1: "tiny", 2: "prefill", 3: "decode", 4: "long", 5: "serving"}.get(config, config)
    if name == "tiny":
        return custom("tiny", [256], num_q_heads=8, num_kv_heads=2, seed=seed,
                      new_tokens=[256], num_pages=16, outlier_scale=20.0)
    if name == "prefill":
        return custom("prefill", [2048] * 32, num_q_heads=32, num_kv_heads=8, seed=seed,
                      new_tokens=[2048] * 32, num_pages=4096, outlier_range=(10.0, 30.0),
                      decode=False)
    if name == "decode":
        lens = _rng(seed, "decode", "lens").integers(512, 8192, size=64, endpoint=True)
        return custom("decode", lens, num_q_heads=32, num_kv_heads=8, seed=seed,
                      outlier_range=(10.0, 30.0))
    if name == "long":
        return custom("long", [32768] * 8, num_q_heads=64, num_kv_heads=8, seed=seed,
                      new_tokens=[0] * 8, num_pages=16384, outlier_scale=20.0)
    if name == "serving":
        raw = _rng(seed, "serving", "lens").lognormal(np.log(1024.0), 1.0, size=256)
        lens = np.clip(np.rint(raw), 64, 16384).astype(np.int32)
        return custom("serving", lens, num_q_heads=32, num_kv_heads=8, seed=seed,
                      outlier_range=(10.0, 30.0))
    raise ValueError(f"unknown workload {config!r}")


# ---- token bookkeeping ------------------------------------------------------------------

def token_index(wl: Workload, which: str = "all"):
    """(seq, pos) int64 arrays of the tokens selected, in seq-major, position order.

    which: 'all' (every cached token), 'history' (tokens cached before the step) or
    'new' (tokens appended by the step)."""
    seqs, poss = [], []
    for s, L in enumerate(wl.seq_lens.tolist()):
        h = L - int(wl.new_tokens[s])
        lo, hi = {"all": (0, L), "history": (0, h), "new": (h, L)}[which]
        poss.append(np.arange(lo, hi, dtype=np.int64))
        seqs.append(np.full(hi - lo, s, dtype=np.int64))
    if not seqs:
        return np.zeros(0, np.int64), np.zeros(0, np.int64)
    return np.concatenate(seqs), np.concatenate(poss)


def slot_mapping(wl: Workload, seq: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Physical slot (page * page_size + offset) of each (seq, pos)."""
    pages = wl.block_table[seq, pos // wl.page_size].astype(np.int64)
    return pages * wl.page_size + pos % wl.page_size


def _flat_offsets(wl: Workload) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(wl.seq_lens.astype(np.int64))])


def kv_values(wl: Workload, which: str = "K", *, tokens: str = "all",
              device="cpu", chunk: int = 4096) -> torch.Tensor:
    """bf16 [T][Hkv][D] values of the selected tokens (see token_index).

    Each token's values depend only on (seed, workload name, K|V, its flat index among all
    cached tokens), so 'history' + 'new' together give exactly 'all', and a sequence's values
    do not depend on how many sequences follow it.  Values are drawn in whole chunks of `chunk`
    flat tokens from per-chunk generators on `device` (the CPU and CUDA generators differ, so
    parity tests draw on the CPU)."""
    Hkv, D = wl.num_kv_heads, wl.head_dim
    seq, pos = token_index(wl, tokens)
    flat = _flat_offsets(wl)[seq] + pos
    out = torch.empty((len(flat), Hkv, D), dtype=torch.bfloat16, device=device)
    if len(flat) == 0:
        return out
    flat_t = torch.as_tensor(flat)
    chan = torch.as_tensor(wl.outlier_channels)
    fac = torch.as_tensor(wl.outlier_scale)
    dev = torch.device(device)
    for c in np.unique(flat // chunk).tolist():
        sel = torch.nonzero((flat_t // chunk) == c).flatten()
        g = torch.Generator(device=dev)
        g.manual_seed(_seed_for(wl.seed, wl.name, which, c))
        vals = torch.randn((chunk, Hkv, D), generator=g, dtype=torch.float32, device=dev)
        if which == "K":
            for h in range(Hkv):
                vals[:, h, chan[h].to(dev)] *= fac[h].to(dev)
        idx = (flat_t[sel] - c * chunk).to(dev)
        out[sel.to(dev)] = vals.index_select(0, idx).to(torch.bfloat16)
    return out


def q_values(wl: Workload, *, device="cpu") -> torch.Tensor:
    """bf16 [S][Hq][D] decode queries, N(0, 1)."""
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(_seed_for(wl.seed, wl.name, "q"))
    q = torch.randn((wl.num_seqs, wl.num_q_heads, wl.head_dim), generator=g,
                    dtype=torch.float32, device=device)
    return q.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view (numpy, on the CPU) of a bf16 tensor's bits."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)

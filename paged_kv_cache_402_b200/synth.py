"""Seeded synthetic inputs for the paged decode path.

This module only draws inputs: context lengths, block-table placements,
query/key/value tensors and the continuous-batching trace.  It computes no
part of the method (no slots, no attention, no allocation decisions); the
tests hand the same draws to the CUDA path and to the oracle.

Every draw comes from numpy's PCG64 (integers, placements, lengths) or from a
seeded ``torch.Generator`` (normal tensors), so a seed fixes a case exactly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAD = -1  # block-table entries past a sequence's last block


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(shape, dtype: torch.dtype, seed: int, device="cpu", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) values, drawn in float32 and rounded once to `dtype`."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def sentinel_(t: torch.Tensor) -> torch.Tensor:
    """Fills a tensor with a quiet-NaN pattern (marks pool blocks no one owns)."""
    if t.dtype == torch.bfloat16:
        t.view(torch.int16).fill_(0x7FC1)
    elif t.dtype == torch.float32:
        t.view(torch.int32).fill_(0x7FC00001)
    else:
        t.fill_(float("nan"))
    return t


@dataclass
class DecodeCase:
    """One decode batch over a paged pool, before the step's append."""

    name: str
    q: torch.Tensor            # [B, Hq, D]
    k_cache: torch.Tensor      # [num_blocks, Hkv, bs, D]
    v_cache: torch.Tensor      # [num_blocks, Hkv, bs, D]
    block_tables: np.ndarray   # [B, max_blocks] int32, PAD past each sequence's blocks
    context_lens: np.ndarray   # [B] int32
    scale: float
    free_blocks: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int32))  # pool blocks no table uses

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def Hq(self):
        return self.q.shape[1]

    @property
    def D(self):
        return self.q.shape[2]

    @property
    def num_blocks(self):
        return self.k_cache.shape[0]

    @property
    def Hkv(self):
        return self.k_cache.shape[1]

    @property
    def block_size(self):
        return self.k_cache.shape[2]


def _tables_from_pool_order(lens, bs, order, max_blocks=None):
    """Gives sequence b the next ceil(len_b / bs) blocks of `order`."""
    need = [-(-int(L) // bs) for L in lens]
    mb = max(1, max(need) if need else 1) if max_blocks is None else max_blocks
    tables = np.full((len(lens), mb), PAD, dtype=np.int32)
    pos = 0
    for b, n in enumerate(need):
        tables[b, :n] = order[pos:pos + n]
        pos += n
    return tables, pos


def tiny_fp32_case(seed: int = 0) -> DecodeCase:
    """4 sequences of lengths 1, 17, 33, 64; 16-token blocks; 2 heads of 64;
    a 16-block pool whose blocks are dealt from a seeded permutation; float32
    N(0,1) data; scale 1/8.  Unowned blocks hold a NaN sentinel."""
    r = rng(seed)
    lens = np.array([1, 17, 33, 64], dtype=np.int32)
    bs, Hkv, Hq, D, NB = 16, 2, 2, 64, 16
    order = r.permutation(NB).astype(np.int32)
    tables, used = _tables_from_pool_order(lens, bs, order)
    k = normal((NB, Hkv, bs, D), torch.float32, seed * 7 + 1)
    v = normal((NB, Hkv, bs, D), torch.float32, seed * 7 + 2)
    free = order[used:]
    for blk in free.tolist():
        sentinel_(k[blk])
        sentinel_(v[blk])
    q = normal((4, Hq, D), torch.float32, seed * 7 + 3)
    return DecodeCase("tiny-fp32", q, k, v, tables, lens, 1.0 / 8.0, free)


def block_table_example_case(seed: int = 0) -> DecodeCase:
    """One 48-token sequence whose logical blocks 0, 1, 2 sit in physical
    blocks 8, 3, 11 of a 12-block pool (the example of "The Block Table
    Map"); float32, 2 heads of 64, 16-token blocks."""
    bs, Hkv, D, NB = 16, 2, 64, 12
    tables = np.array([[8, 3, 11]], dtype=np.int32)
    k = normal((NB, Hkv, bs, D), torch.float32, seed * 5 + 1)
    v = normal((NB, Hkv, bs, D), torch.float32, seed * 5 + 2)
    q = normal((1, 2, D), torch.float32, seed * 5 + 3)
    free = np.array([b for b in range(NB) if b not in (8, 3, 11)], dtype=np.int32)
    return DecodeCase("table-8-3-11", q, k, v, tables, np.array([48], np.int32), 1.0 / 8.0, free)


def random_case(seed: int, B: int, Hq: int, Hkv: int, D: int, bs: int, lens, dtype=torch.bfloat16,
                pool_factor: float = 2.0, scale: float | None = None, device="cpu",
                sentinel: bool = True, extra_blocks: int = 0) -> DecodeCase:
    """A batch with the given context lengths; the pool holds pool_factor x
    the blocks needed (at least one more), and each sequence's blocks are
    dealt from a seeded shuffle of the whole pool.  Q/K/V ~ N(0,1) and the
    scale is 1/sqrt(D) unless given."""
    r = rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    need = int(sum(-(-int(L) // bs) for L in lens))
    NB = max(need + 1 + extra_blocks, int(math.ceil(need * pool_factor)) + extra_blocks)
    order = r.permutation(NB).astype(np.int32)
    tables, used = _tables_from_pool_order(lens, bs, order)
    k = normal((NB, Hkv, bs, D), dtype, seed * 7 + 1, device=device)
    v = normal((NB, Hkv, bs, D), dtype, seed * 7 + 2, device=device)
    free = order[used:]
    if sentinel and len(free):
        idx = torch.as_tensor(free.astype(np.int64), device=device)
        fill = sentinel_(torch.empty((len(free), Hkv, bs, D), dtype=dtype, device=device))
        k.index_copy_(0, idx, fill)
        v.index_copy_(0, idx, fill)
    q = normal((len(lens), Hq, D), dtype, seed * 7 + 3, device=device)
    return DecodeCase(f"random-B{len(lens)}", q, k, v, tables, lens,
                      (1.0 / math.sqrt(D)) if scale is None else scale, free)


def gqa_lengths(seed: int, B: int = 32, lo: int = 128, hi: int = 4096) -> np.ndarray:
    """Context lengths uniform on the integers [lo, hi]."""
    return rng(seed).integers(lo, hi + 1, size=B).astype(np.int32)


def shared_prefix_layout(seed: int, groups: int = 32, group_size: int = 8, prefix: int = 512,
                         median: float = 800.0, sigma: float = 1.0, clip: int = 8192,
                         bs: int = 16, pool_factor: float = 1.25, prefix_tail: bool = False):
    """Groups of sequences that share their first `prefix` tokens' blocks.

    Each sequence adds a private suffix with lognormal length (given median,
    sigma 1) clipped to [1, clip].  With prefix_tail, each group's prefix is
    prefix + r_g tokens, r_g uniform in [1, bs-1], so the prefix ends inside a
    block that all the group's members share.  Returns (prefix_lens [groups],
    suffix_lens [groups*group_size], block order of the pool, num_blocks).
    """
    r = rng(seed)
    pl = np.full(groups, prefix, dtype=np.int64)
    if prefix_tail:
        pl += r.integers(1, bs, size=groups)
    suffix = np.clip(np.round(r.lognormal(math.log(median), sigma, size=groups * group_size)), 1, clip)
    suffix = suffix.astype(np.int64)
    need = int(sum(-(-int(p) // bs) for p in pl)) + int(
        sum(-(-int(pl[i // group_size] + s) // bs) for i, s in enumerate(suffix)))
    NB = int(math.ceil(need * pool_factor)) + groups * group_size + 1
    order = r.permutation(NB).astype(np.int32)
    return pl, suffix, order, NB


def long_context_lengths(seed: int, B: int = 8, lo: int = 32768, hi: int = 131072) -> np.ndarray:
    return rng(seed).integers(lo, hi + 1, size=B).astype(np.int32)


def long_context_lengths_small(seed: int) -> np.ndarray:
    """The first two lengths of long_context_lengths(seed): a batch small
    enough for a profiler capture, drawn from the same distribution."""
    return long_context_lengths(seed)[:2]


def scattered_blocks(seed: int, lens, bs: int, num_blocks: int) -> np.ndarray:
    """Block tables whose entries are drawn without replacement, uniformly
    from a pool of num_blocks."""
    r = rng(seed)
    need = [-(-int(L) // bs) for L in lens]
    total = int(sum(need))
    if total > num_blocks:
        raise ValueError("pool too small")
    picks = r.choice(num_blocks, size=total, replace=False).astype(np.int32)
    tables, _ = _tables_from_pool_order(lens, bs, picks)
    return tables


# ---------------------------------------------------------------------------
# continuous-batching trace


@dataclass
class TraceEvent:
    step: int
    arrivals: list      # [(prompt_len, output_len)] new beam groups this step
    reselect: list      # per running group index i (position in the running list), True if a beam is re-forked


def trace(seed: int, steps: int = 1000, mean_arrivals: float = 4.0, prompt_median: float = 512.0,
          prompt_sigma: float = 1.0, prompt_max: int = 4096, output_mean: float = 256.0,
          reselect_p: float = 0.25, max_groups: int = 4096):
    """Draws a continuous-batching trace: Poisson arrivals per step, lognormal
    prompt lengths clipped to [1, prompt_max], geometric output lengths with
    the given mean (support >= 1), and for each running group a Bernoulli
    draw per step saying whether one beam is replaced by a fork of another.
    The re-selection draws are made for max_groups slots per step; a consumer
    uses the first len(running) of them."""
    r = rng(seed)
    out = []
    p = 1.0 / output_mean
    for s in range(steps):
        n = int(r.poisson(mean_arrivals))
        pls = np.clip(np.round(r.lognormal(math.log(prompt_median), prompt_sigma, size=n)), 1, prompt_max)
        ols = r.geometric(p, size=n)
        res = r.random(max_groups) < reselect_p
        victims = r.integers(0, 4, size=max_groups)
        donors = r.integers(0, 3, size=max_groups)
        out.append(dict(step=s, arrivals=[(int(a), int(b)) for a, b in zip(pls, ols)],
                        reselect=res, victim=victims, donor=donors))
    return out

"""The seeded input generators draw the workloads' stated shapes (no GPU).

Each workload is synthetic: lengths, placements and the trace's arrivals come
from seeded numpy draws.  These tests hold the generators to their recipe:
ranges, medians and means over enough draws that a wrong parameter (a mean
of 2 arrivals instead of 4, a median of 256 instead of 512, an unclipped
tail) shows, and pool layouts that every sequence fits in.
"""
import math

import numpy as np

from paged_kv_cache_402_b200 import synth


def test_gqa_and_long_context_lengths_cover_their_ranges():
    g = np.concatenate([synth.gqa_lengths(s) for s in range(200)])
    assert g.min() >= 128 and g.max() <= 4096
    assert abs(g.mean() - (128 + 4096) / 2) < 0.02 * 4096
    lc = np.concatenate([synth.long_context_lengths(s) for s in range(500)])
    assert lc.min() >= 32768 and lc.max() <= 131072
    assert abs(lc.mean() - (32768 + 131072) / 2) < 0.02 * 131072
    assert (synth.long_context_lengths_small(4) == synth.long_context_lengths(4)[:2]).all()


def test_shared_prefix_layout_fits_and_ends_inside_a_block():
    bs, groups, gsz = 16, 32, 8
    pl, suffix, order, NB = synth.shared_prefix_layout(11, groups=groups, group_size=gsz, prefix=512,
                                                       median=800, clip=8192, bs=bs, prefix_tail=True)
    assert len(pl) == groups and len(suffix) == groups * gsz
    assert ((pl - 512 >= 1) & (pl - 512 <= bs - 1)).all()  # the prefix ends inside a shared block
    assert suffix.min() >= 1 and suffix.max() <= 8192
    assert sorted(order.tolist()) == list(range(NB))
    need = sum(-(-int(p) // bs) for p in pl) + sum(-(-int(pl[i // gsz] + s) // bs) for i, s in enumerate(suffix))
    assert NB >= need + groups * gsz  # room for every sequence and a copy per member
    # suffix median over many draws
    many = np.concatenate([synth.shared_prefix_layout(s, median=800)[1] for s in range(40)])
    assert abs(np.median(many) / 800 - 1) < 0.1


def test_scattered_blocks_are_distinct_pool_blocks():
    lens = synth.gqa_lengths(3)
    NB = 2 * sum(-(-int(L) // 16) for L in lens)
    t = synth.scattered_blocks(5, lens, 16, NB)
    used = np.concatenate([t[b, :-(-int(L) // 16)] for b, L in enumerate(lens)])
    assert len(np.unique(used)) == len(used) and used.min() >= 0 and used.max() < NB
    assert all((t[b, -(-int(L) // 16):] == -1).all() for b, L in enumerate(lens))


def test_trace_draws_follow_the_recipe():
    steps = 4000
    d = synth.trace(7, steps=steps)
    n = np.array([len(e["arrivals"]) for e in d])
    prompts = np.array([a for e in d for a, _ in e["arrivals"]])
    outs = np.array([b for e in d for _, b in e["arrivals"]])
    # Poisson(4) arrivals a step: mean and variance both 4
    assert abs(n.mean() - 4) < 0.15 and abs(n.var() - 4) < 0.4
    # lognormal prompts, median 512, clipped to [1, 4096]
    assert prompts.min() >= 1 and prompts.max() <= 4096
    assert abs(np.median(prompts) / 512 - 1) < 0.06
    assert abs(np.std(np.log(prompts[prompts < 4096])) - 1) < 0.1
    # geometric outputs, mean 256, support from 1
    assert outs.min() >= 1 and abs(outs.mean() / 256 - 1) < 0.05
    # re-selection with probability 0.25 per running group
    res = np.concatenate([e["reselect"][:64] for e in d])
    assert abs(res.mean() - 0.25) < 0.01
    # same seed, same trace
    again = synth.trace(7, steps=20)
    assert [e["arrivals"] for e in again] == [e["arrivals"] for e in d[:20]]


def test_normal_draws_are_seeded_standard_normals():
    import torch
    a = synth.normal((4096, 64), torch.float32, 3)
    assert torch.equal(a, synth.normal((4096, 64), torch.float32, 3))
    assert not torch.equal(a, synth.normal((4096, 64), torch.float32, 4))
    assert abs(float(a.mean())) < 0.01 and abs(float(a.std()) - 1) < 0.01
    b = synth.normal((4096, 64), torch.bfloat16, 3)
    assert torch.equal(b, a.to(torch.bfloat16))  # drawn in fp32, rounded once
    assert math.isclose(float(synth.normal((1 << 16,), torch.float32, 9, std=0.5).std()), 0.5, rel_tol=0.02)

"""The step the benchmark times, at the workloads' full sizes, against the
oracle on every output row.

Each test builds its workload the way the benchmark does (the C++ allocator
deals the blocks, the pool holds seeded N(0,1) values drawn by torch), then
runs the benchmark's step: one token per sequence through the allocator, the
sharing plan (pa_share_plan), the copy-on-write sources (pa_cow_sources), and
one pa_decode_shared call that copies, appends and decodes.  The oracle's
allocator model makes the same decisions, the oracle copies and appends on a
host pool, and decodes every (sequence, query head) row in float64.  The
appended rows and copies must match bit for bit; every output row must be
within the bf16 bound |gpu - ref| <= 2e-2 + 1e-2 |ref|.

Workloads ("The Block Table Map": attention reads each sequence through its
table; "pagedattention" glossary entry, paragraph 5: sharers point at the
same blocks and are copied when they write):
  * long context: 8 sequences of 32768..131072 tokens scattered over an
    80 GiB K+V pool, 32 query / 8 kv heads;
  * shared prefix: 256 sequences in groups of 8 sharing a 512 + r token
    prefix, lognormal private suffixes (median 800, up to 8192), 64 query /
    8 kv heads;
  * copy-on-write step: the same groups before their suffixes, so the step's
    append copies each group's shared partial block for 7 of 8 members.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

from .test_gpu_parity import assert_attn_close, host_pool, same_bits

pytestmark = pytest.mark.gpu


def _host_step(A, seqs, dev, bs):
    """The benchmark's host work for a step: one token per sequence, the
    tables and lengths, the copy-on-write sources and the sharing plan."""
    slots, pairs = A.batch_append(seqs, np.ones(len(seqs), np.int32))
    mb = max(A.seq_len(s)[1] for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    cow = pa.cow_sources(pairs, tables, lens, bs)
    plan = pa.share_plan(tables, lens, bs).to(dev)
    return slots, pairs, tables, lens, cow, plan


def _device_step(dev, cache, Hq, seed, pairs, tables, lens, cow, plan):
    """The benchmark's device call for a step (one pa_decode_shared with the
    plan, the copy sources and the new rows); returns (out, k, v, q), the
    new rows and queries on the host."""
    Hkv, D, dt = cache.num_kv_heads, cache.head_dim, cache.dtype
    n = len(lens)
    kn = synth.normal((n, Hkv, D), dt, seed)
    vn = synth.normal((n, Hkv, D), dt, seed + 1)
    q = synth.normal((n, Hq, D), dt, seed + 2)
    out = pa.pa_decode_shared(q.to(dev), cache, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                              int(lens.max()), 1 / math.sqrt(D), plan=plan, k_new=kn.to(dev), v_new=vn.to(dev),
                              cow_src=torch.from_numpy(cow).to(dev) if len(pairs) else None)
    assert pa.pa_read_device_error() == 0
    return out, kn, vn, q


def _grouped_pool(seed, groups, gsz, suffix_median, dev, NB_extra=0, with_suffix=True):
    """Groups of gsz sequences that share a 512 + r token prefix (r in
    [1, 15]); with_suffix, each member then grows a lognormal suffix, which
    copies the shared partial block for all members but the last.  Returns
    (library allocator, model, sequences, device pool, host pool k, v)."""
    Hkv, D, bs = 8, 128, 16
    pl, suffix, order, NB = synth.shared_prefix_layout(seed, groups=groups, group_size=gsz, prefix=512,
                                                       median=suffix_median, clip=8192, bs=bs, pool_factor=1.25,
                                                       prefix_tail=True)
    NB += NB_extra
    order = np.concatenate([order, np.arange(len(order), NB)]).astype(np.int32)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    k = synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 2, device=dev)
    v = synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 3, device=dev)
    hk, hv = host_pool(k), host_pool(v)
    roots = [A.new_seq() for _ in range(groups)]
    assert [M.new_seq() for _ in range(groups)] == roots
    A.batch_append(roots, pl)
    M.batch_append(roots, pl)
    seqs = []
    for r in roots:
        seqs.append(r)
        for _ in range(gsz - 1):
            c = A.fork(r)
            assert M.fork(r) == c
            seqs.append(c)
    if with_suffix:
        _, pairs = A.batch_append(seqs, suffix)
        _, mpairs = M.batch_append(seqs, suffix)
        assert pairs.tolist() == [list(p) for p in mpairs] and len(pairs) == groups * (gsz - 1)
        # the suffix copies, made by torch on the device (an independent
        # route) and by the oracle on the host
        src = torch.as_tensor(pairs[:, 0].astype(np.int64), device=dev)
        dst = torch.as_tensor(pairs[:, 1].astype(np.int64), device=dev)
        k.index_copy_(0, dst, k.index_select(0, src))
        v.index_copy_(0, dst, v.index_select(0, src))
        oracle.copy_blocks(hk, hv, mpairs)
    return A, M, seqs, pa.KVCache(k, v), hk, hv


def _check_grouped_step(A, M, seqs, cache, hk, hv, dev, Hq, seed, expect_copies):
    slots, pairs, tables, lens, cow, plan = _host_step(A, seqs, dev, cache.block_size)
    out, kn, vn, q = _device_step(dev, cache, Hq, seed, pairs, tables, lens, cow, plan)
    mslots, mpairs = M.batch_append(seqs, [1] * len(seqs))
    assert slots.tolist() == mslots and pairs.tolist() == [list(p) for p in mpairs]
    assert len(pairs) == expect_copies
    assert plan.n_groups == 2 * (len(seqs) // 8), "each group of 8 forms two plan groups of 4"
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    ref = oracle.decode(q, hk, hv, tables, lens, 1 / math.sqrt(cache.head_dim))
    assert_attn_close(out, ref, torch.bfloat16)


def test_shared_prefix_full_size_every_row(cuda_device):
    """256 sequences, 16 384 rows, the cascade plan over each group's shared
    partition, every row against the oracle, the pool bit for bit."""
    A, M, seqs, cache, hk, hv = _grouped_pool(11, 32, 8, 800, cuda_device, NB_extra=256 * 2)
    _check_grouped_step(A, M, seqs, cache, hk, hv, cuda_device, 64, 14, expect_copies=0)
    del cache
    torch.cuda.empty_cache()


def test_cow_step_full_size_every_row(cuda_device):
    """The copy-on-write step: 32 groups of 8 whose 512 + r token prefix ends
    in a shared block; the step copies it for 7 members of each group (224
    copies inside the decode call), every row against the oracle, the pool
    bit for bit."""
    A, M, seqs, cache, hk, hv = _grouped_pool(21, 32, 8, 800, cuda_device, NB_extra=256 * 2, with_suffix=False)
    _check_grouped_step(A, M, seqs, cache, hk, hv, cuda_device, 64, 24, expect_copies=32 * 7)
    del cache
    torch.cuda.empty_cache()


def test_long_context_full_size_every_row(cuda_device):
    """8 sequences of 32768..131072 tokens whose blocks are dealt from a
    seeded shuffle of an 80 GiB K+V pool, the fused append + decode step,
    every one of the 256 rows against the oracle.  The oracle sees each
    sequence's blocks gathered into a compact host pool (read before the
    step: values drawn by torch), appends the new row there itself, and the
    gathered blocks after the step must equal its pool bit for bit."""
    dev = cuda_device
    B, Hq, Hkv, D, bs = 8, 32, 8, 128, 16
    NB = 80 * 2**30 // (2 * Hkv * bs * D * 2)
    lens0 = synth.long_context_lengths(4)
    order = synth.rng(5).permutation(NB).astype(np.int32)
    A = pa.Allocator(NB, bs, order)
    seqs = [A.new_seq() for _ in range(B)]
    A.batch_append(seqs, lens0)
    k = torch.empty(NB, Hkv, bs, D, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    # the step's new block, if a sequence starts one, comes from the free
    # list's next entries: fill those too, so every gathered block is defined
    need = int(sum(-(-(int(L) + 1) // bs) for L in lens0)) + B
    idx = torch.as_tensor(order[:need].astype(np.int64), device=dev)
    for i in range(0, len(idx), 65536):
        part = idx[i:i + 65536]
        k.index_copy_(0, part, synth.normal((len(part), Hkv, bs, D), torch.bfloat16, 100 + i, device=dev))
        v.index_copy_(0, part, synth.normal((len(part), Hkv, bs, D), torch.bfloat16, 200 + i, device=dev))
    cache = pa.KVCache(k, v)
    slots, pairs, tables, lens, cow, plan = _host_step(A, seqs, dev, bs)
    assert len(pairs) == 0 and plan.n_groups == 0 and (lens == lens0 + 1).all()
    # each sequence's blocks as torch drew them, gathered before the step
    nbs = [-(-int(L) // bs) for L in lens]
    before = []
    for b in range(B):
        blocks = torch.as_tensor(tables[b, :nbs[b]].astype(np.int64), device=dev)
        before.append((host_pool(k.index_select(0, blocks)), host_pool(v.index_select(0, blocks))))
    out, kn, vn, q = _device_step(dev, cache, Hq, 41, pairs, tables, lens, cow, plan)
    got = out.float().cpu().double().numpy()
    scale = 1 / math.sqrt(D)
    for b in range(B):
        hk, hv = before[b]
        # the oracle's append of the new row into its compact pool (block j
        # of the sequence is block j of the compact pool)
        oracle.append_kv(hk, hv, kn[b:b + 1], vn[b:b + 1], [int(lens[b]) - 1])
        blocks = torch.as_tensor(tables[b, :nbs[b]].astype(np.int64), device=dev)
        assert same_bits(host_pool(k.index_select(0, blocks)), hk), f"sequence {b}: k pool differs"
        assert same_bits(host_pool(v.index_select(0, blocks)), hv), f"sequence {b}: v pool differs"
        ref = oracle.decode(q[b:b + 1], hk, hv, np.arange(nbs[b], dtype=np.int32)[None, :],
                            np.array([lens[b]], np.int32), scale)
        g = got[b:b + 1]
        assert (np.abs(g - ref) <= 2e-2 + 1e-2 * np.abs(ref)).all(), f"sequence {b}: rows out of tolerance"
    del k, v, cache
    torch.cuda.empty_cache()

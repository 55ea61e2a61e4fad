"""pa_decode_shared (cascade over the blocks a sharing plan's groups hold in
common) against the oracle's decode of the same pool, and against the
library's own pa_decode / pa_append_decode without a plan.

Attention within the bf16 bound |gpu - ref| <= 2e-2 + 1e-2 |ref| of the
float64 oracle; with a fused append the pool bit for bit.  A member whose
shared blocks end on a partition boundary gets its statistics over each
partition from the same tiles and the same per-column arithmetic as without
the plan, so its outputs must also be bit-identical to the plan-free call;
where the shared blocks end inside a partition, that partition's statistics
come in two pieces, and the output is held to the oracle's bound.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

from .test_gpu_fused import _fork_groups, _pool, _prefill
from .test_gpu_parity import assert_attn_close, host_pool, same_bits

pytestmark = pytest.mark.gpu


def _groups_layout(A, M, dev, cache, hk, hv, dt, prompt_lens, fanout, seed):
    roots = _prefill(A, M, list(prompt_lens), dev, cache, hk, hv, dt, seed)
    return _fork_groups(A, M, roots, fanout)


@pytest.mark.parametrize("G,bs,prompt", [
    (8, 16, 1300),   # 81 shared blocks, groups of 8 forks -> plan groups of 4
    (8, 16, 1024),   # the first prompt's blocks end on a partition boundary
    (4, 16, 700),    # one shared partition and a piece of the next
    (2, 8, 1600),    # three shared partitions and a piece, small blocks
    (1, 32, 2100),   # four shared partitions and a piece, large blocks
    (4, 16, 200),    # shared blocks inside the first partition, some members of one partition
])
def test_shared_decode_matches_oracle_and_plain(cuda_device, G, bs, prompt):
    dt, Hkv, D = torch.bfloat16, 4, 128
    Hq = G * Hkv
    prompts = [prompt, prompt + 37, prompt // 2 + 600]
    NB = 3 * 8 * (-(-(prompt + 700) // bs)) + 64
    order = synth.rng(61).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
    seqs = _groups_layout(A, M, cuda_device, cache, hk, hv, dt, prompts, 8, 62)
    # every member grows a private suffix of its own length
    extra = synth.rng(63).integers(1, 300, size=len(seqs))
    slots, pairs = A.batch_append(seqs, extra.tolist())
    mslots, mpairs = M.batch_append(seqs, extra.tolist())
    assert slots.tolist() == mslots
    kn = synth.normal((int(extra.sum()), Hkv, D), dt, 64)
    vn = synth.normal((int(extra.sum()), Hkv, D), dt, 65)
    if len(pairs):
        pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(pairs)).to(cuda_device), cache)
    pa.pa_append_kv(kn.to(cuda_device), vn.to(cuda_device), torch.from_numpy(slots).to(cuda_device), cache)
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    plan = pa.share_plan(tables, lens, bs)
    assert plan.n_groups == 3 * 2 and (plan.first_token >= pa.PA_SHARE_MIN_TOKENS).all()
    plan.to(cuda_device)
    q = synth.normal((len(seqs), Hq, D), dt, 66)
    td, ld, qd = (torch.from_numpy(tables).to(cuda_device), torch.from_numpy(lens).to(cuda_device),
                  q.to(cuda_device))
    scale = 1 / math.sqrt(D)
    out = pa.pa_decode_shared(qd, cache, td, ld, int(lens.max()), scale, plan=plan)
    assert pa.pa_read_device_error() == 0
    ref = oracle.decode(q, hk, hv, tables, lens, scale)
    assert_attn_close(out, ref, dt)
    plain = pa.pa_decode(qd, cache, td, ld, int(lens.max()), scale)
    aligned = torch.from_numpy(plan.first_token % cache.partition_tokens == 0).to(cuda_device)
    assert torch.equal(out[aligned].view(torch.int16), plain[aligned].view(torch.int16))
    if prompt == 1024:
        assert bool(aligned.any())


def test_shared_fused_step_copy_on_write(cuda_device):
    """The shared-prefix step with its copies, appends and plan in one call:
    groups of 8 share a 512 + r prefix (its last block partly filled and
    shared), so every member but the last copies that block; the first
    blocks are read once per plan group."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 8, 128, 16, 64
    groups, gsz = 4, 8
    pl, _, order, NB = synth.shared_prefix_layout(9, groups=groups, group_size=gsz, prefix=512,
                                                  median=60, clip=300, prefix_tail=True)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
    roots = _prefill(A, M, pl.tolist(), cuda_device, cache, hk, hv, dt, 10)
    seqs = _fork_groups(A, M, roots, gsz)
    n = len(seqs)
    slots, pairs = A.batch_append(seqs, [1] * n)
    mslots, mpairs = M.batch_append(seqs, [1] * n)
    assert slots.tolist() == mslots and len(pairs) == groups * (gsz - 1)
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    cow = pa.cow_sources(pairs, tables, lens, bs)
    plan = pa.share_plan(tables, lens, bs).to(cuda_device)
    assert plan.n_groups == groups * 2
    kn = synth.normal((n, Hkv, D), dt, 13)
    vn = synth.normal((n, Hkv, D), dt, 14)
    q = synth.normal((n, Hq, D), dt, 12)
    scale = 1 / math.sqrt(D)
    out = pa.pa_decode_shared(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                              torch.from_numpy(lens).to(cuda_device), int(lens.max()), scale, plan=plan,
                              k_new=kn.to(cuda_device), v_new=vn.to(cuda_device),
                              cow_src=torch.from_numpy(cow).to(cuda_device))
    assert pa.pa_read_device_error() == 0
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    ref = oracle.decode(q, hk, hv, tables, lens, scale)
    assert_attn_close(out, ref, dt)


@pytest.mark.parametrize("bad", [1090, 7 * 512])
def test_shared_plan_that_does_not_fit(cuda_device, bad):
    """A first_token that is not a whole number of blocks, or lies past a
    sequence's end, sets PA_DEVERR_PLAN and that sequence is computed whole:
    the output stays right."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 2, 128, 16, 8
    A = pa.Allocator(400, bs, list(range(400)))
    r = A.new_seq()
    A.batch_append([r], [1100])
    seqs = [r] + [A.fork(r) for _ in range(3)]
    A.batch_append(seqs, [5, 9, 1, 30])
    tables, lens = A.build_block_tables(seqs, 80)
    plan = pa.share_plan(tables, lens, bs)
    assert plan.shared_tokens.tolist() == [1088]
    plan.first_token[1] = bad
    plan.to(cuda_device)
    case_k = synth.normal((400, Hkv, bs, D), dt, 70)
    case_v = synth.normal((400, Hkv, bs, D), dt, 71)
    cache = pa.KVCache(case_k.to(cuda_device), case_v.to(cuda_device))
    q = synth.normal((4, Hq, D), dt, 72)
    scale = 1 / math.sqrt(D)
    out = pa.pa_decode_shared(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                              torch.from_numpy(lens).to(cuda_device), int(lens.max()), scale, plan=plan)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_PLAN
    ref = oracle.decode(q, host_pool(case_k), host_pool(case_v), tables, lens, scale)
    assert_attn_close(out, ref, dt)


def test_shared_plan_across_batch_slices(cuda_device):
    """1101 sequences (more than the partition kernel's per-sequence tables:
    its coarse form, entries of 8 sequences) in groups of 3 forks, one group
    straddling sequence 1024; with the fused append."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 2, 128, 16, 8
    roots_n, fan = 367, 3
    prompts = (600 + synth.rng(101).integers(0, 400, size=roots_n)).tolist()
    NB = sum(-(-p // bs) for p in prompts) + roots_n * fan * 3 + 16
    order = synth.rng(102).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
    roots = _prefill(A, M, prompts, cuda_device, cache, hk, hv, dt, 103)
    seqs = _fork_groups(A, M, roots, fan)
    n = len(seqs)
    assert n == 1101
    slots, pairs = A.batch_append(seqs, [1] * n)
    mslots, mpairs = M.batch_append(seqs, [1] * n)
    assert slots.tolist() == mslots
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    cow = pa.cow_sources(pairs, tables, lens, bs)
    plan = pa.share_plan(tables, lens, bs)
    assert plan.n_groups == roots_n
    assert any(min(g) < 1024 <= max(g) for g in plan.members.tolist())
    plan.to(cuda_device)
    kn = synth.normal((n, Hkv, D), dt, 104)
    vn = synth.normal((n, Hkv, D), dt, 105)
    q = synth.normal((n, Hq, D), dt, 106)
    scale = 1 / math.sqrt(D)
    out = pa.pa_decode_shared(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                              torch.from_numpy(lens).to(cuda_device), int(lens.max()), scale, plan=plan,
                              k_new=kn.to(cuda_device), v_new=vn.to(cuda_device),
                              cow_src=torch.from_numpy(cow).to(cuda_device) if len(pairs) else None)
    assert pa.pa_read_device_error() == 0
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    rows = [(b, h) for b in list(range(1016, 1032)) + list(range(0, 1101, 37)) for h in (0, 7)]
    ref = oracle.decode(q, hk, hv, tables, lens, scale, rows=rows)
    assert_attn_close(torch.stack([out[b, h] for b, h in rows]), ref, dt)

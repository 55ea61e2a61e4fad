"""Head-packed passes of the tensor-core partition kernel against the oracle.

With a group size of at most 4 and a multiple of 4 kv heads, a sequence's
short partial last partition goes through the kernel as passes of 4 kv
heads, 32 rows of each 128-row K and V tile per head; the query tile holds
the 4 heads' query rows and a score counts only where the row's head is the
column's.  The kernel packs a partition of len tokens when that takes fewer
chunks, ceil(len / 32) < 4 ceil(len / 128): up to 96 tokens, 129 to 224, and
so on.  These tests put tails on both sides of those bounds, on sequences of
one partition (output written by the pass itself) and of several (partial
statistics through the reduce), for every block size, and through the fused
copy-on-write step.  Attention within the bf16 bound |gpu - ref| <= 2e-2 +
1e-2 |ref| of the float64 oracle; the pool bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

from .test_gpu_fused import _fork_groups, _fused_step, _pool, _prefill
from .test_gpu_parity import assert_attn_close, decode_case, host_pool, same_bits

pytestmark = pytest.mark.gpu

TAILS = [1, 17, 31, 32, 33, 64, 65, 95, 96, 97, 127, 128, 129, 200, 224, 225, 300, 511]


@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_packed_tails_decode(cuda_device, G, bs):
    """Tails of every length class, alone (one partition) and after one or
    two whole partitions."""
    Hkv = 8
    lens = np.array(TAILS + [512 + t for t in TAILS[::2]] + [1024 + t for t in TAILS[1::3]], np.int32)
    case = synth.random_case(700 + 10 * G + bs, B=len(lens), Hq=G * Hkv, Hkv=Hkv, D=128, bs=bs, lens=lens,
                             dtype=torch.bfloat16)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.bfloat16)


@pytest.mark.parametrize("G", [2, 4])
def test_packed_heads_of_four(cuda_device, G):
    """Four kv heads: one packed pass covers all of them."""
    Hkv = 4
    lens = np.array([3, 40, 90, 150, 600, 700, 1100, 1600], np.int32)
    case = synth.random_case(760 + G, B=len(lens), Hq=G * Hkv, Hkv=Hkv, D=128, bs=16, lens=lens,
                             dtype=torch.bfloat16)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.bfloat16)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_packed_fused_copy_on_write(cuda_device, bs):
    """Groups of 4 forks of prompts that end inside a block: each step copies
    the shared partial block for 3 of 4 members inside the packed passes
    (every head's copy and newest row), three steps in a row."""
    dt, Hkv, D, G = torch.bfloat16, 8, 128, 4
    Hq = G * Hkv
    prompts = [bs * 3 + 5, 91, 201, 533, 1000 + bs // 2 + 1]
    NB = 4 * sum(-(-(p + 8) // bs) for p in prompts) + 64
    order = synth.rng(771 + bs).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
    roots = _prefill(A, M, prompts, cuda_device, cache, hk, hv, dt, 772)
    seqs = _fork_groups(A, M, roots, 4)
    copies = 0
    for step in range(3):
        q = synth.normal((len(seqs), Hq, D), dt, 780 + step)
        out, ref, n = _fused_step(A, M, seqs, cuda_device, cache, hk, hv, q, dt, 790 + 2 * step, 1 / math.sqrt(D))
        copies += n
        assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
        assert_attn_close(out, ref, dt)
    assert copies == 3 * len(prompts)


def test_packed_shared_step(cuda_device):
    """The sharing plan's cascade over each group's full blocks, then the
    partition kernel's packed passes over the members' private tokens, in
    one fused call: against the oracle and the pool bit for bit."""
    dt, Hkv, D, G, bs = torch.bfloat16, 8, 128, 4, 16
    Hq = G * Hkv
    prompts = [300, 700, 1333]
    NB = 4 * sum(-(-(p + 64) // bs) for p in prompts) + 64
    order = synth.rng(801).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
    roots = _prefill(A, M, prompts, cuda_device, cache, hk, hv, dt, 802)
    seqs = _fork_groups(A, M, roots, 4)
    extra = synth.rng(803).integers(1, 120, size=len(seqs))
    slots, pairs = A.batch_append(seqs, extra.tolist())
    mslots, mpairs = M.batch_append(seqs, extra.tolist())
    kn = synth.normal((int(extra.sum()), Hkv, D), dt, 804)
    vn = synth.normal((int(extra.sum()), Hkv, D), dt, 805)
    if len(pairs):
        pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(pairs)).to(cuda_device), cache)
    pa.pa_append_kv(kn.to(cuda_device), vn.to(cuda_device), torch.from_numpy(slots).to(cuda_device), cache)
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    n = len(seqs)
    slots, pairs = A.batch_append(seqs, [1] * n)
    mslots, mpairs = M.batch_append(seqs, [1] * n)
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    cow = pa.cow_sources(pairs, tables, lens, bs)
    plan = pa.share_plan(tables, lens, bs).to(cuda_device)
    assert plan.n_groups == len(prompts)
    k1 = synth.normal((n, Hkv, D), dt, 806)
    v1 = synth.normal((n, Hkv, D), dt, 807)
    q = synth.normal((n, Hq, D), dt, 808)
    out = pa.pa_decode_shared(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                              torch.from_numpy(lens).to(cuda_device), int(lens.max()), 1 / math.sqrt(D), plan=plan,
                              k_new=k1.to(cuda_device), v_new=v1.to(cuda_device),
                              cow_src=torch.from_numpy(cow).to(cuda_device) if len(pairs) else None)
    assert pa.pa_read_device_error() == 0
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, k1, v1, mslots)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    ref = oracle.decode(q, hk, hv, tables, lens, 1 / math.sqrt(D))
    assert_attn_close(out, ref, dt)

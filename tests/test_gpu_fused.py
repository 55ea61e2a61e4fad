"""pa_append_decode (copy on write + append of each sequence's newest token +
decode, one call) against the oracle's copy, append and decode, and against
the library's three separate calls on the same state.

The pool must match bit for bit (unowned blocks hold a NaN sentinel); the
output within the decode tolerances (fp32 max-abs 1e-5; bf16
|gpu - ref| <= 2e-2 + 1e-2 |ref|); and the fused output must equal the
separate calls' output bit for bit, since both run the same decode over the
same pool.
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


def _prefill(A, M, lens, dev, cache, hk, hv, dtype, seed):
    seqs = []
    Hkv, D = cache.num_kv_heads, cache.head_dim
    for _ in lens:
        s = A.new_seq()
        assert M.new_seq() == s
        seqs.append(s)
    slots, pairs = A.batch_append(seqs, lens)
    mslots, _ = M.batch_append(seqs, lens)
    assert slots.tolist() == mslots and len(pairs) == 0
    total = int(np.sum(lens))
    kn = synth.normal((total, Hkv, D), dtype, seed)
    vn = synth.normal((total, Hkv, D), dtype, seed + 1)
    pa.pa_append_kv(kn.to(dev), vn.to(dev), torch.from_numpy(slots).to(dev), cache)
    oracle.append_kv(hk, hv, kn, vn, slots)
    return seqs


def _fork_groups(A, M, roots, gsz):
    seqs = []
    for r in roots:
        seqs.append(r)
        for _ in range(gsz - 1):
            c = A.fork(r)
            assert M.fork(r) == c
            seqs.append(c)
    return seqs


def _fused_step(A, M, seqs, dev, cache, hk, hv, q, dtype, seed, scale):
    """One step on both sides: one token per sequence through both
    allocators; the GPU runs pa_append_decode, the oracle copy + append +
    decode.  Returns (gpu out, oracle out, number of copies)."""
    Hkv, D, bs = cache.num_kv_heads, cache.head_dim, cache.block_size
    n = len(seqs)
    slots, pairs = A.batch_append(seqs, [1] * n)
    mslots, mpairs = M.batch_append(seqs, [1] * n)
    assert slots.tolist() == mslots
    assert [tuple(p) for p in pairs.tolist()] == mpairs
    kn = synth.normal((n, Hkv, D), dtype, seed)
    vn = synth.normal((n, Hkv, D), dtype, seed + 1)
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    cow = pa.cow_sources(pairs, tables, lens, bs)
    assert int((cow >= 0).sum()) == len(pairs)
    out = pa.pa_append_decode(kn.to(dev), vn.to(dev), q.to(dev), cache, torch.from_numpy(tables).to(dev),
                              torch.from_numpy(lens).to(dev), int(lens.max()), scale,
                              cow_src=torch.from_numpy(cow).to(dev) if len(pairs) else None)
    assert pa.pa_read_device_error() == 0
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    ref = oracle.decode(q, hk, hv, tables, lens, scale)
    return out, ref, len(pairs)


def _pool(NB, Hkv, bs, D, dt, dev):
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    return pa.KVCache(k0.to(dev), v0.to(dev)), host_pool(k0), host_pool(v0)


@pytest.mark.parametrize("dtype,D,G,bs", [
    (torch.bfloat16, 128, 4, 16),   # tensor-core path
    (torch.bfloat16, 128, 1, 8),
    (torch.bfloat16, 128, 2, 32),
    (torch.bfloat16, 128, 8, 16),
    (torch.bfloat16, 64, 4, 16),    # CUDA-core path (append kernel + decode)
    (torch.float32, 128, 4, 16),
    (torch.float32, 64, 2, 8),
])
def test_fused_step_matches_oracle(cuda_device, dtype, D, G, bs):
    """Ragged lengths (one of them on a block boundary, so the step opens a
    new block) through a seeded shuffled pool: three fused steps in a row."""
    Hkv = 4
    Hq = G * Hkv
    lens = synth.rng(21).integers(1, 1400, size=12).astype(int)
    lens[0] = 2 * bs  # the next token starts a new block
    lens[1] = 511      # the next token completes a 512-token partition
    lens[2] = 512      # the next token opens a second partition
    NB = 2 * int(sum(-(-(int(L) + 4) // bs) for L in lens))
    order = synth.rng(22).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dtype, cuda_device)
    seqs = _prefill(A, M, lens.tolist(), cuda_device, cache, hk, hv, dtype, 23)
    for step in range(3):
        q = synth.normal((len(seqs), Hq, D), dtype, 30 + step)
        out, ref, _ = _fused_step(A, M, seqs, cuda_device, cache, hk, hv, q, dtype, 40 + 2 * step,
                                  1 / math.sqrt(D))
        assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
        assert_attn_close(out, ref, dtype)


@pytest.mark.parametrize("dtype,G", [(torch.bfloat16, 8), (torch.float32, 4)])
def test_fused_step_copy_on_write(cuda_device, dtype, G):
    """Groups share a prefix ending inside a block: the step copies that block
    for every member but the last (in the same launch as the appends and the
    decode on the tensor-core path).  Shared full blocks stay bit-identical."""
    Hkv, D, bs = 8, 128, 16
    Hq = G * Hkv
    groups, gsz = 4, 8
    pl, _, order, NB = synth.shared_prefix_layout(9, groups=groups, group_size=gsz, prefix=512,
                                                  median=60, clip=300, prefix_tail=True)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dtype, cuda_device)
    roots = _prefill(A, M, pl.tolist(), cuda_device, cache, hk, hv, dtype, 10)
    seqs = _fork_groups(A, M, roots, gsz)
    shared_full = {b for r in roots for b in M.block_table(r)[:-1]}
    snap = {b: (hk[b].copy(), hv[b].copy()) for b in shared_full}
    q = synth.normal((len(seqs), Hq, D), dtype, 12)
    out, ref, ncopies = _fused_step(A, M, seqs, cuda_device, cache, hk, hv, q, dtype, 13, 1 / math.sqrt(D))
    assert ncopies == groups * (gsz - 1)
    gk, gv = host_pool(cache.k), host_pool(cache.v)
    assert same_bits(gk, hk) and same_bits(gv, hv)
    for b, (sk, sv) in snap.items():
        assert same_bits(gk[b], sk) and same_bits(gv[b], sv)
    assert_attn_close(out, ref, dtype)
    # a second step: the copies are private now, nothing is copied
    q = synth.normal((len(seqs), Hq, D), dtype, 14)
    out, ref, ncopies = _fused_step(A, M, seqs, cuda_device, cache, hk, hv, q, dtype, 15, 1 / math.sqrt(D))
    assert ncopies == 0
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    assert_attn_close(out, ref, dtype)


def test_fused_equals_separate_calls(cuda_device):
    """The same state through pa_copy_blocks + pa_append_kv + pa_decode and
    through pa_append_decode: pools and outputs identical bit for bit."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 8, 128, 16, 64
    pl, _, order, NB = synth.shared_prefix_layout(5, groups=3, group_size=4, prefix=512, median=900,
                                                  clip=3000, prefix_tail=True)
    A1, A2 = pa.Allocator(NB, bs, order), pa.Allocator(NB, bs, order)
    k0 = synth.normal((NB, Hkv, bs, D), dt, 50)
    v0 = synth.normal((NB, Hkv, bs, D), dt, 51)
    c1 = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    c2 = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    seqs = []
    for A in (A1, A2):
        roots = [A.new_seq() for _ in pl]
        A.batch_append(roots, pl.tolist())
        seqs = [s for r in roots for s in [r] + [A.fork(r) for _ in range(3)]]
    n = len(seqs)
    for step in range(2):
        s1, p1 = A1.batch_append(seqs, [1] * n)
        s2, p2 = A2.batch_append(seqs, [1] * n)
        assert np.array_equal(s1, s2) and np.array_equal(p1, p2)
        mb = max(len(A1.block_table(s)) for s in seqs)
        tables, lens = A1.build_block_tables(seqs, mb)
        kn = synth.normal((n, Hkv, D), dt, 60 + step).to(cuda_device)
        vn = synth.normal((n, Hkv, D), dt, 70 + step).to(cuda_device)
        q = synth.normal((n, Hq, D), dt, 80 + step).to(cuda_device)
        td, ld = torch.from_numpy(tables).to(cuda_device), torch.from_numpy(lens).to(cuda_device)
        if len(p1):
            pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(p1)).to(cuda_device), c1)
        pa.pa_append_kv(kn, vn, torch.from_numpy(s1).to(cuda_device), c1)
        o1 = pa.pa_decode(q, c1, td, ld, int(lens.max()), 1 / math.sqrt(D))
        cow = pa.cow_sources(p2, tables, lens, bs)
        o2 = pa.pa_append_decode(kn, vn, q, c2, td, ld, int(lens.max()), 1 / math.sqrt(D),
                                 cow_src=torch.from_numpy(cow).to(cuda_device))
        assert pa.pa_read_device_error() == 0
        assert torch.equal(c1.k.view(torch.int16), c2.k.view(torch.int16))
        assert torch.equal(c1.v.view(torch.int16), c2.v.view(torch.int16))
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fused_empty_and_bad_rows(cuda_device, dtype):
    """A zero length appends nothing and gives a zero row; a copy source
    outside the pool sets PA_DEVERR_PAIR and is skipped (the append and the
    decode of that sequence still happen)."""
    Hkv, D, bs, Hq = 2, 128, 16, 8
    case = synth.random_case(31, B=5, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=np.array([0, 17, 300, 1, 600], np.int32),
                             dtype=dtype, device="cpu", sentinel=True)
    dev = cuda_device
    hk, hv = host_pool(case.k_cache), host_pool(case.v_cache)
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev))
    kn = synth.normal((5, Hkv, D), dtype, 32)
    vn = synth.normal((5, Hkv, D), dtype, 33)
    tables, lens = case.block_tables, case.context_lens
    cow = np.full(5, -1, np.int32)
    cow[2] = case.k_cache.shape[0] + 3  # outside the pool
    out = pa.pa_append_decode(kn.to(dev), vn.to(dev), case.q.to(dev), cache, torch.from_numpy(tables).to(dev),
                              torch.from_numpy(lens).to(dev), int(lens.max()), case.scale,
                              cow_src=torch.from_numpy(cow).to(dev))
    assert pa.pa_read_device_error() == pa.PA_DEVERR_PAIR
    slots = np.array([-1 if L == 0 else int(tables[i, (L - 1) // bs]) * bs + (L - 1) % bs
                      for i, L in enumerate(lens)], np.int64)
    oracle.append_kv(hk, hv, kn, vn, slots)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    ref = oracle.decode(case.q, hk, hv, tables, lens, case.scale)
    assert_attn_close(out, ref, dtype)
    assert not out[0].any()


def test_fused_many_sequences_coarse(cuda_device):
    """2100 sequences run as one launch of the tensor-core kernel's coarse
    form (its tables count whole entries of 8 sequences), which places each
    sequence's new row and copy source from those tables.  Some sequences
    copy a block of another sequence (a full first block) over their last
    block."""
    B, Hq, Hkv, D, bs = 2100, 8, 2, 128, 16
    dt = torch.bfloat16
    lens = synth.rng(48).integers(1, 80, size=B).astype(np.int32)
    case = synth.random_case(48, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=lens, dtype=dt, sentinel=True)
    tables = case.block_tables
    donors = np.flatnonzero(lens > bs)
    r = synth.rng(49)
    cow = np.full(B, -1, np.int32)
    for b in r.choice(B, size=300, replace=False):
        d = int(r.choice(donors))
        if d != b:
            cow[b] = tables[d, 0]
    kn = synth.normal((B, Hkv, D), dt, 50)
    vn = synth.normal((B, Hkv, D), dt, 51)
    hk, hv = host_pool(case.k_cache), host_pool(case.v_cache)
    dev = cuda_device
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev))
    out = pa.pa_append_decode(kn.to(dev), vn.to(dev), case.q.to(dev), cache, torch.from_numpy(tables).to(dev),
                              torch.from_numpy(lens).to(dev), int(lens.max()), case.scale,
                              cow_src=torch.from_numpy(cow).to(dev))
    assert pa.pa_read_device_error() == 0
    last = tables[np.arange(B), (lens - 1) // bs]
    oracle.copy_blocks(hk, hv, [(int(cow[b]), int(last[b])) for b in range(B) if cow[b] >= 0])
    oracle.append_kv(hk, hv, kn, vn, last.astype(np.int64) * bs + (lens - 1) % bs)
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    ref = oracle.decode(case.q, hk, hv, tables, lens, case.scale)
    assert_attn_close(out, ref, dt)

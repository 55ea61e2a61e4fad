"""Pins the oracle's allocator model, append and block copy (no GPU).

Facts used ("PagedAttention Internals", "Fixed-Size KV Blocks" and "The
Block Table Map"; the "pagedattention" glossary entry, comparison table and
paragraph 5, sharing): a sequence holds ceil(n / bs) blocks
after n tokens; any free block can take the next portion; waste is confined to
the last block; shared blocks are copied only when a sharer writes them.
"""
import numpy as np
import pytest

import oracle
from paged_kv_cache_402_b200 import synth


def _caches(NB, Hkv, bs, D, seed=0):
    r = synth.rng(seed)
    k = r.integers(0, 2**16, size=(NB, Hkv, bs, D), dtype=np.uint16)
    v = r.integers(0, 2**16, size=(NB, Hkv, bs, D), dtype=np.uint16)
    return k, v


def test_blocks_after_n_appends():
    for bs in (1, 2, 8, 16):
        A = oracle.AllocatorModel(64, bs)
        sid = A.new_seq()
        for n in range(1, 60):
            A.append(sid, 1)
            assert len(A.block_table(sid)) == -(-n // bs)
            assert A.seq_waste(sid) < bs


def test_table_follows_free_order():
    """With the free list dealt 8, 3, 11, ... a 48-token sequence gets the
    table of the example in "The Block Table Map"."""
    order = [8, 3, 11] + [b for b in range(12) if b not in (8, 3, 11)]
    A = oracle.AllocatorModel(12, 16, order)
    sid = A.new_seq()
    slots, cow = A.append(sid, 48)
    assert A.block_table(sid) == [8, 3, 11]
    assert slots == [8 * 16 + i for i in range(16)] + [3 * 16 + i for i in range(16)] + [11 * 16 + i for i in range(16)]
    assert cow is None


def test_block_count_conserved_and_refcounts_match_tables():
    r = synth.rng(5)
    A = oracle.AllocatorModel(200, 4, r.permutation(200))
    live = []
    for step in range(400):
        op = r.integers(0, 4)
        if op == 0 or not live:
            live.append(A.new_seq())
        elif op == 1:
            live.append(A.fork(live[r.integers(len(live))]))
        elif op == 2 and len(live) > 1:
            A.free_seq(live.pop(r.integers(len(live))))
        else:
            sid = live[r.integers(len(live))]
            try:
                A.append(sid, int(r.integers(1, 6)))
            except oracle.OutOfBlocks:
                pass
        refs = np.zeros(200, int)
        for t in A.tables.values():
            for blk in t:
                refs[blk] += 1
        assert refs.tolist() == A.ref
        assert A.used_blocks() + len(A.free) == 200
        assert int((refs > 0).sum()) == A.used_blocks()
        for sid in A.tables:
            assert 0 <= A.seq_waste(sid) < 4
        u = A.usage()
        assert u.allocated == 4 * A.used_blocks()


def test_exhaustion_leaves_state_unchanged():
    A = oracle.AllocatorModel(4, 4)
    s = A.new_seq()
    A.append(s, 10)  # 3 blocks
    before = (list(A.free), list(A.ref), {k: list(v) for k, v in A.tables.items()}, dict(A.lens))
    with pytest.raises(oracle.OutOfBlocks):
        A.append(s, 7)  # needs 2 more, 1 free
    assert (list(A.free), list(A.ref), {k: list(v) for k, v in A.tables.items()}, dict(A.lens)) == before
    t = A.new_seq()
    with pytest.raises(oracle.OutOfBlocks):
        A.batch_append([s, t], [3, 4])  # one new block each, one free
    assert dict(A.lens) == {s: 10, t: 0}


def test_fork_shares_until_write_then_copies():
    bs, NB = 4, 16
    A = oracle.AllocatorModel(NB, bs, synth.rng(1).permutation(NB))
    k, v = _caches(NB, 2, bs, 8)
    p = A.new_seq()
    A.append(p, 6)  # 2 blocks, the second half full
    c = A.fork(p)
    assert A.block_table(c) == A.block_table(p)
    assert all(A.ref[b] == 2 for b in A.block_table(p))
    shared = A.block_table(p)
    snap_k, snap_v = k[shared].copy(), v[shared].copy()
    # the parent writes into the shared, partially filled last block -> copy
    slots, cow = A.append(p, 1)
    assert cow is not None and cow[0] == shared[1]
    assert A.ref[shared[1]] == 1 and A.ref[cow[1]] == 1
    assert A.block_table(p) == [shared[0], cow[1]]
    assert A.block_table(c) == shared
    oracle.copy_blocks(k, v, [cow])
    r = synth.rng(2)
    newk = r.integers(0, 2**16, size=(1, 2, 8), dtype=np.uint16)
    newv = r.integers(0, 2**16, size=(1, 2, 8), dtype=np.uint16)
    oracle.append_kv(k, v, newk, newv, slots)
    # shared blocks are bit-unchanged
    assert np.array_equal(k[shared], snap_k) and np.array_equal(v[shared], snap_v)
    # the copy holds the same first two tokens, then the parent's new token
    assert np.array_equal(k[cow[1], :, :2], snap_k[1, :, :2])
    assert np.array_equal(k[cow[1], :, 2], newk[0])
    assert np.array_equal(v[cow[1], :, 2], newv[0])
    # the child now owns the old block alone and writes in place
    slots_c, cow_c = A.append(c, 1)
    assert cow_c is None and slots_c == [shared[1] * bs + 2]


def test_full_shared_block_never_copied():
    A = oracle.AllocatorModel(16, 4)
    p = A.new_seq()
    A.append(p, 8)  # two full blocks
    c = A.fork(p)
    _, cow = A.append(p, 1)
    assert cow is None
    _, cow = A.append(c, 1)
    assert cow is None
    assert A.block_table(p)[:2] == A.block_table(c)[:2]
    assert A.block_table(p)[2] != A.block_table(c)[2]


def test_k_sharers_make_k_minus_1_copies():
    """k sequences share a partial last block; one batch appends to all: the
    first k-1 copy it, the last (reference count 1 by then) writes in place."""
    for k in (2, 3, 8):
        A = oracle.AllocatorModel(64, 16)
        root = A.new_seq()
        A.append(root, 21)
        sids = [root] + [A.fork(root) for _ in range(k - 1)]
        last = A.block_table(root)[-1]
        slots, cows = A.batch_append(sids, [1] * k)
        assert len(cows) == k - 1
        assert all(c[0] == last for c in cows)
        assert A.block_table(sids[-1])[-1] == last
        assert slots[-1] == last * 16 + 5
        assert A.ref[last] == 1


def test_copy_on_write_counts_against_the_free_list():
    """A write into a shared partial block takes a free block for its copy,
    so a batch is refused, state unchanged, when the copies do not fit; k
    sharers need k - 1 copies, not k (the last writer owns the block by its
    turn)."""
    for k in (2, 3, 5):
        # root: 5 tokens in 2 blocks of 4, the second shared by all k
        for spare in (k - 2, k - 1):
            A = oracle.AllocatorModel(2 + spare, 4)
            root = A.new_seq()
            A.append(root, 5)
            sids = [root] + [A.fork(root) for _ in range(k - 1)]
            assert len(A.free) == spare
            before = (list(A.free), list(A.ref), {s: list(t) for s, t in A.tables.items()}, dict(A.lens))
            if spare < k - 1:
                with pytest.raises(oracle.OutOfBlocks):
                    A.batch_append(sids, [1] * k)
                assert (list(A.free), list(A.ref), {s: list(t) for s, t in A.tables.items()},
                        dict(A.lens)) == before
            else:
                _, cows = A.batch_append(sids, [1] * k)
                assert len(cows) == k - 1 and not A.free


def test_free_returns_blocks_lifo():
    A = oracle.AllocatorModel(8, 2, [0, 1, 2, 3, 4, 5, 6, 7])
    a = A.new_seq()
    A.append(a, 4)  # blocks 0, 1
    b = A.new_seq()
    A.append(b, 2)  # block 2
    A.free_seq(a)   # pushes 0 then 1
    c = A.new_seq()
    A.append(c, 4)
    assert A.block_table(c) == [1, 0]


def test_append_and_copy_bit_exact_and_padding_skipped():
    NB, Hkv, bs, D = 6, 2, 4, 8
    k, v = _caches(NB, Hkv, bs, D, seed=3)
    k0, v0 = k.copy(), v.copy()
    r = synth.rng(4)
    nk = r.integers(0, 2**16, size=(3, Hkv, D), dtype=np.uint16)
    nv = r.integers(0, 2**16, size=(3, Hkv, D), dtype=np.uint16)
    oracle.append_kv(k, v, nk, nv, [9, -1, 22])
    # slot s is row s % bs of block s // bs, every kv head
    for (blk, off), i in (((2, 1), 0), ((5, 2), 2)):
        assert np.array_equal(k[blk, :, off], nk[i]) and np.array_equal(v[blk, :, off], nv[i])
    for cache, before in ((k, k0), (v, v0)):
        changed = np.argwhere((cache != before).any(axis=-1))
        assert {(int(a), int(c)) for a, _, c in changed} <= {(2, 1), (5, 2)}
    with pytest.raises(IndexError):
        oracle.append_kv(k, v, nk[:1], nv[:1], [NB * bs])
    # block 4 becomes what block 1 held; block 1 and the rest stay as they were
    k1, v1 = k.copy(), v.copy()
    oracle.copy_blocks(k, v, [(1, 4)])
    for cache, before in ((k, k1), (v, v1)):
        assert np.array_equal(cache[4], before[1])
        assert all(np.array_equal(cache[b], before[b]) for b in range(NB) if b != 4)


# ------------------------------------------------------------------ usage under sharing
#
# The fragmentation measure is the one of the learn-ml-visualized chapter
# "inference-acceleration-pagedattention-vllm" (fragmentation worked example):
# waste = allocated - used, fragmentation = waste / allocated.  With shared
# blocks the allocation is physical: a block in use counts once however many
# tables hold it, and its tokens once.  The counts below are worked out by
# hand, not by the model.


def test_usage_reproduces_the_paged_worked_example():
    """Lengths 1, 4, 2 grown through the allocator in pages of 2: 8 slots held,
    7 used, the single wasted slot in the length-1 sequence's half-empty page."""
    A = oracle.AllocatorModel(16, 2)
    for L in (1, 4, 2):
        A.append(A.new_seq(), L)
    u = A.usage()
    assert (u.allocated, u.used, u.wasted) == (8, 7, 1)
    assert u.fragmentation == 1 / 8


def test_usage_of_a_shared_partial_block_by_hand():
    """Block size 4.  A root of 6 tokens holds block 10 (4 tokens) and block
    11 (2 tokens); two forks share both (reference count 3).  Physically:
    8 slots held, 6 used.  One token is then appended to the root, the first
    fork and the second fork, in that order: the root copies 11 into 12, the
    first fork copies 11 into 13, and the second fork, by then the only
    holder of 11, writes into it in place.  Physically: 10 (4 tokens, shared
    by three), 11, 12 and 13 (3 tokens each): 16 slots held, 13 used, 3
    wasted."""
    A = oracle.AllocatorModel(32, 4, [10, 11, 12, 13] + [b for b in range(32) if b not in (10, 11, 12, 13)])
    root = A.new_seq()
    A.append(root, 6)
    kids = [A.fork(root), A.fork(root)]
    u = A.usage()
    assert (u.allocated, u.used) == (8, 6)
    assert u.fragmentation == 2 / 8
    slots, cows = A.batch_append([root] + kids, [1, 1, 1])
    assert cows == [(11, 12), (11, 13)]
    assert slots == [12 * 4 + 2, 13 * 4 + 2, 11 * 4 + 2]
    u = A.usage()
    assert (u.allocated, u.used, u.wasted) == (16, 13, 3)
    assert u.fragmentation == 3 / 16


def test_usage_of_full_shared_blocks_by_hand():
    """Block size 4.  A root of 8 tokens fills blocks 10 and 11; two forks
    share them.  One token appended to each of the three takes a fresh
    block each (12, 13, 14; full blocks are never copied).  Physically: 10
    and 11 (4 tokens each, counted once), 12, 13, 14 (1 token each): 20
    slots held, 11 used.  Freeing the root then releases only its own block
    12: 16 held, 10 used."""
    A = oracle.AllocatorModel(32, 4, list(range(10, 32)) + list(range(10)))
    root = A.new_seq()
    A.append(root, 8)
    kids = [A.fork(root), A.fork(root)]
    u = A.usage()
    assert (u.allocated, u.used) == (8, 8)
    _, cows = A.batch_append([root] + kids, [1, 1, 1])
    assert cows == []
    assert [A.block_table(s) for s in [root] + kids] == [[10, 11, 12], [10, 11, 13], [10, 11, 14]]
    u = A.usage()
    assert (u.allocated, u.used, u.wasted) == (20, 11, 9)
    A.free_seq(root)
    u = A.usage()
    assert (u.allocated, u.used) == (16, 10)
    assert A.ref[10] == 2 and A.ref[12] == 0

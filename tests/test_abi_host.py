"""The C ABI on the host (no GPU): exported symbols, argument checks that
return before any launch, the copy-pair check, and the C++ allocator against
the oracle's allocator model."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def _declared():
    names = set()
    for f in os.listdir(HEADER_DIR):
        if f.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, f)).read()
            names |= set(re.findall(r"PA_API\s+[\w\s\*]*?\b(pa_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("pa_append_kv", "pa_decode", "pa_copy_blocks", "pa_decode_workspace_size",
                     "pa_read_device_error", "pa_alloc_create", "pa_seq_append", "pa_seq_fork"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(L, n)]
    assert not missing, f"not exported: {missing}"


def test_no_internal_symbols_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True).stdout
    ours = {l.split()[-1] for l in out.splitlines() if l.split() and l.split()[-1].startswith("pa_")}
    assert ours == set(_declared())


def test_header_constants_match_the_binding():
    """Every numeric #define of the header that the binding mirrors has the
    same value there."""
    hdr = open(os.path.join(os.path.dirname(__file__), "..", "include", "pagedattn.h")).read()
    found = {}
    for name, val in re.findall(r"^#define (PA_[A-Z_]+) \(?([0-9xu<> ]+)\)?", hdr, re.M):
        val = val.replace("u", "").strip()
        found[name] = eval(val, {})
    mirrored = [n for n in found if hasattr(pa, n)]
    assert {"PA_PARTITION_TOKENS", "PA_SHARE_MIN_TOKENS", "PA_STATIC_WORKSPACE_BYTES",
            "PA_DEVERR_PLAN"} <= set(mirrored)
    for n in mirrored:
        assert getattr(pa, n) == found[n], n


def test_status_strings_and_version():
    assert pa.lib().pa_status_string(pa.PA_OK) == b"ok"
    assert pa.lib().pa_status_string(pa.PA_ERR_OUT_OF_BLOCKS) == b"out of free blocks"
    assert pa.lib().pa_version().count(b".") == 2
    # no CUDA call of the library has failed on this thread
    assert pa.lib().pa_last_cuda_error() == 0
    assert pa.lib().pa_cuda_error_string(0) == b"no error"
    assert pa.lib().pa_cuda_error_string(2) == b"out of memory"


def _cache_struct(**kw):
    d = dict(k=16, v=32, dtype=pa.PA_DTYPE_BF16, num_blocks=8, block_size=16, num_kv_heads=2, head_dim=128)
    d.update(kw)
    return pa.pa_cache_t(**d)


@pytest.mark.parametrize("kw,expect", [
    (dict(dtype=7), pa.PA_ERR_UNSUPPORTED),
    (dict(block_size=12), pa.PA_ERR_UNSUPPORTED),
    (dict(head_dim=96), pa.PA_ERR_UNSUPPORTED),
    (dict(num_blocks=0), pa.PA_ERR_INVALID_ARG),
    (dict(k=0), pa.PA_ERR_INVALID_ARG),
    (dict(k=17), pa.PA_ERR_INVALID_ARG),  # misaligned pool
])
def test_bad_cache_rejected_before_launch(kw, expect):
    c = _cache_struct(**kw)
    L = pa.lib()
    assert L.pa_append_kv(16, 16, 16, 1, ctypes.byref(c), None) == expect
    assert L.pa_copy_blocks(16, 1, ctypes.byref(c), None) == expect
    assert L.pa_decode(16, ctypes.byref(c), 16, 4, 16, 1, 2, 64, 1.0, 16, None, 0, None) == expect


def test_decode_argument_checks():
    c = _cache_struct()
    L = pa.lib()
    args = lambda **o: [o.get("q", 16), ctypes.byref(c), 16, o.get("mb", 4), 16, o.get("B", 1), o.get("Hq", 2),
                        o.get("ml", 64), o.get("scale", 1.0), o.get("out", 16), o.get("ws", None),
                        o.get("wsb", 0), None]
    assert L.pa_decode(*args(Hq=3)) == pa.PA_ERR_INVALID_ARG          # not a multiple of Hkv
    assert L.pa_decode(*args(Hq=6)) == pa.PA_ERR_UNSUPPORTED           # group size 3
    assert L.pa_decode(*args(Hq=32)) == pa.PA_ERR_UNSUPPORTED          # group size 16
    assert L.pa_decode(*args(ml=65)) == pa.PA_ERR_INVALID_ARG          # 65 tokens > 4 blocks x 16
    assert L.pa_decode(*args(scale=float("nan"))) == pa.PA_ERR_INVALID_ARG
    assert L.pa_decode(*args(q=0)) == pa.PA_ERR_INVALID_ARG
    assert L.pa_decode(*args(out=8)) == pa.PA_ERR_INVALID_ARG          # misaligned
    # a context past one partition needs a workspace
    assert L.pa_decode(*args(mb=64, ml=1000)) == pa.PA_ERR_INVALID_ARG
    need = L.pa_decode_workspace_size(1, 2, 1000, 128)
    assert L.pa_decode(*args(mb=64, ml=1000, ws=16, wsb=need - 16)) == pa.PA_ERR_TOO_SMALL
    assert L.pa_decode(*args(B=0)) == pa.PA_OK                         # nothing to do, no launch


def test_append_decode_argument_checks():
    c = _cache_struct()
    L = pa.lib()
    args = lambda **o: [o.get("k", 16), o.get("v", 16), o.get("cow", None), o.get("q", 16), ctypes.byref(c), 16,
                        o.get("mb", 4), 16, o.get("B", 1), o.get("Hq", 2), o.get("ml", 64), 1.0, o.get("out", 16),
                        None, 0, None]
    assert L.pa_append_decode(*args(k=0)) == pa.PA_ERR_INVALID_ARG      # no new key rows
    assert L.pa_append_decode(*args(v=8)) == pa.PA_ERR_INVALID_ARG      # misaligned
    assert L.pa_append_decode(*args(Hq=6)) == pa.PA_ERR_UNSUPPORTED     # group size 3, as pa_decode
    assert L.pa_append_decode(*args(ml=65)) == pa.PA_ERR_INVALID_ARG    # 65 tokens > 4 blocks x 16
    assert L.pa_append_decode(*args(out=0)) == pa.PA_ERR_INVALID_ARG
    assert L.pa_append_decode(*args(B=0)) == pa.PA_OK                   # nothing to do, no launch


def test_cow_sources():
    tables = np.array([[4, 9, -1], [4, 7, -1], [5, 6, 2]], np.int32)
    lens = np.array([20, 17, 33], np.int32)  # last blocks 9, 7, 2 at block size 16
    assert pa.cow_sources([[3, 7]], tables, lens, 16).tolist() == [-1, 3, -1]
    assert pa.cow_sources(np.zeros((0, 2)), tables, lens, 16).tolist() == [-1, -1, -1]
    with pytest.raises(pa.PagedAttnError):
        pa.cow_sources([[3, 8]], tables, lens, 16)           # 8 is no sequence's last block
    with pytest.raises(pa.PagedAttnError):
        pa.cow_sources([[3, 7], [1, 7]], tables, lens, 16)   # a repeated destination


def test_cow_sources_of_an_allocator_step():
    """Four sharers of a partly filled block each append one token: the first
    three copy it (in batch order), the last writes in place."""
    A = pa.Allocator(64, 16, list(range(64)))
    r = A.new_seq()
    A.batch_append([r], [20])
    shared = A.block_table(r)[-1]
    seqs = [r] + [A.fork(r) for _ in range(3)]
    _, pairs = A.batch_append(seqs, [1] * 4)
    tables, lens = A.build_block_tables(seqs, 4)
    cow = pa.cow_sources(pairs, tables, lens, 16)
    assert cow.tolist() == [shared, shared, shared, -1]
    assert [int(tables[i, 1]) for i in range(3)] == [int(p[1]) for p in pairs]


def test_cow_sources_walks_the_table_in_c():
    """The library finds each sequence's last block itself: the newest
    token's table entry, (len - 1) / bs; a length of 0 has none, and a
    newest token past the table's width is an argument error."""
    L = pa.lib()
    tables = np.array([[4, 9, -1], [4, 7, -1], [5, 6, 2], [8, -1, -1]], np.int32)
    lens = np.array([20, 17, 33, 0], np.int32)
    pairs = np.array([[3, 7], [1, 2]], np.int32)
    out = np.full(4, 99, np.int32)
    assert L.pa_cow_sources(pairs.ctypes.data, 2, tables.ctypes.data, 3, lens.ctypes.data, 4, 16,
                            out.ctypes.data) == pa.PA_OK
    assert out.tolist() == [-1, 3, 1, -1]
    assert L.pa_cow_sources(pairs.ctypes.data, 2, tables.ctypes.data, 3, lens.ctypes.data, 4, 8,
                            out.ctypes.data) == pa.PA_ERR_INVALID_ARG   # 33 tokens need entry 4 at bs 8
    assert L.pa_cow_sources(pairs.ctypes.data, 1, tables.ctypes.data, 3, lens.ctypes.data, 4, 0,
                            out.ctypes.data) == pa.PA_ERR_INVALID_ARG


def test_fragmentation_of_a_shared_step_by_hand():
    """The C++ allocator's fragmentation on the hand-counted case of the
    oracle's pins (learn-ml-visualized worked example's measure, waste over
    allocated): a root of 6 tokens at block size 4 forked twice holds 8
    slots with 6 used (0.25); after one token each (two copies on write) 16
    slots with 13 used (3/16)."""
    A = pa.Allocator(32, 4, [10, 11, 12, 13] + [b for b in range(32) if b not in (10, 11, 12, 13)])
    root = A.new_seq()
    A.append(root, 6)
    kids = [A.fork(root), A.fork(root)]
    st = A.stats()
    assert (st["allocated_slots"], st["used_slots"], st["fragmentation"]) == (8, 6, 0.25)
    _, pairs = A.batch_append([root] + kids, [1, 1, 1])
    assert pairs.tolist() == [[11, 12], [11, 13]]
    st = A.stats()
    assert (st["allocated_slots"], st["used_slots"], st["fragmentation"]) == (16, 13, 3 / 16)
    frag = ctypes.c_double(-1.0)
    assert pa.lib().pa_alloc_fragmentation(A._h, ctypes.byref(frag)) == pa.PA_OK
    assert frag.value == 3 / 16
    empty = pa.Allocator(8, 4)
    assert empty.stats()["fragmentation"] == 0.0
    assert pa.lib().pa_alloc_fragmentation(None, ctypes.byref(frag)) == pa.PA_ERR_INVALID_ARG


def test_wrappers_check_q_and_out_before_any_launch():
    """The Python wrappers refuse a q whose head_dim is not the cache's, or an
    out of another shape, before the library is called (the C side writes
    B x Hq x head_dim elements of out)."""
    import types
    import torch
    cache = types.SimpleNamespace(head_dim=128, num_kv_heads=2, dtype=torch.bfloat16)
    q64 = torch.zeros(2, 4, 64, dtype=torch.bfloat16)
    q = torch.zeros(2, 4, 128, dtype=torch.bfloat16)
    t = torch.zeros(2, 4, dtype=torch.int32)
    n = torch.zeros(2, dtype=torch.int32)
    for fn in (pa.pa_decode, pa.pa_decode_static_workspace, pa.pa_decode_shared):
        with pytest.raises(ValueError, match="head_dim"):
            fn(q64, cache, t, n, 16, 0.1)
        with pytest.raises(ValueError, match="out must"):
            fn(q, cache, t, n, 16, 0.1, out=torch.zeros(1, 4, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="head_dim"):
        pa.pa_append_decode(q, q, q64, cache, t, n, 16, 0.1)


def test_workspace_size_of_huge_lengths():
    """A length near INT32_MAX sizes its partitions without wrapping."""
    ws = pa.pa_decode_workspace_size(1, 1, 2**31 - 1, 128)
    parts = -(-(2**31 - 1) // 512)
    assert ws == 2 * ((parts * 4 + 15) // 16 * 16) + parts * 128 * 4


def test_step_layout():
    """The staging area of one decode step: q, new rows, then the int32
    arrays the step's host work writes, each 16-byte aligned, in order."""
    L = pa.pa_step_layout_t()
    c = _cache_struct(num_kv_heads=8)
    assert pa.lib().pa_step_layout(32, 32, ctypes.byref(c), 257, 4, ctypes.byref(L)) == pa.PA_OK
    offs = [L.q, L.k_new, L.v_new, L.tables, L.lens, L.cow_src, L.first_token, L.members, L.shared_tokens,
            L.bytes]
    assert offs == sorted(offs) and all(o % 16 == 0 for o in offs)
    assert L.k_new - L.q == 32 * 32 * 128 * 2 and L.v_new - L.k_new == 32 * 8 * 128 * 2
    assert L.lens - L.tables >= 32 * 257 * 4 and L.shared_tokens - L.members >= 16 * 4 * 4
    assert pa.lib().pa_step_layout(32, 32, ctypes.byref(c), 257, 5, ctypes.byref(L)) == pa.PA_ERR_INVALID_ARG


def test_decode_step_refuses_before_the_allocator_moves():
    """Argument errors of pa_decode_step come before the allocator's step: a
    slot without buffers, or a workspace too small, leaves every sequence as
    it was."""
    A = pa.Allocator(64, 16)
    s = A.new_seq()
    A.append(s, 600)
    seqs = np.array([s], np.int32)
    nc, ng, ml = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    c = _cache_struct(num_blocks=64, num_kv_heads=2)
    slot = pa.pa_step_slot_t()
    args = lambda sl: (A._h, seqs.ctypes.data, 1, 64, 0, ctypes.byref(c), 8, ctypes.c_float(0.1), ctypes.byref(sl),
                       None, None, None, ctypes.byref(nc), ctypes.byref(ng), ctypes.byref(ml))
    assert pa.lib().pa_decode_step(*args(slot)) == pa.PA_ERR_INVALID_ARG
    slot = pa.pa_step_slot_t(16, 32, 48, 64, None, 0, 1, 2, 3)  # fake addresses, no workspace
    assert pa.lib().pa_decode_step(*args(slot)) == pa.PA_ERR_TOO_SMALL  # 64 x 16 tokens of room need a workspace
    assert A.seq_len(s) == (600, 38)


def test_share_plan_block_granular():
    """The plan's unit of sharing is the block, whatever the partition size:
    two sequences whose first 600 tokens sit in the same blocks, the 38th
    only partly (copied on write when they diverged), share 37 blocks."""
    bs = 16
    common = np.arange(100, 100 + 600 // bs + 1, dtype=np.int32)
    t = np.full((2, 80), -1, np.int32)
    t[0, :38] = common[:38]
    t[1, :38] = common[:38]
    t[0, 37:70] = np.arange(500, 533)
    t[1, 37:70] = np.arange(600, 633)
    lens = np.array([1100, 1090], np.int32)
    plan = pa.share_plan(t, lens, bs)
    assert plan.n_groups == 1 and plan.shared_tokens.tolist() == [37 * bs]
    assert plan.first_token.tolist() == [37 * bs, 37 * bs]
    for bad_bs in (12, 64):
        with pytest.raises(pa.PagedAttnError):
            pa.share_plan(t, lens, bad_bs)


def test_shared_workspace_size():
    """With a plan, the scratch holds one more row per (sequence, query head)
    than the plain decode's (the piece of the partition a shared prefix ends
    in), and is needed even when every sequence fits one partition."""
    rows = lambda r: 2 * ((r * 4 + 15) // 16 * 16) + r * 128 * 4
    ws, wss = pa.pa_decode_workspace_size, pa.pa_decode_shared_workspace_size
    assert ws(2, 8, 1000, 128, 256) == rows(2 * 8 * 4)
    assert wss(2, 8, 1000, 128, 256) == rows(2 * 8 * 5)
    assert wss(3, 4, 1000, 128, 512) == rows(3 * 4 * 3)
    assert ws(3, 4, 500, 128, 512) == 0 and wss(3, 4, 500, 128, 512) == rows(3 * 4 * 2)
    assert wss(3, 4, 500, 128, 384) == 0 and wss(0, 4, 500, 128, 512) == 0
    assert ws(2, 8, 1000, 128, 1024) == 0 and ws(2, 8, 1000, 128, 384) == 0
    assert ws(2, 8, 1000, 128) == ws(2, 8, 1000, 128, 512)


def test_workspace_size():
    ws = pa.pa_decode_workspace_size
    assert ws(4, 8, 512, 128) == 0
    rows = 4 * 8 * 2
    assert ws(4, 8, 513, 128) == 2 * ((rows * 4 + 15) // 16 * 16) + rows * 128 * 4
    assert ws(8, 32, 131072, 128) == 2 * 8 * 32 * 256 * 4 + 8 * 32 * 256 * 128 * 4


def test_check_copy_pairs():
    assert pa.pa_check_copy_pairs([[1, 2], [3, 4]], 8)
    assert not pa.pa_check_copy_pairs([[1, 2], [3, 2]], 8)   # repeated destination
    assert not pa.pa_check_copy_pairs([[1, 2], [2, 4]], 8)   # destination is a source
    assert not pa.pa_check_copy_pairs([[1, 8]], 8)           # outside the pool
    assert pa.pa_check_copy_pairs(np.zeros((0, 2)), 8)


# ------------------------------------------------------------- allocator


def test_allocator_basics_match_model():
    order = [8, 3, 11] + [b for b in range(12) if b not in (8, 3, 11)]
    A = pa.Allocator(12, 16, order)
    M = oracle.AllocatorModel(12, 16, order)
    s, m = A.new_seq(), M.new_seq()
    slots, cow = A.append(s, 48)
    mslots, mcow = M.append(m, 48)
    assert slots.tolist() == mslots and cow is None and mcow is None
    assert A.block_table(s) == [8, 3, 11]
    with pytest.raises(pa.OutOfBlocks):
        A.append(s, 16 * 10)
    assert A.seq_len(s) == (48, 3)


def test_allocator_rejects_bad_input():
    with pytest.raises(pa.PagedAttnError):
        pa.Allocator(4, 16, [0, 1, 1, 2])
    A = pa.Allocator(4, 4)
    with pytest.raises(pa.PagedAttnError):
        A.append(99, 1)
    s = A.new_seq()
    with pytest.raises(pa.PagedAttnError):
        A.batch_append([s, s], [1, 1])


@pytest.mark.parametrize("seed", range(4))
def test_allocator_random_trace_matches_model(seed):
    """Random new / fork / free / (batch) append traces: the C++ allocator and
    the oracle's model agree on every slot, copy pair, table, refcount and
    usage figure, and on every out-of-blocks refusal."""
    r = synth.rng(100 + seed)
    NB, bs = 96, int(r.choice([1, 2, 4, 8, 16]))
    order = r.permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    live = []
    for step in range(500):
        op = int(r.integers(0, 6))
        if op == 0 or not live:
            a, m = A.new_seq(), M.new_seq()
            assert a == m
            live.append(a)
        elif op == 1:
            p = live[int(r.integers(len(live)))]
            a, m = A.fork(p), M.fork(p)
            assert a == m
            live.append(a)
        elif op == 2 and len(live) > 1:
            s = live.pop(int(r.integers(len(live))))
            A.free_seq(s)
            M.free_seq(s)
        elif op == 3:
            s = live[int(r.integers(len(live)))]
            n = int(r.integers(0, 3 * bs))
            try:
                got = A.append(s, n)
                ok = True
            except pa.OutOfBlocks:
                ok = False
            try:
                want = M.append(s, n)
                assert ok
                assert got[0].tolist() == want[0] and got[1] == want[1]
            except oracle.OutOfBlocks:
                assert not ok
        else:
            k = int(r.integers(1, len(live) + 1))
            sel = [int(x) for x in r.choice(live, size=k, replace=False)]
            ns = [int(x) for x in r.integers(0, 2 * bs, size=k)]
            try:
                gs, gp = A.batch_append(sel, ns)
                ok = True
            except pa.OutOfBlocks:
                ok = False
            try:
                ws, wp = M.batch_append(sel, ns)
                assert ok
                assert gs.tolist() == ws
                assert [tuple(x) for x in gp.tolist()] == wp
            except oracle.OutOfBlocks:
                assert not ok
        for s in live:
            assert A.block_table(s) == M.block_table(s)
            assert A.seq_len(s)[0] == M.lens[s]
        st = A.stats()
        u = M.usage()
        assert st["used_slots"] == u.used and st["allocated_slots"] == u.allocated
        assert st["free_blocks"] == len(M.free)
        for b in range(NB):
            assert A.refcount(b) == M.ref[b]


def test_allocator_copies_count_against_the_free_list():
    """k sharers of a partial last block appending in one batch need k - 1
    copy blocks: with one fewer free the library refuses the batch and its
    tables, lengths and refcounts stay as they were, like the model's; with
    exactly k - 1 both make the same copies."""
    for k in (2, 3, 5):
        for spare in (k - 2, k - 1):
            A, M = pa.Allocator(2 + spare, 4), oracle.AllocatorModel(2 + spare, 4)
            root = A.new_seq()
            assert M.new_seq() == root
            A.append(root, 5)
            M.append(root, 5)
            sids = [root] + [A.fork(root) for _ in range(k - 1)]
            assert [M.fork(root) for _ in range(k - 1)] == sids[1:]
            before = [(A.block_table(s), A.seq_len(s)[0]) for s in sids], [A.refcount(b) for b in range(2 + spare)]
            if spare < k - 1:
                with pytest.raises(pa.OutOfBlocks):
                    A.batch_append(sids, [1] * k)
                with pytest.raises(oracle.OutOfBlocks):
                    M.batch_append(sids, [1] * k)
                assert ([(A.block_table(s), A.seq_len(s)[0]) for s in sids],
                        [A.refcount(b) for b in range(2 + spare)]) == before
            else:
                gs, gp = A.batch_append(sids, [1] * k)
                ws, wp = M.batch_append(sids, [1] * k)
                assert gs.tolist() == ws and [tuple(x) for x in gp.tolist()] == wp and len(wp) == k - 1
                assert A.stats()["free_blocks"] == 0


def test_build_block_tables():
    A = pa.Allocator(32, 4)
    s = [A.new_seq() for _ in range(3)]
    for i, n in zip(s, (1, 9, 4)):
        A.append(i, n)
    tables, lens = A.build_block_tables(s, 4, pad=-1)
    assert lens.tolist() == [1, 9, 4]
    for row, i in zip(tables, s):
        t = A.block_table(i)
        assert row[:len(t)].tolist() == t and (row[len(t):] == -1).all()
    with pytest.raises(pa.PagedAttnError):
        A.build_block_tables(s, 2)


def test_fragmentation_example_through_the_allocator():
    """The worked example's paged layout (lengths 1, 4, 2; page size 2) in the
    C++ allocator: 8 slots allocated, 1 wasted."""
    A = pa.Allocator(16, 2)
    for n in (1, 4, 2):
        A.append(A.new_seq(), n)
    st = A.stats()
    assert st["allocated_slots"] == 8 and st["used_slots"] == 7
    assert st["fragmentation"] == pytest.approx(0.125)


def test_seqs_max_len():
    A = pa.Allocator(64, 8)
    s = [A.new_seq() for _ in range(3)]
    for i, n in zip(s, (5, 30, 17)):
        A.append(i, n)
    assert A.max_len(s) == (30, 4)
    assert A.max_len(s[:1]) == (5, 1)
    assert A.max_len([]) == (0, 0)


def test_share_plan_groups():
    """Buckets by the first block, groups of at most max_members in sequence
    order, a lone leftover in no group; the shared blocks stop where the
    tables part or before a member's last block, and a group that would
    share fewer than PA_SHARE_MIN_TOKENS tokens is dropped."""
    t = np.full((7, 96), -1, np.int32)
    for i in (0, 1, 2):                       # share 40 blocks, then private
        t[i, :40] = np.arange(40)
        t[i, 40:50] = 100 + 10 * i + np.arange(10)
    t[3, :60] = 200 + np.arange(60)           # alone
    t[4, :40] = np.arange(40)                 # joins 0..2 (same first block)
    t[4, 40:45] = 500 + np.arange(5)
    for i in (5, 6):                          # share 70 blocks
        t[i, :70] = 1000 + np.arange(70)
        t[i, 70:80] = 2000 + 10 * i + np.arange(10)
    lens = np.array([50 * 16, 49 * 16 + 3, 45 * 16, 60 * 16, 1024, 80 * 16, 75 * 16], np.int32)
    pl = pa.share_plan(t, lens, 16)
    assert pl.members.tolist() == [[0, 1, 2, 4], [5, 6, -1, -1]]
    assert pl.shared_tokens.tolist() == [640, 1120]
    assert pl.first_token.tolist() == [640, 640, 640, 0, 640, 1120, 1120]
    pl3 = pa.share_plan(t, lens, 16, max_members=3)       # 0, 1, 2 | 4 alone
    assert pl3.members.tolist() == [[0, 1, 2], [5, 6, -1]]
    assert pl3.first_token.tolist() == [640, 640, 640, 0, 0, 1120, 1120]
    short = lens.copy()
    short[6] = 1024                           # 64 blocks: 63 before 6's last
    assert pa.share_plan(t, short, 16).shared_tokens.tolist() == [640, 1008]
    short[6] = 8 * 16                         # 7 blocks before the last: under the minimum
    pl = pa.share_plan(t, short, 16)
    assert pl.members.tolist() == [[0, 1, 2, 4]] and pl.first_token[5] == 0 and pl.first_token[6] == 0
    short[6] = 9 * 16                         # 8 blocks: exactly the minimum
    assert pa.share_plan(t, short, 16).shared_tokens.tolist() == [640, 128]
    short[6] = 16                             # one block: nothing before its last
    assert pa.share_plan(t, short, 16).n_groups == 1


def test_share_plan_of_allocator_forks():
    """Forks of a 1300-token prompt share its 81 full blocks (the 82nd, the
    fork point's partial block, is copied on write by all but one)."""
    A = pa.Allocator(256, 16, list(range(256)))
    r = A.new_seq()
    A.batch_append([r], [1300])
    seqs = [r] + [A.fork(r) for _ in range(5)]
    A.batch_append(seqs, [1] * 6)
    tables, lens = A.build_block_tables(seqs, 90)
    pl = pa.share_plan(tables, lens, 16)
    assert pl.members.tolist() == [seqs[:4], seqs[4:] + [-1, -1]]
    assert pl.shared_tokens.tolist() == [1296, 1296] and pl.first_token.tolist() == [1296] * 6


def test_decode_shared_argument_checks():
    c = _cache_struct()
    L = pa.lib()
    plan = pa.pa_share_plan_t(16, 16, 16, 1, 5)
    args = lambda **o: [None, None, None, 16, ctypes.byref(c), 16, o.get("mb", 64), 16, 1, 2, o.get("ml", 1000),
                        1.0, ctypes.byref(o.get("plan", plan)), 16, 16, 1 << 20, None]
    assert L.pa_decode_shared(*args()) == pa.PA_ERR_INVALID_ARG                 # 5 members > 4
    bad = pa.pa_share_plan_t(0, 16, 16, 1, 4)
    assert L.pa_decode_shared(*args(plan=bad)) == pa.PA_ERR_INVALID_ARG         # no member array
    bad = pa.pa_share_plan_t(16, 0, 16, 1, 4)
    assert L.pa_decode_shared(*args(plan=bad)) == pa.PA_ERR_INVALID_ARG         # no shared tokens
    # with groups the scratch has the extra row: the plain decode's size is
    # too small, even for one partition (500 tokens)
    ok_plan = pa.pa_share_plan_t(16, 16, 16, 1, 4)
    for ml, mb in ((1000, 64), (500, 32)):
        plain = max(16, pa.pa_decode_workspace_size(1, 2, ml, 128))
        a = args(plan=ok_plan, ml=ml, mb=mb)
        a[15] = plain
        assert L.pa_decode_shared(*a) == pa.PA_ERR_TOO_SMALL


def test_decode_step_prepare_equals_the_separate_calls():
    """One call gives what batch_append + build_block_tables + cow_sources +
    share_plan give on an identical allocator: forks with copies on write,
    sharing groups, fresh blocks, and all-or-nothing on a full pool."""
    def state(seed):
        A = pa.Allocator(600, 16, synth.rng(seed).permutation(600))
        roots = [A.new_seq() for _ in range(5)]
        A.batch_append(roots, [600, 700, 37, 512, 1030])
        seqs = roots + [A.fork(roots[0]) for _ in range(3)] + [A.fork(roots[4]) for _ in range(2)]
        return A, seqs
    A1, seqs = state(3)
    A2, _ = state(3)
    for _ in range(3):
        got = A1.decode_step(seqs, 80)
        slots, pairs = A2.batch_append(seqs, [1] * len(seqs))
        tables, lens = A2.build_block_tables(seqs, 80)
        cow = pa.cow_sources(pairs, tables, lens, 16)
        plan = pa.share_plan(tables, lens, 16)
        assert np.array_equal(got["lens"], lens)
        for i, L in enumerate(lens):  # entries past a sequence's blocks are not written
            nb = -(-int(L) // 16)
            assert np.array_equal(got["tables"][i, :nb], tables[i, :nb])
        assert np.array_equal(got["cow_src"], cow) and got["n_copies"] == len(pairs)
        assert np.array_equal(got["members"], plan.members)
        assert np.array_equal(got["shared_tokens"], plan.shared_tokens)
        assert np.array_equal(got["first_token"], plan.first_token) and got["n_groups"] == plan.n_groups
        assert got["max_len"] == int(lens.max())
    assert A1.stats() == A2.stats()
    nogroups = A1.decode_step(seqs, 80, share_max_members=0)
    assert nogroups["n_groups"] == 0 and not nogroups["first_token"].any()
    with pytest.raises(pa.PagedAttnError):
        A1.decode_step(seqs, 40)  # 1030 tokens do not fit 40 blocks: nothing changes
    before = A1.stats()
    small = pa.Allocator(70, 16, list(range(70)))
    r = small.new_seq()
    small.batch_append([r], [16 * 70])
    with pytest.raises(pa.OutOfBlocks):
        small.decode_step([r], 80)
    assert small.seq_len(r)[0] == 16 * 70 and A1.stats() == before

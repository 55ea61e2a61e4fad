"""Pins the oracle to facts fixed outside itself (no GPU).

Each test checks the oracle against something it does not compute: numbers
the pages print, closed forms, invariants the pages state, a library softmax
on data laid out densely by a different route, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_402_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- fragmentation


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden("fragmentation.json")["cases"], ids=lambda c: f"{c['scheme']}-{c['lengths']}")
def test_fragmentation_golden(case):
    if case["scheme"] == "naive":
        u = oracle.naive_usage(case["lengths"], case["reserve"])
    else:
        u = oracle.paged_usage(case["lengths"], case["page"])
    assert u.allocated == case["allocated"]
    assert u.used == sum(case["lengths"])
    assert u.wasted == case["wasted"]
    if "fragmentation_3dp" in case:
        assert round(u.fragmentation, 3) == case["fragmentation_3dp"]
    else:
        assert u.fragmentation == pytest.approx(case["fragmentation"], abs=1e-15)


def test_naive_rejects_overlong():
    with pytest.raises(ValueError):
        oracle.naive_usage([5], 4)


def test_paged_waste_under_one_page_any_length():
    """A paged sequence wastes fewer than one page of slots, whatever its
    length; the naive waste can approach the whole reservation."""
    r = synth.rng(3)
    for page in (1, 2, 8, 16, 32):
        for L in r.integers(1, 5000, size=200).tolist():
            u = oracle.paged_usage([L], page)
            assert 0 <= u.wasted < page
            assert u.allocated % page == 0
    assert oracle.naive_usage([1], 4096).wasted == 4095


# ---------------------------------------------------------------- attention


def _dense_case(seed, lens, Hq, Hkv, D, bs, dtype=torch.float64, extra=3):
    """Draws dense per-sequence K/V ([L, Hkv, D]) first, then scatters them
    block by block into a pool along a seeded placement.  Returns the paged
    inputs and the dense tensors they came from."""
    r = synth.rng(seed)
    need = [-(-L // bs) for L in lens]
    NB = sum(need) + extra
    order = r.permutation(NB)
    g = torch.Generator().manual_seed(seed)
    kd = [torch.randn(L, Hkv, D, generator=g, dtype=torch.float64).to(dtype) for L in lens]
    vd = [torch.randn(L, Hkv, D, generator=g, dtype=torch.float64).to(dtype) for L in lens]
    q = torch.randn(len(lens), Hq, D, generator=g, dtype=torch.float64).to(dtype)
    kc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=dtype)
    vc = torch.full((NB, Hkv, bs, D), float("nan"), dtype=dtype)
    tables = np.full((len(lens), max(need + [1])), -1, np.int32)
    pos = 0
    for b, L in enumerate(lens):
        for j in range(need[b]):
            blk = int(order[pos])
            pos += 1
            tables[b, j] = blk
            n = min(bs, L - j * bs)
            kc[blk, :, :n, :] = kd[b][j * bs:j * bs + n].transpose(0, 1)
            vc[blk, :, :n, :] = vd[b][j * bs:j * bs + n].transpose(0, 1)
    return q, kc, vc, tables, np.array(lens, np.int32), kd, vd


def _torch_dense_attention(q, kd, vd, scale):
    """softmax(scale q K^T) V per sequence with torch in float64; query head h
    uses KV head h // G (repeat_interleave over contiguous groups)."""
    B, Hq, D = q.shape
    out = torch.zeros(B, Hq, D, dtype=torch.float64)
    for b in range(B):
        if kd[b].shape[0] == 0:
            continue
        Hkv = kd[b].shape[1]
        K = kd[b].double().repeat_interleave(Hq // Hkv, dim=1).transpose(0, 1)  # [Hq, L, D]
        V = vd[b].double().repeat_interleave(Hq // Hkv, dim=1).transpose(0, 1)
        s = torch.einsum("hd,hld->hl", q[b].double(), K) * scale
        out[b] = torch.einsum("hl,hld->hd", torch.softmax(s, dim=-1), V)
    return out.numpy()


def test_block_table_example_matches_dense():
    """Logical blocks 0, 1, 2 in physical blocks 8, 3, 11 ("The Block Table
    Map"): paged attention equals dense attention over the contiguous rows."""
    bs, Hkv, D, L = 16, 2, 64, 48
    g = torch.Generator().manual_seed(11)
    kd = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64)
    vd = torch.randn(L, Hkv, D, generator=g, dtype=torch.float64)
    q = torch.randn(1, 2, D, generator=g, dtype=torch.float64)
    kc = torch.full((12, Hkv, bs, D), float("nan"), dtype=torch.float64)
    vc = kc.clone()
    for j, blk in enumerate((8, 3, 11)):
        kc[blk] = kd[j * bs:(j + 1) * bs].transpose(0, 1)
        vc[blk] = vd[j * bs:(j + 1) * bs].transpose(0, 1)
    out = oracle.decode(q, kc, vc, [[8, 3, 11]], [L], 0.125)
    ref = _torch_dense_attention(q, [kd], [vd], 0.125)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_paged_equals_dense_gqa(seed):
    lens = [1, 5, 16, 17, 40, 0, 63]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(seed, lens, Hq=8, Hkv=2, D=16, bs=4)
    out = oracle.decode(q, kc, vc, tables, lens_a, 0.3)
    ref = _torch_dense_attention(q, kd, vd, 0.3)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_permutation_invariance_exact():
    """Two placements of the same logical content give bit-identical results:
    the oracle sums in logical order whatever the physical order."""
    lens = [7, 33, 20]
    outs = []
    for seed in (5, 6, 7):
        g = torch.Generator().manual_seed(99)  # same dense content every time
        bs, Hkv, D = 8, 1, 8
        kd = [torch.randn(L, Hkv, D, generator=g, dtype=torch.float64) for L in lens]
        vd = [torch.randn(L, Hkv, D, generator=g, dtype=torch.float64) for L in lens]
        q = torch.randn(3, 2, D, generator=g, dtype=torch.float64)
        need = [-(-L // bs) for L in lens]
        NB = sum(need) + 4
        order = synth.rng(seed).permutation(NB)
        kc = torch.zeros(NB, Hkv, bs, D, dtype=torch.float64)
        vc = torch.zeros_like(kc)
        tables = np.full((3, max(need)), -1, np.int32)
        pos = 0
        for b, L in enumerate(lens):
            for j in range(need[b]):
                blk = int(order[pos]); pos += 1
                tables[b, j] = blk
                n = min(bs, L - j * bs)
                kc[blk, :, :n] = kd[b][j * bs:j * bs + n].transpose(0, 1)
                vc[blk, :, :n] = vd[b][j * bs:j * bs + n].transpose(0, 1)
        outs.append(oracle.decode(q, kc, vc, tables, lens, 0.7))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_bruteforce_with_allocator_slots():
    """The C table walk equals pure-Python loops over the slots the allocator
    model handed out as the tokens were appended (no table involved)."""
    bs, Hkv, Hq, D, NB = 4, 2, 4, 8, 24
    order = synth.rng(21).permutation(NB)
    A = oracle.AllocatorModel(NB, bs, order)
    lens = [1, 6, 9, 12]
    slot_lists = []
    for L in lens:
        sid = A.new_seq()
        slots = []
        for _ in range(L):  # one token at a time, as decoding grows it
            s, cow = A.append(sid, 1)
            assert cow is None
            slots += s
        slot_lists.append(slots)
    g = torch.Generator().manual_seed(4)
    kc = torch.randn(NB, Hkv, bs, D, generator=g, dtype=torch.float32)
    vc = torch.randn(NB, Hkv, bs, D, generator=g, dtype=torch.float32)
    q = torch.randn(len(lens), Hq, D, generator=g, dtype=torch.float32)
    mb = max(len(A.block_table(s)) for s in range(len(lens)))
    tables = np.full((len(lens), mb), -1, np.int32)
    for s in range(len(lens)):
        t = A.block_table(s)
        tables[s, :len(t)] = t
    out = oracle.decode(q, kc, vc, tables, lens, 0.5)
    ref = oracle.decode_bruteforce(q, kc, vc, slot_lists, 0.5)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_context_of_one_returns_that_value_row():
    q, kc, vc, tables, lens, kd, vd = _dense_case(1, [1, 1], Hq=2, Hkv=1, D=32, bs=16)
    out = oracle.decode(q, kc, vc, tables, lens, 3.0)
    for b in range(2):
        for h in range(2):
            assert np.array_equal(out[b, h], vd[b][0, 0].numpy())


def test_zero_scale_gives_mean_of_values():
    lens = [5, 37]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(2, lens, Hq=2, Hkv=2, D=8, bs=8)
    out = oracle.decode(q, kc, vc, tables, lens_a, 0.0)
    for b in range(2):
        mean = vd[b].numpy().mean(axis=0)  # [Hkv, D]
        np.testing.assert_allclose(out[b], mean, rtol=0, atol=1e-14)


def test_equal_keys_give_mean_of_values():
    lens = [9]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(3, lens, Hq=1, Hkv=1, D=8, bs=4)
    for j in range(tables.shape[1]):
        kc[tables[0, j]] = 0.25  # every key the same vector
    out = oracle.decode(q, kc, vc, tables, lens_a, 1.0)
    np.testing.assert_allclose(out[0, 0], vd[0][:, 0].numpy().mean(axis=0), rtol=0, atol=1e-14)


def test_dominant_key_selects_its_value():
    """One logit at least 50 above all others: the weight of every other row
    is below e^-50, so the output is that row's value vector."""
    lens = [40]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(4, lens, Hq=1, Hkv=1, D=8, bs=8)
    q[:] = 0
    q[0, 0, 0] = 1.0
    for j in range(tables.shape[1]):
        kc[tables[0, j], :, :, 0] = 0.0
    hot = 29
    kc[tables[0, hot // 8], 0, hot % 8, 0] = 60.0
    out = oracle.decode(q, kc, vc, tables, lens_a, 1.0)
    np.testing.assert_allclose(out[0, 0], vd[0][hot, 0].numpy(), rtol=0, atol=1e-20 + 1e-12)


def test_empty_context_gives_zeros():
    q, kc, vc, tables, lens, kd, vd = _dense_case(5, [0, 3], Hq=2, Hkv=1, D=4, bs=4)
    out = oracle.decode(q, kc, vc, tables, lens, 1.0)
    assert np.array_equal(out[0], np.zeros((2, 4)))


def test_softmax_shift_and_scale():
    """Adding a constant to every key logit leaves the output unchanged; with
    D=1 and q=1 that is a constant shift of the keys (exact in closed form)."""
    lens = [12]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(6, lens, Hq=1, Hkv=1, D=1, bs=4)
    q[:] = 1.0
    base = oracle.decode(q, kc, vc, tables, lens_a, 1.0)
    for j in range(tables.shape[1]):
        kc[tables[0, j]] += 7.0
    shifted = oracle.decode(q, kc, vc, tables, lens_a, 1.0)
    np.testing.assert_allclose(base, shifted, rtol=1e-13, atol=0)


def test_bf16_widening_known_patterns():
    pats = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x4049], dtype=np.uint16)
    vals = oracle.widen(pats)
    assert vals.tolist() == [1.0, -2.0, 1.0078125, 0.0, -0.0, 3.140625]


def test_bf16_inputs_match_widened_f64():
    case = synth.random_case(8, B=3, Hq=4, Hkv=2, D=16, bs=8, lens=[3, 20, 31], dtype=torch.bfloat16)
    out_bf = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    out_64 = oracle.decode(oracle.widen(case.q), oracle.widen(case.k_cache), oracle.widen(case.v_cache),
                           case.block_tables, case.context_lens, case.scale)
    assert np.array_equal(out_bf, out_64)


@pytest.mark.parametrize("part", [1, 4, 16, 32, 1000])
def test_partitioned_merge_equals_single_pass(part):
    """The split-context form (per-partition max/sum/accumulator, merged by a
    log-sum-exp combine) is an identity: it equals the one-pass softmax."""
    lens = [1, 16, 17, 64, 100, 0]
    q, kc, vc, tables, lens_a, kd, vd = _dense_case(7, lens, Hq=4, Hkv=2, D=8, bs=4)
    m, l, acc, np_ = oracle.decode_partials(q, kc, vc, tables, lens_a, 0.9, part)
    merged = oracle.merge_partials(m, l, acc, np_)
    full = oracle.decode(q, kc, vc, tables, lens_a, 0.9)
    np.testing.assert_allclose(merged, full, rtol=0, atol=1e-12)
    assert np_.tolist() == [-(-L // part) for L in lens]
    # each partition's statistics are those of its own tokens' logits,
    # recomputed here from the dense rows with torch
    G = 4 // 2
    for b, L in enumerate(lens):
        for h in range(4):
            s = (kd[b][:, h // G, :].double() @ q[b, h].double()).numpy() * 0.9
            for p in range(np_[b]):
                seg = s[p * part:(p + 1) * part]
                assert m[b, h, p] == pytest.approx(seg.max(), abs=1e-13)
                assert l[b, h, p] == pytest.approx(np.exp(seg - seg.max()).sum(), rel=1e-13)
                w = np.exp(seg - seg.max())
                ref_acc = w @ vd[b][p * part:(p + 1) * part, h // G, :].double().numpy()
                np.testing.assert_allclose(acc[b, h, p], ref_acc, rtol=0, atol=1e-12)


def test_rows_subset_matches_full():
    case = synth.tiny_fp32_case(0)
    full = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    rows = [(3, 1), (0, 0), (2, 1)]
    sub = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale, rows=rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(sub[i], full[b, h])


def test_bad_table_entry_rejected():
    case = synth.tiny_fp32_case(0)
    t = case.block_tables.copy()
    t[3, 0] = 999
    with pytest.raises(ValueError):
        oracle.decode(case.q, case.k_cache, case.v_cache, t, case.context_lens, case.scale)


def test_tiny_case_reads_no_unowned_block():
    """Unowned pool blocks hold NaN; a finite output shows the walk never
    touched them."""
    case = synth.tiny_fp32_case(0)
    out = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert np.isfinite(out).all()


# ------------------------------------------------------------- prefill


def _torch_dense_causal(qrows, kd, vd, starts, lens, scale):
    """For every sequence b, its last n_b tokens' queries against its dense
    keys with a causal mask (query i of the chunk sees keys 0 .. L - n + i),
    softmax and weighted values by torch in float64."""
    outs = []
    for b in range(len(lens)):
        L, n = int(lens[b]), int(starts[b + 1] - starts[b])
        if n == 0:
            continue
        Q = qrows[starts[b]:starts[b + 1]].double()                    # [n, Hq, D]
        Hq, Hkv = Q.shape[1], kd[b].shape[1]
        K = kd[b].double().repeat_interleave(Hq // Hkv, dim=1)           # [L, Hq, D]
        V = vd[b].double().repeat_interleave(Hq // Hkv, dim=1)
        s = torch.einsum("ihd,thd->hit", Q, K) * scale                   # [Hq, n, L]
        pos = torch.arange(L - n, L).view(1, n, 1)
        s = s.masked_fill(torch.arange(L).view(1, 1, L) > pos, float("-inf"))
        outs.append(torch.einsum("hit,thd->ihd", torch.softmax(s, dim=-1), V))
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_prefill_equals_dense_causal(seed):
    """Chunks of new tokens (a whole prompt, a chunk after a cached prefix, a
    single token, none) against torch's masked softmax over the dense keys."""
    lens = [40, 17, 70, 9]
    news = [40, 5, 33, 0]
    q0, kc, vc, tables, lens_a, kd, vd = _dense_case(seed, lens, Hq=6, Hkv=2, D=16, bs=4)
    starts = np.concatenate([[0], np.cumsum(news)]).astype(np.int32)
    g = torch.Generator().manual_seed(100 + seed)
    qrows = torch.randn(int(starts[-1]), 6, 16, generator=g, dtype=torch.float64)
    out = oracle.prefill(qrows, kc, vc, tables, lens_a, starts, 0.4)
    ref = _torch_dense_causal(qrows, kd, vd, starts, lens_a, 0.4)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_prefill_is_causal():
    """Changing the keys and values after a new token's position changes
    nothing for it, and changes the tokens that see them."""
    lens = [30]
    q0, kc, vc, tables, lens_a, kd, vd = _dense_case(3, lens, Hq=2, Hkv=1, D=8, bs=4)
    starts = np.array([0, 12], np.int32)  # positions 18 .. 29 are new
    qrows = torch.randn(12, 2, 8, generator=torch.Generator().manual_seed(7), dtype=torch.float64)
    before = oracle.prefill(qrows, kc, vc, tables, lens_a, starts, 0.5)
    blk, off = int(tables[0, 25 // 4]), 25 % 4  # token 25
    kc[blk, :, off] += 3.0
    vc[blk, :, off] -= 2.0
    after = oracle.prefill(qrows, kc, vc, tables, lens_a, starts, 0.5)
    np.testing.assert_array_equal(before[:25 - 18], after[:25 - 18])
    assert np.abs(before[25 - 18:] - after[25 - 18:]).min() > 0


def test_prefill_last_token_is_bruteforce_decode():
    """The chunk's last token sees the whole context: the pure-Python loop
    over the allocator's slots (no table) gives the same row."""
    bs, Hkv, Hq, D, NB = 4, 2, 4, 8, 24
    A = oracle.AllocatorModel(NB, bs, synth.rng(31).permutation(NB))
    lens = [9, 14]
    slot_lists = []
    for L in lens:
        sid = A.new_seq()
        slots, cow = A.append(sid, L)
        assert cow is None
        slot_lists.append(slots)
    g = torch.Generator().manual_seed(32)
    kc = torch.randn(NB, Hkv, bs, D, generator=g, dtype=torch.float64)
    vc = torch.randn(NB, Hkv, bs, D, generator=g, dtype=torch.float64)
    news = [3, 14]
    starts = np.array([0, 3, 17], np.int32)
    qrows = torch.randn(17, Hq, D, generator=g, dtype=torch.float64)
    tables = np.full((2, 4), -1, np.int32)
    for s in range(2):
        t = A.block_table(s)
        tables[s, :len(t)] = t
    out = oracle.prefill(qrows, kc, vc, tables, lens, starts, 0.6)
    for b in range(2):
        last = int(starts[b + 1]) - 1
        ref = oracle.decode_bruteforce(qrows[last:last + 1], kc, vc, [slot_lists[b]], 0.6)
        np.testing.assert_allclose(out[last], ref[0], rtol=0, atol=1e-12)
        # and the chunk's first token sees only the tokens up to its position
        first = int(starts[b])
        p = lens[b] - news[b]
        ref = oracle.decode_bruteforce(qrows[first:first + 1], kc, vc, [slot_lists[b][:p + 1]], 0.6)
        np.testing.assert_allclose(out[first], ref[0], rtol=0, atol=1e-12)

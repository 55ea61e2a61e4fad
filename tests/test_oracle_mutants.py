"""Plants plausible mistakes in the oracle and checks that the pins catch
every one (no GPU; nothing here touches the product path).

Each mutant is one small edit: in a copy of the C attention oracle (a wrong
index, a dropped term, a flipped sign, a transposed layout, a wrong head
mapping), or in one Python function or method of the oracle, swapped in for
the test (the append and the block copy, the allocator model, the usage and
fragmentation measures).  The pins of test_oracle_pins and
test_oracle_allocator must fail on each, or the pins are too weak.
"""
import ctypes
import inspect
import os
import subprocess
import textwrap

import numpy as np
import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

MUTANTS = {
    "offset-index": ("int off = t % bs;", "int off = (t / bs) % bs;"),
    "dropped-scale": ("s[t] = scale * dot;", "s[t] = dot;"),
    "flipped-exponent": ("double p = exp(s[t] - m);", "double p = exp(m - s[t]);"),
    "head-mapping": ("int g = h / G;\n  int n = lens[b];", "int g = h % Hkv;\n  int n = lens[b];"),
    "dropped-normalisation": ("for (int d = 0; d < D; ++d) out_row[d] /= denom;", ""),
    "transposed-layout": ("return ((blk * Hkv + g) * bs + off) * (int64_t)D;",
                          "return ((blk * bs + off) * Hkv + g) * (int64_t)D;"),
    "merge-missing-rescale": ("L += l[i * max_parts + p] * w;", "L += l[i * max_parts + p];"),
    "partial-max-skipped": ("if (s[t - t0] > m) m = s[t - t0];", "m = 0.0;"),
    "prefill-causal-limit": ("for (int t = 0; t <= p; ++t) {\n      int64_t kr", "for (int t = 0; t < p; ++t) {\n      int64_t kr"),
    "prefill-dropped-scale": ("s[t] = dot * scale;", "s[t] = dot;"),
    "prefill-no-prefix": ("const int p = lens[b] - n + (int)(j - qstart[b]);", "const int p = (int)(j - qstart[b]);"),
    "prefill-query-row": ("const int64_t qoff = (j * Hq + h) * D;", "const int64_t qoff = ((int64_t)b * Hq + h) * D;"),
    "bf16-wrong-half": ("uint32_t u = ((uint32_t)((const uint16_t *)base)[i]) << 16;",
                        "uint32_t u = ((uint32_t)((const uint16_t *)base)[i]);"),
}

PIN_TESTS = [
    pins.test_block_table_example_matches_dense,
    lambda: [pins.test_paged_equals_dense_gqa(s) for s in (0, 1)],
    pins.test_bruteforce_with_allocator_slots,
    pins.test_zero_scale_gives_mean_of_values,
    pins.test_dominant_key_selects_its_value,
    lambda: [pins.test_partitioned_merge_equals_single_pass(p) for p in (4, 16)],
    pins.test_bf16_inputs_match_widened_f64,
    lambda: [pins.test_prefill_equals_dense_causal(s) for s in (0, 1)],
    pins.test_prefill_is_causal,
    pins.test_prefill_last_token_is_bruteforce_decode,
]


def _usage_per_sharer(self):
    """A plausible mistake: every table's blocks counted, so a block shared
    by k sequences is held k times and its tokens used k times."""
    bs = self.block_size
    return oracle.Usage(allocated=bs * sum(len(t) for t in self.tables.values()), used=sum(self.lens.values()))


def _usage_tokens_per_sharer(self):
    """A plausible mistake: physical blocks counted once, but every
    sequence's tokens counted, so shared tokens are used several times."""
    bs = self.block_size
    blocks = {b for t in self.tables.values() for b in t}
    return oracle.Usage(allocated=bs * len(blocks), used=sum(self.lens.values()))


USAGE_MUTANTS = {"usage-per-sharer": _usage_per_sharer, "usage-tokens-per-sharer": _usage_tokens_per_sharer}


def _usage_pins():
    from tests import test_oracle_allocator as alloc_pins
    return [alloc_pins.test_usage_reproduces_the_paged_worked_example,
            alloc_pins.test_usage_of_a_shared_partial_block_by_hand,
            alloc_pins.test_usage_of_full_shared_blocks_by_hand]


def _append_transposed_offset(k_cache, v_cache, k, v, slot_mapping):
    """A plausible mistake: block and row of a slot swapped."""
    ka, _ = oracle.host_array(k)
    va, _ = oracle.host_array(v)
    bs = k_cache.shape[2]
    for i, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s >= 0:
            off, blk = divmod(s, bs)
            k_cache[blk, :, off, :] = ka[i]
            v_cache[blk, :, off, :] = va[i]


def _append_padding_written(k_cache, v_cache, k, v, slot_mapping):
    """A plausible mistake: a negative (padding) slot is not skipped and
    lands, by negative indexing, in the last block."""
    ka, _ = oracle.host_array(k)
    va, _ = oracle.host_array(v)
    NB, bs = k_cache.shape[0], k_cache.shape[2]
    for i, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s >= NB * bs:
            raise IndexError(s)
        blk, off = divmod(s, bs)
        k_cache[blk, :, off, :] = ka[i]
        v_cache[blk, :, off, :] = va[i]


def _append_key_as_value(k_cache, v_cache, k, v, slot_mapping):
    """A plausible mistake: the key row written into both caches."""
    ka, _ = oracle.host_array(k)
    bs = k_cache.shape[2]
    for i, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s >= 0:
            blk, off = divmod(s, bs)
            if blk >= k_cache.shape[0]:
                raise IndexError(s)
            k_cache[blk, :, off, :] = ka[i]
            v_cache[blk, :, off, :] = ka[i]


def _copy_reversed(k_cache, v_cache, pairs):
    """A plausible mistake: the pair read as (dst, src)."""
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        k_cache[src] = k_cache[dst]
        v_cache[src] = v_cache[dst]


def _copy_keys_only(k_cache, v_cache, pairs):
    """A plausible mistake: the value block left behind."""
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        k_cache[dst] = k_cache[src]


APPEND_COPY_MUTANTS = {
    "append-transposed-offset": ("append_kv", _append_transposed_offset),
    "append-padding-written": ("append_kv", _append_padding_written),
    "append-key-as-value": ("append_kv", _append_key_as_value),
    "copy-reversed": ("copy_blocks", _copy_reversed),
    "copy-keys-only": ("copy_blocks", _copy_keys_only),
}


def _append_copy_pins():
    from tests import test_oracle_allocator as alloc_pins
    return [alloc_pins.test_append_and_copy_bit_exact_and_padding_skipped]


@pytest.mark.parametrize("name", sorted(APPEND_COPY_MUTANTS))
def test_append_copy_mutant_is_caught(name, monkeypatch):
    for t in _append_copy_pins():
        t()  # the oracle as it stands passes every pin
    attr, fn = APPEND_COPY_MUTANTS[name]
    monkeypatch.setattr(oracle, attr, fn)
    caught = 0
    for t in _append_copy_pins():
        try:
            t()
        except (AssertionError, IndexError):
            caught += 1
    assert caught > 0, f"no pin fails on mutant {name}"


# Mistakes planted in one method of the allocator model: (method, the
# original text, its replacement).
ALLOCATOR_MUTANTS = {
    "fork-takes-no-reference": ("fork", "self.ref[blk] += 1", "pass"),
    "free-list-fifo": ("free_seq", "self.free.append(blk)", "self.free.insert(0, blk)"),
    "copy-keeps-reference": ("batch_append", "self.ref[last] -= 1", "pass"),
    "copy-unshared-block": ("batch_append", "if self.ref[last] > 1:", "if self.ref[last] >= 1:"),
    "copy-pair-reversed": ("batch_append", "cows.append((last, new))", "cows.append((new, last))"),
    "slot-drops-offset": ("batch_append", "slots.append(table[pos // bs] * bs + pos % bs)",
                          "slots.append(table[pos // bs] * bs)"),
    "need-ignores-copies": ("_blocks_needed", "need += 1", "pass"),
    "need-counts-every-sharer": ("_blocks_needed", "self.ref[last] - ref_taken.get(last, 0) > 1",
                                 "self.ref[last] > 1"),
}


def _mutated_method(name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(oracle.AllocatorModel, name)))
    assert src.count(old) == 1, f"mutation site in {name} not unique"
    ns = {}
    exec(src.replace(old, new), vars(oracle), ns)
    return ns[name]


def _allocator_pins():
    from tests import test_oracle_allocator as alloc_pins
    return [getattr(alloc_pins, n) for n in sorted(dir(alloc_pins))
            if n.startswith("test_") and not inspect.signature(getattr(alloc_pins, n)).parameters]


@pytest.mark.parametrize("name", sorted(ALLOCATOR_MUTANTS))
def test_allocator_mutant_is_caught(name, monkeypatch):
    for t in _allocator_pins():
        t()  # the model as it stands passes every pin
    method, old, new = ALLOCATOR_MUTANTS[name]
    monkeypatch.setattr(oracle.AllocatorModel, method, _mutated_method(method, old, new))
    caught = 0
    for t in _allocator_pins():
        try:
            t()
        except (AssertionError, IndexError, oracle.OutOfBlocks, pytest.fail.Exception):
            caught += 1
    assert caught > 0, f"no pin fails on mutant {name}"


# Mistakes planted in the fragmentation measures (learn-ml-visualized,
# fragmentation worked example): (function, original text, replacement).
FRAGMENTATION_MUTANTS = {
    "paged-rounds-down": ("paged_usage", "-(-L // page_size)", "L // page_size"),
    "paged-extra-page": ("paged_usage", "-(-L // page_size)", "L // page_size + 1"),
    "naive-one-reservation": ("naive_usage", "allocated=reserve * len(lengths)", "allocated=reserve"),
    "naive-reserves-the-longest": ("naive_usage", "allocated=reserve * len(lengths)",
                                   "allocated=max(lengths) * len(lengths)"),
}


def _mutated_function(name, old, new):
    src = inspect.getsource(getattr(oracle, name))
    assert src.count(old) == 1, f"mutation site in {name} not unique"
    ns = {}
    exec(src.replace(old, new), vars(oracle), ns)
    return ns[name]


def _fragmentation_pins():
    return ([lambda c=c: pins.test_fragmentation_golden(c) for c in pins._golden("fragmentation.json")["cases"]]
            + [pins.test_naive_rejects_overlong, pins.test_paged_waste_under_one_page_any_length])


@pytest.mark.parametrize("name", sorted(FRAGMENTATION_MUTANTS) + ["waste-over-used"])
def test_fragmentation_mutant_is_caught(name, monkeypatch):
    for t in _fragmentation_pins():
        t()  # the measures as they stand pass every pin
    if name == "waste-over-used":
        # the fraction taken over the slots used instead of those allocated
        monkeypatch.setattr(oracle.Usage, "fragmentation", property(lambda u: u.wasted / u.used))
    else:
        fn, old, new = FRAGMENTATION_MUTANTS[name]
        monkeypatch.setattr(oracle, fn, _mutated_function(fn, old, new))
    caught = 0
    for t in _fragmentation_pins():
        try:
            t()
        except (AssertionError, pytest.fail.Exception):
            caught += 1
    assert caught > 0, f"no pin fails on mutant {name}"


@pytest.mark.parametrize("name", sorted(USAGE_MUTANTS))
def test_usage_mutant_is_caught(name, monkeypatch):
    for t in _usage_pins():
        t()  # the model as it stands passes every pin
    monkeypatch.setattr(oracle.AllocatorModel, "usage", USAGE_MUTANTS[name])
    caught = 0
    for t in _usage_pins():
        try:
            t()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin fails on mutant {name}"


def _build_mutant(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / f"m_{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"m_{name}.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", str(path), "-o", str(so), "-lm"], check=True)
    return str(so)


def test_original_passes_all_pins():
    for t in PIN_TESTS:
        t()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name, monkeypatch):
    old, new = MUTANTS[name]
    so = _build_mutant(tmp_path, name, old, new)
    monkeypatch.setattr(oracle, "_lib", oracle.load(so))
    caught = 0
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, f"no pin fails on mutant {name}"

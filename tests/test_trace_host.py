"""The continuous-batching trace driver on the host (no GPU): the C++
allocator and the oracle's allocator model, driven by the same draws, make
identical plans step after step (same sequence ids, slots, copy pairs), and
the allocator's invariants hold throughout (paged waste under one block per
sequence, blocks conserved)."""
import numpy as np
import pytest

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth
from paged_kv_cache_402_b200.trace import BeamTrace


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_trace_plans_match_model(bs):
    NB = 6000
    order = synth.rng(30 + bs).permutation(NB)
    A = pa.Allocator(NB, bs, order)
    M = oracle.AllocatorModel(NB, bs, order)
    draws = synth.trace(31, steps=150, mean_arrivals=1.0, prompt_median=64, prompt_max=512,
                        output_mean=20, max_groups=256)
    ta = BeamTrace(A, lambda: A.stats()["free_blocks"], bs, draws)
    tm = BeamTrace(M, lambda: len(M.free), bs, draws)
    total_cow = 0
    for step in range(150):
        pa_ = ta.step()
        pm = tm.step()
        assert pa_.prompt_seqs == pm.prompt_seqs
        assert pa_.decode_seqs == pm.decode_seqs
        assert np.array_equal(pa_.prompt_slots, pm.prompt_slots)
        assert np.array_equal(pa_.decode_slots, pm.decode_slots)
        assert np.array_equal(pa_.cow_pairs, pm.cow_pairs)
        assert pa.pa_check_copy_pairs(pa_.cow_pairs, NB)
        total_cow += len(pa_.cow_pairs)
        st = A.stats()
        assert st["free_blocks"] == len(M.free)
        assert st["used_slots"] == M.usage().used
        for s in pa_.decode_seqs:
            assert M.seq_waste(s) < bs
    assert total_cow > 0  # beams of a fresh group share a partial prompt block
    assert len(ta.running) > 0

"""The whole path under continuous batching, step by step, against the oracle.

A short seeded trace of beam-search requests (Poisson arrivals, lognormal
prompts, geometric outputs, beams re-forked copy-on-write) drives the C++
allocator and the oracle's allocator model in lockstep.  Every step the device
runs the copy-on-write block copies, the prompt and decode appends and the
decode of every running beam; the oracle does the same on a host pool.  The
pools must match bit for bit (checked every few steps, and at the end), and
sampled decode rows within the bf16 tolerance, every step."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth
from paged_kv_cache_402_b200.trace import BeamTrace

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_trace_step_by_step(cuda_device, bs):
    dev = cuda_device
    Hq, Hkv, D, NB, steps = 32, 8, 128, 3000, 36
    dt = torch.bfloat16
    order = synth.rng(60 + bs).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    draws = synth.trace(61 + bs, steps=steps, mean_arrivals=1.2, prompt_median=80, prompt_max=300,
                        output_mean=10, max_groups=512)
    ta = BeamTrace(A, lambda: A.stats()["free_blocks"], bs, draws)
    tm = BeamTrace(M, lambda: len(M.free), bs, draws)
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    cache = pa.KVCache(k0.to(dev), v0.to(dev))
    hk = oracle.host_array(k0)[0].copy()
    hv = oracle.host_array(v0)[0].copy()
    scale = 1 / math.sqrt(D)
    r = synth.rng(62 + bs)
    checked = 0
    for s in range(steps):
        pa_, pm = ta.step(), tm.step()
        assert pa_.decode_seqs == pm.decode_seqs
        assert np.array_equal(pa_.prompt_slots, pm.prompt_slots)
        assert np.array_equal(pa_.decode_slots, pm.decode_slots)
        assert np.array_equal(pa_.cow_pairs, pm.cow_pairs)
        n_prompt, n_dec = len(pa_.prompt_slots), len(pa_.decode_slots)
        if n_prompt:  # prompt rows: written before the decode tokens
            kp = synth.normal((n_prompt, Hkv, D), dt, 1000 * s + 1)
            vp = synth.normal((n_prompt, Hkv, D), dt, 1000 * s + 2)
            pa.pa_append_kv(kp.to(dev), vp.to(dev), torch.from_numpy(pa_.prompt_slots).to(dev), cache)
            oracle.append_kv(hk, hv, kp, vp, pm.prompt_slots)
        if n_dec == 0:
            continue
        if len(pa_.cow_pairs):
            pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(pa_.cow_pairs)).to(dev), cache)
            oracle.copy_blocks(hk, hv, pm.cow_pairs)
        kd = synth.normal((n_dec, Hkv, D), dt, 1000 * s + 3)
        vd = synth.normal((n_dec, Hkv, D), dt, 1000 * s + 4)
        pa.pa_append_kv(kd.to(dev), vd.to(dev), torch.from_numpy(pa_.decode_slots).to(dev), cache)
        oracle.append_kv(hk, hv, kd, vd, pm.decode_slots)
        mb = max(len(M.block_table(q)) for q in pm.decode_seqs)
        tables, lens = A.build_block_tables(pa_.decode_seqs, mb)
        q = synth.normal((n_dec, Hq, D), dt, 1000 * s + 5)
        out = pa.pa_decode(q.to(dev), cache, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                           int(lens.max()), scale)
        assert pa.pa_read_device_error() == 0
        rows = [(int(b), int(h)) for b, h in zip(r.integers(0, n_dec, 12), r.integers(0, Hq, 12))]
        mt = np.full((n_dec, mb), -1, np.int32)
        for i, sq in enumerate(pm.decode_seqs):
            t = M.block_table(sq)
            mt[i, :len(t)] = t
        assert np.array_equal(mt, tables)
        ref = oracle.decode(q, hk, hv, mt, np.array([M.lens[sq] for sq in pm.decode_seqs], np.int32), scale, rows=rows)
        got = out.float().cpu().double().numpy()
        for i, (b, h) in enumerate(rows):
            assert (np.abs(got[b, h] - ref[i]) <= 2e-2 + 1e-2 * np.abs(ref[i])).all(), f"step {s} row {(b, h)}"
        checked += len(rows)
        if s % 8 == 7 or s == steps - 1:
            gk = oracle.host_array(cache.k.cpu())[0]
            gv = oracle.host_array(cache.v.cpu())[0]
            assert np.array_equal(gk, hk) and np.array_equal(gv, hv), f"pools differ after step {s}"
    assert checked > 0 and len(ta.running) > 0


@pytest.mark.parametrize("bs,part", [(8, 512), (16, 512), (32, 512), (16, 1024), (16, 256)])
def test_trace_measured_step(cuda_device, bs, part):
    """The trace step exactly as the benchmark times it, step by step against
    the oracle: the prompts' rows through pa_append_kv, then one
    pa_decode_shared call per step with the sharing plan (pa_share_plan) of
    the running beams, their copy-on-write sources (pa_cow_sources) and
    their decode tokens' rows.  Beams of one request share the prompt's
    blocks and are copied when they write ("pagedattention" glossary entry,
    paragraph 5); beams whose prompts hold enough full blocks make the
    plan's groups.  Every decode row of every step is checked against the
    oracle, the pools bit for bit every 4 steps and at the end.  The
    partition sizes the trace sweep compares at 16-token blocks run too
    (1024: the sweep's choice on the full trace)."""
    dev = cuda_device
    Hq, Hkv, D, steps = 32, 8, 128, 40
    NB = 65536 // bs
    dt = torch.bfloat16
    order = synth.rng(70 + bs).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    draws = synth.trace(71 + bs, steps=steps, mean_arrivals=0.8, prompt_median=700, prompt_max=2000,
                        output_mean=14, max_groups=512)
    ta = BeamTrace(A, lambda: A.stats()["free_blocks"], bs, draws)
    tm = BeamTrace(M, lambda: len(M.free), bs, draws)
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    cache = pa.KVCache(k0.to(dev), v0.to(dev), partition_tokens=part)
    hk = oracle.host_array(k0)[0].copy()
    hv = oracle.host_array(v0)[0].copy()
    scale = 1 / math.sqrt(D)
    grouped_steps = copy_steps = rows_checked = 0
    for s in range(steps):
        pa_, pm = ta.step(), tm.step()
        assert pa_.decode_seqs == pm.decode_seqs
        assert np.array_equal(pa_.prompt_slots, pm.prompt_slots)
        assert np.array_equal(pa_.decode_slots, pm.decode_slots)
        assert np.array_equal(pa_.cow_pairs, pm.cow_pairs)
        n_prompt, n = len(pa_.prompt_slots), len(pa_.decode_seqs)
        if n_prompt:
            kp = synth.normal((n_prompt, Hkv, D), dt, 1000 * s + 1)
            vp = synth.normal((n_prompt, Hkv, D), dt, 1000 * s + 2)
            pa.pa_append_kv(kp.to(dev), vp.to(dev), torch.from_numpy(pa_.prompt_slots).to(dev), cache)
            oracle.append_kv(hk, hv, kp, vp, pm.prompt_slots)
        if n == 0:
            continue
        max_ctx, mb = A.max_len(pa_.decode_seqs)
        tables, lens = A.build_block_tables(pa_.decode_seqs, mb)
        plan = pa.share_plan(tables, lens, bs).to(dev)
        has_pairs = len(pa_.cow_pairs) > 0
        cow = pa.cow_sources(pa_.cow_pairs, tables, lens, bs) if has_pairs else None
        kd = synth.normal((n, Hkv, D), dt, 1000 * s + 3)
        vd = synth.normal((n, Hkv, D), dt, 1000 * s + 4)
        q = synth.normal((n, Hq, D), dt, 1000 * s + 5)
        out = pa.pa_decode_shared(q.to(dev), cache, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                                  max_ctx, scale, plan=plan, k_new=kd.to(dev), v_new=vd.to(dev),
                                  cow_src=torch.from_numpy(cow).to(dev) if has_pairs else None)
        assert pa.pa_read_device_error() == 0
        grouped_steps += plan.n_groups > 0
        copy_steps += has_pairs
        # the oracle: copies, then the decode tokens' rows, then the decode
        oracle.copy_blocks(hk, hv, pm.cow_pairs)
        oracle.append_kv(hk, hv, kd, vd, pm.decode_slots)
        mt = np.full((n, mb), -1, np.int32)
        for i, sq in enumerate(pm.decode_seqs):
            t = M.block_table(sq)
            mt[i, :len(t)] = t
        ml = np.array([M.lens[sq] for sq in pm.decode_seqs], np.int32)
        assert np.array_equal(mt, tables) and np.array_equal(ml, lens)
        ref = oracle.decode(q, hk, hv, mt, ml, scale)
        got = out.float().cpu().double().numpy()
        bad = np.abs(got - ref) > 2e-2 + 1e-2 * np.abs(ref)
        assert not bad.any(), f"step {s}: {int(bad.sum())} elements out of tolerance"
        rows_checked += n * Hq
        if s % 4 == 3 or s == steps - 1:
            gk = oracle.host_array(cache.k.cpu())[0]
            gv = oracle.host_array(cache.v.cpu())[0]
            assert np.array_equal(gk, hk) and np.array_equal(gv, hv), f"pools differ after step {s}"
    assert grouped_steps > 0, "no step had a sharing plan"
    assert copy_steps > 0, "no step copied on write"
    assert rows_checked > 0

"""pa_decode_step (through pa.DecodeStepper): a whole decode step from pinned
host buffers in one call, against the oracle, several steps in a row with two
alternating step slots.

Every step the library's allocator and the oracle's model append one token
per sequence; the oracle copies on write, appends and decodes on its host
pool.  The output the step copies back to pinned host memory must be within
the bf16 bound |gpu - ref| <= 2e-2 + 1e-2 |ref| (fp32: max-abs 1e-5), the
pool bit for bit at the end.  The batch shares prompt blocks (forks of a
root whose prompt ends inside a block, so the first step copies on write),
so the sharing plan has groups over the prompts' full blocks.
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


@pytest.mark.parametrize("dtype,D,G,bs,share", [
    (torch.bfloat16, 128, 4, 16, 4),   # tensor-core path with the cascade plan
    (torch.bfloat16, 128, 8, 8, 2),
    (torch.bfloat16, 128, 2, 32, 0),   # no plan
    (torch.float32, 64, 2, 16, 4),     # CUDA-core path (the plan is not used)
])
def test_decode_step_matches_oracle(cuda_device, dtype, D, G, bs, share):
    dev = cuda_device
    Hkv = 2
    Hq = G * Hkv
    prompts = [1300, 700, 45, 9]
    NB = 4 * 4 * (-(-(max(prompts) + 40) // bs)) + 64
    order = synth.rng(81).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dtype, dev)
    roots = _prefill(A, M, prompts, dev, cache, hk, hv, dtype, 82)
    seqs = _fork_groups(A, M, roots, 4)
    n = len(seqs)
    steps = 7
    mb = max(len(M.block_table(s)) for s in seqs) + steps
    scale = 1 / math.sqrt(D)
    stepper = pa.DecodeStepper(A, cache, n, Hq, mb, scale, share_max_members=share)
    pending = {}
    copies = groups = 0
    for s in range(steps):
        k = stepper.next_slot
        if k in pending:  # the slot's previous step: its output is on the host now
            stepper.wait(k)
            ref, dt_ = pending.pop(k)
            assert_attn_close(stepper.output(k), ref, dt_)
        q_h, k_h, v_h = stepper.inputs()
        q = synth.normal((n, Hq, D), dtype, 90 + 3 * s)
        kn = synth.normal((n, Hkv, D), dtype, 91 + 3 * s)
        vn = synth.normal((n, Hkv, D), dtype, 92 + 3 * s)
        q_h.copy_(q)
        k_h.copy_(kn)
        v_h.copy_(vn)
        info = stepper.step(seqs)
        assert info["slot"] == k
        mslots, mpairs = M.batch_append(seqs, [1] * n)
        assert info["n_copies"] == len(mpairs)
        copies += info["n_copies"]
        groups += info["n_groups"]
        oracle.copy_blocks(hk, hv, mpairs)
        oracle.append_kv(hk, hv, kn, vn, mslots)
        tables = np.full((n, mb), -1, np.int32)
        for i, sq in enumerate(seqs):
            t = M.block_table(sq)
            tables[i, :len(t)] = t
        lens = np.array([M.lens[sq] for sq in seqs], np.int32)
        assert info["max_len"] == int(lens.max())
        pending[k] = (oracle.decode(q, hk, hv, tables, lens, scale), dtype)
    for k, (ref, dt_) in pending.items():
        stepper.wait(k)
        assert_attn_close(stepper.output(k), ref, dt_)
    stepper.close()
    assert pa.pa_read_device_error() == 0
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    assert copies > 0, "no step copied on write"
    if share and dtype == torch.bfloat16:
        assert groups > 0, "no step had a sharing plan"

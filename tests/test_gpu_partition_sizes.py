"""Decode with split-context partitions of 256 and 1024 tokens (the pool's
partition_tokens), against the oracle.

The partition size only changes how a context is cut for the log-sum-exp
reduce and what a sharing plan can share; the result is the same attention
(bf16: |gpu - ref| <= 2e-2 + 1e-2 |ref|, fp32: max-abs 1e-5 against the
float64 oracle).  The workspace statistics per partition are checked against
the oracle's partials of the same partition size.
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

PARTS = [256, 1024]


def _case_dev(case, dev, part):
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev), partition_tokens=part)
    return (cache, case.q.to(dev), torch.from_numpy(case.block_tables).to(dev),
            torch.from_numpy(case.context_lens).to(dev))


@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("dtype,G,D", [(torch.bfloat16, 1, 128), (torch.bfloat16, 4, 128), (torch.bfloat16, 8, 128),
                                       (torch.float32, 4, 128), (torch.bfloat16, 2, 64)])
def test_decode_partition_size(cuda_device, part, dtype, G, D):
    Hkv = 2
    lens = [1, part - 1, part, part + 1, 2 * part + 1, 3000, 129, 4 * part + 7]
    case = synth.random_case(300 + part + G, B=len(lens), Hq=G * Hkv, Hkv=Hkv, D=D, bs=16, lens=lens, dtype=dtype)
    cache, q, tables, lens_d = _case_dev(case, cuda_device, part)
    out = pa.pa_decode(q, cache, tables, lens_d, int(case.context_lens.max()), case.scale)
    assert pa.pa_read_device_error() == 0
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, dtype)


@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_partials_partition_size(cuda_device, part, dtype):
    """The workspace rows: per partition, the normalised partial output
    acc / l and the partition's log-sum-exp m ln 2 + ln l (m is kept in
    base-2 units against a reference that may lag the exact maximum, so the
    pair (m, l) is compared through that invariant)."""
    lens = [part + 300, part + 1, 3 * part - 5]
    B, Hq, Hkv, D = 3, 8, 2, 128
    case = synth.random_case(46 + part, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=16, lens=lens, dtype=dtype)
    cache, q, tables, lens_d = _case_dev(case, cuda_device, part)
    max_ctx = int(case.context_lens.max())
    P = -(-max_ctx // part)
    need = pa.pa_decode_workspace_size(B, Hq, max_ctx, D, part)
    ws = torch.zeros(need, dtype=torch.uint8, device=cuda_device)
    pa.pa_decode(q, cache, tables, lens_d, max_ctx, case.scale, workspace=ws)
    torch.cuda.synchronize()
    assert pa.pa_read_device_error() == 0
    rows = B * Hq * P
    wsf = ws.view(torch.float32).cpu()
    off = (rows * 4 + 15) // 16 * 16 // 4
    gm = wsf[:rows].view(B, Hq, P).double().numpy() * math.log(2.0)
    gl = wsf[off:off + rows].view(B, Hq, P).double().numpy()
    gacc = wsf[2 * off:2 * off + rows * D].view(B, Hq, P, D).double().numpy()
    m, l, acc, np_ = oracle.decode_partials(case.q, case.k_cache, case.v_cache, case.block_tables,
                                            case.context_lens, case.scale, part)
    for b in range(B):
        for p in range(np_[b]):
            np.testing.assert_allclose(gm[b, :, p] + np.log(gl[b, :, p]), m[b, :, p] + np.log(l[b, :, p]),
                                       rtol=0, atol=1e-4)
            got = gacc[b, :, p] / gl[b, :, p][:, None]
            want = acc[b, :, p] / l[b, :, p][:, None]
            if dtype == torch.float32:
                np.testing.assert_allclose(got, want, rtol=0, atol=1e-5)
            else:
                assert (np.abs(got - want) <= 2e-2 + 1e-2 * np.abs(want)).all()


@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("off", [0, 37])
def test_shared_fused_step_partition_size(cuda_device, part, off):
    """Groups of 8 forks share a prompt of several partitions; one fused step
    (copies on write, appends, the cascade over the plan's shared blocks cut
    at partitions of this size) against the oracle, the pool bit for bit.
    With off = 0 the shared blocks end on a partition boundary and the
    output is bit-identical to the same step without the plan; with off = 37
    they end 32 tokens into a partition, which then comes in two pieces."""
    dt, Hkv, D, bs, G = torch.bfloat16, 2, 128, 16, 4
    Hq = G * Hkv
    prompts = [2 * part + 5 + off, 3 * part + 9 + off, part + 3 + off]
    NB = 3 * 8 * (-(-(max(prompts) + 64) // bs)) + 64
    order = synth.rng(91).permutation(NB)
    outs = []
    for use_plan in (True, False):
        A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
        cache, hk, hv = _pool(NB, Hkv, bs, D, dt, cuda_device)
        cache = pa.KVCache(cache.k, cache.v, partition_tokens=part)
        roots = _prefill(A, M, prompts, cuda_device, cache, hk, hv, dt, 92)
        seqs = _fork_groups(A, M, roots, 8)
        n = len(seqs)
        slots, pairs = A.batch_append(seqs, [1] * n)
        mslots, mpairs = M.batch_append(seqs, [1] * n)
        assert slots.tolist() == mslots and len(pairs) > 0
        mb = max(len(M.block_table(s)) for s in seqs)
        tables, lens = A.build_block_tables(seqs, mb)
        cow = pa.cow_sources(pairs, tables, lens, bs)
        plan = pa.share_plan(tables, lens, bs).to(cuda_device) if use_plan else None
        if use_plan:
            # two plan groups of 4 forks per prompt, sharing the prompt's full
            # blocks before its partly filled (copied) last block
            assert plan.n_groups == 6
            sh = 32 if off else 0
            assert sorted(set(plan.shared_tokens.tolist())) == [part + sh, 2 * part + sh, 3 * part + sh]
        kn = synth.normal((n, Hkv, D), dt, 93)
        vn = synth.normal((n, Hkv, D), dt, 94)
        q = synth.normal((n, Hq, D), dt, 95)
        out = pa.pa_decode_shared(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                                  torch.from_numpy(lens).to(cuda_device), int(lens.max()), 1 / math.sqrt(D), plan=plan,
                                  k_new=kn.to(cuda_device), v_new=vn.to(cuda_device),
                                  cow_src=torch.from_numpy(cow).to(cuda_device))
        assert pa.pa_read_device_error() == 0
        oracle.copy_blocks(hk, hv, mpairs)
        oracle.append_kv(hk, hv, kn, vn, mslots)
        assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
        ref = oracle.decode(q, hk, hv, tables, lens, 1 / math.sqrt(D))
        assert_attn_close(out, ref, dt)
        outs.append(out)
    if off == 0:
        assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


@pytest.mark.parametrize("part", [256])
def test_decode_step_partition_size(cuda_device, part):
    """The one-call step over a pool of 256-token partitions (its plan and
    workspace follow the pool's size), three steps, against the oracle."""
    dev, dt, Hkv, D, bs, G = cuda_device, torch.bfloat16, 2, 128, 16, 4
    Hq = G * Hkv
    prompts = [700, 300]
    NB = 2 * 4 * 64 + 64
    order = synth.rng(97).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    cache, hk, hv = _pool(NB, Hkv, bs, D, dt, dev)
    cache = pa.KVCache(cache.k, cache.v, partition_tokens=part)
    roots = _prefill(A, M, prompts, dev, cache, hk, hv, dt, 98)
    seqs = _fork_groups(A, M, roots, 4)
    n = len(seqs)
    mb = max(len(M.block_table(s)) for s in seqs) + 4
    stepper = pa.DecodeStepper(A, cache, n, Hq, mb, 1 / math.sqrt(D))
    groups = 0
    for s in range(3):
        q_h, k_h, v_h = stepper.inputs()
        q = synth.normal((n, Hq, D), dt, 99 + 3 * s)
        kn = synth.normal((n, Hkv, D), dt, 100 + 3 * s)
        vn = synth.normal((n, Hkv, D), dt, 101 + 3 * s)
        q_h.copy_(q)
        k_h.copy_(kn)
        v_h.copy_(vn)
        info = stepper.step(seqs)
        groups += info["n_groups"]
        mslots, mpairs = M.batch_append(seqs, [1] * n)
        oracle.copy_blocks(hk, hv, mpairs)
        oracle.append_kv(hk, hv, kn, vn, mslots)
        tables = np.full((n, mb), -1, np.int32)
        for i, sq in enumerate(seqs):
            t = M.block_table(sq)
            tables[i, :len(t)] = t
        lens = np.array([M.lens[sq] for sq in seqs], np.int32)
        stepper.wait(info["slot"])
        assert_attn_close(stepper.output(info["slot"]), oracle.decode(q, hk, hv, tables, lens, 1 / math.sqrt(D)), dt)
    stepper.close()
    assert groups > 0

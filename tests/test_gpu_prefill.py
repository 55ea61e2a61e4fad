"""pa_prefill (paged chunked-prefill attention) against the oracle's float64
prefill on the same seeded pools: every new token of a chunk attends
causally to its sequence through the block table.  bf16 bound
|gpu - ref| <= 2e-2 + 1e-2 |ref|."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

from .test_gpu_parity import assert_attn_close

pytestmark = pytest.mark.gpu


def _chunk_case(seed, cached, new, Hq, Hkv, bs, dev, D=128):
    """Sequences with `cached` tokens already in the pool and `new` tokens
    appended for this chunk (K/V for all of them through pa_append_kv, on a
    seeded shuffled pool).  Returns the device inputs and host mirrors."""
    dt = torch.bfloat16
    lens = np.asarray(cached, np.int64) + np.asarray(new, np.int64)
    NB = 2 * int(sum(-(-int(L) // bs) for L in lens)) + 8
    order = synth.rng(seed).permutation(NB)
    A = pa.Allocator(NB, bs, order)
    seqs = [A.new_seq() for _ in lens]
    slots, _ = A.batch_append(seqs, lens.tolist())
    kn = synth.normal((int(lens.sum()), Hkv, D), dt, seed + 1)
    vn = synth.normal((int(lens.sum()), Hkv, D), dt, seed + 2)
    cache = pa.KVCache.empty(NB, Hkv, bs, D, dt, dev)
    pa.pa_append_kv(kn.to(dev), vn.to(dev), torch.from_numpy(slots).to(dev), cache)
    mb = max(1, max(len(A.block_table(s)) for s in seqs))
    tables, lens32 = A.build_block_tables(seqs, mb)
    starts = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    q = synth.normal((int(starts[-1]), Hq, D), dt, seed + 3)
    return cache, q, tables, lens32, starts


def _run(cache, q, tables, lens, starts, dev, scale):
    out = pa.pa_prefill(q.to(dev), cache, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                        torch.from_numpy(starts).to(dev), int(lens.max()), scale,
                        max_query_len=int(np.diff(starts).max()))
    assert pa.pa_read_device_error() == 0
    return out


@pytest.mark.parametrize("G,bs", [(1, 16), (2, 8), (4, 16), (8, 32), (4, 8), (8, 16)])
def test_prefill_matches_oracle(cuda_device, G, bs):
    """Whole prompts, chunks after a cached prefix, ragged query tiles, one
    new token, and a sequence with no new token."""
    Hkv = 2
    Hq = G * Hkv
    cached = [0, 300, 0, 77, 1000, 5, 40]
    new = [200, 129, 1, 64, 70, 0, 257]
    cache, q, tables, lens, starts = _chunk_case(71 + G + bs, cached, new, Hq, Hkv, bs, cuda_device)
    scale = 1 / math.sqrt(128)
    out = _run(cache, q, tables, lens, starts, cuda_device, scale)
    hk, _ = oracle.host_array(cache.k.cpu())
    hv, _ = oracle.host_array(cache.v.cpu())
    ref = oracle.prefill(q, hk, hv, tables, lens, starts, scale)
    assert_attn_close(out, ref, torch.bfloat16)


def test_prefill_long_prompts_sampled(cuda_device):
    """Prompts of the trace's shape (lognormal, median 512, up to 4096), 32/8
    heads: sampled rows of every sequence against the oracle, including each
    chunk's first and last tokens."""
    Hq, Hkv, bs = 32, 8, 16
    r = synth.rng(81)
    new = np.clip(np.round(np.exp(r.normal(math.log(512), 1.0, size=12))), 1, 4096).astype(int)
    cached = np.zeros(12, int)
    cache, q, tables, lens, starts = _chunk_case(82, cached, new, Hq, Hkv, bs, cuda_device)
    scale = 1 / math.sqrt(128)
    out = _run(cache, q, tables, lens, starts, cuda_device, scale)
    rows = []
    for b in range(12):
        idx = {int(starts[b]), int(starts[b + 1]) - 1} | set(
            int(x) for x in r.integers(starts[b], starts[b + 1], size=6))
        rows += [(j, h) for j in sorted(idx) for h in (0, 5, 31)]
    hk, _ = oracle.host_array(cache.k.cpu())
    hv, _ = oracle.host_array(cache.v.cpu())
    ref = oracle.prefill(q, hk, hv, tables, lens, starts, scale, rows=rows)
    got = torch.stack([out[j, h] for j, h in rows])
    assert_attn_close(got, ref, torch.bfloat16)


def test_prefill_single_new_token_is_decode(cuda_device):
    """One new token per sequence is the decode step: the prefill output
    agrees with pa_decode on the same pool within the bf16 bound of the
    oracle, and both with the oracle's decode."""
    Hq, Hkv, bs = 32, 8, 16
    cached = [100, 511, 1500, 3]
    new = [1, 1, 1, 1]
    cache, q, tables, lens, starts = _chunk_case(91, cached, new, Hq, Hkv, bs, cuda_device)
    scale = 1 / math.sqrt(128)
    out = _run(cache, q, tables, lens, starts, cuda_device, scale)
    dec = pa.pa_decode(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                       torch.from_numpy(lens).to(cuda_device), int(lens.max()), scale)
    hk, _ = oracle.host_array(cache.k.cpu())
    hv, _ = oracle.host_array(cache.v.cpu())
    ref = oracle.decode(q, hk, hv, tables, lens, scale)
    assert_attn_close(out, ref, torch.bfloat16)
    assert_attn_close(dec, ref, torch.bfloat16)


def test_prefill_bad_chunk_length_is_reported(cuda_device):
    """A chunk longer than its sequence sets PA_DEVERR_LEN; the other
    sequences are still right."""
    Hq, Hkv, bs = 8, 2, 16
    cache, q, tables, lens, starts = _chunk_case(95, [10, 0], [20, 30], Hq, Hkv, bs, cuda_device)
    bad = lens.copy()
    bad[1] = 12  # 30 new tokens in a 12-token sequence
    out = pa.pa_prefill(q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device),
                        torch.from_numpy(bad).to(cuda_device), torch.from_numpy(starts).to(cuda_device),
                        int(lens.max()), 0.1, max_query_len=30)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_LEN
    hk, _ = oracle.host_array(cache.k.cpu())
    hv, _ = oracle.host_array(cache.v.cpu())
    ref = oracle.prefill(q[:20], hk, hv, tables[:1], lens[:1], starts[:2], 0.1)
    assert_attn_close(out[:20], ref, torch.bfloat16)


def test_prefill_many_short_units_no_timeout(cuda_device):
    """Hundreds of one-chunk units per CTA, repeated: every softmax warp must
    have read a unit before its Q slot is reused (a lagging warp once saw the
    slot's barrier two phases ahead and gave up waiting).  No error bit, and
    the output still matches the oracle."""
    Hq, Hkv, bs = 32, 8, 16
    r = synth.rng(97)
    new = r.integers(1, 64, size=400)
    cached = r.integers(0, 40, size=400)
    cache, q, tables, lens, starts = _chunk_case(98, cached, new, Hq, Hkv, bs, cuda_device)
    scale = 1 / math.sqrt(128)
    args = (q.to(cuda_device), cache, torch.from_numpy(tables).to(cuda_device), torch.from_numpy(lens).to(cuda_device),
            torch.from_numpy(starts).to(cuda_device), int(lens.max()), scale)
    out = None
    for _ in range(30):
        out = pa.pa_prefill(*args, max_query_len=int(new.max()))
    assert pa.pa_read_device_error() == 0
    rows = [(int(j), h) for j in r.integers(0, int(starts[-1]), size=40) for h in (0, 17)]
    hk, _ = oracle.host_array(cache.k.cpu())
    hv, _ = oracle.host_array(cache.v.cpu())
    ref = oracle.prefill(q, hk, hv, tables, lens, starts, scale, rows=rows)
    assert_attn_close(torch.stack([out[j, h] for j, h in rows]), ref, torch.bfloat16)

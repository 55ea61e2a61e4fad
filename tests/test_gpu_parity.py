"""CUDA path against the oracle, element by element, on the same seeded inputs.

Append and block copy must match bit for bit over the whole pool (unowned
blocks hold a NaN sentinel, so a stray write shows).  Attention must match
within max-abs 1e-5 for fp32 and |gpu - ref| <= 2e-2 + 1e-2 |ref| for bf16
(the oracle runs in float64 on the same, widened inputs).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

pytestmark = pytest.mark.gpu

F32_ATOL = 1e-5
BF16_ATOL, BF16_RTOL = 2e-2, 1e-2


def assert_attn_close(gpu: torch.Tensor, ref: np.ndarray, dtype):
    g = gpu.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape
    assert np.isfinite(g).all(), "non-finite output"
    err = np.abs(g - ref)
    if dtype == torch.float32:
        assert err.max() <= F32_ATOL, f"max abs err {err.max():.3g}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), f"{bad.sum()} elements out of tolerance, worst {(err - bound).max():.3g}"


def host_pool(t: torch.Tensor) -> np.ndarray:
    """Host copy of a pool in the oracle's element form (uint16 patterns for
    bf16, float32 for fp32)."""
    a, _ = oracle.host_array(t.cpu())
    return a.copy()


def same_bits(a: np.ndarray, b: np.ndarray) -> bool:
    """Bit-for-bit equality (NaN sentinels included)."""
    if a.dtype == np.float32:
        a, b = a.view(np.uint32), b.view(np.uint32)
    return a.shape == b.shape and np.array_equal(a, b)


def to_dev(case: synth.DecodeCase, dev):
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev))
    return (cache, case.q.to(dev), torch.from_numpy(case.block_tables).to(dev),
            torch.from_numpy(case.context_lens).to(dev))


def decode_case(case: synth.DecodeCase, dev, scale=None):
    cache, q, tables, lens = to_dev(case, dev)
    out = pa.pa_decode(q, cache, tables, lens, int(case.context_lens.max()), case.scale if scale is None else scale)
    assert pa.pa_read_device_error() == 0
    return out


# ------------------------------------------------------------------ decode


def test_tiny_fp32_decode(cuda_device):
    case = synth.tiny_fp32_case(0)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.float32)


def test_block_table_example_fp32(cuda_device):
    case = synth.block_table_example_case(1)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.float32)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_group_sizes(cuda_device, dtype, G, D):
    Hkv = 2
    lens = [1, 15, 16, 17, 100, 511, 512, 513, 1200, 0, 2049]
    case = synth.random_case(10 + G + D, B=len(lens), Hq=G * Hkv, Hkv=Hkv, D=D, bs=16, lens=lens, dtype=dtype)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, dtype)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_decode_block_sizes(cuda_device, bs):
    lens = [3, bs, bs + 1, 513, 1000, 1537]
    case = synth.random_case(30 + bs, B=len(lens), Hq=8, Hkv=2, D=128, bs=bs, lens=lens, dtype=torch.bfloat16)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.bfloat16)


def test_decode_peaked_softmax(cuda_device):
    """Scale x 8: large logit gaps exercise the max subtraction."""
    lens = [700, 64, 1800]
    case = synth.random_case(41, B=3, Hq=8, Hkv=2, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    out = decode_case(case, cuda_device, scale=8.0 / math.sqrt(128))
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, 8.0 / math.sqrt(128))
    assert_attn_close(out, ref, torch.bfloat16)


def test_decode_context_one_and_zero(cuda_device):
    case = synth.random_case(42, B=3, Hq=4, Hkv=2, D=128, bs=16, lens=[1, 0, 1], dtype=torch.float32)
    out = decode_case(case, cuda_device).cpu()
    assert torch.equal(out[1], torch.zeros_like(out[1]))
    for b in (0, 2):
        blk = int(case.block_tables[b, 0])
        for h in range(4):
            assert torch.equal(out[b, h], case.v_cache[blk, h // 2, 0])


def test_decode_permutation_invariance(cuda_device):
    """The same logical rows placed through two different tables give the
    same result within rounding."""
    lens = [900, 40]
    a = synth.random_case(43, B=2, Hq=8, Hkv=2, D=128, bs=16, lens=lens, dtype=torch.bfloat16, sentinel=False)
    # move every block of a to a new place
    perm = synth.rng(44).permutation(a.num_blocks)
    k2 = torch.empty_like(a.k_cache)
    v2 = torch.empty_like(a.v_cache)
    k2[torch.as_tensor(perm)] = a.k_cache
    v2[torch.as_tensor(perm)] = a.v_cache
    t2 = np.where(a.block_tables >= 0, perm[np.maximum(a.block_tables, 0)], -1).astype(np.int32)
    b = synth.DecodeCase("moved", a.q, k2, v2, t2, a.context_lens, a.scale)
    oa = decode_case(a, cuda_device).float()
    ob = decode_case(b, cuda_device).float()
    assert torch.equal(oa, ob)


def test_gqa_bf16_full_size(cuda_device):
    """bf16 GQA decode at full size: 32 sequences, 32 query / 8 kv heads,
    head_dim 128, 16-token blocks, lengths uniform in [128, 4096], a pool of
    twice the needed blocks dealt from a seeded shuffle; every output row."""
    lens = synth.gqa_lengths(2)
    case = synth.random_case(2, B=32, Hq=32, Hkv=8, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.bfloat16)


def test_partials_match_oracle_partials(cuda_device):
    """The split-context workspace itself: per-partition max (base-2 units on
    the device), sum and accumulator against the oracle's partials."""
    lens = [1100, 513, 2000]
    case = synth.random_case(45, B=3, Hq=8, Hkv=2, D=128, bs=16, lens=lens, dtype=torch.float32)
    cache, q, tables, lens_d = to_dev(case, cuda_device)
    B, Hq, D, P = 3, 8, 128, 4
    need = pa.pa_decode_workspace_size(B, Hq, 2000, D)
    ws = torch.zeros(need, dtype=torch.uint8, device=cuda_device)
    pa.pa_decode(q, cache, tables, lens_d, 2000, case.scale, workspace=ws)
    torch.cuda.synchronize()
    rows = B * Hq * P
    wsf = ws.view(torch.float32).cpu()
    off = (rows * 4 + 15) // 16 * 16 // 4
    gm = wsf[:rows].view(B, Hq, P).double().numpy() * math.log(2.0)
    gl = wsf[off:off + rows].view(B, Hq, P).double().numpy()
    gacc = wsf[2 * off:2 * off + rows * D].view(B, Hq, P, D).double().numpy()
    m, l, acc, np_ = oracle.decode_partials(case.q, case.k_cache, case.v_cache, case.block_tables,
                                            case.context_lens, case.scale, 512)
    for b in range(B):
        for p in range(np_[b]):
            np.testing.assert_allclose(gm[b, :, p], m[b, :, p], rtol=0, atol=1e-5)
            np.testing.assert_allclose(gl[b, :, p], l[b, :, p], rtol=1e-5)
            np.testing.assert_allclose(gacc[b, :, p], acc[b, :, p], rtol=1e-5, atol=1e-4)


# ------------------------------------------------------------- append / copy


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_append_bit_exact(cuda_device, dtype):
    NB, Hkv, bs, D, N = 40, 4, 16, 128, 300
    r = synth.rng(50)
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dtype))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dtype))
    slots = r.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[::7] = -1  # padding
    kn = synth.normal((N, Hkv, D), dtype, 51)
    vn = synth.normal((N, Hkv, D), dtype, 52)
    cache = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    pa.pa_append_kv(kn.to(cuda_device), vn.to(cuda_device), torch.from_numpy(slots).to(cuda_device), cache)
    assert pa.pa_read_device_error() == 0
    hk, hv = host_pool(k0), host_pool(v0)
    oracle.append_kv(hk, hv, kn, vn, slots)
    assert same_bits(host_pool(cache.k), hk)
    assert same_bits(host_pool(cache.v), hv)


def test_copy_blocks_bit_exact(cuda_device):
    NB, Hkv, bs, D = 64, 8, 16, 128
    k0 = synth.normal((NB, Hkv, bs, D), torch.bfloat16, 60)
    v0 = synth.normal((NB, Hkv, bs, D), torch.bfloat16, 61)
    perm = synth.rng(62).permutation(NB)
    pairs = np.stack([perm[:20], perm[20:40]], axis=1).astype(np.int32)
    assert pa.pa_check_copy_pairs(pairs, NB)
    cache = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    pa.pa_copy_blocks(torch.from_numpy(pairs).to(cuda_device), cache)
    assert pa.pa_read_device_error() == 0
    hk, hv = host_pool(k0), host_pool(v0)
    oracle.copy_blocks(hk, hv, pairs)
    assert same_bits(host_pool(cache.k), hk)
    assert same_bits(host_pool(cache.v), hv)


# ------------------------------------------------------------- device errors


def test_device_errors_are_reported_not_trapped(cuda_device):
    NB, Hkv, bs, D = 8, 2, 16, 64
    cache = pa.KVCache.empty(NB, Hkv, bs, D, torch.float32, cuda_device)
    cache.k.zero_()
    cache.v.zero_()
    kn = torch.ones(2, Hkv, D, device=cuda_device)
    pa.pa_append_kv(kn, kn, torch.tensor([NB * bs, 3], device=cuda_device), cache)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_SLOT
    assert float(cache.k[0, :, 3].sum()) == Hkv * D  # the good row landed
    pa.pa_copy_blocks(torch.tensor([[0, NB]], dtype=torch.int32, device=cuda_device), cache)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_PAIR
    q = torch.ones(1, 2, D, device=cuda_device)
    tables = torch.tensor([[0, 99]], dtype=torch.int32, device=cuda_device)
    pa.pa_decode(q, cache, tables, torch.tensor([20], dtype=torch.int32, device=cuda_device), 32, 1.0)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_TABLE
    out = pa.pa_decode(q, cache, tables[:, :1], torch.tensor([17], dtype=torch.int32, device=cuda_device), 16, 1.0)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_LEN
    assert torch.equal(out, torch.zeros_like(out))
    assert pa.pa_read_device_error() == 0


# ------------------------------------------------------------- full step


def _prefill(A, M, lens, dev, cache, hk, hv, dtype, seed):
    """Creates the sequences through both allocators and writes their prompt
    rows with pa_append_kv (GPU) and the oracle's append (host)."""
    seqs = []
    Hkv, D = cache.num_kv_heads, cache.head_dim
    for i, L in enumerate(lens):
        s = A.new_seq()
        assert M.new_seq() == s
        seqs.append(s)
    slots, pairs = A.batch_append(seqs, lens)
    mslots, mpairs = M.batch_append(seqs, lens)
    assert slots.tolist() == mslots and len(pairs) == 0 == len(mpairs)
    total = int(np.sum(lens))
    kn = synth.normal((total, Hkv, D), dtype, seed)
    vn = synth.normal((total, Hkv, D), dtype, seed + 1)
    pa.pa_append_kv(kn.to(dev), vn.to(dev), torch.from_numpy(slots).to(dev), cache)
    oracle.append_kv(hk, hv, kn, vn, slots)
    return seqs


def _step(A, M, seqs, dev, cache, hk, hv, q, dtype, seed, scale):
    """One decode step on both sides: allocate one token per sequence, copy
    on write, append, decode.  Returns (gpu out, oracle out)."""
    Hkv, D = cache.num_kv_heads, cache.head_dim
    n = len(seqs)
    slots, pairs = A.batch_append(seqs, [1] * n)
    mslots, mpairs = M.batch_append(seqs, [1] * n)
    assert slots.tolist() == mslots
    assert [tuple(p) for p in pairs.tolist()] == mpairs
    kn = synth.normal((n, Hkv, D), dtype, seed)
    vn = synth.normal((n, Hkv, D), dtype, seed + 1)
    if len(pairs):
        assert pa.pa_check_copy_pairs(pairs, cache.num_blocks)
        pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(pairs)).to(dev), cache)
    pa.pa_append_kv(kn.to(dev), vn.to(dev), torch.from_numpy(slots).to(dev), cache)
    oracle.copy_blocks(hk, hv, mpairs)
    oracle.append_kv(hk, hv, kn, vn, mslots)
    mb = max(len(M.block_table(s)) for s in seqs)
    tables, lens = A.build_block_tables(seqs, mb)
    out = pa.pa_decode(q.to(dev), cache, torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev),
                       int(lens.max()), scale)
    assert pa.pa_read_device_error() == 0
    mt = np.full((n, mb), -1, np.int32)
    for i, s in enumerate(seqs):
        t = M.block_table(s)
        mt[i, :len(t)] = t
    assert np.array_equal(tables, mt)
    ref = oracle.decode(q, hk, hv, mt, np.array([M.lens[s] for s in seqs], np.int32), scale)
    return out, ref


def test_full_step_gqa_bf16(cuda_device):
    """Allocator + append + decode for the bf16 GQA batch (32 sequences,
    32/8 heads, head_dim 128, 16-token blocks, lengths uniform in [128, 4096]);
    the pool (twice the needed blocks) is dealt from a seeded shuffle."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 8, 128, 16, 32
    lens = synth.gqa_lengths(3)
    NB = 2 * int(sum(-(-(int(L) + 1) // bs) for L in lens))
    order = synth.rng(4).permutation(NB)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    cache = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    hk, hv = host_pool(k0), host_pool(v0)
    seqs = _prefill(A, M, lens.tolist(), cuda_device, cache, hk, hv, dt, 5)
    q = synth.normal((len(seqs), Hq, D), dt, 7)
    out, ref = _step(A, M, seqs, cuda_device, cache, hk, hv, q, dt, 8, 1 / math.sqrt(D))
    assert same_bits(host_pool(cache.k), hk) and same_bits(host_pool(cache.v), hv)
    assert_attn_close(out, ref, dt)


def test_full_step_shared_prefix_cow(cuda_device):
    """Groups share a prefix that ends inside a block; one append step makes
    every group member but the last copy that block (copy on write), then all
    decode.  Shared full blocks stay bit-identical; the whole pool matches
    the oracle bit for bit."""
    dt, Hkv, D, bs, Hq = torch.bfloat16, 8, 128, 16, 64
    groups, gsz = 4, 8
    pl, suffix, order, NB = synth.shared_prefix_layout(9, groups=groups, group_size=gsz, prefix=512,
                                                       median=60, clip=300, prefix_tail=True)
    A, M = pa.Allocator(NB, bs, order), oracle.AllocatorModel(NB, bs, order)
    k0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    v0 = synth.sentinel_(torch.empty(NB, Hkv, bs, D, dtype=dt))
    cache = pa.KVCache(k0.to(cuda_device), v0.to(cuda_device))
    hk, hv = host_pool(k0), host_pool(v0)
    roots = _prefill(A, M, pl.tolist(), cuda_device, cache, hk, hv, dt, 10)
    seqs = []
    for r in roots:
        seqs.append(r)
        for _ in range(gsz - 1):
            c = A.fork(r)
            assert M.fork(r) == c
            seqs.append(c)
    shared_full = {b for r in roots for b in M.block_table(r)[:-1]}
    snap = {b: (hk[b].copy(), hv[b].copy()) for b in shared_full}
    q = synth.normal((len(seqs), Hq, D), dt, 12)
    out, ref = _step(A, M, seqs, cuda_device, cache, hk, hv, q, dt, 13, 1 / math.sqrt(D))
    gk, gv = host_pool(cache.k), host_pool(cache.v)
    assert same_bits(gk, hk) and same_bits(gv, hv)
    for b, (sk, sv) in snap.items():
        assert same_bits(gk[b], sk) and same_bits(gv[b], sv)
    assert_attn_close(out, ref, dt)


# ------------------------------------------------------------- bf16 / head_dim 128 specifics


def test_bf16_context_one_is_exact(cuda_device):
    """ctx = 1: the single weight is exactly 1, so the output is the value
    row itself, bit for bit (bf16, head_dim 128)."""
    case = synth.random_case(46, B=3, Hq=8, Hkv=2, D=128, bs=16, lens=[1, 0, 1], dtype=torch.bfloat16)
    out = decode_case(case, cuda_device).cpu()
    assert torch.equal(out[1], torch.zeros_like(out[1]))
    for b in (0, 2):
        blk = int(case.block_tables[b, 0])
        for h in range(8):
            assert torch.equal(out[b, h], case.v_cache[blk, h // 4, 0])


@pytest.mark.parametrize("B", [300, 2100])
def test_many_sequences(cuda_device, B):
    """More sequences than one thread's share of the in-kernel prefix sums
    (300), and more than one launch of the bf16 kernel takes (2100 runs as
    two slices); lengths include zeros and several partitions."""
    lens = synth.rng(47 + B).integers(0, 1300 if B < 1000 else 80, size=B).astype(np.int32)
    case = synth.random_case(47, B=B, Hq=8, Hkv=2, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    out = decode_case(case, cuda_device)
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out, ref, torch.bfloat16)


def test_bf16_device_errors(cuda_device):
    """A table entry outside the pool and a length past max_context_len on
    the bf16 head_dim-128 path: reported in the error word, no trap; the
    other sequences are still right."""
    lens = [700, 40, 1300]
    case = synth.random_case(48, B=3, Hq=8, Hkv=2, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    cache, q, tables, lens_d = to_dev(case, cuda_device)
    bad = tables.clone()
    bad[0, 3] = case.num_blocks + 5
    out = pa.pa_decode(q, cache, bad, lens_d, 1300, case.scale)
    assert pa.pa_read_device_error() & pa.PA_DEVERR_TABLE
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(out[1:], ref[1:], torch.bfloat16)
    lens_bad = lens_d.clone()
    lens_bad[1] = 5000
    out = pa.pa_decode(q, cache, tables, lens_bad, 1300, case.scale)
    assert pa.pa_read_device_error() == pa.PA_DEVERR_LEN
    assert torch.equal(out[1].float().cpu(), torch.zeros(8, 128))
    assert_attn_close(out[[0, 2]], ref[[0, 2]], torch.bfloat16)
    assert pa.pa_read_device_error() == 0

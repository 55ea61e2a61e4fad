"""pa_decode_static_workspace, the decode entry point that allocates nothing.

Some callers cannot allocate device memory while they decode: a serving
process that sized its paged KV pool to take nearly all free HBM (so even a
small workspace allocation can fail), or code behind a plugin or runtime
interface that offers no device allocator.  For them the library keeps the
split-context scratch in one fixed array of its own.  These tests call that
entry point through the C ABI on two calls in a row with different shapes
(the second call's layout of the scratch differs from the first's, and the
first leaves its contents behind), and check each against pa_decode, which
takes a caller workspace, and against the float64 oracle.  Sizes past the
array are refused before any launch.

This file is collected last on purpose, so that a run that stops at the
first failure has run every other test first.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

pytestmark = pytest.mark.gpu

BF16_ATOL, BF16_RTOL = 2e-2, 1e-2  # the bf16 tolerance of the parity tests


def _inputs(seed, B, max_len, dev):
    lens = synth.rng(seed).integers(1, max_len, size=B).astype(np.int32)
    lens[0] = max_len  # several 512-token partitions: the scratch is used
    case = synth.random_case(seed, B=B, Hq=32, Hkv=8, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev))
    return (case, cache, case.q.to(dev), torch.from_numpy(case.block_tables).to(dev),
            torch.from_numpy(case.context_lens).to(dev))


def _close(got: torch.Tensor, want: np.ndarray, what: str):
    g = got.float().cpu().double().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    bad = np.abs(g - want) > BF16_ATOL + BF16_RTOL * np.abs(want)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance"


def test_static_workspace_two_calls_match_pa_decode_and_oracle(cuda_device):
    L = pa.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # a larger layout first (32 sequences, 8 partitions per row), then a
    # smaller one (8 sequences, 3 partitions per row): the second call reads
    # only what it wrote itself, never the first call's leftovers
    for seed, B, max_len in ((71, 32, 4000), (72, 8, 1500)):
        case, cache, q, tables, lens = _inputs(seed, B, max_len, cuda_device)
        max_ctx = int(case.context_lens.max())
        assert 0 < pa.pa_decode_workspace_size(B, 32, max_ctx, 128) <= pa.PA_STATIC_WORKSPACE_BYTES
        want = pa.pa_decode(q, cache, tables, lens, max_ctx, case.scale)
        got = torch.full_like(q, float("nan"))
        st = L.pa_decode_static_workspace(q.data_ptr(), cache.ref(), tables.data_ptr(), tables.shape[1],
                                          lens.data_ptr(), B, 32, max_ctx, ctypes.c_float(case.scale),
                                          got.data_ptr(), stream)
        assert st == pa.PA_OK, L.pa_status_string(st)
        assert pa.pa_read_device_error() == 0
        _close(got, want.float().cpu().double().numpy(), f"B={B} against pa_decode")
        ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
        _close(got, ref, f"B={B} against the oracle")


def test_static_workspace_python_wrapper(cuda_device):
    case, cache, q, tables, lens = _inputs(73, 16, 2999, cuda_device)
    got = pa.pa_decode_static_workspace(q, cache, tables, lens, int(case.context_lens.max()), case.scale)
    assert pa.pa_read_device_error() == 0
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    _close(got, ref, "wrapper against the oracle")
    with pytest.raises(ValueError):  # a q whose head_dim is not the cache's, refused before any launch
        pa.pa_decode_static_workspace(q[..., :64].contiguous(), cache, tables, lens, 2999, case.scale)
    with pytest.raises(ValueError):  # an out of another shape
        pa.pa_decode_static_workspace(q, cache, tables, lens, 2999, case.scale, out=q[:8].clone())


def test_static_workspace_refuses_oversize(cuda_device):
    L = pa.lib()
    cache = pa.KVCache.empty(8, 8, 16, 128, torch.bfloat16, cuda_device)
    q = torch.zeros(8, 32, 128, dtype=torch.bfloat16, device=cuda_device)
    tables = torch.zeros(8, 8192, dtype=torch.int32, device=cuda_device)
    lens = torch.zeros(8, dtype=torch.int32, device=cuda_device)
    need = pa.pa_decode_workspace_size(8, 32, 131072, 128)
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    st = L.pa_decode_static_workspace(q.data_ptr(), cache.ref(), tables.data_ptr(), 8192, lens.data_ptr(), 8, 32,
                                      131072, ctypes.c_float(1 / math.sqrt(128)), q.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == pa.PA_ERR_TOO_SMALL
    # a length near INT32_MAX is an argument error, not a wrapped size
    st = L.pa_decode_static_workspace(q.data_ptr(), cache.ref(), tables.data_ptr(), 8192, lens.data_ptr(), 8, 32,
                                      2**31 - 1, ctypes.c_float(1 / math.sqrt(128)), q.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == pa.PA_ERR_INVALID_ARG
    assert pa.pa_read_device_error() == 0

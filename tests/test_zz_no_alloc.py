"""pa_decode_static_workspace, the decode entry point that allocates nothing.

Some callers cannot allocate device memory while they decode: a serving
process that sized its paged KV pool to take nearly all free HBM (so even a
small workspace allocation can fail), or code behind a plugin or runtime
interface that offers no device allocator.  For them the library keeps the
split-context scratch in one fixed array of its own.  These tests call that
entry point through the C ABI and check it against pa_decode, which takes a
caller workspace, on two calls in a row with different inputs, and check
that sizes past the array are refused before any launch.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

pytestmark = pytest.mark.gpu

BF16_ATOL, BF16_RTOL = 2e-2, 1e-2  # the bf16 tolerance of the parity tests


def _inputs(seed, dev):
    lens = synth.rng(seed).integers(1, 3000, size=16).astype(np.int32)
    lens[0] = 2999  # several 512-token partitions: the scratch is used
    case = synth.random_case(seed, B=16, Hq=32, Hkv=8, D=128, bs=16, lens=lens, dtype=torch.bfloat16)
    cache = pa.KVCache(case.k_cache.to(dev), case.v_cache.to(dev))
    return (case, cache, case.q.to(dev), torch.from_numpy(case.block_tables).to(dev),
            torch.from_numpy(case.context_lens).to(dev))


def test_static_workspace_matches_pa_decode_on_two_calls(cuda_device):
    L = pa.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (71, 72):
        case, cache, q, tables, lens = _inputs(seed, cuda_device)
        max_ctx = int(case.context_lens.max())
        assert 0 < pa.pa_decode_workspace_size(16, 32, max_ctx, 128) <= pa.PA_STATIC_WORKSPACE_BYTES
        want = pa.pa_decode(q, cache, tables, lens, max_ctx, case.scale)
        got = torch.full_like(q, float("nan"))
        st = L.pa_decode_static_workspace(q.data_ptr(), cache.ref(), tables.data_ptr(), tables.shape[1],
                                          lens.data_ptr(), 16, 32, max_ctx, ctypes.c_float(case.scale),
                                          got.data_ptr(), stream)
        assert st == pa.PA_OK, L.pa_status_string(st)
        assert pa.pa_read_device_error() == 0
        g = got.float().cpu().double().numpy()
        w = want.float().cpu().double().numpy()
        assert np.isfinite(g).all()
        assert (np.abs(g - w) <= BF16_ATOL + BF16_RTOL * np.abs(w)).all()


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
    assert pa.pa_read_device_error() == 0

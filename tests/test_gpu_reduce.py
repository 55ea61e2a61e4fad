"""The partition merge (log-sum-exp reduce) kernels against the oracle and
against each other.

A call whose rows have at most 32 partitions merges one row per warp
(decode_reduce_rows, sized for 4, 8 or 16 partitions, and
decode_reduce_rows_wide up to 32); a longer declared maximum context takes
the one-CTA-per-row decode_reduce.  All merge in the same order with the
same arithmetic, so for the same partition statistics their outputs must
agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_402_b200 as pa
from paged_kv_cache_402_b200 import synth

from .test_gpu_parity import assert_attn_close, to_dev

pytestmark = pytest.mark.gpu

PART = 512


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16).cpu()


@pytest.mark.parametrize("parts", [2, 4, 8, 16, 17, 24, 32])
@pytest.mark.parametrize("G,dtype,D", [(1, torch.bfloat16, 128), (4, torch.bfloat16, 128),
                                       (8, torch.bfloat16, 128), (2, torch.float32, 128),
                                       (4, torch.float32, 64)])
def test_row_reduce_matches_block_reduce_bits(cuda_device, parts, G, dtype, D):
    """Lengths from 1 token to exactly `parts` partitions: the call with the
    true maximum merges with a warp-per-row kernel, the call declaring 33
    partitions with the one-CTA-per-row kernel; same bits, and within the
    bound of the oracle."""
    Hkv = 2
    top = parts * PART
    lens = np.array([top, 1, PART, PART + 1, top - 1, max(top - PART + 1, 1), 0, (top + 1) // 2], np.int32)
    case = synth.random_case(80 + G + parts, B=len(lens), Hq=G * Hkv, Hkv=Hkv, D=D, bs=16, lens=lens,
                             dtype=dtype)
    cache, q, tables, lens_d = to_dev(case, cuda_device)
    # wide enough a table for the longer declared maximum to be a valid call
    long_max = 32 * PART + 1
    cols = -(-long_max // 16)
    tables = torch.cat([tables, torch.full_like(tables[:, :1], -1).expand(-1, cols - tables.shape[1])],
                       dim=1).contiguous()
    rows_path = pa.pa_decode(q, cache, tables, lens_d, top, case.scale)
    assert pa.pa_read_device_error() == 0
    block_path = pa.pa_decode(q, cache, tables, lens_d, long_max, case.scale)
    assert pa.pa_read_device_error() == 0
    assert torch.equal(_bits(rows_path), _bits(block_path))
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert_attn_close(rows_path, ref, dtype)


@pytest.mark.parametrize("B,G", [(1100, 4), (1500, 8), (8300, 1)])
def test_row_reduce_many_rows(cuda_device, B, G):
    """More sequences than the tensor-core kernel's per-sequence tables hold
    (1024): 1100 and 1500 take its coarse tables (entries of 8 sequences) in
    one launch, 8300 two launches (8192 + 108) before one reduce; 1500 x 16
    query heads = 24000 rows is more than the grid-stride reduce has warps.
    Every fifth sequence (every 25th of 8300) has 2 to 4 partitions.
    Sampled rows against the oracle."""
    Hkv = 2
    r = synth.rng(95 + B)
    lens = r.integers(1, 64, size=B).astype(np.int32)
    multi = np.arange(0, B, 5 if B < 4096 else 25)
    lens[multi] = r.integers(PART + 1, 4 * PART, size=len(multi))
    lens[1020:1030] = 4 * PART - 3
    if B > 8192:
        lens[8188:8196] = 4 * PART - 5
    case = synth.random_case(95, B=B, Hq=G * Hkv, Hkv=Hkv, D=128, bs=16, lens=lens, dtype=torch.bfloat16,
                             pool_factor=1.05)
    cache, q, tables, lens_d = to_dev(case, cuda_device)
    out = pa.pa_decode(q, cache, tables, lens_d, int(lens.max()), case.scale)
    assert pa.pa_read_device_error() == 0
    seqs = sorted(set(list(range(0, B, 15)) + list(range(1016, 1032)) +
                      (list(range(8184, 8200)) if B > 8192 else [])))
    rows = [(b, h) for b in seqs for h in (0, G * Hkv - 1)]
    ref = oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale,
                        rows=rows)
    assert_attn_close(torch.stack([out[b, h] for b, h in rows]), ref, torch.bfloat16)

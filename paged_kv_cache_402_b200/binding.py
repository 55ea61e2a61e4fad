"""Python binding of libpagedattn (the paged KV-cache decode path, sm_100a).

Thin ctypes marshalling over the C ABI of ``include/pagedattn.h``: every step
runs in the library's CUDA kernels (append, block copy, decode partition and
reduce) or its C++ allocator.  PyTorch supplies device memory and streams
only.  There is no fallback: if the library is missing, importing this
module raises.

Names follow the C ABI: ``pa_append_kv``, ``pa_decode``, ``pa_copy_blocks``,
``pa_decode_workspace_size``, ``pa_read_device_error``,
``pa_check_copy_pairs``; ``Allocator`` wraps the ``pa_alloc_*`` / ``pa_seq_*``
calls and ``KVCache`` holds the two pools.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_OUT_OF_BLOCKS = 0, 1, 2, 3
PA_ERR_CUDA, PA_ERR_NOT_FOUND, PA_ERR_TOO_SMALL = 4, 5, 6
PA_DTYPE_F32, PA_DTYPE_BF16 = 0, 1
PA_DEVERR_SLOT, PA_DEVERR_TABLE, PA_DEVERR_PAIR, PA_DEVERR_TIMEOUT, PA_DEVERR_LEN, PA_DEVERR_PLAN = 1, 2, 4, 8, 16, 32
PA_PARTITION_TOKENS = 512
PA_SHARE_MIN_TOKENS = 128  # shortest shared prefix a plan group takes

_DTYPES = {torch.float32: PA_DTYPE_F32, torch.bfloat16: PA_DTYPE_BF16}


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {_lib.pa_status_string(status).decode()} (status {status})"
        if status == PA_ERR_CUDA:
            code = _lib.pa_last_cuda_error()
            msg += f": CUDA error {code} ({_lib.pa_cuda_error_string(code).decode()})"
        super().__init__(msg)


class OutOfBlocks(PagedAttnError):
    pass


class pa_cache_t(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("partition_tokens", ctypes.c_int32)]


class pa_step_layout_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("q", "k_new", "v_new", "tables", "lens", "cow_src", "first_token",
                                             "members", "shared_tokens", "bytes")]


class pa_step_slot_t(ctypes.Structure):
    _fields_ = [("host", ctypes.c_void_p), ("dev", ctypes.c_void_p), ("out_host", ctypes.c_void_p),
                ("out_dev", ctypes.c_void_p), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("ev_in", ctypes.c_void_p), ("ev_kernel", ctypes.c_void_p), ("ev_out", ctypes.c_void_p)]


class pa_share_plan_t(ctypes.Structure):
    _fields_ = [("members", ctypes.c_void_p), ("shared_tokens", ctypes.c_void_p), ("first_token", ctypes.c_void_p),
                ("n_groups", ctypes.c_int32), ("max_members", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_402_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    # host int32 / int64 arrays go in as plain addresses (_i32p / _i64p check
    # their dtype and layout), which ctypes converts far faster than typed
    # pointers; ctypes.byref() results are accepted there too
    i32p, i64p = vp, vp
    cp = ctypes.POINTER(pa_cache_t)
    st = ctypes.c_int
    sigs = {
        "pa_append_kv": (st, [vp, vp, vp, i32, cp, vp]),
        "pa_decode": (st, [vp, cp, vp, i32, vp, i32, i32, i32, f32, vp, vp, sz, vp]),
        "pa_decode_workspace_size": (sz, [i32, i32, i32, i32]),
        "pa_decode_workspace_size_p": (sz, [i32, i32, i32, i32, i32]),
        "pa_decode_shared_workspace_size": (sz, [i32, i32, i32, i32, i32]),
        "pa_decode_static_workspace": (st, [vp, cp, vp, i32, vp, i32, i32, i32, f32, vp, vp]),
        "pa_append_decode": (st, [vp, vp, vp, vp, cp, vp, i32, vp, i32, i32, i32, f32, vp, vp, sz, vp]),
        "pa_cow_sources": (st, [i32p, i32, i32p, i32, i32p, i32, i32, i32p]),
        "pa_decode_shared": (st, [vp, vp, vp, vp, cp, vp, i32, vp, i32, i32, i32, f32,
                                  ctypes.POINTER(pa_share_plan_t), vp, vp, sz, vp]),
        "pa_share_plan": (st, [i32p, i32, i32p, i32, i32, i32, i32p, i32p, i32p, i32p]),
        "pa_prefill": (st, [vp, cp, vp, i32, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp]),
        "pa_decode_step_prepare": (st, [vp, i32p, i32, i32, i32, i32p, i32p, i32p, i32p, i32p, i32p,
                                        i32p, i32p, i32p]),
        "pa_step_layout": (st, [i32, i32, cp, i32, i32, ctypes.POINTER(pa_step_layout_t)]),
        "pa_step_slot_events": (st, [ctypes.POINTER(pa_step_slot_t)]),
        "pa_step_slot_release": (st, [ctypes.POINTER(pa_step_slot_t)]),
        "pa_step_slot_wait": (st, [ctypes.POINTER(pa_step_slot_t)]),
        "pa_decode_step": (st, [vp, i32p, i32, i32, i32, cp, i32, f32, ctypes.POINTER(pa_step_slot_t), vp, vp,
                                vp, i32p, i32p, i32p]),
        "pa_copy_blocks": (st, [vp, i32, cp, vp]),
        "pa_check_copy_pairs": (st, [i32p, i32, i32]),
        "pa_read_device_error": (st, [vp, i32p]),
        "pa_read_wait_timeout": (st, [vp, ctypes.POINTER(ctypes.c_uint32)]),
        "pa_status_string": (ctypes.c_char_p, [st]),
        "pa_last_cuda_error": (ctypes.c_int32, []),
        "pa_cuda_error_string": (ctypes.c_char_p, [ctypes.c_int32]),
        "pa_version": (ctypes.c_char_p, []),
        "pa_alloc_create": (st, [i32, i32, i32p, ctypes.POINTER(vp)]),
        "pa_alloc_destroy": (None, [vp]),
        "pa_seq_new": (st, [vp, i32p]),
        "pa_seq_fork": (st, [vp, i32, i32p]),
        "pa_seq_free": (st, [vp, i32]),
        "pa_seq_append": (st, [vp, i32, i32, i64p, i32p, i32p]),
        "pa_batch_append": (st, [vp, i32p, i32p, i32, i64p, i32p, i32p]),
        "pa_seq_len": (st, [vp, i32, i32p, i32p]),
        "pa_seq_block_table": (st, [vp, i32, i32p, i32, i32p]),
        "pa_build_block_tables": (st, [vp, i32p, i32, i32, i32, i32p, i32p]),
        "pa_seqs_max_len": (st, [vp, i32p, i32, i32p, i32p]),
        "pa_alloc_stats": (st, [vp, i64p, i64p, i32p, i32p]),
        "pa_alloc_fragmentation": (st, [vp, ctypes.POINTER(ctypes.c_double)]),
        "pa_block_refcount": (st, [vp, i32, i32p]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        if status == PA_ERR_OUT_OF_BLOCKS:
            raise OutOfBlocks(status, what)
        raise PagedAttnError(status, what)


def _stream_ptr(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev(t: torch.Tensor, what: str, dtype=None) -> int:
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _i32p(a: np.ndarray) -> int:
    """Address of a C-contiguous int32 host array."""
    if a.dtype != np.int32 or not a.flags.c_contiguous:
        raise TypeError("expected a C-contiguous int32 array")
    return a.ctypes.data


def _i64p(a: np.ndarray) -> int:
    """Address of a C-contiguous int64 host array."""
    if a.dtype != np.int64 or not a.flags.c_contiguous:
        raise TypeError("expected a C-contiguous int64 array")
    return a.ctypes.data


def _check_q_out(q: torch.Tensor, out, cache) -> None:
    """q must be [B, Hq, head_dim] of the cache; a given out must have q's
    shape (the library writes B x Hq x head_dim elements there)."""
    if q.dim() != 3 or q.shape[2] != cache.head_dim:
        raise ValueError(f"q must be [B, Hq, {cache.head_dim}] (the cache's head_dim), got {list(q.shape)}")
    if out is not None and tuple(out.shape) != tuple(q.shape):
        raise ValueError(f"out must have q's shape {list(q.shape)}, got {list(out.shape)}")


# --------------------------------------------------------------------------
# the pools


class KVCache:
    """The paged pools: k and v of shape [num_blocks, num_kv_heads, block_size, head_dim];
    partition_tokens is the split-context partition of the decode calls over
    them (256, 512 or 1024)."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, partition_tokens: int = PA_PARTITION_TOKENS):
        if k.shape != v.shape or k.dtype != v.dtype or k.dim() != 4:
            raise ValueError("k and v must be [num_blocks, Hkv, block_size, head_dim] of one dtype")
        if k.dtype not in _DTYPES:
            raise TypeError(f"unsupported cache dtype {k.dtype}")
        _dev(k, "k_cache")
        _dev(v, "v_cache")
        if partition_tokens not in (256, 512, 1024):
            raise ValueError("partition_tokens must be 256, 512 or 1024")
        self.k, self.v = k, v
        self.partition_tokens = int(partition_tokens)
        self.struct = pa_cache_t(k.data_ptr(), v.data_ptr(), _DTYPES[k.dtype], k.shape[0], k.shape[2],
                                 k.shape[1], k.shape[3], self.partition_tokens)

    @classmethod
    def empty(cls, num_blocks, num_kv_heads, block_size, head_dim, dtype=torch.bfloat16, device="cuda",
              partition_tokens: int = PA_PARTITION_TOKENS):
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        return cls(torch.empty(shape, dtype=dtype, device=device), torch.empty(shape, dtype=dtype, device=device),
                   partition_tokens)

    @property
    def num_blocks(self):
        return self.k.shape[0]

    @property
    def num_kv_heads(self):
        return self.k.shape[1]

    @property
    def block_size(self):
        return self.k.shape[2]

    @property
    def head_dim(self):
        return self.k.shape[3]

    @property
    def dtype(self):
        return self.k.dtype

    def ref(self):
        return ctypes.byref(self.struct)


# --------------------------------------------------------------------------
# kernels


def pa_append_kv(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor, cache: KVCache, stream=None) -> None:
    """Scatters new key/value rows [N, Hkv, D] into the pools at slot_mapping [N] (int64)."""
    n = slot_mapping.numel()
    if k.shape != (n, cache.num_kv_heads, cache.head_dim) or v.shape != k.shape:
        raise ValueError("k, v must be [num_tokens, num_kv_heads, head_dim]")
    _check(_lib.pa_append_kv(_dev(k, "k", cache.dtype), _dev(v, "v", cache.dtype),
                             _dev(slot_mapping, "slot_mapping", torch.int64), n, cache.ref(),
                             _stream_ptr(stream)), "pa_append_kv")


def pa_decode_workspace_size(num_seqs: int, num_q_heads: int, max_context_len: int, head_dim: int,
                             partition_tokens: int = PA_PARTITION_TOKENS) -> int:
    return int(_lib.pa_decode_workspace_size_p(num_seqs, num_q_heads, max_context_len, head_dim,
                                               int(partition_tokens)))


def pa_decode_shared_workspace_size(num_seqs: int, num_q_heads: int, max_context_len: int, head_dim: int,
                                    partition_tokens: int = PA_PARTITION_TOKENS) -> int:
    """Scratch of pa_decode_shared with a plan that has groups (one more row
    per (sequence, query head) than pa_decode_workspace_size)."""
    return int(_lib.pa_decode_shared_workspace_size(num_seqs, num_q_heads, max_context_len, head_dim,
                                                    int(partition_tokens)))


def pa_decode(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor, context_lens: torch.Tensor,
              max_context_len: int, scale: float, out: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Paged decode attention; returns out [B, Hq, D] in the cache dtype."""
    _check_q_out(q, out, cache)
    B, Hq, D = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    need = pa_decode_workspace_size(B, Hq, int(max_context_len), D, cache.partition_tokens)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode(_dev(q, "q", cache.dtype), cache.ref(), _dev(block_tables, "block_tables", torch.int32),
                          block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32), B, Hq,
                          int(max_context_len), float(scale), _dev(out, "out", cache.dtype), ws_ptr, ws_bytes,
                          _stream_ptr(stream)), "pa_decode")
    return out


def pa_append_decode(k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, cache: KVCache,
                     block_tables: torch.Tensor, context_lens: torch.Tensor, max_context_len: int, scale: float,
                     cow_src: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step in one call: per sequence b, the copy of block
    cow_src[b] over b's last block (cow_src int32 [B], -1 for none; None for
    no copies), the append of b's newest token (k_new, v_new [B, Hkv, D],
    written at position context_lens[b] - 1 through b's block table) and the
    decode.  Returns out [B, Hq, D]."""
    _check_q_out(q, out, cache)
    B, Hq, D = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    row_shape = (B, cache.num_kv_heads, D)
    if tuple(k_new.shape) != row_shape or tuple(v_new.shape) != row_shape:
        raise ValueError(f"k_new and v_new must be {list(row_shape)}")
    if cow_src is not None and cow_src.shape != (B,):
        raise ValueError("cow_src must be [B]")
    if out is None:
        out = torch.empty_like(q)
    need = pa_decode_workspace_size(B, Hq, int(max_context_len), D, cache.partition_tokens)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_append_decode(
        _dev(k_new, "k_new", cache.dtype), _dev(v_new, "v_new", cache.dtype),
        _dev(cow_src, "cow_src", torch.int32) if cow_src is not None else None,
        _dev(q, "q", cache.dtype), cache.ref(), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32), B, Hq, int(max_context_len),
        float(scale), _dev(out, "out", cache.dtype), ws_ptr, ws_bytes, _stream_ptr(stream)), "pa_append_decode")
    return out


def cow_sources(pairs, tables: np.ndarray, lens: np.ndarray, block_size: int,
                out: np.ndarray | None = None) -> np.ndarray:
    """Host: the per-sequence copy sources pa_append_decode takes, from a
    step's copy pairs [k, 2] and the host tables / lengths after the append
    (pa_cow_sources)."""
    pairs = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    tables = np.ascontiguousarray(np.asarray(tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    n = len(lens)
    if tables.ndim != 2 or tables.shape[0] != n:
        raise ValueError("tables must be [n_seqs, max_blocks]")
    res = out if out is not None else np.empty(n, dtype=np.int32)
    _check(_lib.pa_cow_sources(_i32p(pairs), pairs.shape[0], _i32p(tables), tables.shape[1], _i32p(lens), n,
                               int(block_size), _i32p(res)), "pa_cow_sources")
    return res


class SharePlan:
    """A sharing plan (groups of sequences that hold the same blocks for their
    leading tokens, a whole number of blocks) as host arrays, plus its device
    copy: members [n_groups, max_members], shared_tokens [n_groups],
    first_token [n_seqs]."""

    def __init__(self, members: np.ndarray, shared_tokens: np.ndarray, first_token: np.ndarray):
        self.members, self.shared_tokens, self.first_token = members, shared_tokens, first_token
        self.n_groups, self.max_members = int(members.shape[0]), int(members.shape[1])
        self._dev = None

    def to(self, device, stream=None) -> "SharePlan":
        """Copies the arrays to the device (kept until the plan is dropped);
        a plan without groups needs none."""
        if self.n_groups > 0:
            self._dev = tuple(torch.from_numpy(np.ascontiguousarray(a)).to(device, non_blocking=True)
                              for a in (self.members, self.shared_tokens, self.first_token))
        return self

    def bind(self, members: torch.Tensor, shared_tokens: torch.Tensor, first_token: torch.Tensor) -> "SharePlan":
        """Uses caller-owned device tensors that already hold (or, in stream
        order before the call that reads them, will hold) this plan's arrays,
        e.g. filled by asynchronous copies from pinned host buffers."""
        if self.n_groups > 0:
            self._dev = (members, shared_tokens, first_token)
        return self

    @property
    def nbytes(self) -> int:
        """Bytes the device copy takes (0 without groups)."""
        return 0 if self.n_groups == 0 else self.members.nbytes + self.shared_tokens.nbytes + self.first_token.nbytes

    def ref(self):
        if self.n_groups == 0:
            return None
        if self._dev is None:
            raise ValueError("SharePlan.to(device) first")
        m, sh, ft = self._dev
        self._struct = pa_share_plan_t(m.data_ptr(), sh.data_ptr(), ft.data_ptr(), self.n_groups, self.max_members)
        return ctypes.byref(self._struct)


def share_plan(tables, lens, block_size: int, max_members: int = 4) -> SharePlan:
    """Host: groups the sequences of a batch whose tables agree on their
    leading blocks (pa_share_plan)."""
    tables = np.ascontiguousarray(np.asarray(tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    n = len(lens)
    cap = max(1, n // 2)
    members = np.empty((cap, max_members), dtype=np.int32)
    shared = np.empty(cap, dtype=np.int32)
    first = np.empty(n, dtype=np.int32)
    ng = ctypes.c_int32(0)
    _check(_lib.pa_share_plan(_i32p(tables), tables.shape[1] if tables.ndim == 2 else 0, _i32p(lens), n,
                              int(block_size), int(max_members), _i32p(members), _i32p(shared),
                              _i32p(first), ctypes.byref(ng)), "pa_share_plan")
    g = ng.value
    return SharePlan(members[:g].copy(), shared[:g].copy(), first)


def pa_decode_shared(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor, context_lens: torch.Tensor,
                     max_context_len: int, scale: float, plan: SharePlan | None = None,
                     k_new: torch.Tensor | None = None, v_new: torch.Tensor | None = None,
                     cow_src: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """pa_decode, or pa_append_decode when k_new / v_new are given, with the
    blocks a plan's groups share read once for all their members."""
    _check_q_out(q, out, cache)
    B, Hq, D = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    row_shape = (B, cache.num_kv_heads, D)
    if k_new is not None and (tuple(k_new.shape) != row_shape or tuple(v_new.shape) != row_shape):
        raise ValueError(f"k_new and v_new must be {list(row_shape)}")
    if out is None:
        out = torch.empty_like(q)
    size = (pa_decode_shared_workspace_size if plan is not None and plan.n_groups > 0
            else pa_decode_workspace_size)
    need = size(B, Hq, int(max_context_len), D, cache.partition_tokens)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode_shared(
        _dev(k_new, "k_new", cache.dtype) if k_new is not None else None,
        _dev(v_new, "v_new", cache.dtype) if v_new is not None else None,
        _dev(cow_src, "cow_src", torch.int32) if cow_src is not None else None,
        _dev(q, "q", cache.dtype), cache.ref(), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32), B, Hq, int(max_context_len),
        float(scale), plan.ref() if plan is not None else None, _dev(out, "out", cache.dtype), ws_ptr, ws_bytes,
        _stream_ptr(stream)), "pa_decode_shared")
    return out


def pa_prefill(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor, context_lens: torch.Tensor,
               query_starts: torch.Tensor, max_context_len: int, scale: float, max_query_len: int | None = None,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Paged chunked-prefill attention: the last query_starts[b+1] -
    query_starts[b] tokens of sequence b (already in the cache) attend
    causally to the sequence; q and out are [total, Hq, 128] bf16."""
    _check_q_out(q, out, cache)
    T, Hq, D = q.shape
    B = context_lens.shape[0]
    if block_tables.dim() != 2 or block_tables.shape[0] != B or query_starts.shape != (B + 1,):
        raise ValueError("block_tables must be [B, max_blocks] and query_starts [B + 1]")
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.pa_prefill(_dev(q, "q", cache.dtype), cache.ref(), _dev(block_tables, "block_tables", torch.int32),
                           block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32),
                           _dev(query_starts, "query_starts", torch.int32), B, Hq, T,
                           int(T if max_query_len is None else max_query_len), int(max_context_len), float(scale),
                           _dev(out, "out", cache.dtype), _stream_ptr(stream)), "pa_prefill")
    return out


PA_STATIC_WORKSPACE_BYTES = 8 << 20


def pa_decode_static_workspace(q: torch.Tensor, cache: KVCache, block_tables: torch.Tensor,
                               context_lens: torch.Tensor, max_context_len: int, scale: float,
                               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """pa_decode with the library's fixed scratch array instead of a
    workspace (for callers that cannot allocate device memory); raises
    PagedAttnError (buffer too small) past PA_STATIC_WORKSPACE_BYTES."""
    _check_q_out(q, out, cache)
    B, Hq, D = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("block_tables must be [B, max_blocks] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.pa_decode_static_workspace(
        _dev(q, "q", cache.dtype), cache.ref(), _dev(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], _dev(context_lens, "context_lens", torch.int32), B, Hq, int(max_context_len),
        float(scale), _dev(out, "out", cache.dtype), _stream_ptr(stream)), "pa_decode_static_workspace")
    return out


def pa_copy_blocks(src_dst_pairs: torch.Tensor, cache: KVCache, stream=None) -> None:
    """Copies whole blocks of both pools: pairs [n, 2] int32 (src, dst) on the device."""
    n = src_dst_pairs.shape[0] if src_dst_pairs.numel() else 0
    if n and (src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2):
        raise ValueError("pairs must be [n, 2]")
    _check(_lib.pa_copy_blocks(_dev(src_dst_pairs, "pairs", torch.int32) if n else None, n, cache.ref(),
                               _stream_ptr(stream)), "pa_copy_blocks")


def pa_check_copy_pairs(pairs, num_blocks: int) -> bool:
    a = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    return _lib.pa_check_copy_pairs(_i32p(a), a.shape[0], int(num_blocks)) == PA_OK


def pa_read_wait_timeout(stream=None) -> list:
    """Synchronises the stream; returns (and clears) [taken, mbarrier shared
    address, parity | block << 1, thread] of the first wait that gave up."""
    info = (ctypes.c_uint32 * 4)()
    _check(_lib.pa_read_wait_timeout(_stream_ptr(stream), info), "pa_read_wait_timeout")
    return list(info)


def pa_read_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error bits."""
    bits = ctypes.c_int32(0)
    _check(_lib.pa_read_device_error(_stream_ptr(stream), ctypes.byref(bits)), "pa_read_device_error")
    return bits.value


# --------------------------------------------------------------------------
# one decode step from pinned host buffers


class DecodeStepper:
    """Decode steps of a fixed batch of sequences from pinned host buffers,
    one native call per step (pa_decode_step): the allocator's step, one
    copy of the inputs to the device, the fused copy-on-write + append +
    decode, and the copy of the output back.  `slots` step slots (default 2)
    alternate, so the host prepares step i + 1 while the device runs step i.

    Per step: ``q, k_new, v_new = stepper.inputs()`` gives the next slot's
    pinned input views (after waiting for that slot's previous step), the
    caller fills them, ``stepper.step(seqs)`` launches, and
    ``stepper.output(slot)`` is that slot's pinned output once
    ``stepper.wait(slot)`` returned."""

    def __init__(self, alloc: "Allocator", cache: KVCache, n_seqs: int, num_q_heads: int, max_blocks: int,
                 scale: float, share_max_members: int = 4, slots: int = 2, stream=None, h2d_stream=None,
                 d2h_stream=None):
        self.alloc, self.cache = alloc, cache
        self.n, self.Hq, self.max_blocks = int(n_seqs), int(num_q_heads), int(max_blocks)
        self.share, self.scale = int(share_max_members), float(scale)
        dev = cache.k.device
        lay = pa_step_layout_t()
        _check(_lib.pa_step_layout(self.n, self.Hq, cache.ref(), self.max_blocks, self.share, ctypes.byref(lay)),
               "pa_step_layout")
        self.layout = lay
        size = pa_decode_shared_workspace_size if self.share > 0 else pa_decode_workspace_size
        ws_bytes = max(16, size(self.n, self.Hq, self.max_blocks * cache.block_size, cache.head_dim,
                                cache.partition_tokens))
        Hkv, D, dt = cache.num_kv_heads, cache.head_dim, cache.dtype
        self._slots = []
        for _ in range(int(slots)):
            host = torch.zeros(lay.bytes, dtype=torch.uint8).pin_memory()
            devb = torch.empty(lay.bytes, dtype=torch.uint8, device=dev)
            out_host = torch.empty(self.n, self.Hq, D, dtype=dt).pin_memory()
            out_dev = torch.empty(self.n, self.Hq, D, dtype=dt, device=dev)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            st = pa_step_slot_t(host.data_ptr(), devb.data_ptr(), out_host.data_ptr(), out_dev.data_ptr(),
                                ws.data_ptr(), ws_bytes, None, None, None)
            _check(_lib.pa_step_slot_events(ctypes.byref(st)), "pa_step_slot_events")

            def view(off, shape):
                nb = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
                return host[off:off + nb].view(dt).view(shape)
            self._slots.append({"struct": st, "keep": (host, devb, out_host, out_dev, ws), "out_host": out_host,
                                "q": view(lay.q, (self.n, self.Hq, D)), "k": view(lay.k_new, (self.n, Hkv, D)),
                                "v": view(lay.v_new, (self.n, Hkv, D))})
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        # inputs and outputs on streams of their own, so that step i + 1's
        # inputs do not queue behind step i's output copy
        self.h2d_stream = h2d_stream if h2d_stream is not None else torch.cuda.Stream(device=dev)
        self.d2h_stream = d2h_stream if d2h_stream is not None else torch.cuda.Stream(device=dev)
        self.i = 0
        self.h2d_bytes = lay.bytes
        self.d2h_bytes = self.n * self.Hq * D * torch.tensor([], dtype=dt).element_size()

    @property
    def next_slot(self) -> int:
        return self.i % len(self._slots)

    def wait(self, slot: int) -> None:
        """Until the slot's last step has its inputs on the device and its
        output on the host."""
        _check(_lib.pa_step_slot_wait(ctypes.byref(self._slots[slot]["struct"])), "pa_step_slot_wait")

    def inputs(self):
        """(q, k_new, v_new) pinned views of the next slot, after waiting for
        its previous step."""
        S = self._slots[self.next_slot]
        self.wait(self.next_slot)
        return S["q"], S["k"], S["v"]

    def output(self, slot: int) -> torch.Tensor:
        return self._slots[slot]["out_host"]

    def step(self, seqs) -> dict:
        """Launches one step through the next slot; returns the slot index,
        the step's copies on write, plan groups and longest context."""
        seqs = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        if len(seqs) != self.n:
            raise ValueError(f"a stepper of {self.n} sequences got {len(seqs)}")
        k = self.next_slot
        nc, ng, ml = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
        _check(_lib.pa_decode_step(self.alloc._h, _i32p(seqs), self.n, self.max_blocks, self.share,
                                   self.cache.ref(), self.Hq, self.scale, ctypes.byref(self._slots[k]["struct"]),
                                   self.stream.cuda_stream, self.h2d_stream.cuda_stream,
                                   self.d2h_stream.cuda_stream, ctypes.byref(nc),
                                   ctypes.byref(ng), ctypes.byref(ml)), "pa_decode_step")
        self.i += 1
        return {"slot": k, "n_copies": nc.value, "n_groups": ng.value, "max_len": ml.value}

    def close(self) -> None:
        """Waits for every slot and releases their events."""
        for k, S in enumerate(self._slots):
            if S["struct"].ev_in:
                self.wait(k)
                _check(_lib.pa_step_slot_release(ctypes.byref(S["struct"])), "pa_step_slot_release")

    def __del__(self):
        try:
            if _lib is not None:
                self.close()
        except Exception:
            pass


# --------------------------------------------------------------------------
# the host allocator


class Allocator:
    """Reference-counted block allocator (C++), copy on write of shared partial blocks."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        h = ctypes.c_void_p()
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if self._order.shape != (self.num_blocks,):
                raise ValueError("free_order must list every block once")
            order = _i32p(self._order)
        _check(_lib.pa_alloc_create(self.num_blocks, self.block_size, order, ctypes.byref(h)), "pa_alloc_create")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.pa_alloc_destroy(h)
            self._h = None

    def decode_step(self, seqs, max_blocks: int, share_max_members: int = 4, out: dict | None = None) -> dict:
        """One decode step's host work in one call (pa_decode_step_prepare):
        one token appended to every sequence, then the tables, lengths,
        copy-on-write sources and sharing plan that pa_decode_shared takes.
        `out` may hold preallocated int32 arrays ("tables" [n, max_blocks],
        "lens", "cow_src", "first_token" [n], "members" [n // 2, m],
        "shared_tokens" [n // 2]); returns them (members / shared_tokens
        trimmed to the groups) with
        "n_groups", "n_copies" and "max_len"."""
        seqs = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        n = len(seqs)
        m = max(int(share_max_members), 1)
        o = out if out is not None else {
            "tables": np.empty((n, max_blocks), np.int32), "lens": np.empty(n, np.int32),
            "cow_src": np.empty(n, np.int32), "first_token": np.empty(n, np.int32),
            "members": np.empty((max(1, n // 2), m), np.int32), "shared_tokens": np.empty(max(1, n // 2), np.int32)}
        ng, nc, ml = ctypes.c_int32(0), ctypes.c_int32(0), ctypes.c_int32(0)
        _check(_lib.pa_decode_step_prepare(self._h, _i32p(seqs), n, int(max_blocks), int(share_max_members),
                                           _i32p(o["tables"]), _i32p(o["lens"]), _i32p(o["cow_src"]),
                                           _i32p(o["members"]), _i32p(o["shared_tokens"]), _i32p(o["first_token"]),
                                           ctypes.byref(ng), ctypes.byref(nc), ctypes.byref(ml)), "pa_decode_step_prepare")
        res = dict(o)
        res["members"], res["shared_tokens"] = o["members"][:ng.value], o["shared_tokens"][:ng.value]
        res.update(n_groups=ng.value, n_copies=nc.value, max_len=ml.value)
        return res

    def new_seq(self) -> int:
        s = ctypes.c_int32()
        _check(_lib.pa_seq_new(self._h, ctypes.byref(s)), "pa_seq_new")
        return s.value

    def fork(self, parent: int) -> int:
        s = ctypes.c_int32()
        _check(_lib.pa_seq_fork(self._h, int(parent), ctypes.byref(s)), "pa_seq_fork")
        return s.value

    def free_seq(self, seq: int) -> None:
        _check(_lib.pa_seq_free(self._h, int(seq)), "pa_seq_free")

    def append(self, seq: int, n: int):
        """Returns (slots int64 [n], cow pair (src, dst) or None)."""
        slots = np.empty(max(n, 1), dtype=np.int64)
        pair = np.empty(2, dtype=np.int32)
        ncow = ctypes.c_int32()
        _check(_lib.pa_seq_append(self._h, int(seq), int(n), _i64p(slots), _i32p(pair), ctypes.byref(ncow)),
               "pa_seq_append")
        return slots[:n], ((int(pair[0]), int(pair[1])) if ncow.value else None)

    def batch_append(self, seqs, n_tokens, out_slots: np.ndarray | None = None, out_pairs: np.ndarray | None = None):
        """Returns (slots int64 [sum n], cow pairs int32 [k, 2])."""
        seqs = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        n_tokens = np.ascontiguousarray(np.asarray(n_tokens, dtype=np.int32))
        total = int(n_tokens.sum())
        slots = out_slots if out_slots is not None else np.empty(max(total, 1), dtype=np.int64)
        pairs = out_pairs if out_pairs is not None else np.empty((max(len(seqs), 1), 2), dtype=np.int32)
        ncow = ctypes.c_int32()
        _check(_lib.pa_batch_append(self._h, _i32p(seqs), _i32p(n_tokens), len(seqs), _i64p(slots),
                                    _i32p(pairs), ctypes.byref(ncow)), "pa_batch_append")
        return slots[:total], pairs[:ncow.value]

    def seq_len(self, seq: int):
        n, nb = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.pa_seq_len(self._h, int(seq), ctypes.byref(n), ctypes.byref(nb)), "pa_seq_len")
        return n.value, nb.value

    def block_table(self, seq: int) -> list:
        _, nb = self.seq_len(seq)
        out = np.empty(max(nb, 1), dtype=np.int32)
        cnt = ctypes.c_int32()
        _check(_lib.pa_seq_block_table(self._h, int(seq), _i32p(out), nb, ctypes.byref(cnt)), "pa_seq_block_table")
        return out[:cnt.value].tolist()

    def max_len(self, seqs):
        """(longest length in tokens, most blocks) over the sequences."""
        seqs = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        ml, mb = ctypes.c_int32(), ctypes.c_int32()
        _check(_lib.pa_seqs_max_len(self._h, _i32p(seqs), len(seqs), ctypes.byref(ml), ctypes.byref(mb)),
               "pa_seqs_max_len")
        return ml.value, mb.value

    def build_block_tables(self, seqs, max_blocks: int, pad: int = -1, out_tables=None, out_lens=None):
        seqs = np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
        tables = out_tables if out_tables is not None else np.empty((len(seqs), max_blocks), dtype=np.int32)
        lens = out_lens if out_lens is not None else np.empty(len(seqs), dtype=np.int32)
        _check(_lib.pa_build_block_tables(self._h, _i32p(seqs), len(seqs), int(max_blocks), int(pad),
                                          _i32p(tables), _i32p(lens)), "pa_build_block_tables")
        return tables, lens

    def stats(self) -> dict:
        used, alloc = ctypes.c_int64(), ctypes.c_int64()
        free, usedb = ctypes.c_int32(), ctypes.c_int32()
        frag = ctypes.c_double()
        _check(_lib.pa_alloc_stats(self._h, ctypes.byref(used), ctypes.byref(alloc), ctypes.byref(free),
                                   ctypes.byref(usedb)), "pa_alloc_stats")
        _check(_lib.pa_alloc_fragmentation(self._h, ctypes.byref(frag)), "pa_alloc_fragmentation")
        return dict(used_slots=used.value, allocated_slots=alloc.value, free_blocks=free.value,
                    used_blocks=usedb.value, fragmentation=frag.value)

    def refcount(self, block: int) -> int:
        r = ctypes.c_int32()
        _check(_lib.pa_block_refcount(self._h, int(block), ctypes.byref(r)), "pa_block_refcount")
        return r.value

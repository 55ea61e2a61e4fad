"""Oracle for the paged KV-cache decode path: plain, slow, obviously correct.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports it, and this package
imports nothing from the product.  It works on host arrays only.

Sources, by page and section:

* "PagedAttention Internals" (wondering.app lesson):
  - "Fixed-Size KV Blocks": a sequence's cache is a list of fixed-size blocks;
    tokens fill the current block and another block is taken when it is full;
    unused capacity is confined to the incomplete last block.
  - "The Block Table Map": a per-sequence table maps logical block n to a
    physical block (the example maps logical 0, 1, 2 to physical 8, 3, 11);
    the attention step reads through the table; the logical order is kept.
  - "Sharing And Dynamic Growth": sequences obtain blocks as they need them
    and release them when they finish.
* "pagedattention" glossary entry (chipfoundryservices.com):
  - paragraph 3 (block tables): blocks of 16 tokens as the example, given to
    a request one at a time as it grows.
  - the comparison table and paragraph 5 (sharing): a common prompt prefix or
    the samples of a beam search point at the same physical blocks and are
    copied on write only when they diverge.
* learn-ml-visualized chapter "inference-acceleration-pagedattention-vllm", the
  fragmentation worked example:
  waste = allocated - used, fragmentation = total waste / total allocated;
  naive scheme reserves a fixed number of slots per sequence, paged scheme
  allocates whole pages of a fixed size as the sequence grows.

Readings where the pages are silent (each also listed in the design notes):

* attention is the textbook scaled dot-product step, softmax(scale q K^T) V,
  taken in float64 as a two-pass softmax;
* query head h reads KV head h // (Hq // Hkv);
* cache layout [num_blocks, Hkv, block_size, head_dim];
* a context length of 0 gives a zero output row; a negative slot is skipped;
* the free list hands blocks out in a caller-given order and takes released
  blocks back last-in first-out; a writer copies a partially filled last block
  iff its reference count is above one at its turn, in batch order.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2

_lib = None


def load(path: str) -> ctypes.CDLL:
    """Loads a build of the C oracle and declares its entry points."""
    L = ctypes.CDLL(path)
    vp, i32p, f64p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)
    L.oracle_decode.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, i32p, ctypes.c_int, i32p,
                                ctypes.c_int, ctypes.c_int, ctypes.c_double, i32p,
                                ctypes.c_int, f64p]
    L.oracle_decode.restype = ctypes.c_int
    L.oracle_decode_partials.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, i32p,
                                         ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_int,
                                         f64p, f64p, f64p]
    L.oracle_decode_partials.restype = ctypes.c_int
    L.oracle_merge_partials.argtypes = [f64p, f64p, f64p, i32p, ctypes.c_int64,
                                        ctypes.c_int, ctypes.c_int, f64p]
    L.oracle_merge_partials.restype = None
    L.oracle_prefill.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                 ctypes.c_int, ctypes.c_int, i32p, ctypes.c_int, i32p, i32p,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_double, i32p, ctypes.c_int, f64p]
    L.oracle_prefill.restype = ctypes.c_int
    L.oracle_set_threads.argtypes = [ctypes.c_int]
    L.oracle_max_threads.restype = ctypes.c_int
    return L


def lib() -> ctypes.CDLL:
    """Loads (building first if needed) the C part of the oracle."""
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_max_threads())


# --------------------------------------------------------------------------
# element access


def host_array(x):
    """Returns (contiguous numpy array, element-type code) for a host tensor.

    bfloat16 data travel as their raw 16-bit patterns (numpy has no bfloat16).
    """
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), BF16
        if x.dtype == torch.float32:
            return x.numpy(), F32
        if x.dtype == torch.float64:
            return x.numpy(), F64
        raise TypeError(f"unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    raise TypeError(f"unsupported dtype {x.dtype}")


def widen(x) -> np.ndarray:
    """Exact float64 copy of a float32 / float64 / bfloat16-pattern array."""
    a, code = host_array(x)
    if code == BF16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# --------------------------------------------------------------------------
# attention


def decode(q, k_cache, v_cache, block_tables, context_lens, scale, rows=None) -> np.ndarray:
    """Paged decode attention in float64 (the C oracle).

    q [B, Hq, D], caches [num_blocks, Hkv, bs, D] (same element type as q),
    block_tables [B, max_blocks] int32, context_lens [B] int32.
    Returns [B, Hq, D] float64, or [len(rows), D] for rows = [(b, h), ...].
    """
    qa, qc = host_array(q)
    ka, kc = host_array(k_cache)
    va, vc = host_array(v_cache)
    if not (qc == kc == vc):
        raise TypeError("q, k_cache and v_cache must share one element type")
    B, Hq, D = qa.shape
    NB, Hkv, bs, D2 = ka.shape
    if D2 != D or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    tables = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    if tables.ndim != 2 or tables.shape[0] != B or lens.shape != (B,):
        raise ValueError("table / length shape mismatch")
    if rows is None:
        out = np.zeros((B, Hq, D), dtype=np.float64)
        rows_a, n_rows = None, 0
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
        n_rows = rows_a.shape[0]
        out = np.zeros((n_rows, D), dtype=np.float64)
    rc = lib().oracle_decode(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, qc, NB, Hkv, bs, D,
        _ptr(tables, ctypes.c_int32), tables.shape[1], _ptr(lens, ctypes.c_int32), B, Hq,
        float(scale), None if rows_a is None else _ptr(rows_a, ctypes.c_int32), n_rows,
        _ptr(out, ctypes.c_double))
    if rc:
        raise ValueError(f"oracle_decode rejected its input (code {rc})")
    return out


def prefill(q, k_cache, v_cache, block_tables, context_lens, query_starts, scale, rows=None) -> np.ndarray:
    """Paged chunked-prefill attention in float64 (the C oracle).

    The last n_b = query_starts[b+1] - query_starts[b] tokens of sequence b
    (context_lens[b] tokens in all) are new; their queries are rows
    query_starts[b] .. query_starts[b+1]-1 of q [total, Hq, D], and each
    attends causally to the sequence's tokens up to its own position.
    Returns [total, Hq, D] float64, or [len(rows), D] for rows = [(j, h), ...].
    """
    qa, qc = host_array(q)
    ka, kc = host_array(k_cache)
    va, vc = host_array(v_cache)
    if not (qc == kc == vc):
        raise TypeError("q, k_cache and v_cache must share one element type")
    T, Hq, D = qa.shape
    NB, Hkv, bs, D2 = ka.shape
    if D2 != D or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    tables = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    qs = np.ascontiguousarray(np.asarray(query_starts, dtype=np.int32))
    B = lens.shape[0]
    if tables.ndim != 2 or tables.shape[0] != B or qs.shape != (B + 1,) or int(qs[-1]) != T:
        raise ValueError("table / length / query start shape mismatch")
    if rows is None:
        out = np.zeros((T, Hq, D), dtype=np.float64)
        rows_a, n_rows = None, 0
    else:
        rows_a = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 2))
        n_rows = rows_a.shape[0]
        out = np.zeros((n_rows, D), dtype=np.float64)
    rc = lib().oracle_prefill(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, qc, NB, Hkv, bs, D,
        _ptr(tables, ctypes.c_int32), tables.shape[1], _ptr(lens, ctypes.c_int32), _ptr(qs, ctypes.c_int32),
        B, Hq, float(scale), None if rows_a is None else _ptr(rows_a, ctypes.c_int32), n_rows,
        _ptr(out, ctypes.c_double))
    if rc:
        raise ValueError(f"oracle_prefill rejected its input (code {rc})")
    return out


def decode_partials(q, k_cache, v_cache, block_tables, context_lens, scale, partition_size):
    """Per-partition (m, l, acc) in float64; see oracle_decode_partials.

    Returns m [B, Hq, P], l [B, Hq, P], acc [B, Hq, P, D] and nparts [B]
    (entries past a sequence's last partition are NaN).
    """
    qa, qc = host_array(q)
    ka, _ = host_array(k_cache)
    va, _ = host_array(v_cache)
    B, Hq, D = qa.shape
    NB, Hkv, bs, _ = ka.shape
    tables = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    nparts = (lens.astype(np.int64) + partition_size - 1) // partition_size
    P = max(1, int(nparts.max()) if B else 1)
    m = np.full((B, Hq, P), np.nan)
    l = np.full((B, Hq, P), np.nan)
    acc = np.full((B, Hq, P, D), np.nan)
    rc = lib().oracle_decode_partials(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, qc, NB, Hkv, bs, D,
        _ptr(tables, ctypes.c_int32), tables.shape[1], _ptr(lens, ctypes.c_int32), B, Hq,
        float(scale), int(partition_size), P, _ptr(m, ctypes.c_double),
        _ptr(l, ctypes.c_double), _ptr(acc, ctypes.c_double))
    if rc:
        raise ValueError(f"oracle_decode_partials rejected its input (code {rc})")
    return m, l, acc, nparts.astype(np.int32)


def merge_partials(m, l, acc, nparts) -> np.ndarray:
    """Log-sum-exp combine of decode_partials' output -> [B, Hq, D] float64."""
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    B, Hq, P, D = acc.shape
    rows_np = np.ascontiguousarray(np.repeat(np.asarray(nparts, dtype=np.int32), Hq))
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lib().oracle_merge_partials(_ptr(m, ctypes.c_double), _ptr(l, ctypes.c_double),
                                _ptr(acc, ctypes.c_double), _ptr(rows_np, ctypes.c_int32),
                                B * Hq, P, D, _ptr(out, ctypes.c_double))
    return out


def decode_bruteforce(q, k_cache, v_cache, slot_lists, scale):
    """Pure-Python loops over explicit per-sequence slot lists (tiny inputs).

    slot_lists[b] lists, in logical order, the flat slots
    (physical block * block_size + offset) of sequence b's tokens.  This path
    never looks at a block table.
    """
    qd, kd, vd = widen(q), widen(k_cache), widen(v_cache)
    B, Hq, D = qd.shape
    _, Hkv, bs, _ = kd.shape
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    for b in range(B):
        slots = list(slot_lists[b])
        for h in range(Hq):
            g = h // G
            if not slots:
                continue
            logits = []
            for s in slots:
                blk, off = divmod(int(s), bs)
                dot = 0.0
                for d in range(D):
                    dot += float(qd[b, h, d]) * float(kd[blk, g, off, d])
                logits.append(scale * dot)
            top = max(logits)
            w = [math.exp(x - top) for x in logits]
            tot = math.fsum(w)
            for d in range(D):
                acc = 0.0
                for wi, s in zip(w, slots):
                    blk, off = divmod(int(s), bs)
                    acc += wi * float(vd[blk, g, off, d])
                out[b, h, d] = acc / tot
    return out


# --------------------------------------------------------------------------
# append and block copy (bit copies)


def append_kv(k_cache: np.ndarray, v_cache: np.ndarray, k, v, slot_mapping) -> None:
    """Writes token i's key/value rows at slot_mapping[i], in place.

    Caches are [num_blocks, Hkv, bs, D] host arrays (bfloat16 as uint16,
    float32 as float32); k, v are [N, Hkv, D] of the same element type.  A
    negative slot is padding and is skipped.  Slots past the pool raise.
    """
    ka, _ = host_array(k)
    va, _ = host_array(v)
    NB, Hkv, bs, D = k_cache.shape
    for i, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s < 0:
            continue
        blk, off = divmod(s, bs)
        if blk >= NB:
            raise IndexError(f"slot {s} is past the pool")
        k_cache[blk, :, off, :] = ka[i]
        v_cache[blk, :, off, :] = va[i]


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs) -> None:
    """Copy-on-write block copies: block dst becomes a copy of block src."""
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]


# --------------------------------------------------------------------------
# fragmentation (the worked example of the learn-ml-visualized chapter)


@dataclass
class Usage:
    allocated: int
    used: int

    @property
    def wasted(self) -> int:
        return self.allocated - self.used

    @property
    def fragmentation(self) -> float:
        return self.wasted / self.allocated if self.allocated else 0.0


def naive_usage(lengths, reserve: int) -> Usage:
    """Every sequence holds a fixed reservation of `reserve` slots."""
    lengths = [int(x) for x in lengths]
    if any(L > reserve or L < 0 for L in lengths):
        raise ValueError("a length exceeds the fixed reservation")
    return Usage(allocated=reserve * len(lengths), used=sum(lengths))


def paged_usage(lengths, page_size: int) -> Usage:
    """Every sequence holds whole pages, as many as its tokens need."""
    lengths = [int(x) for x in lengths]
    if any(L < 0 for L in lengths):
        raise ValueError("negative length")
    pages = sum(-(-L // page_size) for L in lengths)
    return Usage(allocated=page_size * pages, used=sum(lengths))


# --------------------------------------------------------------------------
# block allocator model


class OutOfBlocks(Exception):
    pass


@dataclass
class AllocatorModel:
    """Reference-counted block allocator, one block at a time, copy on write.

    free_order: the order in which never-used blocks are handed out (a
    permutation of range(num_blocks)); released blocks are handed out again
    before those, most recently released first.
    """

    num_blocks: int
    block_size: int
    free_order: list | None = None
    free: list = field(init=False)
    ref: list = field(init=False)
    tables: dict = field(init=False, default_factory=dict)
    lens: dict = field(init=False, default_factory=dict)
    next_id: int = field(init=False, default=0)

    def __post_init__(self):
        order = list(range(self.num_blocks)) if self.free_order is None else [int(x) for x in self.free_order]
        if sorted(order) != list(range(self.num_blocks)):
            raise ValueError("free_order must be a permutation of the blocks")
        self.free = list(reversed(order))  # top of the stack is the end
        self.ref = [0] * self.num_blocks

    # -- sequences
    def new_seq(self) -> int:
        sid = self.next_id
        self.next_id += 1
        self.tables[sid] = []
        self.lens[sid] = 0
        return sid

    def fork(self, parent: int) -> int:
        sid = self.new_seq()
        self.tables[sid] = list(self.tables[parent])
        self.lens[sid] = self.lens[parent]
        for blk in self.tables[sid]:
            self.ref[blk] += 1
        return sid

    def free_seq(self, sid: int) -> None:
        for blk in self.tables.pop(sid):
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
        del self.lens[sid]

    def _blocks_needed(self, sid: int, n: int, ref_taken: dict) -> int:
        if n <= 0:
            return 0
        pos, bs = self.lens[sid], self.block_size
        need = -(-(pos + n) // bs) - (-(-pos // bs))
        if pos % bs:
            last = self.tables[sid][-1]
            if self.ref[last] - ref_taken.get(last, 0) > 1:
                need += 1
                ref_taken[last] = ref_taken.get(last, 0) + 1
        return need

    def append(self, sid: int, n: int):
        """Appends n tokens; returns (slots, cow_pair or None)."""
        slots, cows = self.batch_append([sid], [n])
        return slots, (cows[0] if cows else None)

    def batch_append(self, sids, ns):
        """Appends ns[i] tokens to sids[i], in order; all or nothing.

        Returns the flat list of slots (sequence by sequence, token by token)
        and the list of (src, dst) copy-on-write pairs in the order made.
        """
        sids = [int(s) for s in sids]
        ns = [int(n) for n in ns]
        if len(set(sids)) != len(sids):
            raise ValueError("a sequence appears twice in one batch")
        taken: dict = {}
        need = sum(self._blocks_needed(s, n, taken) for s, n in zip(sids, ns))
        if need > len(self.free):
            raise OutOfBlocks(f"need {need} blocks, {len(self.free)} free")
        bs = self.block_size
        slots, cows = [], []
        for sid, n in zip(sids, ns):
            table = self.tables[sid]
            for _ in range(n):
                pos = self.lens[sid]
                if pos % bs == 0:
                    blk = self.free.pop()
                    self.ref[blk] = 1
                    table.append(blk)
                else:
                    last = table[-1]
                    if self.ref[last] > 1:
                        new = self.free.pop()
                        self.ref[new] = 1
                        self.ref[last] -= 1
                        table[-1] = new
                        cows.append((last, new))
                slots.append(table[pos // bs] * bs + pos % bs)
                self.lens[sid] = pos + 1
        return slots, cows

    # -- views
    def block_table(self, sid: int) -> list:
        return list(self.tables[sid])

    def used_blocks(self) -> int:
        return self.num_blocks - len(self.free)

    def usage(self) -> Usage:
        """Physical usage: each block in use counted once, with its fill."""
        bs = self.block_size
        fill: dict = {}
        for sid, table in self.tables.items():
            L = self.lens[sid]
            for j, blk in enumerate(table):
                f = min(bs, L - j * bs)
                if fill.setdefault(blk, f) != f:
                    raise AssertionError("sharers disagree on a shared block's fill")
        return Usage(allocated=bs * len(fill), used=sum(fill.values()))

    def seq_waste(self, sid: int) -> int:
        return self.block_size * len(self.tables[sid]) - self.lens[sid]

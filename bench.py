"""Benchmark of the paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa|shared-prefix|long-context|trace]

One step = one pass of the hot path over one batch: copy-on-write block
copies (when the allocator made any), the slot-mapped KV append of one new
token per sequence, and paged decode attention (partition kernel + LSE
reduce).  The host allocator's decisions for every step are made before the
timed region (their host time is reported separately and included in `e2e`).

Default workload: bf16 GQA decode, 32 sequences, 32 query / 8 KV heads,
head_dim 128, 16-token blocks, context lengths uniform in [128, 4096], a pool
of twice the needed blocks dealt from a seeded shuffle.  L2 (126 MB) is
defeated by rotating independent batch instances whose KV together exceed it
several times over.

value = KV bytes read by decode per second over the whole step (GB/s);
tokens/s and the roofline of the decode launch (partition + reduce) ride
along.  `--impl reference` times the float64 CPU oracle instead, on a bounded
sample of the same workload.

Multi-GPU: every rank runs its own independent replica (its own pool,
allocator and sequences; no collective on the data path) and value is the sum
over ranks divided by the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
METRIC = "paged decode KV-read GB/s (% of HBM peak) and decode tokens/s at 1 B200"


# ----------------------------------------------------------------- helpers


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s of this machine's B200s (burst: a kernel timed alone),
    from MEASURED_PEAKS.json, else the fallback figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the sources the partition kernel and its reduce are built from
    (not the cascade's, which they do not include); ties an ncu traffic
    figure to them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_402_b200", "csrc")
    for f in ("pa_decode_tc.cuh", "pa_decode_simt.cuh", "pa_device.cuh", "pa_tc.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, algo_bytes_per_launch: float):
    """Per-launch DRAM traffic (read + write bytes) of the step's kernels as an
    ncu capture of the current decode sources measured it, applied to this
    run's launches: the captured traffic / algorithmic-bytes ratio times this
    run's mean algorithmic bytes per launch (traffic grows in proportion to
    the K/V read).  None when no capture matches the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("kernel_hash") != kernel_source_hash():
        return None
    cap = rec["captured_launch"]
    ratio = (cap["dram_read_bytes"] + cap["dram_write_bytes"]) / cap["algorithmic_bytes"]
    return int(round(ratio * algo_bytes_per_launch))


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML by a thread as fast
    as NVML answers (every ~0.1 ms) while the timed region runs: the region
    is K steps of a few hundred microseconds each, so a slower rate would
    leave only a handful of samples."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, dev):
        self.dev = dev
        self.samples = []
        self.reason_bits = 0
        self.max_mhz = None
        self.error = None
        self._stop = None
        self._thread = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def __enter__(self):
        import threading
        try:
            nv, h = self._handle()
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            # the first calls of a query are slow: make them before the region
            nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception as e:  # NVML missing: report it, keep timing
            self.error = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    self.reason_bits |= nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception as e:
                    self.error = str(e)
                    return
                time.sleep(0.0001)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        time.sleep(0.005)
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        reasons = sorted(k for k, bit in self.REASONS.items() if self.reason_bits & bit)
        if self.error and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.error]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


def bandwidth_probes(dev, nbytes: int = 4 << 30, reps: int = 6):
    """HBM bandwidth measured in this job, outside the timed region, on a
    4 GiB buffer (32x the L2): a read-only stream (torch's sum of float32
    values: every byte read once, nothing written but the scalar) and a copy
    (read + write bytes of copy_ into a second buffer).  Best of three runs
    of `reps` launches each, CUDA events on the current stream.  Returns
    (read GB/s, copy GB/s)."""
    x = torch.ones(nbytes // 4, dtype=torch.float32, device=dev)
    y = torch.empty_like(x)
    acc = torch.empty((), dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def best(fn, bytes_per_rep):
        for _ in range(2):
            fn()
        out = 0.0
        for _ in range(3):
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            out = max(out, reps * bytes_per_rep / (e0.elapsed_time(e1) / 1e3) / 1e9)
        return out

    read = best(lambda: torch.sum(x, dim=0, dtype=torch.float32, out=acc), nbytes)
    copy = best(lambda: y.copy_(x), 2 * nbytes)
    del x, y
    torch.cuda.empty_cache()
    return read, copy


# ----------------------------------------------------------------- workload


def _fill_blocks_normal(cache, blocks, seed, dev, chunk=65536):
    """N(0,1) bf16 values in the listed pool blocks only (a pool much larger
    than what the batch uses is never read anywhere else)."""
    from paged_kv_cache_402_b200 import synth
    idx = torch.as_tensor(np.asarray(blocks, dtype=np.int64), device=dev)
    shape = tuple(cache.k.shape[1:])
    for i in range(0, len(idx), chunk):
        part = idx[i:i + chunk]
        cache.k.index_copy_(0, part, synth.normal((len(part),) + shape, torch.bfloat16, seed * 7919 + i, device=dev))
        cache.v.index_copy_(0, part, synth.normal((len(part),) + shape, torch.bfloat16, seed * 7919 + i + 1, device=dev))


def setup_independent(seed, wl, uses, dev):
    """Sequences of the workload's lengths; the pool is dealt from a seeded
    shuffle of all its blocks (pool_factor x the needed blocks, or a fixed
    pool size)."""
    import paged_kv_cache_402_b200 as pa
    from paged_kv_cache_402_b200 import synth
    B, Hkv, D, bs = wl["B"], wl["Hkv"], wl["D"], wl["bs"]
    lens = wl["lengths"](seed)
    need = int(sum(-(-(int(L) + uses) // bs) for L in lens))
    NB = wl.get("num_blocks") or int(math.ceil(need * wl.get("pool_factor", 2.0))) + 1
    order = synth.rng(seed + 1).permutation(NB)
    alloc = pa.Allocator(NB, bs, order)
    if wl.get("fill_used_only"):
        cache = pa.KVCache.empty(NB, Hkv, bs, D, torch.bfloat16, dev, partition_tokens=wl["part"])
        _fill_blocks_normal(cache, order[:need], seed, dev)
    else:
        cache = pa.KVCache(synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 2, device=dev),
                           synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 3, device=dev), wl["part"])
    seqs = [alloc.new_seq() for _ in range(B)]
    alloc.batch_append(seqs, lens)  # prompt blocks; the pool's contents stand in for the prompt rows
    return alloc, cache, [seqs]


def setup_shared_prefix(seed, wl, uses, dev):
    """Groups of 8 that share the blocks of a 512 + r token prefix (r in
    [1, 15], so the prefix ends inside a shared block); each member then
    appends its own lognormal suffix, which makes 7 members per group copy
    that block (the copies are made on the device here, in set-up)."""
    import paged_kv_cache_402_b200 as pa
    from paged_kv_cache_402_b200 import synth
    Hkv, D, bs, gsz = wl["Hkv"], wl["D"], wl["bs"], wl["group_size"]
    groups = wl["B"] // gsz
    pl, suffix, order, NB = synth.shared_prefix_layout(seed, groups=groups, group_size=gsz, prefix=512,
                                                       median=800, clip=8192, bs=bs, pool_factor=1.25,
                                                       prefix_tail=True)
    NB += wl["B"] * (-(-uses // bs) + 1)
    order = np.concatenate([order, np.arange(len(order), NB)]).astype(np.int32)
    alloc = pa.Allocator(NB, bs, order)
    cache = pa.KVCache(synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 2, device=dev),
                       synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 3, device=dev), wl["part"])
    roots = [alloc.new_seq() for _ in range(groups)]
    alloc.batch_append(roots, pl)
    seqs = []
    for r in roots:
        seqs += [r] + [alloc.fork(r) for _ in range(gsz - 1)]
    _, pairs = alloc.batch_append(seqs, suffix)
    if len(pairs):
        pa.pa_copy_blocks(torch.from_numpy(np.ascontiguousarray(pairs)).to(dev), cache)
    return alloc, cache, [seqs]


def setup_cow_steps(seed, wl, uses, dev):
    """One fresh set of groups per step: each group's 8 members share a
    512 + r token prefix that ends inside a block, so the step's append of
    one token to every member copies that block for 7 of them."""
    import paged_kv_cache_402_b200 as pa
    from paged_kv_cache_402_b200 import synth
    Hkv, D, bs, gsz = wl["Hkv"], wl["D"], wl["bs"], wl["group_size"]
    groups = wl["B"] // gsz
    per_set = groups * (-(-(512 + bs) // bs) + gsz)
    NB = uses * per_set + 1
    order = synth.rng(seed + 1).permutation(NB)
    alloc = pa.Allocator(NB, bs, order)
    cache = pa.KVCache(synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 2, device=dev),
                       synth.normal((NB, Hkv, bs, D), torch.bfloat16, seed + 3, device=dev), wl["part"])
    r = synth.rng(seed + 5)
    sets = []
    for _ in range(uses):
        roots = [alloc.new_seq() for _ in range(groups)]
        alloc.batch_append(roots, 512 + r.integers(1, bs, size=groups))
        seqs = []
        for root in roots:
            seqs += [root] + [alloc.fork(root) for _ in range(gsz - 1)]
        sets.append(seqs)
    return alloc, cache, sets


class Instance:
    """One independent workload instance: pool, allocator, sequences, and the
    inputs of `uses` steps (slots, copy pairs, tables, lengths, q and new
    rows), all made before any timing."""

    def __init__(self, seed: int, wl: dict, uses: int, dev, extra: int = 0):
        import paged_kv_cache_402_b200 as pa
        from paged_kv_cache_402_b200 import synth

        self.wl = wl
        B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
        dt = torch.bfloat16
        t0 = time.perf_counter()
        self.alloc, self.cache, self.sets = wl["setup"](seed, wl, uses + extra, dev)
        self.uses = uses
        torch.cuda.synchronize()
        self.setup_s = time.perf_counter() - t0
        lens_now = [self.alloc.seq_len(q)[0] for q in self.sets[0]]
        self.lens0 = np.array(lens_now, dtype=np.int32)
        self.max_blocks = int(-(-(int(max(max(self.alloc.seq_len(q)[0] for q in st) for st in self.sets))
                                  + uses + extra + 1) // bs))
        self.steps = []
        self.host_alloc_s = 0.0
        row_bytes = 2 * Hkv * D * 2
        for u in range(uses):
            seqs = self.sets[u % len(self.sets)]
            t1 = time.perf_counter()
            slots, pairs = self.alloc.batch_append(seqs, np.ones(B, np.int32))
            tables, lens = self.alloc.build_block_tables(seqs, self.max_blocks)
            cow = pa.cow_sources(pairs, tables, lens, bs)
            plan = pa.share_plan(tables, lens, bs)
            self.host_alloc_s += time.perf_counter() - t1
            nblk = (lens.astype(np.int64) + bs - 1) // bs
            # unique bytes: every physical block once, with its fill
            fill = {}
            for i in range(B):
                for j in range(int(nblk[i])):
                    fill.setdefault(int(tables[i, j]), min(bs, int(lens[i]) - j * bs))
            st = {
                "seqs": seqs,
                "slots": torch.from_numpy(slots.copy()).to(dev),
                "pairs": torch.from_numpy(np.ascontiguousarray(pairs)).to(dev) if len(pairs) else None,
                "cow": torch.from_numpy(cow).to(dev) if len(pairs) else None,
                "plan": plan.to(dev),
                "n_pairs": len(pairs),
                "tables": torch.from_numpy(tables).to(dev),
                "lens": torch.from_numpy(lens).to(dev),
                "max_ctx": int(lens.max()),
                "kv_bytes": int(lens.astype(np.int64).sum()) * row_bytes,
                "kv_unique_bytes": int(sum(fill.values())) * row_bytes,
                "q": synth.normal((B, Hq, D), dt, seed * 1000 + 10 + 3 * u, device=dev),
                "k": synth.normal((B, Hkv, D), dt, seed * 1000 + 11 + 3 * u, device=dev),
                "v": synth.normal((B, Hkv, D), dt, seed * 1000 + 12 + 3 * u, device=dev),
            }
            # the decode's bytes: unique K/V, q and out, lengths and table entries
            st["algo_bytes"] = st["kv_unique_bytes"] + 2 * B * Hq * D * 2 + B * 4 + int(nblk.sum()) * 4
            # the fused step also reads and writes each new row, and reads and
            # writes each copied block
            st["algo_bytes_fused"] = (st["algo_bytes"] + 2 * B * Hkv * D * 2 * 2
                                      + len(pairs) * 2 * bs * Hkv * D * 2 * 2 + (B * 4 if len(pairs) else 0))
            self.steps.append(st)
        top = max(st["max_ctx"] for st in self.steps)
        ws = torch.empty(max(16, pa.pa_decode_shared_workspace_size(B, Hq, top + 64, D, wl["part"])),
                         dtype=torch.uint8, device=dev)
        out = torch.empty(B, Hq, D, dtype=dt, device=dev)
        for st in self.steps:
            st["ws"], st["out"] = ws, out


def _lengths(fn_name):
    def f(seed):
        from paged_kv_cache_402_b200 import synth
        return getattr(synth, fn_name)(seed)
    return f


WORKLOADS = {
    "gqa": dict(
        name="bf16 GQA decode: 32 seqs, 32 q / 8 kv heads, head_dim 128, 16-token blocks, "
             "context ~U[128,4096] +1 appended token per step, pool 2x needed (seeded shuffle)",
        B=32, Hq=32, Hkv=8, D=128, bs=16, lengths=_lengths("gqa_lengths"), setup=setup_independent,
        rotate=3, max_uses=32),
    "shared-prefix": dict(
        name="bf16 shared-prefix decode: 256 seqs in groups of 8 sharing a 512+r token prefix (refcounted "
             "blocks, copied on write), lognormal suffix median 800 clipped to 8192, 64 q / 8 kv heads, "
             "head_dim 128, 16-token blocks, +1 token per step",
        B=256, Hq=64, Hkv=8, D=128, bs=16, group_size=8, setup=setup_shared_prefix, rotate=2, max_uses=32),
    "long-context": dict(
        name="bf16 long-context decode: 8 seqs, context ~U[32768,131072], 32 q / 8 kv heads, head_dim 128, "
             "16-token blocks scattered over an 80 GiB K+V pool, 512-token partitions + LSE reduce, +1 token per step",
        B=8, Hq=32, Hkv=8, D=128, bs=16, lengths=_lengths("long_context_lengths"), setup=setup_independent,
        num_blocks=80 * 2**30 // (2 * 8 * 16 * 128 * 2), fill_used_only=True, rotate=1, max_uses=100000),
    "long-context-small": dict(
        name="bf16 long-context decode, profiler-sized: the first 2 of the long-context lengths (context "
             "~U[32768,131072]), 32 q / 8 kv heads, head_dim 128, 16-token blocks scattered over a 4 GiB K+V pool, "
             "512-token partitions + LSE reduce, +1 token per step",
        B=2, Hq=32, Hkv=8, D=128, bs=16, lengths=_lengths("long_context_lengths_small"), setup=setup_independent,
        num_blocks=4 * 2**30 // (2 * 8 * 16 * 128 * 2), fill_used_only=True, rotate=1, max_uses=100000),
    "cow-step": dict(
        name="bf16 copy-on-write step: 256 seqs in groups of 8 sharing a 512+r token prefix; each step's "
             "append copies the shared partial block for 7 of 8 members (224 pairs), then decodes; "
             "64 q / 8 kv heads, head_dim 128, 16-token blocks",
        B=256, Hq=64, Hkv=8, D=128, bs=16, group_size=8, setup=setup_cow_steps, rotate=1, max_uses=100000,
        fresh_sets=True),
}


def decode_launches(n_seqs: int, max_ctx: int, part: int, n_groups: int = 0) -> int:
    """Kernel launches of one decode call: with a plan that has groups, the
    cascade (one launch per 1024 groups); the partition kernel (one per slice
    of at most 8192 sequences, or 1024 when the batch holds no more, whose
    whole partitions fit 20 bits); the log-sum-exp reduce (more than one
    partition, or a plan)."""
    max_parts = max(-(-max_ctx // part), 1)
    per_launch = max(min(1024 if n_seqs <= 1024 else 8192, ((1 << 20) - 1) // max_parts), 1)
    n = -(-n_seqs // per_launch)
    if n_groups:
        n += -(-n_groups // 1024)
    if max_parts > 1 or n_groups:
        n += 1
    return n


def aggregate_ranks(world: int, ms: float, kv_gb: float, tokens: float, e2e_s: float, e2e_gb: float, device):
    """Whole-job figures of the replicas: the slowest rank's times, the sum
    of every rank's work.  Returns (ms, GB, tokens, end-to-end GB/s).  Every
    rank takes the same two collectives in the same order."""
    t = torch.tensor([ms, e2e_s], dtype=torch.float64, device=device)
    w = torch.tensor([kv_gb, tokens, e2e_gb], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        torch.distributed.all_reduce(w, op=torch.distributed.ReduceOp.SUM)
    return float(t[0]), float(w[0]), float(w[1]), float(w[2]) / float(t[1])


def run_ours(args, rank: int, world: int, dev):
    import paged_kv_cache_402_b200 as pa

    wl = dict(WORKLOADS[args.workload], part=args.partition)
    total = args.warmup + args.steps
    # enough instances that none is used more than max_uses times (each use
    # grows every sequence by one token)
    R = args.rotate or max(wl["rotate"], -(-total // wl["max_uses"]))
    uses = -(-total // R)
    # instance 0 keeps room (and, for fresh-set workloads, sets) for the
    # end-to-end leg's steps
    insts = [Instance(1000 * rank + 17 * i + 1, wl, uses, dev, extra=args.steps if i == 0 else 0)
             for i in range(R)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(s, strm, ev=None):
        inst = insts[s % R]
        st = inst.steps[s // R]
        n = 0
        scale = 1.0 / math.sqrt(wl["D"])
        if args.unfused:
            if st["pairs"] is not None:
                pa.pa_copy_blocks(st["pairs"], inst.cache, strm)
                n += 1
            pa.pa_append_kv(st["k"], st["v"], st["slots"], inst.cache, strm)
            n += 1
        if ev is not None:
            ev[0].record(strm)
        if args.unfused:
            pa.pa_decode(st["q"], inst.cache, st["tables"], st["lens"], st["max_ctx"], scale,
                         out=st["out"], workspace=st["ws"], stream=strm)
        elif not args.no_share_plan:
            pa.pa_decode_shared(st["q"], inst.cache, st["tables"], st["lens"], st["max_ctx"], scale,
                                plan=st["plan"], k_new=st["k"], v_new=st["v"], cow_src=st["cow"],
                                out=st["out"], workspace=st["ws"], stream=strm)
        else:
            pa.pa_append_decode(st["k"], st["v"], st["q"], inst.cache, st["tables"], st["lens"], st["max_ctx"],
                                scale, cow_src=st["cow"], out=st["out"], workspace=st["ws"], stream=strm)
        if ev is not None:
            ev[1].record(strm)
        groups = st["plan"].n_groups if (st["plan"] is not None and not args.unfused and not args.no_share_plan) else 0
        n += decode_launches(len(st["lens"]), st["max_ctx"], wl["part"], groups)
        return n, st

    for s in range(args.warmup):
        step(s, stream)
    bits = pa.pa_read_device_error()
    if bits != 0:
        raise RuntimeError(f"device error during warm-up (device error bits {bits:#x})")

    # The K timed steps (inputs precomputed, resident) are captured once into
    # a CUDA graph and replayed, so the host's launch rate does not bound the
    # device-side measurement.  With the separate calls, each step's decode
    # call is bracketed by events captured inside the graph; with the fused
    # call the step is that one call, so its duration is the timed region / K
    # (events between the steps would only serialise them).
    per_step_events = args.unfused
    # external: inside a captured graph the records become event-record nodes
    dec_events = [(torch.cuda.Event(enable_timing=True, external=True),
                   torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
    launches = 0
    kv_bytes = 0       # distinct physical K/V bytes (what HBM must serve)
    kv_logical = 0     # per-sequence K/V bytes (shared blocks counted per sharer)
    pairs = 0
    algo_bytes = []
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = torch.cuda.current_stream()
            for i in range(args.steps):
                n, st = step(args.warmup + i, cap, dec_events[i] if per_step_events else None)
                launches += n
                kv_bytes += st["kv_unique_bytes"]
                kv_logical += st["kv_bytes"]
                pairs += st["n_pairs"]
                algo_bytes.append(st["algo_bytes"] if args.unfused else st["algo_bytes_fused"])
        graph.replay()  # one untimed replay: the graph's own warm-up
        torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t_start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                n, st = step(args.warmup + i, stream, dec_events[i] if per_step_events else None)
                launches += n
                kv_bytes += st["kv_unique_bytes"]
                kv_logical += st["kv_bytes"]
                pairs += st["n_pairs"]
                algo_bytes.append(st["algo_bytes"] if args.unfused else st["algo_bytes_fused"])
        t_end.record(stream)
        torch.cuda.synchronize()
    if graph is not None:
        del graph
    if world > 1:
        torch.distributed.barrier()
    ms = t_start.elapsed_time(t_end)
    dec_ms = [a.elapsed_time(b) for a, b in dec_events] if per_step_events else [ms / args.steps]
    bits = pa.pa_read_device_error()
    if bits != 0:
        raise RuntimeError(f"device error during the timed steps (device error bits {bits:#x})")
    clocks = clk.summary()

    # end to end through the public API with pinned host buffers
    e2e = run_e2e(args, insts, wl, dev, stream)
    read_gbs, copy_gbs = bandwidth_probes(dev)

    ms_all, gb_all, tok_all, e2e_value = aggregate_ranks(world, ms, kv_bytes / 1e9, float(args.steps * wl["B"]),
                                                         e2e["seconds"], e2e["kv_gb"], dev)

    peak, peak_kind = measured_peaks()
    dec_avg_s = statistics.mean(dec_ms) / 1e3
    achieved = statistics.mean(algo_bytes) / dec_avg_s / 1e9
    host_alloc_us = 1e6 * statistics.mean([i.host_alloc_s / len(i.steps) for i in insts])
    line = {
        "metric": METRIC,
        "value": round(gb_all / (ms_all / 1e3), 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_all / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v; seeded lengths and block placement)",
        "config": {"workload": wl["name"], "global_batch": wl["B"] * world, "block_size": wl["bs"],
                   "q_heads": wl["Hq"], "kv_heads": wl["Hkv"], "head_dim": wl["D"],
                   "partition_tokens": wl["part"],
                   "l2": f"{R} rotating batch instances per rank (KV per step ~{kv_bytes / args.steps / 1e6:.0f} MB, "
                         f"working set ~{R * kv_bytes / args.steps / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}",
                   "timing": "eager launches" if args.no_graph else "CUDA graph replay of the K steps",
                   "step": ("pa_copy_blocks + pa_append_kv + pa_decode" if args.unfused else
                            "pa_append_decode (copy on write + append + decode in one call)" if args.no_share_plan
                            else "pa_decode_shared (copy on write + append + decode in one call; partitions "
                                 "that a group of sequences holds in the same blocks read once per group of "
                                 "up to 4)"),
                   "share_groups_per_step": round(statistics.mean(
                       insts[0].steps[i]["plan"].n_groups for i in range(len(insts[0].steps))), 2)},
        "tokens_per_s": round(tok_all / (ms_all / 1e3), 1),
        "kv_logical_gbs": round(kv_logical * world / 1e9 / (ms_all / 1e3), 2),
        "copy_pairs_per_step": round(pairs / args.steps, 2),
        "kv_frac_of_hbm_peak": round(gb_all / (ms_all / 1e3) / peak, 4),
        "kv_frac_of_8tbs_nominal": round(gb_all / (ms_all / 1e3) / NOMINAL_HBM_GBS, 4),
        "kv_frac_of_read_peak": round(gb_all / (ms_all / 1e3) / (read_gbs * world), 4),
        "probes": {"read_gbs": round(read_gbs, 1), "copy_gbs": round(copy_gbs, 1),
                   "how": "this job, after the timed region: torch sum (read-only) and copy_ over 4 GiB, "
                          "best of 3 x 6 launches"},
        "host_alloc_us_per_step": round(host_alloc_us, 2),
        "roofline": {"bound": "hbm",
                     "kernel": ("pa_decode (partition + LSE reduce)" if args.unfused else
                                "pa_append_decode (copy + append + partition in one kernel, + LSE reduce)"
                                if args.no_share_plan else
                                "pa_decode_shared (cascade over shared partitions + fused copy/append/partition"
                                " + LSE reduce)"),
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": profiled_traffic(args.workload, statistics.mean(algo_bytes)),
                     "decode_us": round(dec_avg_s * 1e6, 2),
                     "duration_from": ("CUDA events around each decode call in the timed graph" if per_step_events
                                       else "CUDA events around the K-step timed region / K (one call per step)"),
                     "algo_bytes_per_launch": int(statistics.mean(algo_bytes))},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(1e3 * e2e["seconds"] / e2e["steps"], 4)},
        "gpu_launches": launches * world,
        "clocks": clocks,
    }
    return line


def unique_kv_bytes(tables: np.ndarray, lens: np.ndarray, bs: int, row_bytes: int) -> int:
    """K/V bytes of the distinct physical blocks a batch reads (each block
    once, with its fill)."""
    fill = {}
    for i in range(len(lens)):
        for j in range(-(-int(lens[i]) // bs)):
            fill.setdefault(int(tables[i, j]), min(bs, int(lens[i]) - j * bs))
    return int(sum(fill.values())) * row_bytes


def run_e2e(args, insts, wl, dev, stream):
    """Each step from host memory, through the public API: the step's host
    work (one allocator call that appends the tokens and writes the tables,
    lengths, copy-on-write sources and sharing plan; with --unfused the
    allocator append and table build), one pinned host -> device copy of
    every input of the step (q, new rows, tables, lengths, copy sources,
    plan; slots and pairs for --unfused), the step's call, and the device ->
    host copy of its output, which the host then reads.  Wall clock over all
    steps.  Pipelined two deep: the host prepares step i + 1 while the device
    runs step i; copies run on their own stream, ordered by events against
    the compute stream, and every buffer has two copies."""
    import paged_kv_cache_402_b200 as pa

    if not args.unfused:
        return run_e2e_native(args, insts, wl, dev, stream)
    B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
    inst = insts[0]
    mb = inst.max_blocks
    n_steps = max(1, args.steps)
    G2 = max(1, B // 2)
    share = 0 if (args.unfused or args.no_share_plan) else 4
    # one packed buffer per step: (name, shape, dtype), each part 16-byte aligned
    parts = [("q", (B, Hq, D), torch.bfloat16), ("k", (B, Hkv, D), torch.bfloat16),
             ("v", (B, Hkv, D), torch.bfloat16), ("tables", (B, mb), torch.int32), ("lens", (B,), torch.int32),
             ("cow_src", (B,), torch.int32), ("first_token", (B,), torch.int32), ("members", (G2, 4), torch.int32),
             ("shared_tokens", (G2,), torch.int32), ("slots", (B,), torch.int64), ("pairs", (B, 2), torch.int32)]
    offs, total = {}, 0
    for name, shape, dt in parts:
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dt).element_size()
        offs[name] = (total, nbytes)
        total += (nbytes + 15) // 16 * 16
    g = torch.Generator().manual_seed(5)
    rows = {"q": torch.randn(B, Hq, D, generator=g).to(torch.bfloat16),
            "k": torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16),
            "v": torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16)}

    def views(buf):
        return {name: buf[offs[name][0]:offs[name][0] + offs[name][1]].view(dt).view(shape)
                for name, shape, dt in parts}

    def make_set():
        h_buf = torch.zeros(total, dtype=torch.uint8).pin_memory()
        d_buf = torch.empty(total, dtype=torch.uint8, device=dev)
        hv = views(h_buf)
        for k in ("q", "k", "v"):
            hv[k].copy_(rows[k])
        np_out = {k: hv[k].numpy() for k in ("tables", "lens", "cow_src", "first_token", "members", "shared_tokens")}
        return {"h_buf": h_buf, "d_buf": d_buf, "h": hv, "d": views(d_buf), "np": np_out,
                "out": torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev),
                "h_out": torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory(),
                "ev_in": torch.cuda.Event(), "ev_kernel": torch.cuda.Event(), "ev_out": torch.cuda.Event(),
                "used": False}

    sets = [make_set(), make_set()]
    copy_stream = torch.cuda.Stream(device=dev)
    ws = torch.empty(max(16, pa.pa_decode_workspace_size(B, Hq, mb * bs, D, wl["part"])), dtype=torch.uint8,
                     device=dev)
    ones = np.ones(B, np.int32)
    scale = 1.0 / math.sqrt(D)
    seen = []
    checksum = 0.0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n_steps):
        S = sets[i % 2]
        h, d = S["h"], S["d"]
        if S["used"]:
            S["ev_in"].synchronize()        # its pinned inputs are free again
            S["ev_out"].synchronize()       # the output of step i - 2 is on the host
            checksum += float(S["h_out"][0, 0, 0])
        seqs = inst.sets[inst.uses + i] if wl.get("fresh_sets") else inst.sets[0]
        if args.unfused:
            _, pairs = inst.alloc.batch_append(seqs, ones, out_slots=h["slots"].numpy(),
                                               out_pairs=h["pairs"].numpy())
            inst.alloc.build_block_tables(seqs, mb, out_tables=S["np"]["tables"], out_lens=S["np"]["lens"])
            npairs, max_len, plan = len(pairs), int(S["np"]["lens"].max()), None
        else:
            st = inst.alloc.decode_step(seqs, mb, share_max_members=share, out=S["np"])
            npairs, max_len = st["n_copies"], st["max_len"]
            plan = pa.SharePlan(st["members"], st["shared_tokens"], st["first_token"])
            if plan.n_groups:
                plan.bind(d["members"][:plan.n_groups], d["shared_tokens"][:plan.n_groups], d["first_token"])
        with torch.cuda.stream(copy_stream):
            if S["used"]:
                copy_stream.wait_event(S["ev_kernel"])   # step i - 2 no longer reads these device inputs
            S["d_buf"].copy_(S["h_buf"], non_blocking=True)
            S["ev_in"].record(copy_stream)
        stream.wait_event(S["ev_in"])
        if S["used"]:
            stream.wait_event(S["ev_out"])               # the output buffer of step i - 2 was copied out
        if args.unfused:
            if npairs:
                pa.pa_copy_blocks(d["pairs"][:npairs], inst.cache, stream)
            pa.pa_append_kv(d["k"], d["v"], d["slots"], inst.cache, stream)
            pa.pa_decode(d["q"], inst.cache, d["tables"], d["lens"], max_len, scale, out=S["out"],
                         workspace=ws, stream=stream)
        else:
            pa.pa_decode_shared(d["q"], inst.cache, d["tables"], d["lens"], max_len, scale, plan=plan,
                                k_new=d["k"], v_new=d["v"], cow_src=d["cow_src"] if npairs else None,
                                out=S["out"], workspace=ws, stream=stream)
        S["ev_kernel"].record(stream)
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(S["ev_kernel"])
            S["h_out"].copy_(S["out"], non_blocking=True)
            S["ev_out"].record(copy_stream)
        S["used"] = True
        seen.append((S["np"]["tables"].copy(), S["np"]["lens"].copy()))
    for S in sets:
        if S["used"]:
            S["ev_out"].synchronize()
            checksum += float(S["h_out"][0, 0, 0])
    seconds = time.perf_counter() - t0
    torch.cuda.synchronize()
    if not math.isfinite(checksum):
        raise RuntimeError("non-finite output in the end-to-end steps")
    kv = sum(unique_kv_bytes(t, l, bs, 2 * Hkv * D * 2) for t, l in seen)
    return {"seconds": seconds, "kv_gb": kv / 1e9, "steps": n_steps, "h2d": total, "d2h": B * Hq * D * 2}


def run_e2e_native(args, insts, wl, dev, stream):
    """The end-to-end leg through the library's one-call step
    (pa.DecodeStepper over pa_decode_step): per step one native call does the
    allocator's step (one token per sequence, tables, lengths, copy-on-write
    sources, sharing plan) into a pinned staging area, one host -> device copy
    of it (q, new rows and the host-built arrays), the fused decode, and the
    device -> host copy of the output; the host reads each output once its
    slot comes round again.  Two slots alternate, so the host prepares step
    i + 1 while the device runs step i.  Wall clock over all steps.

    The K/V bytes of each step: its lengths are read from the slot's staging
    area (B ints); the bytes the batch's sharers hold in common are taken
    from the batch's tables after the loop, which stay valid for every step
    because no step of these workloads changes what is shared (asserted: no
    step copies on write, except in fresh-set workloads, whose every set is
    stepped once and is read after the loop as the step left it)."""
    import paged_kv_cache_402_b200 as pa

    B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
    inst = insts[0]
    mb = inst.max_blocks
    n_steps = max(1, args.steps)
    share = 0 if args.no_share_plan else 4
    row = 2 * Hkv * D * 2
    stepper = pa.DecodeStepper(inst.alloc, inst.cache, B, Hq, mb, 1.0 / math.sqrt(D), share_max_members=share,
                               stream=stream)
    g = torch.Generator().manual_seed(5)
    rows = (torch.randn(B, Hq, D, generator=g).to(torch.bfloat16),
            torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16),
            torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16))
    for _ in range(2):  # the rows of both slots (the values do not change the work)
        for dst, src in zip(stepper.inputs(), rows):
            dst.copy_(src)
        stepper.i += 1
    stepper.i = 0
    lens_view = [stepper._slots[k]["keep"][0][stepper.layout.lens:stepper.layout.lens + 4 * B].view(torch.int32).numpy()
                 for k in range(2)]
    fresh = bool(wl.get("fresh_sets"))
    logical = np.zeros(n_steps, np.int64)
    copies = 0
    checksum = 0.0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n_steps):
        k = stepper.next_slot
        if i >= 2:
            stepper.wait(k)
            checksum += float(stepper.output(k)[0, 0, 0])
        seqs = inst.sets[inst.uses + i] if fresh else inst.sets[0]
        info = stepper.step(seqs)
        copies += info["n_copies"]
        logical[i] = int(lens_view[k].sum(dtype=np.int64))
    for k in range(min(2, n_steps)):
        stepper.wait((n_steps - 1 - k) % 2)
        checksum += float(stepper.output((n_steps - 1 - k) % 2)[0, 0, 0])
    seconds = time.perf_counter() - t0
    torch.cuda.synchronize()
    stepper.close()
    if not math.isfinite(checksum):
        raise RuntimeError("non-finite output in the end-to-end steps")
    if fresh:
        kv = 0
        for i in range(n_steps):
            tables, lens = inst.alloc.build_block_tables(inst.sets[inst.uses + i], mb)
            kv += unique_kv_bytes(tables, lens, bs, row)
    else:
        if copies:
            raise RuntimeError("a step copied on write: the shared bytes changed during the end-to-end leg")
        tables, lens = inst.alloc.build_block_tables(inst.sets[0], mb)
        shared_excess = int(lens.astype(np.int64).sum()) * row - unique_kv_bytes(tables, lens, bs, row)
        kv = int(logical.sum()) * row - n_steps * shared_excess
    return {"seconds": seconds, "kv_gb": kv / 1e9, "steps": n_steps, "h2d": stepper.h2d_bytes,
            "d2h": stepper.d2h_bytes}


def run_prefill(args, rank: int, world: int, dev):
    """Chunked-prefill attention over batches of new prompts (the trace's
    prompt shape: lognormal lengths, median 512, clipped to [1, 4096]), 32 q
    / 8 kv heads, head_dim 128, 16-token blocks.  A step appends every
    prompt's K/V rows (pa_append_kv) and runs pa_prefill over them; the
    metric is causal attention FLOP/s (QK^T and PV, 4 * D per visible key
    per query row and head) against the measured bf16 tensor peak."""
    import paged_kv_cache_402_b200 as pa
    from paged_kv_cache_402_b200 import synth

    B, Hq, Hkv, D, bs = 32, 32, 8, 128, 16
    dt = torch.bfloat16
    R = 2
    insts = []
    for i in range(R):
        seed = 1000 * rank + 31 * i + args.seed
        r = synth.rng(seed)
        n = np.clip(np.round(np.exp(r.normal(math.log(512), 1.0, size=B))), 1, 4096).astype(np.int64)
        NB = 2 * int(sum(-(-int(x) // bs) for x in n)) + 8
        A = pa.Allocator(NB, bs, synth.rng(seed + 1).permutation(NB))
        seqs = [A.new_seq() for _ in range(B)]
        slots, _ = A.batch_append(seqs, n.tolist())
        mb = max(len(A.block_table(s_)) for s_ in seqs)
        tables, lens = A.build_block_tables(seqs, mb)
        starts = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
        T = int(starts[-1])
        insts.append({
            "cache": pa.KVCache.empty(NB, Hkv, bs, D, dt, dev),
            "k": synth.normal((T, Hkv, D), dt, seed + 2, device=dev),
            "v": synth.normal((T, Hkv, D), dt, seed + 3, device=dev),
            "q": synth.normal((T, Hq, D), dt, seed + 4, device=dev),
            "out": torch.empty(T, Hq, D, dtype=dt, device=dev),
            "slots": torch.from_numpy(slots).to(dev), "tables": torch.from_numpy(tables).to(dev),
            "lens": torch.from_numpy(lens).to(dev), "starts": torch.from_numpy(starts).to(dev),
            "max_ctx": int(lens.max()), "max_q": int(n.max()), "tokens": T,
            # visible keys per query row: position + 1 (whole prompts)
            "flops": 4 * D * Hq * int(sum(x * (x + 1) // 2 for x in n)),
        })
    stream = torch.cuda.current_stream()

    def step(s_, strm):
        it = insts[s_ % R]
        pa.pa_append_kv(it["k"], it["v"], it["slots"], it["cache"], strm)
        pa.pa_prefill(it["q"], it["cache"], it["tables"], it["lens"], it["starts"], it["max_ctx"],
                      1.0 / math.sqrt(D), max_query_len=it["max_q"], out=it["out"], stream=strm)
        return it

    for s_ in range(args.warmup):
        step(s_, stream)
    torch.cuda.synchronize()
    bits = pa.pa_read_device_error()
    if bits != 0:
        raise RuntimeError(f"device error during warm-up (device error bits {bits:#x}, "
                           f"first wait given up: {pa.pa_read_wait_timeout()})")
    flops = sum(insts[(args.warmup + i) % R]["flops"] for i in range(args.steps))
    tokens = sum(insts[(args.warmup + i) % R]["tokens"] for i in range(args.steps))
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            cap = torch.cuda.current_stream()
            for i in range(args.steps):
                step(args.warmup + i, cap)
        graph.replay()
        torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                step(args.warmup + i, stream)
        t1.record(stream)
        torch.cuda.synchronize()
    del graph
    if world > 1:
        torch.distributed.barrier()
    ms = t0.elapsed_time(t1)
    bits = pa.pa_read_device_error()
    if bits != 0:
        raise RuntimeError(f"device error during the timed steps (device error bits {bits:#x}, "
                           f"first wait given up: {pa.pa_read_wait_timeout()})")
    ms_all, fl_all, tok_all, _ = aggregate_ranks(world, ms, flops / 1e12, float(tokens), 1.0, 0.0, dev)
    peak, kind = measured_tensor_peak()
    tflops = fl_all / (ms_all / 1e3)
    return {
        "metric": "paged chunked-prefill attention TFLOP/s (causal, bf16 in, fp32 accumulate) at 1 B200",
        "workload": "prefill", "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_all / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v; seeded prompt lengths and block placement)",
        "config": {"workload": "bf16 paged prefill: 32 prompts, lengths lognormal (median 512, clipped to "
                               "[1, 4096]), 32 q / 8 kv heads, head_dim 128, 16-token blocks; step = append of "
                               "the prompts' K/V + causal attention of every prompt token",
                   "global_batch": B * world, "l2": f"{R} rotating batch instances",
                   "timing": "eager launches" if args.no_graph else "CUDA graph replay of the K steps",
                   "parallelism": f"replicas x{world}"},
        "tokens_per_s": round(tok_all / (ms_all / 1e3), 1),
        "roofline": {"bound": "tensor", "kernel": "pa_append_kv + pa_prefill", "achieved": round(tflops, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "peak_source": f"{kind} bf16_tflops (dense, burst)", "traffic": None},
        "clocks": clk.summary(),
        "gpu_launches": 2 * args.steps,
    }


def choose_block_size(lines, frag_budget: float):
    """The block-size and partition-size choice from a trace sweep.

    Block size: the pages' trade-off is that smaller blocks waste less of
    the last block of every sequence, larger ones cost less bookkeeping and
    fewer, larger copies per key range ("pagedattention" glossary entry,
    paragraph 6).  Among the layouts of the default partition size, the
    fastest in decode tokens per second of wall time (bookkeeping included)
    whose mean fragmentation stays within the budget; the smallest block size
    if none does.

    Partition size: the grain of the split-context decode and of sharing (a
    smaller one lets a plan share more of a common prefix, at more work
    units per step).  It changes only device work, so among the layouts of
    the chosen block size, the one of least device time per step."""
    base = [d for d in lines if d["config"].get("partition_tokens", 512) == 512] or lines
    ok = [d for d in base if d["fragmentation_mean"] is not None and d["fragmentation_mean"] <= frag_budget]
    bs_pick = (max(ok, key=lambda d: d["tokens_per_s"]) if ok
               else min(base, key=lambda d: d["config"]["block_size"]))["config"]["block_size"]
    same_bs = [d for d in lines if d["config"]["block_size"] == bs_pick]
    pick = min(same_bs, key=lambda d: d["device_ms_per_step"])

    def key(d):
        return f"bs{d['config']['block_size']}/p{d['config'].get('partition_tokens', 512)}"
    return {
        "workload": "trace-sweep",
        "block_size_choice": bs_pick,
        "partition_choice": pick["config"].get("partition_tokens", 512),
        "rule": (f"block size: fastest wall-clock decode tokens/s with mean fragmentation <= {frag_budget:.0%}; "
                 "partition size: least device time per step at that block size"),
        "per_layout": {key(d): {
            "tokens_per_s": d["tokens_per_s"], "device_gbs_unique": d["value"],
            "fragmentation_mean": d["fragmentation_mean"], "device_ms_per_step": d["device_ms_per_step"]}
            for d in lines},
    }


def run_trace(args, dev):
    """Continuous batching of beam-search requests over a 16 GiB K+V pool, one
    JSON line per block size: per step the host trace driver (allocator
    calls), host -> device copies of the step's tables / lengths / slots /
    copy pairs, copy-on-write copies, prompt and decode appends, the decode of
    every running beam, and the device -> host read of the output."""
    import paged_kv_cache_402_b200 as pa
    from paged_kv_cache_402_b200 import synth
    from paged_kv_cache_402_b200.trace import BeamTrace

    Hq, Hkv, D = 32, 8, 128
    dt = torch.bfloat16
    row = 2 * Hkv * D * 2
    stream = torch.cuda.current_stream()
    lines = []
    if args.block_size or args.partition != 512:
        layouts = [(args.block_size or 16, args.partition)]
    else:  # block sizes at the default partition, then partition sizes at 16-token blocks
        layouts = [(8, 512), (16, 512), (32, 512), (16, 256), (16, 1024)]
    draws = synth.trace(args.seed, steps=args.trace_steps)
    # random rows to draw prompt / decode K, V and q from (values do not
    # change the work; the pool of rows is reused cyclically)
    src = synth.normal((1 << 16, Hkv, D), dt, 901, device=dev)
    qsrc = synth.normal((8192, Hq, D), dt, 902, device=dev)
    for bs, part in layouts:
        NB = 16 * 2**30 // (2 * Hkv * bs * D * 2)
        order = synth.rng(args.seed + bs).permutation(NB)
        A = pa.Allocator(NB, bs, order)
        cache = pa.KVCache.empty(NB, Hkv, bs, D, dt, dev, partition_tokens=part)
        drv = BeamTrace(A, lambda: A.stats()["free_blocks"], bs, draws)
        out = torch.empty(8192, Hq, D, dtype=dt, device=dev)
        ws = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.trace_steps)]
        host_s = dec_ms = 0.0
        wall = 0.0
        uniq = logical = 0
        beams = 0
        frag = []
        h2d = d2h = 0
        launches = 0
        torch.cuda.synchronize()
        for s_ in range(args.trace_steps):
            t0 = time.perf_counter()
            plan = drv.step()
            n = len(plan.decode_seqs)
            if n:
                max_ctx, mb = A.max_len(plan.decode_seqs)
                tables, lens = A.build_block_tables(plan.decode_seqs, mb)
                splan = (pa.share_plan(tables, lens, bs)
                         if not (args.unfused or args.no_share_plan) else None)
            host_s += time.perf_counter() - t0
            if n == 0:
                wall += time.perf_counter() - t0
                continue
            npr = len(plan.prompt_slots)
            h = [torch.from_numpy(plan.prompt_slots).pin_memory() if npr else None,
                 torch.from_numpy(plan.decode_slots).pin_memory() if args.unfused else None,
                 (torch.from_numpy(np.ascontiguousarray(plan.cow_pairs)).pin_memory()
                  if len(plan.cow_pairs) and args.unfused else None),
                 torch.from_numpy(tables).pin_memory(), torch.from_numpy(lens).pin_memory(),
                 (torch.from_numpy(pa.cow_sources(plan.cow_pairs, tables, lens, bs)).pin_memory()
                  if len(plan.cow_pairs) and not args.unfused else None)]
            d_ = [x.to(dev, non_blocking=True) if x is not None else None for x in h]
            # everything but the library's own calls is set up before the
            # step's first event: inputs, plan, workspace, q and out
            dplan = splan.to(dev) if splan is not None else None
            kd = src[(s_ * 131) % ((1 << 16) - n):][:n]
            need = (pa.pa_decode_shared_workspace_size if splan is not None and splan.n_groups
                    else pa.pa_decode_workspace_size)(n, Hq, max_ctx, D, part)
            if need > ws.numel():
                ws = torch.empty(need * 5 // 4, dtype=torch.uint8, device=dev)
            q = qsrc[:n] if n <= 8192 else synth.normal((n, Hq, D), dt, s_, device=dev)
            o = out[:n] if n <= 8192 else torch.empty(n, Hq, D, dtype=dt, device=dev)
            if npr:
                i0 = (s_ * 977) % ((1 << 16) - npr) if npr < (1 << 16) else 0
                kk = src[i0:i0 + npr]
            ev[s_][0].record(stream)
            if npr:
                pa.pa_append_kv(kk, kk, d_[0], cache, stream)
                launches += 1
            if args.unfused:
                if d_[2] is not None:
                    pa.pa_copy_blocks(d_[2], cache, stream)
                    launches += 1
                pa.pa_append_kv(kd, kd, d_[1], cache, stream)
                pa.pa_decode(q, cache, d_[3], d_[4], max_ctx, 1 / math.sqrt(D), out=o, workspace=ws, stream=stream)
                launches += 1 + decode_launches(n, max_ctx, part)
            elif args.no_share_plan:
                pa.pa_append_decode(kd, kd, q, cache, d_[3], d_[4], max_ctx, 1 / math.sqrt(D), cow_src=d_[5],
                                    out=o, workspace=ws, stream=stream)
                launches += decode_launches(n, max_ctx, part)
            else:
                pa.pa_decode_shared(q, cache, d_[3], d_[4], max_ctx, 1 / math.sqrt(D), plan=dplan,
                                    k_new=kd, v_new=kd, cow_src=d_[5], out=o, workspace=ws, stream=stream)
                launches += decode_launches(n, max_ctx, part, splan.n_groups)
                h2d += splan.nbytes
            ev[s_][1].record(stream)
            res = o[:1].to("cpu", non_blocking=True)
            torch.cuda.synchronize()
            wall += time.perf_counter() - t0
            dec_ms += ev[s_][0].elapsed_time(ev[s_][1])
            st = A.stats()
            uniq += st["used_slots"] * row
            logical += int(lens.astype(np.int64).sum()) * row
            beams += n
            frag.append(st["fragmentation"])
            h2d += sum(x.numel() * x.element_size() for x in h if x is not None)
            d2h += res.numel() * res.element_size()
        bits = pa.pa_read_device_error()
        if bits != 0:
            raise RuntimeError(f"device error in the trace (device error bits {bits:#x})")
        peak, peak_kind = measured_peaks()
        steps = args.trace_steps
        line = {
            "metric": METRIC, "workload": "trace",
            "value": round(uniq / 1e9 / (dec_ms / 1e3), 2), "unit": "GB/s",
            "n_gpus": 1, "steps": steps, "warmup": 0, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic trace (seeded)",
            "config": {"workload": "bf16 continuous-batching trace: Poisson(4) arrivals per step, prompts "
                                   "lognormal (median 512, max 4096), outputs geometric (mean 256), beam "
                                   "groups of 4 re-forked copy-on-write, 32 q / 8 kv heads, head_dim 128, "
                                   "16 GiB K+V pool",
                       "block_size": bs, "partition_tokens": part, "trace_steps": steps,
                       "timing": "device: CUDA events around each step's kernels; wall: whole step incl. host"},
            "kv_logical_gbs": round(logical / 1e9 / (dec_ms / 1e3), 2),
            "kv_frac_of_hbm_peak": round(uniq / 1e9 / (dec_ms / 1e3) / peak, 4),
            "tokens_per_s": round(beams / wall, 1),
            "device_ms_per_step": round(dec_ms / steps, 4), "wall_ms_per_step": round(1e3 * wall / steps, 4),
            "host_driver_ms_per_step": round(1e3 * host_s / steps, 4),
            "mean_running_beams": round(beams / steps, 1),
            "fragmentation_mean": round(float(np.mean(frag)), 5) if frag else None,
            "fragmentation_last": round(frag[-1], 5) if frag else None,
            "e2e": {"value": round(uniq / 1e9 / wall, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d // steps,
                    "d2h_bytes_per_step": d2h // steps},
            "gpu_launches": launches,
        }
        lines.append(line)
        del cache, A, drv
        torch.cuda.empty_cache()
    return lines


# ----------------------------------------------------------------- CPU oracle


ORACLE_CASE_BYTES = 768 << 20  # K/V the host-side case of the oracle holds at most


def oracle_case(wl, seed: int):
    """The oracle's host-side case: the workload's batch (its lengths, +1 for
    the step's appended token), cut to its first sequences when the whole
    batch would hold more than ORACLE_CASE_BYTES of K/V (the long-context
    batch holds 2.7 GB).  Returns (case, lengths, description of the cut)."""
    from paged_kv_cache_402_b200 import synth

    B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
    lens = wl["lengths"](seed) + 1
    row = 2 * Hkv * D * 2
    n = 1
    while n < B and int(lens[:n + 1].astype(np.int64).sum()) * row <= ORACLE_CASE_BYTES:
        n += 1
    lens = lens[:n]
    case = synth.random_case(seed, B=n, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=lens, dtype=torch.bfloat16,
                             sentinel=False, pool_factor=1.0 if n < B else 2.0)
    cut = "the whole batch" if n == B else f"its first {n} of {B} sequences"
    return case, lens, cut


def _oracle_rows(order, start, count, Hkv, G):
    chunk = [int(order[(start + i) % len(order)]) for i in range(count)]
    return chunk, [(u // Hkv, (u % Hkv) * G + gi) for u in chunk for gi in range(G)]


def oracle_sample(wl, seed: int, budget_s: float, min_s: float, threads: int | None = None):
    """Times the float64 oracle on the host over whole (sequence, kv head)
    groups of one batch of the workload until about budget_s of work, on
    `threads` OpenMP threads (all of them by default).  Returns (GB/s of KV
    processed, seconds, threads, description)."""
    import oracle

    Hq, Hkv, D = wl["Hq"], wl["Hkv"], wl["D"]
    case, lens, cut = oracle_case(wl, seed)
    G = Hq // Hkv
    order = synth_rng(seed + 9).permutation(len(lens) * Hkv)
    prev = oracle.max_threads()
    if threads is not None:
        oracle.set_threads(threads)
    used = oracle.max_threads()
    try:
        done_bytes, t_total, groups, pos = 0, 0.0, 0, 0
        while t_total < budget_s:
            chunk, rows = _oracle_rows(order, pos, min(len(order), max(1, 2 * used)), Hkv, G)
            pos += len(chunk)
            t0 = time.perf_counter()
            oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale,
                          rows=rows)
            t_total += time.perf_counter() - t0
            done_bytes += sum(int(lens[u // Hkv]) * 2 * D * 2 for u in chunk)
            groups += len(chunk)
            if t_total >= min_s and groups >= len(order):
                break
    finally:
        oracle.set_threads(prev)
    desc = (f"{groups} (sequence, kv head) groups ({groups * G} query rows) of {cut} of one batch of the "
            f"workload, {t_total:.1f} s of oracle time on {used} thread(s)")
    return done_bytes / 1e9 / t_total, t_total, used, desc


def synth_rng(seed):
    from paged_kv_cache_402_b200 import synth
    return synth.rng(seed)


def run_reference(args):
    """The oracle as it stands on the host cores: W untimed and K timed steps,
    each step a bounded sample of the workload (whole (sequence, kv head)
    groups of one batch, eight per oracle thread, taken round-robin)."""
    import oracle

    wl = WORKLOADS[args.workload] if args.workload in WORKLOADS else WORKLOADS["long-context"]
    if "lengths" not in wl:
        wl = WORKLOADS["long-context"]
    Hq, Hkv, D = wl["Hq"], wl["Hkv"], wl["D"]
    G = Hq // Hkv
    case, lens, cut = oracle_case(wl, 1)
    order = synth_rng(10).permutation(len(lens) * Hkv)
    threads = oracle.max_threads()
    per_step = min(8 * threads, len(order))
    pos = 0
    total_bytes, total_s, groups = 0, 0.0, 0
    for s in range(args.warmup + args.steps):
        chunk, rows = _oracle_rows(order, pos, per_step, Hkv, G)
        pos += per_step
        t0 = time.perf_counter()
        oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale, rows=rows)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            total_s += dt
            total_bytes += sum(int(lens[u // Hkv]) * 2 * D * 2 for u in chunk)
            groups += len(chunk)
    gbs = total_bytes / 1e9 / total_s
    seq_bytes = float(np.mean(lens)) * 2 * Hkv * D * 2
    desc = (f"{args.steps} steps of {per_step} (sequence, kv head) groups ({per_step * G} query rows) each, "
            f"round-robin over {cut} of one batch of the workload; {total_s:.1f} s timed")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(gbs, 4),
        "unit": "GB/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * total_s / args.steps, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/k/v; seeded lengths and block placement)",
        "config": {"workload": wl["name"], "global_batch": wl["B"], "block_size": wl["bs"],
                   "q_heads": wl["Hq"], "kv_heads": wl["Hkv"], "head_dim": wl["D"]},
        "tokens_per_s": round(gbs * 1e9 / seq_bytes, 3),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------- main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["trace", "prefill"], default="long-context")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rotate", type=int, default=0, help="batch instances to rotate (0: the workload's default)")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly instead of from a CUDA graph")
    ap.add_argument("--no-share-plan", action="store_true",
                    help="fused step without the cascade over shared partitions (pa_append_decode)")
    ap.add_argument("--unfused", action="store_true",
                    help="run each step as pa_copy_blocks + pa_append_kv + pa_decode instead of pa_append_decode")
    ap.add_argument("--block-size", type=int, default=0, help="trace workload: one block size (0: 8, 16 and 32)")
    ap.add_argument("--partition", type=int, default=512, choices=[256, 512, 1024],
                    help="tokens per split-context partition of the decode (trace: with the default 512 the sweep "
                         "also runs 256 and 1024 at 16-token blocks)")
    ap.add_argument("--trace-steps", type=int, default=1000)
    ap.add_argument("--frag-budget", type=float, default=0.05,
                    help="trace sweep: largest mean fragmentation a block-size choice may have")
    ap.add_argument("--seed", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    try:
        if args.workload == "prefill":
            line = run_prefill(args, rank, world, dev)
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        if args.workload == "trace":  # one trace, on rank 0; the other ranks only join the exit
            if rank == 0:
                lines = run_trace(args, dev)
                for line in lines:
                    print(json.dumps(line), flush=True)
                if len(lines) > 1:
                    print(json.dumps(choose_block_size(lines, args.frag_budget)), flush=True)
            if world > 1:
                torch.distributed.barrier()
            return
        line = run_ours(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline and "lengths" in WORKLOADS[args.workload]:
            wl = WORKLOADS[args.workload]
            gbs, secs, threads, desc = oracle_sample(wl, seed=1, budget_s=args.cpu_budget, min_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                    "sample": desc}
            # the same oracle on one host core, beside the all-core figure
            gbs1, _, _, desc1 = oracle_sample(wl, seed=1, budget_s=args.cpu_budget / 4, min_s=0.0, threads=1)
            line["cpu_baseline"]["single_core"] = {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                                                   "sample": desc1}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

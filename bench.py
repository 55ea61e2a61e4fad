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


def kernel_source_hash() -> str:
    """Hash of the decode kernel sources; ties an ncu traffic figure to them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_402_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.startswith("pa_decode") or f == "pa_device.cuh":
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """Per-launch DRAM traffic (bytes) recorded by an ncu capture of the
    current decode kernel, scaled to the workload, or None when no capture
    matches the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("kernel_hash") != kernel_source_hash():
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML by a thread about
    every millisecond while the timed region runs (the region is short)."""

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
                time.sleep(0.001)

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


# ----------------------------------------------------------------- workload


class Instance:
    """One independent batch: pool, allocator, sequences, and per-step inputs
    (slots, copy pairs, tables, lengths, q and new rows) for `uses` steps."""

    def __init__(self, seed: int, wl: dict, uses: int, dev, pin: bool = True):
        import paged_kv_cache_402_b200 as pa
        from paged_kv_cache_402_b200 import synth

        self.wl = wl
        B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
        dt = torch.bfloat16
        self.lens0 = wl["lengths"](seed)
        need = int(sum(-(-(int(L) + uses) // bs) for L in self.lens0))
        NB = int(math.ceil(need * wl.get("pool_factor", 2.0))) + 1
        order = synth.rng(seed + 1).permutation(NB)
        self.alloc = pa.Allocator(NB, bs, order)
        self.cache = pa.KVCache(synth.normal((NB, Hkv, bs, D), dt, seed + 2, device=dev),
                                synth.normal((NB, Hkv, bs, D), dt, seed + 3, device=dev))
        t0 = time.perf_counter()
        self.seqs = [self.alloc.new_seq() for _ in range(B)]
        self.alloc.batch_append(self.seqs, self.lens0)  # prompt blocks; the pool's contents stand in for them
        self.max_blocks = int(-(-(int(self.lens0.max()) + uses) // bs))
        self.steps = []
        self.host_alloc_s = 0.0
        for u in range(uses):
            t1 = time.perf_counter()
            slots, pairs = self.alloc.batch_append(self.seqs, np.ones(B, np.int32))
            tables, lens = self.alloc.build_block_tables(self.seqs, self.max_blocks)
            self.host_alloc_s += time.perf_counter() - t1
            st = {
                "slots": torch.from_numpy(slots.copy()).to(dev),
                "pairs": torch.from_numpy(np.ascontiguousarray(pairs)).to(dev) if len(pairs) else None,
                "tables": torch.from_numpy(tables).to(dev),
                "lens": torch.from_numpy(lens).to(dev),
                "max_ctx": int(lens.max()),
                "kv_bytes": int(lens.astype(np.int64).sum()) * 2 * Hkv * D * 2,
                "q": synth.normal((B, Hq, D), dt, seed * 1000 + 10 + 3 * u, device=dev),
                "k": synth.normal((B, Hkv, D), dt, seed * 1000 + 11 + 3 * u, device=dev),
                "v": synth.normal((B, Hkv, D), dt, seed * 1000 + 12 + 3 * u, device=dev),
            }
            st["ws"] = torch.empty(max(16, pa.pa_decode_workspace_size(B, Hq, st["max_ctx"], D)),
                                   dtype=torch.uint8, device=dev)
            st["out"] = torch.empty(B, Hq, D, dtype=dt, device=dev)
            st["algo_bytes"] = (st["kv_bytes"] + 2 * B * Hq * D * 2 + B * 4
                                + int(((lens.astype(np.int64) + bs - 1) // bs).sum()) * 4)
            self.steps.append(st)
        self.setup_s = time.perf_counter() - t0


WORKLOADS = {
    "gqa": dict(
        name="bf16 GQA decode: 32 seqs, 32 q / 8 kv heads, head_dim 128, 16-token blocks, "
             "context ~U[128,4096] +1 appended token per step, pool 2x needed (seeded shuffle)",
        B=32, Hq=32, Hkv=8, D=128, bs=16,
        lengths=lambda seed: __import__("paged_kv_cache_402_b200.synth", fromlist=["x"]).gqa_lengths(seed),
        rotate=3),
}


def run_ours(args, rank: int, world: int, dev):
    import paged_kv_cache_402_b200 as pa

    wl = WORKLOADS[args.workload]
    R = args.rotate or wl["rotate"]
    total = args.warmup + args.steps
    uses = -(-total // R)
    insts = [Instance(1000 * rank + 17 * i + 1, wl, uses, dev) for i in range(R)]
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(s, ev=None):
        inst = insts[s % R]
        st = inst.steps[s // R]
        n = 0
        if st["pairs"] is not None:
            pa.pa_copy_blocks(st["pairs"], inst.cache, stream)
            n += 1
        pa.pa_append_kv(st["k"], st["v"], st["slots"], inst.cache, stream)
        n += 1
        if ev is not None:
            ev[0].record(stream)
        pa.pa_decode(st["q"], inst.cache, st["tables"], st["lens"], st["max_ctx"], 1.0 / math.sqrt(wl["D"]),
                     out=st["out"], workspace=st["ws"], stream=stream)
        if ev is not None:
            ev[1].record(stream)
        n += 2 if st["max_ctx"] > pa.PA_PARTITION_TOKENS else 1
        return n, st

    for s in range(args.warmup):
        step(s)
    if pa.pa_read_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    dec_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    kv_bytes = 0
    algo_bytes = []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            n, st = step(args.warmup + i, dec_events[i])
            launches += n
            kv_bytes += st["kv_bytes"]
            algo_bytes.append(st["algo_bytes"])
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = t_start.elapsed_time(t_end)
    dec_ms = [a.elapsed_time(b) for a, b in dec_events]
    if pa.pa_read_device_error() != 0:
        raise RuntimeError("device error during the timed steps")
    clocks = clk.summary()

    # end to end through the public API with pinned host buffers
    e2e = run_e2e(args, insts, wl, dev, stream)

    t = torch.tensor([ms, kv_bytes / 1e9, float(args.steps * wl["B"])], dtype=torch.float64, device=dev)
    if world > 1:
        tmax = t[:1].clone()
        torch.distributed.all_reduce(tmax, op=torch.distributed.ReduceOp.MAX)
        tsum = t[1:].clone()
        torch.distributed.all_reduce(tsum, op=torch.distributed.ReduceOp.SUM)
        ms_all, gb_all, tok_all = float(tmax[0]), float(tsum[0]), float(tsum[1])
        e2e_t = torch.tensor([e2e["seconds"]], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(e2e_t, op=torch.distributed.ReduceOp.MAX)
        e2e_gb = torch.tensor([e2e["kv_gb"]], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(e2e_gb, op=torch.distributed.ReduceOp.SUM)
        e2e_value = float(e2e_gb[0]) / float(e2e_t[0])
    else:
        ms_all, gb_all, tok_all = ms, kv_bytes / 1e9, float(args.steps * wl["B"])
        e2e_value = e2e["kv_gb"] / e2e["seconds"]

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
                   "partition_tokens": pa.PA_PARTITION_TOKENS,
                   "l2": f"{R} rotating batch instances per rank (KV per step ~{kv_bytes / args.steps / 1e6:.0f} MB, "
                         f"working set ~{R * kv_bytes / args.steps / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "tokens_per_s": round(tok_all / (ms_all / 1e3), 1),
        "kv_frac_of_hbm_peak": round(gb_all / (ms_all / 1e3) / peak, 4),
        "kv_frac_of_8tbs_nominal": round(gb_all / (ms_all / 1e3) / NOMINAL_HBM_GBS, 4),
        "host_alloc_us_per_step": round(host_alloc_us, 2),
        "roofline": {"bound": "hbm", "kernel": "pa_decode (partition + LSE reduce)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": profiled_traffic(args.workload),
                     "decode_us": round(dec_avg_s * 1e6, 2),
                     "algo_bytes_per_launch": int(statistics.mean(algo_bytes))},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(1e3 * e2e["seconds"] / e2e["steps"], 4)},
        "gpu_launches": launches * world,
        "clocks": clocks,
    }
    return line


def run_e2e(args, insts, wl, dev, stream):
    """Each step from host memory: allocator call, pinned host -> device copies
    of the step's inputs, copy / append / decode, device -> host of the output."""
    import paged_kv_cache_402_b200 as pa

    B, Hq, Hkv, D = wl["B"], wl["Hq"], wl["Hkv"], wl["D"]
    inst = insts[0]
    mb = inst.max_blocks + args.steps + args.warmup
    h = {
        "q": torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory(),
        "k": torch.empty(B, Hkv, D, dtype=torch.bfloat16).pin_memory(),
        "v": torch.empty(B, Hkv, D, dtype=torch.bfloat16).pin_memory(),
        "slots": torch.empty(B, dtype=torch.int64).pin_memory(),
        "pairs": torch.empty(B, 2, dtype=torch.int32).pin_memory(),
        "tables": torch.empty(B, mb, dtype=torch.int32).pin_memory(),
        "lens": torch.empty(B, dtype=torch.int32).pin_memory(),
        "out": torch.empty(B, Hq, D, dtype=torch.bfloat16).pin_memory(),
    }
    g = torch.Generator().manual_seed(5)
    h["q"].copy_(torch.randn(B, Hq, D, generator=g).to(torch.bfloat16))
    h["k"].copy_(torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16))
    h["v"].copy_(torch.randn(B, Hkv, D, generator=g).to(torch.bfloat16))
    d = {k: torch.empty(v.shape, dtype=v.dtype, device=dev) for k, v in h.items() if k != "out"}
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
    # grow capacity: a second, larger pool would be needed for long runs; the
    # instance pool was sized for warmup + steps uses per instance
    n_steps = max(1, min(args.steps, len(inst.steps)))
    ws = torch.empty(max(16, pa.pa_decode_workspace_size(B, Hq, int(inst.lens0.max()) + 2 * mb, D)),
                     dtype=torch.uint8, device=dev)
    slots_np, pairs_np = h["slots"].numpy(), h["pairs"].numpy()
    tables_np, lens_np = h["tables"].numpy(), h["lens"].numpy()
    kv_gb = 0.0
    h2d = d2h = 0
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n_steps):
        _, pairs = inst.alloc.batch_append(inst.seqs, np.ones(B, np.int32), out_slots=slots_np, out_pairs=pairs_np)
        inst.alloc.build_block_tables(inst.seqs, mb, out_tables=tables_np, out_lens=lens_np)
        npairs = len(pairs)
        for k in ("q", "k", "v", "slots", "tables", "lens"):
            d[k].copy_(h[k], non_blocking=True)
        if npairs:
            d["pairs"][:npairs].copy_(h["pairs"][:npairs], non_blocking=True)
            pa.pa_copy_blocks(d["pairs"][:npairs], inst.cache, stream)
        pa.pa_append_kv(d["k"], d["v"], d["slots"], inst.cache, stream)
        max_ctx = int(lens_np.max())
        pa.pa_decode(d["q"], inst.cache, d["tables"], d["lens"], max_ctx, 1.0 / math.sqrt(D), out=out,
                     workspace=ws, stream=stream)
        h["out"].copy_(out, non_blocking=True)
        torch.cuda.synchronize()
        kv_gb += float(lens_np.astype(np.int64).sum()) * 2 * Hkv * D * 2 / 1e9
        if i == 0:
            h2d = sum(h[k].numel() * h[k].element_size() for k in ("q", "k", "v", "slots", "tables", "lens"))
            h2d += npairs * 8
            d2h = h["out"].numel() * h["out"].element_size()
    seconds = time.perf_counter() - t0
    return {"seconds": seconds, "kv_gb": kv_gb, "steps": n_steps, "h2d": h2d, "d2h": d2h}


# ----------------------------------------------------------------- CPU oracle


def oracle_sample(wl, seed: int, budget_s: float, min_s: float):
    """Times the float64 oracle on the host over whole (sequence, kv head)
    groups of one batch of the workload until about budget_s of work.
    Returns (GB/s of KV processed, seconds, threads, description)."""
    import oracle
    from paged_kv_cache_402_b200 import synth

    B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
    lens = wl["lengths"](seed) + 1
    case = synth.random_case(seed, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=lens, dtype=torch.bfloat16, sentinel=False)
    G = Hq // Hkv
    order = synth.rng(seed + 9).permutation(B * Hkv)
    threads = oracle.max_threads()
    done_bytes, t_total, groups = 0, 0.0, 0
    i = 0
    while t_total < budget_s:
        chunk = order[i % len(order): i % len(order) + max(1, 2 * threads)]
        i += len(chunk)
        rows = [(int(u) // Hkv, (int(u) % Hkv) * G + gi) for u in chunk for gi in range(G)]
        t0 = time.perf_counter()
        oracle.decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale, rows=rows)
        t_total += time.perf_counter() - t0
        done_bytes += sum(int(lens[int(u) // Hkv]) * 2 * D * 2 for u in chunk)
        groups += len(chunk)
        if t_total >= min_s and groups >= len(order):
            break
    desc = (f"{groups} (sequence, kv head) groups ({groups * G} query rows) of one batch of the workload, "
            f"{t_total:.1f} s of oracle time")
    return done_bytes / 1e9 / t_total, t_total, threads, desc


def run_reference(args):
    """The oracle as it stands on the host cores: W untimed and K timed steps,
    each step a bounded sample of the workload (whole (sequence, kv head)
    groups of one batch, two per oracle thread, taken round-robin)."""
    import oracle
    from paged_kv_cache_402_b200 import synth

    wl = WORKLOADS[args.workload]
    B, Hq, Hkv, D, bs = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["bs"]
    G = Hq // Hkv
    lens = wl["lengths"](1) + 1
    case = synth.random_case(1, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=lens, dtype=torch.bfloat16, sentinel=False)
    order = synth.rng(10).permutation(B * Hkv)
    threads = oracle.max_threads()
    per_step = 2 * threads
    pos = 0
    total_bytes, total_s, groups = 0, 0.0, 0
    for s in range(args.warmup + args.steps):
        chunk = [int(order[(pos + i) % len(order)]) for i in range(per_step)]
        pos += per_step
        rows = [(u // Hkv, (u % Hkv) * G + gi) for u in chunk for gi in range(G)]
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
            f"round-robin over one batch of the workload; {total_s:.1f} s timed")
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
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="gqa")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rotate", type=int, default=0, help="batch instances to rotate (0: the workload's default)")
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
        line = run_ours(args, rank, world, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            wl = WORKLOADS[args.workload]
            gbs, secs, threads, desc = oracle_sample(wl, seed=1, budget_s=args.cpu_budget, min_s=min(5.0, args.cpu_budget))
            line["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                    "sample": desc}
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

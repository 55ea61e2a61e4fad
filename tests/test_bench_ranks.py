"""The replica path of bench.py on the host: two gloo ranks aggregate their
timings (slowest rank's time, summed work), and the reference arm prints one
line from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # rank r: 10 + r ms, (r + 1) GB, 100 tokens, e2e 2 + r s for (r + 1) GB
        res = bench.aggregate_ranks(world, 10.0 + rank, rank + 1.0, 100.0, 2.0 + rank, rank + 1.0,
                                    torch.device("cpu"))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        ms, gb, tok, e2e = json.load(open(tmp_path / f"r{r}.json"))
        assert ms == 11.0 and gb == 3.0 and tok == 200.0
        assert e2e == pytest.approx(3.0 / 3.0)


def test_single_rank_aggregation_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_ranks(1, 5.0, 2.0, 7.0, 4.0, 2.0, torch.device("cpu")) == (5.0, 2.0, 7.0, 0.5)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []


def test_block_size_choice_rule():
    """The fastest layout (block size, partition size) within the
    fragmentation budget; the smallest block size when none fits."""
    sys.path.insert(0, ROOT)
    import bench
    mk = lambda bs, tps, fr: {"config": {"block_size": bs}, "tokens_per_s": tps, "fragmentation_mean": fr,
                              "value": 1.0, "device_ms_per_step": 1.0}
    lines = [mk(8, 350e3, 0.014), mk(16, 530e3, 0.028), mk(32, 650e3, 0.056)]
    assert bench.choose_block_size(lines, 0.05)["block_size_choice"] == 16
    assert bench.choose_block_size(lines, 0.06)["block_size_choice"] == 32
    assert bench.choose_block_size(lines, 0.01)["block_size_choice"] == 8
    assert set(bench.choose_block_size(lines, 0.05)["per_layout"]) == {"bs8/p512", "bs16/p512", "bs32/p512"}
    # the partition size is the one of least device time at the chosen block
    # size, whatever the wall clock (host noise) says
    lines.append(dict(mk(16, 600e3, 0.028), config={"block_size": 16, "partition_tokens": 256},
                      device_ms_per_step=0.9))
    lines.append(dict(mk(16, 700e3, 0.028), config={"block_size": 16, "partition_tokens": 1024},
                      device_ms_per_step=1.1))
    pick = bench.choose_block_size(lines, 0.05)
    assert (pick["block_size_choice"], pick["partition_choice"]) == (16, 256)
    lines[-2]["device_ms_per_step"] = 1.2
    assert bench.choose_block_size(lines, 0.05)["partition_choice"] == 512


def test_traffic_record_follows_the_kernel_sources(tmp_path, monkeypatch):
    """The roofline's ncu traffic is reported only while the partition
    kernel's sources hash to the ones the record was captured on: a record of
    other sources gives None, and the hash moves when one of those sources
    does.  It is the captured traffic / algorithmic ratio applied to this
    run's algorithmic bytes per launch."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.profiled_traffic("no-such-workload", 1e9) is None
    # a copy of the kernel sources with records of its own
    root = tmp_path / "tree"
    csrc = root / "paged_kv_cache_402_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    for f in ("pa_decode_tc.cuh", "pa_decode_simt.cuh", "pa_device.cuh", "pa_tc.cuh"):
        (csrc / f).write_bytes(open(os.path.join(ROOT, "paged_kv_cache_402_b200", "csrc", f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.kernel_source_hash()
    rec = {"kernel_hash": h0,
           "captured_launch": {"dram_read_bytes": 1010, "dram_write_bytes": 10, "algorithmic_bytes": 1000}}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"gqa": rec}))
    assert bench.profiled_traffic("gqa", 5000) == 5100
    (root / "profiles" / "traffic.json").write_text(json.dumps({"gqa": dict(rec, kernel_hash="0" * 16)}))
    assert bench.profiled_traffic("gqa", 5000) is None
    (root / "profiles" / "traffic.json").write_text(json.dumps({"gqa": rec}))
    with open(csrc / "pa_decode_tc.cuh", "a") as f:
        f.write("\n")
    assert bench.kernel_source_hash() != h0
    assert bench.profiled_traffic("gqa", 5000) is None


def test_decode_launch_count():
    """gpu_launches counts every kernel of a decode call: the partition
    kernel once per slice (1024 sequences in its fine form, 8192 in its
    coarse form, fewer when the whole partitions would overflow 20 bits),
    the cascade once per 1024 plan groups, and the reduce when a row can
    have more than one partition or a plan is given."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.decode_launches(8, 131072, 512) == 2            # long context: partition + reduce
    assert bench.decode_launches(32, 400, 512) == 1              # one partition a row: no reduce
    assert bench.decode_launches(256, 8000, 512, n_groups=64) == 3   # cascade + partition + reduce
    assert bench.decode_launches(1024, 500, 1024, n_groups=1) == 3   # a plan alone needs the reduce
    assert bench.decode_launches(3000, 4000, 1024, n_groups=800) == 3  # coarse form: one partition launch
    assert bench.decode_launches(9000, 1000, 1024, n_groups=2100) == 2 + 3 + 1  # 2 slices, 3 cascades
    # 2^20 - 1 whole partitions at most per launch: 256 partitions a row -> 4095 sequences
    assert bench.decode_launches(5000, 256 * 512, 512) == 2 + 1

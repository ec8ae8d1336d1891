"""Host logic of bench.py: byte and op counts, roofline entries, the traffic table, and the
max-over-ranks reduction across two processes (gloo, CPU)."""
import os

import pytest
import torch.multiprocessing as mp

import bench
from rank_residual_w4a4_b200 import _build, twq


def test_weight_bytes_match_the_abi_size_query():
    _build.build()
    for m, n, r in ((512, 512, 32), (4096, 4096, 128), (14336, 4096, 256), (5120, 25600, 0)):
        assert bench.weight_bytes(m, n, r) == sum(twq.weights_sizes(m, n, r))
        b = 16
        xq, sx = twq.act_sizes(b, m)
        assert bench.act_bytes(b, m, n) == xq + sx + 2 * b * n


def test_op_counts():
    assert bench.int8_ops(2048, 4096, 14336, 128) == 2 * 2048 * 4096 * 14336 + 2 * 2048 * 4096 * 128
    assert bench.bf16_flops(2048, 14336, 128) == 2 * 2048 * 128 * 14336


def test_roofline_entries():
    peaks = (6453.7, 1686.7, 1412.9, "measured")
    d = bench.roofline_entry("decode16", 13.3e-6, peaks, None)
    assert d["bound"] == "hbm" and d["unit"] == "GB/s"
    assert abs(d["achieved"] - d["algorithmic_bytes"] / 13.3e-6 / 1e9) < 0.1
    assert abs(d["frac"] - d["achieved"] / 6453.7) < 1e-4
    p = bench.roofline_entry("gateup", 500e-6, peaks, 123)
    assert p["bound"] == "tensor" and p["peak"] == round(1686.7 * 2, 1) and p["traffic"] == 123


def test_traffic_table_is_tied_to_the_kernel_sources():
    path = os.path.join(bench.ROOT, "profiles", "fused_kernel_traffic.txt")
    lines = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    for wl, nbytes, hh in lines:
        h = bench.kernel_source_hash(bench.kernel_kind(wl))
        got = bench.profiled_traffic(wl)
        assert got == (int(nbytes) if hh == h else None)
    assert bench.kernel_kind("decode16_x") == "decode" and bench.kernel_kind("gateup") == "pair"
    assert bench.profiled_traffic("large") is not None  # captured from the committed sources


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    v = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
    bench.barrier(world)
    out[rank] = v
    dist.destroy_process_group()


def test_max_over_ranks_two_processes():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.0, 1: 2.0}


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference (the CPU oracle on the host cores) prints one JSON line
    with the keys of the benchmark contract."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, check=True).stdout.strip().splitlines()
    line = json.loads(out[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"] and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "workload" in line["config"]


def test_sample_rows_cover_every_row_block():
    for b in (1, 16, 129, 2048, 8192):
        rows = bench.sample_rows(b)
        assert rows.min() >= 0 and rows.max() == b - 1
        assert set(rows // 128) == set(range((b + 127) // 128))


def test_output_check_flags_a_wrong_row():
    import numpy as np
    rng = np.random.default_rng(1)
    y = rng.standard_normal((4, 256)).astype(np.float32)
    bits = (y.view(np.uint32) >> 16).astype(np.uint16)  # truncation: within one ulp
    assert bench.compare_rows(bits, bits)["ok"]
    bad = bits.copy()
    bad[2, 7] ^= 0x4000  # a large error in one element
    assert not bench.compare_rows(bad, bits)["ok"]


def test_kernel_timing_covers_at_least_200_launches():
    class P:
        pass
    for b, copies in ((16, 26), (8192, 4), (2048, 2)):
        p = P()
        p.b, p.copies = b, copies
        per, replays = bench.launch_plan(p)
        assert per % copies == 0 and per * replays >= bench.MIN_TIMED_LAUNCHES and replays >= 5


def test_gpus_flag_must_match_the_launched_ranks(monkeypatch):
    import sys
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "2", "--steps", "3", "--warmup", "3"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "ranks" in str(e.value)

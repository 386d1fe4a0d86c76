"""Host-side logic of bench.py, on CPU: FLOP and byte accounting, clock
parsing, max-over-ranks aggregation with gloo (world size 2), and the
reference (oracle) arm, including its rank-0-only behaviour under torchrun."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_prefill_flops_accounting():
    w = synth.LLAMA8B_PREFILL_16K
    n = w.n_q
    visited = w.B * w.Hq * n * (n + 1) // 2
    f = bench.prefill_flops(w, visited, 0)
    assert f["dense"] == pytest.approx(4 * 32 * 128 * (16384 * 16385 / 2))
    # Executed work counts whole tiles, including the masked half of the diagonal.
    assert f["executed"] == pytest.approx(2 * 128 * 128 * 128 * 2 * visited)
    assert f["dense"] < f["executed"] < f["dense"] * (1 + 1.0 / n)
    g = bench.prefill_flops(w, visited, visited // 2)
    assert g["executed"] == pytest.approx(f["executed"] * 0.75)


def test_decode_bytes_accounting():
    w = synth.DecodeWorkload(name="t", B=2, Hq=4, Hkv=2, Lmax=200, Lmin=1, d=128, Bc=64,
                             num_splits=2, tsf=1.0, seed=0)
    lens = np.array([200, 70])
    st = np.zeros((2, 2, 4), np.uint8)
    st[0, :, :4] = 1          # all four tiles of sequence 0 kept (64+64+64+8 keys)
    st[1, 0, :2] = [1, 2]     # sequence 1 head 0: tile 0 kept (64 keys), tile 1 skipped
    st[1, 1, :2] = [1, 1]     # head 1: both kept (64 + 6 keys)
    b = bench.decode_bytes(w, lens, st)
    assert b["k"] == (200 + 70) * 2 * 128 * 2
    assert b["v"] == (2 * 200 + 64 + 70) * 128 * 2
    assert b["total_dense"] - b["total"] == (b["k"] - b["v"])


def test_parse_clock_lines():
    lines = ["1965, 1965, 700.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "1800, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "1700, 1965, 1001.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "garbage"]
    r = bench.parse_clock_lines(lines)
    assert r["sm_mhz"] == 1800 and r["sm_max_mhz"] == 1965 and r["samples"] == 3
    assert r["reasons"] == ["sw_power_cap"]


def _reduce_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    got = bench.reduce_max([float(rank + 1), 10.0 - rank], world)
    out[rank] = got
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = 29611
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_reduce_worker, args=(2, port, out), nprocs=2, join=True)
        assert out[0] == [2.0, 10.0] and out[1] == [2.0, 10.0]
    assert bench.reduce_max([3.0], 1) == [3.0]


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--prefill", synth.TINY_PREFILL.name],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["unit"] == "TFLOP/s"
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_prints_on_rank0_only():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29612",
           os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference", "--steps", "1",
           "--warmup", "3", "--prefill", synth.TINY_PREFILL.name]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


def test_spread_units_and_leg_names():
    w = synth.LLAMA70B_PREFILL_128K
    u = bench.oracle_spread_units(w, 32)
    assert len(u) == 32 and u[0].tolist() == [0, 0, 0] and u[-1].tolist() == [0, 0, w.n_q - 1]
    assert np.all(np.diff(u[:, 2]) > 0)
    tiny = bench.oracle_spread_units(synth.TINY_PREFILL, 100)
    assert len(tiny) == synth.TINY_PREFILL.n_q  # never more tiles than the workload has
    assert set(bench.SHORT) == set(synth.PREFILL_WORKLOADS)
    assert set(bench.ORACLE_SAMPLE_TILES) == set(bench.SHORT.values())


def test_report_headline_and_legs():
    """report() on made-up leg timings: the headline value, roofline and
    per-leg fields come from the headline leg's executed FLOPs and time."""
    args = bench.main.__globals__["argparse"].Namespace(
        steps=10, warmup=3, gpus=1, reading="lit", only="all", no_cpu_baseline=True,
        extra_prefill=synth.LLAMA8B_PREFILL_16K.name, decode=synth.DECODE_B64_32K.name,
        decode_batch=0)
    w, w16 = synth.LLAMA70B_PREFILL_128K, synth.LLAMA8B_PREFILL_16K
    dw = synth.DECODE_B64_32K
    n = w.n_q
    vis = w.Hq * n * (n + 1) // 2
    legs = [
        {"name": "prefill_128k_lit", "key": "128k_lit", "kind": "prefill", "reading": "lit",
         "w": w, "launches": 1, "headline": True,
         "stats": {"skipped": 0, "visited": vis, **bench.prefill_flops(w, vis, 0)}},
        {"name": "prefill_16k_rms", "key": "16k_rms", "kind": "prefill", "reading": "rms",
         "w": w16, "launches": 1,
         "stats": {"skipped": 50, "visited": 100, **bench.prefill_flops(w16, 100, 50)}},
    ]
    ms = {"prefill_128k_lit": 280.0, "prefill_16k_rms": 1.0}
    ms_dense = {"prefill_128k_lit": 280.0, "prefill_16k_rms": 1.5}
    peaks = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    line = bench.report(args, w, dw, 1, legs, ms, ms_dense, {}, (0, 0), peaks, "measured",
                        {"sm_mhz": 1965})
    ex = 2.0 * 128 * 128 * 128 * 2 * vis
    assert line["value"] == pytest.approx(ex / 0.280 / 1e12)
    assert line["roofline"]["frac"] == pytest.approx(line["value"] / 1600.0)
    assert line["roofline"]["leg"] == "128k_lit" and line["config"]["workload"] == w.name
    p = line["prefill"]["16k_rms"]
    assert p["skip_fraction"] == 0.5 and p["speedup_vs_skip_disabled"] == pytest.approx(1.5)
    assert p["ideal_speedup"] == pytest.approx(1 / 0.75)
    assert line["gpu_launches"] == 2 * 10

#!/usr/bin/env python
"""Benchmark of Skip-Softmax tiled attention on B200.

One step = one pass of the whole hot path over one batch of synthetic input of
every workload (each leg its own kernel launch, L2 flushed before it):
  * prefill on the Llama-3.3-70B-layer-shaped long workload (B=1, Hq=64,
    Hkv=8, L=131072, d=128, causal, Br=Bc=128, threshold_scale_factor=1000),
    literal generator reading (|u| = 1, as the workload is written) -- the
    headline -- and the rms reading (|u| = sqrt(d)) where planted tiles
    dominate;
  * prefill on the Llama-3.1-8B-shaped 16K workload (both readings, also with
    the per-warp 32-row vote), the video-DiT-shaped non-causal d=64 workload
    and the tiny 1K workload;
  * split-KV decode on the batch-64 GQA workload (Hq=32, Hkv=8, d=128, KV
    lengths uniform in [16K, 32K], Bc=64, 16 splits, tsf=500) followed by the
    log-sum-exp merge, both readings.

Every leg is also timed with skipping disabled (factor 0, same kernel) and
carries its CPU-oracle figure on a sample of whole query tiles.

`value` is the headline prefill throughput in executed TFLOP/s (tensor work
actually issued: 2 Br Bc d per visited tile for Q K^T plus 2 Br Bc d per kept
tile for P V), over all ranks. Dense-equivalent TFLOP/s, skip fractions and
the decode GB/s on bytes actually moved are reported beside it. `e2e` is the
same metric through the library's host-memory calls (sskip_attn_prefill_host,
which overlaps the copies with the kernels, and sskip_attn_decode_host),
pinned host inputs in and outputs out inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Other modes (one GPU): --sweep (speed vs skip over threshold factors on the
128K workload), --calibrate (factors calibrated to target skip ratios),
--reorder (video workload in raster vs Hilbert token order), --step (one
serving step with a factor per phase, eager and CUDA-graph replay).

For N > 1 launch under torch.distributed.run: every rank runs an independent
replica (the method has no cross-GPU exchange), times are maxed over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the headline
workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "prefill TFLOPS (dense-equiv & executed, % bf16 peak); decode GB/s (% HBM); skip %"
PROFILE_DIR = os.path.join(ROOT, "profiles")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- host logic
def prefill_flops(w, visited: int, skipped: int) -> dict:
    """Dense-equivalent and executed FLOPs of one prefill call."""
    P = w.L * (w.L + 1) // 2 if w.causal else w.L * w.L
    dense = 4.0 * w.B * w.Hq * w.d * P
    executed = 2.0 * w.Br * w.Bc * w.d * (2 * visited - skipped)
    return {"dense": dense, "executed": executed}


def decode_bytes(w, seqlens: np.ndarray, tile_state: np.ndarray) -> dict:
    """Bytes one decode call actually moves: every valid K row, the V rows of
    kept tiles, q, o, lse, seqlens, and the split partials (written + read)."""
    lens = np.asarray(seqlens, np.int64)
    k_bytes = int(lens.sum()) * w.Hkv * w.d * 2
    n_k = tile_state.shape[-1]
    keys_in_tile = np.clip(lens[:, None] - np.arange(n_k)[None, :] * w.Bc, 0, w.Bc)  # [B, n_k]
    kept = tile_state == 1                                                           # [B,Hkv,n_k]
    v_bytes = int((kept * keys_in_tile[:, None, :]).sum()) * w.d * 2
    v_dense = k_bytes
    small = w.B * w.Hq * w.d * 2 * 2 + w.B * w.Hq * 4 + w.B * 4
    partials = w.B * w.Hq * w.num_splits * (w.d + 1) * 4 * 2
    return {"k": k_bytes, "v": v_bytes, "v_dense": v_dense, "other": small + partials,
            "total": k_bytes + v_bytes + small + partials,
            "total_dense": k_bytes + v_dense + small + partials}


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "prefill_kernel": ("prefill_sm100.cuh", "sm100_ptx.cuh", "sm100_tmem.cuh", "skip_rule.cuh"),
    "decode_split_kernel": ("decode_sm100.cuh", "sm100_ptx.cuh", "skip_rule.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources one kernel is compiled from (its ncu record is
    stale as soon as they change)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_long_tiled_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(PROFILE_DIR, "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return float(rec["dram_bytes_per_launch"])


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def reduce_max(values: list[float], world: int, device=None) -> list[float]:
    """Max over ranks (identity for one rank)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        return parse_clock_lines(self.lines)


def parse_clock_lines(lines: list[str]) -> dict:
    sm, mx, reasons = [], [], set()
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 8:
            continue
        try:
            sm.append(float(parts[0]))
            mx.append(float(parts[1]))
        except ValueError:
            continue
        for name, val in zip(names, parts[4:8]):
            if val.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- oracle arm
def oracle_sample_units(w, heads: int, stride: int = 1) -> np.ndarray:
    """Whole query tiles of the first `heads` query heads (every `stride`-th tile)."""
    return np.array([(0, h, i) for h in range(heads) for i in range(0, w.n_q, stride)], np.int32)


def oracle_spread_units(w, n: int) -> np.ndarray:
    """n whole query tiles of query head 0 spread evenly over the query axis
    (for a causal workload: over the diagonal, light and heavy tiles alike)."""
    i = np.unique(np.linspace(0, w.n_q - 1, min(n, w.n_q)).round().astype(int))
    return np.array([(0, 0, int(t)) for t in i], np.int32)


# Short leg names of the prefill workloads.
SHORT = {synth.LLAMA70B_PREFILL_128K.name: "128k", synth.LLAMA8B_PREFILL_16K.name: "16k",
         synth.VIDEO_DIT_PREFILL.name: "video", synth.TINY_PREFILL.name: "tiny"}

# Whole query tiles per leg for the CPU-oracle figure (a few seconds each).
ORACLE_SAMPLE_TILES = {"128k": 8, "16k": 32, "video": 16, "tiny": 16}


def time_oracle(w, x, units: np.ndarray, nthreads: int) -> dict:
    import oracle  # CPU oracle: the baseline leg only
    t0 = time.perf_counter()
    out = oracle.prefill(x["q"], x["k"], x["v"], causal=w.causal, sm_scale=w.scale, tsf=w.tsf,
                         Br=w.Br, Bc=w.Bc, units=units, nthreads=nthreads)
    dt = time.perf_counter() - t0
    fl = 2.0 * w.Br * w.Bc * w.d * (2 * out["visited"] - out["skipped"])
    return {"seconds": dt, "executed_flops": fl, "visited": out["visited"],
            "skipped": out["skipped"]}


def run_reference(args, w, rank: int):
    """CPU oracle as the reference arm: each step is a bounded sample of the
    workload (32 whole query tiles of one query head, spread over the query
    axis)."""
    if rank != 0:
        return
    x = synth.prefill_inputs(w, args.reading)
    threads = os.cpu_count() or 1
    step_units = oracle_spread_units(w, 32)
    for _ in range(args.warmup):
        time_oracle(w, x, step_units, threads)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        r = time_oracle(w, x, step_units, threads)
        secs += r["seconds"]
        flops += r["executed_flops"]
    value = flops / secs / 1e12
    sample = (f"per step {len(step_units)} whole {w.Br}-row query tiles of query head 0 spread "
              f"evenly over the query axis, of {w.name}, {args.reading} reading")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_block(w, args),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(w, args) -> dict:
    dw = decode_workload(args)
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "d": w.d,
            "causal": w.causal, "Br": w.Br, "Bc": w.Bc, "threshold_scale_factor": w.tsf,
            "generator_reading": args.reading,
            "other_prefill_workloads": [n for n in args.extra_prefill.split(",")
                                        if n and n != w.name],
            "decode_workload": dw.name,
            "decode_threshold_scale_factor": dw.tsf, "decode_num_splits": dw.num_splits,
            "l2": "flushed before every timed kernel (256 MiB write)",
            "only": args.only, "parallelism": f"replicas x{args.gpus}"}


# ----------------------------------------------------------------- GPU arm
def run_gpu(args, w, rank: int, world: int, local_rank: int):
    import torch
    import block_sparse_long_tiled_b200 as sk

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(
            torch.bfloat16)

    readings = [r for r in args.readings.split(",") if r]
    if args.reading not in readings:
        readings.insert(0, args.reading)
    warp_readings = [r for r in args.warp_vote_readings.split(",") if r]
    dw = decode_workload(args)

    # ---- legs of the step: every prefill workload per generator reading,
    # then decode. The video workload has one reading (its generator has no
    # planted direction).
    works = [w] + [synth.PREFILL_WORKLOADS[n] for n in args.extra_prefill.split(",")
                   if n and n != w.name]
    legs = []
    if args.only != "decode":
        for wk in works:
            short = SHORT[wk.name]
            for rd in (["lit"] if wk.kind == "video" else readings):
                x = synth.prefill_inputs(wk, rd)
                t = {"q": to_dev(x["q"]), "k": to_dev(x["k"]), "v": to_dev(x["v"])}
                t["o"] = torch.empty_like(t["q"])
                t["lse"] = torch.empty((wk.B, wk.Hq, wk.L), dtype=torch.float32, device=dev)
                t["cnt"] = torch.zeros(2, dtype=torch.int64, device=dev)

                def run(t=t, wk=wk, tsf=None, tiles=None):
                    sk.sskip_attn_prefill(t["q"], t["k"], t["v"], t["o"], t["lse"],
                                          causal=wk.causal, sm_scale=wk.scale,
                                          threshold_scale_factor=wk.tsf if tsf is None else tsf,
                                          Br=wk.Br, Bc=wk.Bc, skip_count=t["cnt"],
                                          tile_state=tiles, stream=stream)
                head = wk is w and rd == args.reading
                legs.append({"name": f"prefill_{short}_{rd}", "key": f"{short}_{rd}",
                             "kind": "prefill", "reading": rd, "t": t, "host": x, "run": run,
                             "launches": 1, "w": wk, "headline": head, "e2e": head})
                if wk.name == args.warp_vote_workload and rd in warp_readings:
                    # Same inputs, vote taken per 32-row warp slice.
                    tw = dict(t, o=torch.empty_like(t["q"]), lse=torch.empty_like(t["lse"]),
                              cnt=torch.zeros(4, dtype=torch.int64, device=dev))

                    def run_w(t=tw, wk=wk, tsf=None, tiles=None):
                        sk.sskip_attn_prefill_vote(
                            t["q"], t["k"], t["v"], t["o"], t["lse"], causal=wk.causal,
                            sm_scale=wk.scale,
                            threshold_scale_factor=wk.tsf if tsf is None else tsf,
                            Br=wk.Br, Bc=wk.Bc, vote_rows=32, counts=t["cnt"], tile_state=tiles,
                            stream=stream)
                    legs.append({"name": f"prefill_{short}_{rd}_warp32",
                                 "key": f"{short}_{rd}_warp32", "kind": "prefill",
                                 "reading": rd, "vote": "warp32", "block_leg": f"prefill_{short}_{rd}",
                                 "t": tw, "host": x, "run": run_w, "launches": 1, "w": wk,
                                 "extra": True})
    if args.only != "prefill":
        for rd in (readings if args.decode_readings == "all" else [args.reading]):
            dx = synth.decode_inputs(dw, rd)
            t = {"q": to_dev(dx["q"]), "kc": to_dev(dx["kcache"]), "vc": to_dev(dx["vcache"]),
                 "lens": torch.from_numpy(dx["seqlens"]).to(dev),
                 "o": torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=dev),
                 "lse": torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=dev),
                 "ws": torch.empty(sk.sskip_attn_decode_workspace_size(dw.B, dw.Hq, dw.d,
                                                                       dw.num_splits),
                                   dtype=torch.uint8, device=dev),
                 "cnt": torch.zeros(2, dtype=torch.int64, device=dev)}

            def run(t=t, tsf=None, tiles=None):
                sk.sskip_attn_decode(t["q"], t["kc"], t["vc"], t["lens"], t["o"], t["lse"],
                                     sm_scale=dw.scale,
                                     threshold_scale_factor=dw.tsf if tsf is None else tsf,
                                     Bc=dw.Bc, num_splits=dw.num_splits, workspace=t["ws"],
                                     skip_count=t["cnt"], tile_state=tiles, stream=stream)
            legs.append({"name": f"decode_{rd}", "key": rd, "kind": "decode", "reading": rd,
                         "t": t, "host": {"q": dx["q"], "seqlens": dx["seqlens"]}, "run": run,
                         "launches": 2, "dw": dw, "e2e": rd == args.reading})
            del dx

    # ---- one untimed pass with tile records: skip counts, FLOPs, bytes moved
    for leg in legs:
        t = leg["t"]
        if leg["kind"] == "prefill":
            wk = leg["w"]
            tiles = torch.empty((wk.B, wk.Hq, wk.n_q, wk.n_k), dtype=torch.uint8, device=dev)
            leg["run"](tiles=tiles)
            c = t["cnt"].cpu().tolist()
            leg["stats"] = {"skipped": c[0], "visited": c[1], **prefill_flops(wk, c[1], c[0])}
            del tiles
            if len(c) == 4:
                leg["stats"].update(slices_skipped=c[2], slices_visited=c[3])
        else:
            tiles = torch.empty((dw.B, dw.Hkv, -(-dw.Lmax // dw.Bc)), dtype=torch.uint8, device=dev)
            leg["run"](tiles=tiles)
            c = t["cnt"].cpu().tolist()
            leg["stats"] = {"skipped": c[0], "visited": c[1],
                            **decode_bytes(dw, leg["host"]["seqlens"], tiles.cpu().numpy())}
    assert sk.sskip_get_status() == sk.SSKIP_OK
    names = [leg["name"] for leg in legs]

    def new_events():
        return {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for n in names}

    def timed(body, steps, only=None):
        """Run `body(events)` steps times after warm-up; device ms per leg
        (the legs in `only`, default all), max over ranks."""
        sel = names if only is None else [n for n in names if n in only]
        for _ in range(args.warmup):
            body(new_events())
        barrier()
        evs = [new_events() for _ in range(steps)]
        for i in range(steps):
            body(evs[i])
        barrier()
        ms = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in evs) / steps for n in sel}
        return dict(zip(sel, reduce_max([ms[n] for n in sel], world, dev)))

    def step(ev, tsf=None):
        for leg in legs:
            if tsf is not None and leg.get("extra"):
                continue  # the control at tsf = 0 is the same for both votes
            flush.zero_()
            ev[leg["name"]][0].record(stream)
            leg["run"](tsf=tsf)
            ev[leg["name"]][1].record(stream)

    props = torch.cuda.get_device_properties(dev)
    gpu_id = None
    if getattr(props, "uuid", None) is not None:
        u = str(props.uuid)
        gpu_id = u if u.startswith("GPU-") else f"GPU-{u}"
    clocks = ClockSampler(gpu_id)
    clocks.start()
    ms = timed(step, args.steps)
    clock_rec = clocks.stop()
    assert sk.sskip_get_status() == sk.SSKIP_OK

    # ---- skip-disabled control: the same kernels and inputs at tsf = 0
    core = [leg["name"] for leg in legs if not leg.get("extra")]
    ms_dense = timed(lambda ev: step(ev, tsf=0.0), max(3, args.steps // 3), only=core) \
        if not args.no_control else {}

    # ---- end to end through the public API: pinned host in, host out
    ems, io_bytes = ({}, (0, 0)) if args.no_e2e else time_e2e(legs, flush, stream, new_events,
                                                             timed, args.steps,
                                                             args.e2e_kv_per_chunk)

    if rank == 0:
        print(json.dumps(report(args, w, dw, world, legs, ms, ms_dense, ems, io_bytes, peaks,
                                peak_kind, clock_rec)), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def time_e2e(legs, flush, stream, new_events, timed, steps, kv_per_chunk=0):
    """Same steps with each leg's inputs copied host->device from pinned memory
    and its outputs copied back inside the timed region."""
    import torch
    legs = [leg for leg in legs if leg.get("e2e")]
    h2d = d2h = 0
    for leg in legs:
        t = leg["t"]
        if leg["kind"] == "prefill":
            leg["pin_in"] = {n: torch.from_numpy(np.ascontiguousarray(leg["host"][n]).view(
                np.int16)).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v")}
            leg["dev_in"] = {n: t[n] for n in ("q", "k", "v")}
        else:
            leg["pin_in"] = {"q": torch.from_numpy(np.ascontiguousarray(leg["host"]["q"]).view(
                np.int16)).view(torch.bfloat16).pin_memory(),
                "lens": torch.from_numpy(leg["host"]["seqlens"]).pin_memory()}
            leg["dev_in"] = {"q": t["q"], "lens": t["lens"]}
        leg["pin_out"] = (torch.empty_like(t["o"], device="cpu").pin_memory(),
                          torch.empty_like(t["lse"], device="cpu").pin_memory())
        h2d += sum(int(v.numel() * v.element_size()) for v in leg["pin_in"].values())
        d2h += sum(int(v.numel() * v.element_size()) for v in leg["pin_out"])

    import block_sparse_long_tiled_b200 as sk

    def e2e_step(ev):
        for leg in legs:
            t = leg["t"]
            flush.zero_()
            ev[leg["name"]][0].record(stream)
            if leg["kind"] == "prefill":
                # Host buffers through the library's overlapped host-memory call.
                w = leg["w"]
                host = dict(leg["pin_in"], o=leg["pin_out"][0], lse=leg["pin_out"][1])
                dev = dict(leg["dev_in"], o=t["o"], lse=t["lse"])
                sk.sskip_attn_prefill_host(host, dev, causal=w.causal, sm_scale=w.scale,
                                           threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc,
                                           kv_per_chunk=kv_per_chunk, skip_count=t["cnt"],
                                           stream=stream)
            else:
                dw = leg["dw"]
                host = {"q": leg["pin_in"]["q"], "seqlens": leg["pin_in"]["lens"],
                        "o": leg["pin_out"][0], "lse": leg["pin_out"][1]}
                dev = {"q": t["q"], "seqlens": t["lens"], "o": t["o"], "lse": t["lse"]}
                sk.sskip_attn_decode_host(host, dev, t["kc"], t["vc"], sm_scale=dw.scale,
                                          threshold_scale_factor=dw.tsf, Bc=dw.Bc,
                                          num_splits=dw.num_splits, workspace=t["ws"],
                                          skip_count=t["cnt"], stream=stream)
            ev[leg["name"]][1].record(stream)

    return timed(e2e_step, steps, only=[leg["name"] for leg in legs]), (h2d, d2h)


def leg_oracle_baseline(leg) -> dict:
    """The CPU oracle on a sample of whole query tiles of the leg's inputs."""
    wk = leg["w"]
    units = oracle_spread_units(wk, ORACLE_SAMPLE_TILES[SHORT[wk.name]])
    threads = os.cpu_count() or 1
    r = time_oracle(wk, leg["host"], units, threads)
    return {"value": r["executed_flops"] / r["seconds"] / 1e12, "unit": "TFLOP/s",
            "cores": threads, "kind": "oracle", "seconds": r["seconds"],
            "sample": (f"{len(units)} whole {wk.Br}-row query tiles of query head 0 spread "
                       f"evenly over the query axis, {wk.name}, {leg['reading']} reading; "
                       f"executed FLOPs / wall time")}


def report(args, w, dw, world, legs, ms, ms_dense, ems, io_bytes, peaks, peak_kind,
           clock_rec) -> dict:
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sustained = float(peaks.get("bf16_tflops_sustained",
                                     FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    K = args.steps
    line = {"metric": METRIC, "value": None, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": sum(ms.values()), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_block(w, args)}
    pre, dec = {}, {}
    cpu_ok = not args.no_cpu_baseline and world == 1
    for leg in legs:
        n, s = leg["name"], leg["stats"]
        t = ms[n] / 1e3
        b = {"ms_per_launch": ms[n], "skip_fraction": s["skipped"] / max(1, s["visited"]),
             "skipped_tiles": s["skipped"], "visited_tiles": s["visited"]}
        if leg["kind"] == "prefill":
            b.update(workload=leg["w"].name, reading=leg["reading"],
                     executed_tflops=s["executed"] / t / 1e12,
                     dense_equiv_tflops=s["dense"] / t / 1e12,
                     executed_frac_of_peak=s["executed"] / t / 1e12 / peak,
                     executed_tflop=s["executed"] / 1e12, dense_equiv_tflop=s["dense"] / 1e12)
            ideal = 1.0 / (1.0 - b["skip_fraction"] / 2.0)
        else:
            b.update(gbs_actually_moved=s["total"] / t / 1e9,
                     frac_of_hbm=s["total"] / t / 1e9 / hbm,
                     bytes_actually_moved=s["total"], bytes_if_no_skip=s["total_dense"])
            ideal = s["total_dense"] / s["total"]
        if n in ms_dense:
            b.update(ms_skip_disabled=ms_dense[n], speedup_vs_skip_disabled=ms_dense[n] / ms[n],
                     ideal_speedup=ideal)
        if n in ems:
            b["e2e_ms"] = ems[n]
        if leg.get("vote"):
            b.update(vote_rows=32, slice_skip_fraction=s["slices_skipped"] / max(1, s["slices_visited"]),
                     slices_skipped=s["slices_skipped"], slices_visited=s["slices_visited"])
            if leg["block_leg"] in ms:
                b["speedup_vs_block_vote"] = ms[leg["block_leg"]] / ms[n]
        elif leg["kind"] == "prefill" and cpu_ok:
            b["cpu_baseline"] = leg_oracle_baseline(leg)
        (pre if leg["kind"] == "prefill" else dec)[leg["key"]] = b
    head = next((leg for leg in legs if leg.get("headline")), None)
    if head is not None:
        hs = head["stats"]
        t = ms[head["name"]] / 1e3
        achieved = hs["executed"] / t / 1e12
        line["value"] = world * achieved
        line["roofline"] = {
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": ncu_traffic("prefill_kernel"),
            "frac_of_sustained": achieved / peak_sustained,
            "kernel": f"prefill_kernel<{w.d},{w.Br},{w.Bc},{'causal' if w.causal else 'full'}>",
            "leg": head["key"],
            "peak_source": f"{peak_kind} bf16_tflops (burst, the conservative figure; the SM "
                           f"clock seen during the step is under clocks)"}
        line["prefill"] = pre
        if head["name"] in ems:
            line["e2e"] = {"value": world * hs["executed"] / (ems[head["name"]] / 1e3) / 1e12,
                           "unit": "TFLOP/s", "h2d_bytes_per_step": io_bytes[0],
                           "d2h_bytes_per_step": io_bytes[1], "leg": head["key"]}
        if "cpu_baseline" in pre[head["key"]]:
            line["cpu_baseline"] = pre[head["key"]]["cpu_baseline"]
    elif pre:
        line["prefill"] = pre
    if dec:
        dkey = args.reading if args.reading in dec else next(iter(dec))
        dstats = next(leg["stats"] for leg in legs if leg["name"] == f"decode_{dkey}")
        gbs = dec[dkey]["gbs_actually_moved"]
        dec["workload"] = dw.name
        dec["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                           "frac": gbs / hbm, "traffic": ncu_traffic("decode_split_kernel"),
                           "reading": dkey, "peak_source": f"{peak_kind} hbm_gbs"}
        line["decode"] = dec
        if head is None:  # decode-only runs report GB/s as the value
            line.update(value=world * gbs, unit="GB/s", roofline=dec["roofline"])
            if f"decode_{dkey}" in ems:
                line["e2e"] = {"value": world * dstats["total"] / (ems[f"decode_{dkey}"] / 1e3) / 1e9,
                               "unit": "GB/s", "h2d_bytes_per_step": io_bytes[0],
                               "d2h_bytes_per_step": io_bytes[1]}
    line["clocks"] = clock_rec
    line["gpu_launches"] = sum(leg["launches"] for leg in legs) * K
    return line


def run_sweep(args):
    """Long-prefill threshold sweep: speed vs skip fraction at each factor."""
    import torch
    import block_sparse_long_tiled_b200 as sk
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    w0 = synth.PREFILL_WORKLOADS[args.prefill]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for rd in [r for r in args.readings.split(",") if r]:
        x = synth.prefill_inputs(w0, rd)
        td = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(
            torch.bfloat16)
        q, k, v = td(x["q"]), td(x["k"]), td(x["v"])
        del x
        base_ms = None
        hx = synth.prefill_inputs(w0, rd) if args.sweep_oracle else None
        for tsf in synth.LLAMA70B_TSF_SWEEP:
            w = w0.replace(tsf=tsf)
            out = sk.prefill(q, k, v, causal=w.causal, sm_scale=w.scale,
                             threshold_scale_factor=tsf, Br=w.Br, Bc=w.Bc)
            c = out["counts"].cpu().tolist()
            ts = []
            for i in range(args.warmup + args.steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                sk.sskip_attn_prefill(q, k, v, out["o"], out["lse"], causal=w.causal,
                                      sm_scale=w.scale, threshold_scale_factor=tsf, Br=w.Br,
                                      Bc=w.Bc)
                b.record()
                torch.cuda.synchronize()
                if i >= args.warmup:
                    ts.append(a.elapsed_time(b))
            ms = float(np.median(ts))
            base_ms = ms if tsf == 0 else base_ms
            f = prefill_flops(w, c[1], c[0])
            s = c[0] / max(1, c[1])
            ora = {}
            if hx is not None:
                # The oracle on a stratified sample of whole query tiles,
                # extrapolated to the call by executed FLOPs (labelled as such).
                units = np.array([(0, h, i) for h in (0, w.Hq // 2)
                                  for i in np.linspace(0, w.n_q - 1, 8).astype(int)], np.int32)
                r = time_oracle(w, hx, units, os.cpu_count() or 1)
                ora = {"oracle_sample_units": int(len(units)), "oracle_sample_s": r["seconds"],
                       "oracle_extrapolated_s": r["seconds"] * f["executed"] / r["executed_flops"],
                       "oracle_cores": os.cpu_count() or 1}
            print(json.dumps({"sweep": w.name, "reading": rd, "threshold_scale_factor": tsf,
                              **ora, "ms": ms, "skip_fraction": s,
                              "executed_tflops": f["executed"] / ms / 1e9,
                              "executed_frac_of_peak": f["executed"] / ms / 1e9 / peak,
                              "dense_equiv_tflops": f["dense"] / ms / 1e9,
                              "speedup_vs_tsf0": (base_ms / ms) if base_ms else None,
                              "ideal_speedup": 1.0 / (1.0 - s / 2.0)}), flush=True)
        del q, k, v
        torch.cuda.empty_cache()


def run_calibration(args):
    """Calibrate the factor to target skip ratios (one recording pass plus
    the host selection), then time the kernel at each calibrated factor."""
    import torch
    import block_sparse_long_tiled_b200 as sk
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    td = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(
        torch.bfloat16)
    targets = [float(t) for t in args.targets.split(",") if t]

    def _unreachable_text(e) -> str:
        # SSKIP_ERR_UNSUPPORTED from the selection: no factor below the
        # smallest context length skips that share (the record holds only
        # while t = factor / L < 1).
        if getattr(e, "status", None) == sk.SSKIP_ERR_UNSUPPORTED:
            return "no factor below the context length reaches this share (t must stay < 1)"
        return str(e)

    def time_it(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    w = synth.PREFILL_WORKLOADS[args.prefill]
    for rd in [r for r in args.readings.split(",") if r]:
        x = synth.prefill_inputs(w, rd)
        q, k, v = td(x["q"]), td(x["k"]), td(x["v"])
        del x
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        cnt = torch.zeros(2, dtype=torch.int64, device=dev)

        def run(f):
            sk.sskip_attn_prefill(q, k, v, o, lse, causal=w.causal, sm_scale=w.scale,
                                  threshold_scale_factor=f, Br=w.Br, Bc=w.Bc, skip_count=cnt)
        dense_ms = time_it(lambda: run(0.0))
        for tgt in targets:
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            try:
                r = sk.calibrate_prefill(q, k, v, causal=w.causal, sm_scale=w.scale,
                                         target_ratio=tgt, Br=w.Br, Bc=w.Bc)
            except sk.SSkipError as e:
                print(json.dumps({"calibration": w.name, "reading": rd, "target": tgt,
                                  "unreachable": _unreachable_text(e)}), flush=True)
                continue
            cal_s = time.perf_counter() - t0
            ms = time_it(lambda: run(r["factor"]))
            c = cnt.cpu().tolist()
            f = prefill_flops(w, c[1], c[0])
            s = c[0] / max(1, c[1])
            print(json.dumps({"calibration": w.name, "reading": rd, "target": tgt,
                              "threshold_scale_factor": r["factor"],
                              "predicted_ratio": r["achieved_ratio"], "skip_fraction": s,
                              "calibration_wall_s": cal_s, "ms": ms, "ms_dense": dense_ms,
                              "speedup_vs_dense": dense_ms / ms,
                              "ideal_speedup": 1.0 / (1.0 - s / 2.0),
                              "executed_tflops": f["executed"] / ms / 1e9,
                              "executed_frac_of_peak": f["executed"] / ms / 1e9 / peak}),
                  flush=True)
        del q, k, v, o
        torch.cuda.empty_cache()

    dw = decode_workload(args)
    for rd in [r for r in args.readings.split(",") if r]:
        dx = synth.decode_inputs(dw, rd)
        q, kc, vc = td(dx["q"]), td(dx["kcache"]), td(dx["vcache"])
        lens = torch.from_numpy(dx["seqlens"]).to(dev)
        o = torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(sk.sskip_attn_decode_workspace_size(dw.B, dw.Hq, dw.d, dw.num_splits),
                         dtype=torch.uint8, device=dev)
        cnt = torch.zeros(2, dtype=torch.int64, device=dev)
        tiles = torch.empty((dw.B, dw.Hkv, -(-dw.Lmax // dw.Bc)), dtype=torch.uint8, device=dev)

        def run_d(f, rec=None):
            sk.sskip_attn_decode(q, kc, vc, lens, o, lse, sm_scale=dw.scale,
                                 threshold_scale_factor=f, Bc=dw.Bc, num_splits=dw.num_splits,
                                 workspace=ws, skip_count=cnt, tile_state=rec)
        dense_ms = time_it(lambda: run_d(0.0))
        for tgt in targets:
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            try:
                r = sk.calibrate_decode(q, kc, vc, lens, sm_scale=dw.scale, target_ratio=tgt,
                                        Bc=dw.Bc, num_splits=dw.num_splits)
            except sk.SSkipError as e:
                print(json.dumps({"calibration": dw.name, "reading": rd, "target": tgt,
                                  "unreachable": _unreachable_text(e)}), flush=True)
                continue
            cal_s = time.perf_counter() - t0
            run_d(r["factor"], tiles)
            by = decode_bytes(dw, dx["seqlens"], tiles.cpu().numpy())
            ms = time_it(lambda: run_d(r["factor"]))
            c = cnt.cpu().tolist()
            print(json.dumps({"calibration": dw.name, "reading": rd, "target": tgt,
                              "threshold_scale_factor": r["factor"],
                              "predicted_ratio": r["achieved_ratio"],
                              "skip_fraction": c[0] / max(1, c[1]), "calibration_wall_s": cal_s,
                              "ms": ms, "ms_dense": dense_ms, "speedup_vs_dense": dense_ms / ms,
                              "ideal_speedup": by["total_dense"] / by["total"],
                              "gbs_actually_moved": by["total"] / ms / 1e6,
                              "frac_of_hbm": by["total"] / ms / 1e6 / hbm}), flush=True)
        del q, kc, vc, dx
        torch.cuda.empty_cache()


def run_reorder(args):
    """Video prefill in raster and in Hilbert token order (block and per-warp
    votes): skip fractions, attention time, and the time and bandwidth of the
    row gathers (Q, K, V) and scatters (O, lse) that reorder the tokens."""
    import torch
    import block_sparse_long_tiled_b200 as sk
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    w = synth.PREFILL_WORKLOADS[args.prefill]
    if args.tsf is not None:
        w = w.replace(tsf=args.tsf)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    td = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(
        torch.bfloat16)
    x = synth.prefill_inputs(w, args.reading)
    q, k, v = td(x["q"]), td(x["k"]), td(x["v"])
    del x
    perm_h = sk.sskip_hilbert3d_order(*w.video_grid, w.L)
    perm = torch.from_numpy(perm_h).to(dev)
    qp, kp, vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    o, op = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    lsep = torch.empty_like(lse)
    cnt = torch.zeros(4, dtype=torch.int64, device=dev)

    def time_it(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    def gather():
        for a, b in ((q, qp), (k, kp), (v, vp)):
            sk.sskip_permute_rows(a, b, perm, scatter=False)

    def scatter():
        sk.sskip_permute_rows(op, o, perm, scatter=True)
        sk.sskip_permute_rows(lsep.unsqueeze(-1), lse.unsqueeze(-1), perm, scatter=True)

    gather()
    g_ms = time_it(gather)
    s_ms = time_it(scatter)
    g_bytes = 3 * 2 * q.numel() * q.element_size()
    s_bytes = 2 * (o.numel() * o.element_size() + lse.numel() * 4)
    rows = []
    for order, (qq, kk, vv, oo, ll) in (("raster", (q, k, v, o, lse)),
                                        ("hilbert", (qp, kp, vp, op, lsep))):
        for vote in (w.Br, 32):
            # The block vote runs the plain kernel; the per-warp vote its own
            # instantiation (sskip_attn_prefill_vote), timed against a dense
            # control of that same instantiation.
            def run(f=w.tsf, vote=vote):
                if vote == w.Br:
                    sk.sskip_attn_prefill(qq, kk, vv, oo, ll, causal=w.causal, sm_scale=w.scale,
                                          threshold_scale_factor=f, Br=w.Br, Bc=w.Bc,
                                          skip_count=cnt)
                else:
                    sk.sskip_attn_prefill_vote(qq, kk, vv, oo, ll, causal=w.causal,
                                               sm_scale=w.scale, threshold_scale_factor=f,
                                               Br=w.Br, Bc=w.Bc, vote_rows=vote, counts=cnt)
            run()
            c = cnt.cpu().tolist()
            ms = time_it(run)
            ms0 = time_it(lambda: run(0.0))
            f = prefill_flops(w, c[1], c[0])
            rows.append({"order": order, "vote_rows": vote, "ms": ms, "ms_dense": ms0,
                         "speedup_vs_dense": ms0 / ms,
                         "skip_fraction": c[0] / c[1],
                         "slice_skip_fraction": (c[2] / c[3]) if vote != w.Br else c[0] / c[1],
                         "executed_tflops": f["executed"] / ms / 1e9,
                         "executed_frac_of_peak": f["executed"] / ms / 1e9 / peak,
                         "dense_equiv_tflops": f["dense"] / ms / 1e9})
    dense_ms = time_it(lambda: sk.sskip_attn_prefill(q, k, v, o, lse, causal=w.causal,
                                                     sm_scale=w.scale, threshold_scale_factor=0.0,
                                                     Br=w.Br, Bc=w.Bc))
    print(json.dumps({"reorder": w.name, "reading": args.reading,
                      "threshold_scale_factor": w.tsf, "ms_dense": dense_ms,
                      "gather_qkv_ms": g_ms, "gather_gbs": g_bytes / g_ms / 1e6,
                      "gather_frac_of_hbm": g_bytes / g_ms / 1e6 / hbm,
                      "scatter_o_lse_ms": s_ms, "scatter_gbs": s_bytes / s_ms / 1e6,
                      "runs": rows}), flush=True)


def run_step_bench(args):
    """One serving step (prefill + decode of one layer, factors 1000 / 500 by
    phase) through sskip_attn_step: eager launches and the same step replayed
    from a CUDA graph."""
    import torch
    import block_sparse_long_tiled_b200 as sk
    dev = torch.device("cuda", 0)
    w = synth.PREFILL_WORKLOADS[args.prefill]
    dw = decode_workload(args)
    td = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(
        torch.bfloat16)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    x = synth.prefill_inputs(w, args.reading)
    P = {"q": td(x["q"]), "k": td(x["k"]), "v": td(x["v"])}
    del x
    P["o"] = torch.empty_like(P["q"])
    P["lse"] = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
    P["count"] = torch.zeros(2, dtype=torch.int64, device=dev)
    dx = synth.decode_inputs(dw, args.reading)
    D = {"q": td(dx["q"]), "kcache": td(dx["kcache"]), "vcache": td(dx["vcache"]),
         "seqlens": torch.from_numpy(dx["seqlens"]).to(dev)}
    del dx
    D["o"] = torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=dev)
    D["lse"] = torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=dev)
    D["workspace"] = torch.empty(sk.sskip_attn_decode_workspace_size(dw.B, dw.Hq, dw.d,
                                                                     dw.num_splits),
                                 dtype=torch.uint8, device=dev)
    D["count"] = torch.zeros(2, dtype=torch.int64, device=dev)
    factors = {"prefill": w.tsf, "decode": dw.tsf}

    def step():
        sk.sskip_attn_step(threshold_scale_factor=factors, sm_scale=w.scale, prefill=P,
                           decode=D, Br=w.Br, Bc=w.Bc, causal=w.causal,
                           num_splits=dw.num_splits)

    def time_it(fn):
        ts = []
        for i in range(args.warmup + args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= args.warmup:
                ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    step()
    torch.cuda.synchronize()
    eager = time_it(step)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        step()
    graph = time_it(g.replay)
    assert sk.sskip_get_status() == sk.SSKIP_OK
    cp, cd = P["count"].cpu().tolist(), D["count"].cpu().tolist()
    print(json.dumps({"step": f"{w.name} + {dw.name}", "reading": args.reading,
                      "threshold_scale_factor": factors, "ms_eager": eager, "ms_graph": graph,
                      "prefill_skip_fraction": cp[0] / cp[1],
                      "decode_skip_fraction": cd[0] / cd[1], "launches": 3}), flush=True)
    del g


def decode_workload(args):
    dw = synth.DECODE_WORKLOADS[args.decode]
    if args.decode_batch:
        dw = dw.replace(B=args.decode_batch)
    return dw


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill", default=None, choices=sorted(synth.PREFILL_WORKLOADS),
                    help="headline prefill workload (default: the 128K workload; --calibrate "
                         "and --step default to the 16K one, --reorder to the video one)")
    ap.add_argument("--extra-prefill", default=",".join(
                        n.name for n in (synth.LLAMA8B_PREFILL_16K, synth.VIDEO_DIT_PREFILL,
                                         synth.TINY_PREFILL)),
                    help="further prefill workloads timed as legs of the step ('' for none)")
    ap.add_argument("--warp-vote-workload", default=synth.LLAMA8B_PREFILL_16K.name,
                    help="the workload whose legs are also timed with the per-warp vote")
    ap.add_argument("--decode", default=synth.DECODE_B64_32K.name,
                    choices=sorted(synth.DECODE_WORKLOADS))
    ap.add_argument("--tsf", type=float, default=None, help="override the prefill factor")
    ap.add_argument("--reading", default="lit", choices=list(synth.READINGS))
    ap.add_argument("--readings", default="lit,rms",
                    help="generator readings timed for prefill (the --reading one is the headline)")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="restrict the step (profiling of one kernel on a small device footprint)")
    ap.add_argument("--decode-batch", type=int, default=0, help="override the decode batch")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-kv-per-chunk", type=int, default=0,
                    help="kv heads per copy/compute group of the host-memory prefill (0: auto)")
    ap.add_argument("--no-control", action="store_true",
                    help="skip the tsf = 0 (skipping disabled) control timing")
    ap.add_argument("--decode-readings", choices=["all", "headline"], default="all")
    ap.add_argument("--warp-vote-readings", default="lit,rms",
                    help="readings also timed with the per-warp (32-row) vote; '' for none")
    ap.add_argument("--sweep", action="store_true",
                    help="threshold sweep of --prefill over 0, 100, 1000, 5000 (pass the 128K workload for the long-prefill sweep)")
    ap.add_argument("--sweep-oracle", action="store_true",
                    help="with --sweep: time the CPU oracle on a sample and extrapolate")
    ap.add_argument("--calibrate", action="store_true",
                    help="calibrate the factors to --targets skip ratios and time them")
    ap.add_argument("--targets", default="0.25,0.5,0.75")
    ap.add_argument("--reorder", action="store_true",
                    help="video prefill in raster vs Hilbert token order")
    ap.add_argument("--step", action="store_true",
                    help="one serving step (prefill + decode, factor per phase), eager and graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.prefill is None:
        args.prefill = (synth.LLAMA8B_PREFILL_16K.name if (args.calibrate or args.step) else
                        synth.VIDEO_DIT_PREFILL.name if args.reorder else
                        synth.LLAMA70B_PREFILL_128K.name)
    w = synth.PREFILL_WORKLOADS[args.prefill]
    if args.tsf is not None:
        w = w.replace(tsf=args.tsf)
    rank, world, local_rank = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.calibrate:
        run_calibration(args)
        return
    if args.reorder:
        run_reorder(args)
        return
    if args.step:
        run_step_bench(args)
        return
    run_gpu(args, w, rank, world, local_rank)


if __name__ == "__main__":
    main()

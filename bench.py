#!/usr/bin/env python
"""Benchmark of Skip-Softmax tiled attention on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * prefill on the Llama-3.1-8B-shaped workload (B=1, Hq=32, Hkv=8, L=16384,
    d=128, causal, Br=Bc=128, threshold_scale_factor=1000), literal generator
    reading (|u| = 1, as the workload is written) -- the headline -- and the
    rms reading (|u| = sqrt(d)) where planted tiles dominate;
  * split-KV decode on the batch-64 GQA workload (Hq=32, Hkv=8, d=128, KV
    lengths uniform in [16K, 32K], Bc=64, 16 splits, tsf=500) followed by the
    log-sum-exp merge.

`value` is the prefill throughput in executed TFLOP/s (tensor work actually
issued: 2 Br Bc d per visited tile for Q K^T plus 2 Br Bc d per kept tile for
P V), over all ranks. Dense-equivalent TFLOP/s, skip fractions and the decode
GB/s on bytes actually moved are reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 launch under torch.distributed.run: every rank runs an independent
replica (the method has no cross-GPU exchange), times are maxed over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same
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
    workload (a stratified quarter of one query head's tiles)."""
    if rank != 0:
        return
    x = synth.prefill_inputs(w, args.reading)
    threads = os.cpu_count() or 1
    step_units = oracle_sample_units(w, heads=1, stride=4)
    for _ in range(args.warmup):
        time_oracle(w, x, step_units, threads)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        r = time_oracle(w, x, step_units, threads)
        secs += r["seconds"]
        flops += r["executed_flops"]
    value = flops / secs / 1e12
    sample = (f"per step {len(step_units)} whole 128-row query tiles (every 4th tile of query "
              f"head 0) of {w.name}, {args.reading} reading")
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
            "generator_reading": args.reading, "decode_workload": dw.name,
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

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

    # ---- inputs (host-generated, seeded), resident in HBM before timing
    readings = [r for r in args.readings.split(",") if r]
    if args.reading not in readings:
        readings.insert(0, args.reading)
    if args.only == "decode":
        readings = []
    pre = {}
    for rd in readings:
        x = synth.prefill_inputs(w, rd)
        d = {"q": to_dev(x["q"]), "k": to_dev(x["k"]), "v": to_dev(x["v"])}
        d["o"] = torch.empty_like(d["q"])
        d["lse"] = torch.empty((w.B, w.Hq, w.L), dtype=torch.float32, device=dev)
        d["cnt"] = torch.zeros(2, dtype=torch.int64, device=dev)
        d["host"] = x
        pre[rd] = d
    dw = decode_workload(args)
    with_dec = args.only != "prefill"
    dx = synth.decode_inputs(dw, args.reading) if with_dec else None
    dec = {} if not with_dec else {
           "q": to_dev(dx["q"]), "kc": to_dev(dx["kcache"]), "vc": to_dev(dx["vcache"]),
           "lens": torch.from_numpy(dx["seqlens"]).to(dev),
           "o": torch.empty((dw.B, dw.Hq, dw.d), dtype=torch.bfloat16, device=dev),
           "lse": torch.empty((dw.B, dw.Hq), dtype=torch.float32, device=dev),
           "ws": torch.empty(sk.sskip_attn_decode_workspace_size(dw.B, dw.Hq, dw.d,
                                                                 dw.num_splits),
                             dtype=torch.uint8, device=dev),
           "cnt": torch.zeros(2, dtype=torch.int64, device=dev)}

    def run_prefill(d):
        sk.sskip_attn_prefill(d["q"], d["k"], d["v"], d["o"], d["lse"], causal=w.causal,
                              sm_scale=w.scale, threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc,
                              skip_count=d["cnt"], stream=stream)

    def run_decode():
        sk.sskip_attn_decode(dec["q"], dec["kc"], dec["vc"], dec["lens"], dec["o"], dec["lse"],
                             sm_scale=dw.scale, threshold_scale_factor=dw.tsf, Bc=dw.Bc,
                             num_splits=dw.num_splits, workspace=dec["ws"],
                             skip_count=dec["cnt"], stream=stream)

    # ---- one untimed pass with tile records: skip counts and V bytes moved
    stats = {}
    for rd, d in pre.items():
        tiles = torch.empty((w.B, w.Hq, w.n_q, w.n_k), dtype=torch.uint8, device=dev)
        sk.sskip_attn_prefill(d["q"], d["k"], d["v"], d["o"], d["lse"], causal=w.causal,
                              sm_scale=w.scale, threshold_scale_factor=w.tsf, Br=w.Br, Bc=w.Bc,
                              skip_count=d["cnt"], tile_state=tiles, stream=stream)
        c = d["cnt"].cpu().tolist()
        stats[rd] = {"skipped": c[0], "visited": c[1], **prefill_flops(w, c[1], c[0])}
    dc, dbytes = None, None
    if with_dec:
        dtiles = torch.empty((dw.B, dw.Hkv, -(-dw.Lmax // dw.Bc)), dtype=torch.uint8, device=dev)
        sk.sskip_attn_decode(dec["q"], dec["kc"], dec["vc"], dec["lens"], dec["o"], dec["lse"],
                             sm_scale=dw.scale, threshold_scale_factor=dw.tsf, Bc=dw.Bc,
                             num_splits=dw.num_splits, workspace=dec["ws"],
                             skip_count=dec["cnt"], tile_state=dtiles, stream=stream)
        dc = dec["cnt"].cpu().tolist()
        dbytes = decode_bytes(dw, dx["seqlens"], dtiles.cpu().numpy())
    assert sk.sskip_get_status() == sk.SSKIP_OK

    seg = list(pre) + (["dec"] if with_dec else [])
    launches_per_step = len(pre) + (2 if with_dec else 0)  # prefill per reading, split + merge

    def step(ev):
        for rd, d in pre.items():
            flush.zero_()
            ev[rd][0].record(stream)
            run_prefill(d)
            ev[rd][1].record(stream)
        if with_dec:
            flush.zero_()
            ev["dec"][0].record(stream)
            run_decode()
            ev["dec"][1].record(stream)

    def new_events():
        return {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for k in seg}

    for _ in range(args.warmup):
        step(new_events())
    props = torch.cuda.get_device_properties(dev)
    gpu_id = None
    if getattr(props, "uuid", None) is not None:
        u = str(props.uuid)
        gpu_id = u if u.startswith("GPU-") else f"GPU-{u}"
    clocks = ClockSampler(gpu_id)
    clocks.start()
    barrier()
    evs = [new_events() for _ in range(args.steps)]
    for i in range(args.steps):
        step(evs[i])
    barrier()
    clock_rec = clocks.stop()
    assert sk.sskip_get_status() == sk.SSKIP_OK

    ms = {k: sum(e[k][0].elapsed_time(e[k][1]) for e in evs) for k in seg}
    keys = list(ms)
    ms = dict(zip(keys, reduce_max([ms[k] for k in keys], world, dev)))
    K = args.steps

    if args.no_e2e:
        ems, hp, ho, hq_dec, hl_dec, ho_dec = None, {}, {}, None, None, None
    else:
        ems, hp, ho, hq_dec, hl_dec, ho_dec = time_e2e(args, pre, dec, dx, with_dec, seg, keys,
                                                      run_prefill, run_decode, flush, stream,
                                                      new_events, barrier, world, dev, K)
    if rank == 0:
        print(json.dumps(report(args, w, world, pre, stats, ms, ems, K, peaks, peak_kind, dw, dbytes,
                                dc, hp, ho, hq_dec, hl_dec, ho_dec, clock_rec,
                                launches_per_step)), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def time_e2e(args, pre, dec, dx, with_dec, seg, keys, run_prefill, run_decode, flush, stream,
             new_events, barrier, world, dev, K):
    """Same steps through the public API with pinned host buffers: H2D of the
    step's inputs and D2H of its outputs inside the timed region."""
    import torch
    hp = {rd: {n: torch.from_numpy(np.ascontiguousarray(pre[rd]["host"][n]).view(np.int16))
               .view(torch.bfloat16).pin_memory() for n in ("q", "k", "v")} for rd in pre}
    ho = {rd: (torch.empty_like(pre[rd]["o"], device="cpu").pin_memory(),
               torch.empty_like(pre[rd]["lse"], device="cpu").pin_memory()) for rd in pre}
    hq_dec = hl_dec = ho_dec = None
    if with_dec:
        hq_dec = torch.from_numpy(np.ascontiguousarray(dx["q"]).view(np.int16)).view(
            torch.bfloat16).pin_memory()
        hl_dec = torch.from_numpy(dx["seqlens"]).pin_memory()
        ho_dec = (torch.empty_like(dec["o"], device="cpu").pin_memory(),
                  torch.empty_like(dec["lse"], device="cpu").pin_memory())

    def e2e_step(ev):
        for rd, d in pre.items():
            flush.zero_()
            ev[rd][0].record(stream)
            for n in ("q", "k", "v"):
                d[n].copy_(hp[rd][n], non_blocking=True)
            run_prefill(d)
            ho[rd][0].copy_(d["o"], non_blocking=True)
            ho[rd][1].copy_(d["lse"], non_blocking=True)
            ev[rd][1].record(stream)
        if with_dec:
            flush.zero_()
            ev["dec"][0].record(stream)
            dec["q"].copy_(hq_dec, non_blocking=True)
            dec["lens"].copy_(hl_dec, non_blocking=True)
            run_decode()
            ho_dec[0].copy_(dec["o"], non_blocking=True)
            ho_dec[1].copy_(dec["lse"], non_blocking=True)
            ev["dec"][1].record(stream)

    for _ in range(args.warmup):
        e2e_step(new_events())
    barrier()
    eevs = [new_events() for _ in range(K)]
    for i in range(K):
        e2e_step(eevs[i])
    barrier()
    ems = {k: sum(e[k][0].elapsed_time(e[k][1]) for e in eevs) for k in keys}
    ems = dict(zip(keys, reduce_max([ems[k] for k in keys], world, dev)))
    return ems, hp, ho, hq_dec, hl_dec, ho_dec


def report(args, w, world, pre, stats, ms, ems, K, peaks, peak_kind, dw, dbytes, dc, hp, ho,
           hq_dec, hl_dec, ho_dec, clock_rec, launches_per_step) -> dict:
    head = args.reading
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {"metric": METRIC, "value": None, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": sum(ms.values()) / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_block(w, args)}

    def prefill_block(rd):
        s = stats[rd]
        t = ms[rd] / K / 1e3
        b = {"ms_per_launch": t * 1e3, "executed_tflops": s["executed"] / t / 1e12,
             "dense_equiv_tflops": s["dense"] / t / 1e12,
             "executed_frac_of_peak": s["executed"] / t / 1e12 / peak,
             "skip_fraction": s["skipped"] / max(1, s["visited"]),
             "skipped_tiles": s["skipped"], "visited_tiles": s["visited"],
             "executed_tflop": s["executed"] / 1e12, "dense_equiv_tflop": s["dense"] / 1e12}
        if ems is not None:
            b["e2e_ms_per_step"] = ems[rd] / K
        return b

    if pre:
        st = stats[head]
        t_launch = ms[head] / K / 1e3  # seconds per prefill launch
        achieved = st["executed"] / t_launch / 1e12
        line["value"] = world * st["executed"] * K / (ms[head] / 1e3) / 1e12
        line["roofline"] = {
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": ncu_traffic("prefill_kernel"),
            "kernel": f"prefill_kernel<{w.d},{w.Br},{w.Bc},{'causal' if w.causal else 'full'}>",
            "peak_source": f"{peak_kind} bf16_tflops (burst; kernel timed alone)"}
        line["prefill"] = {rd: prefill_block(rd) for rd in pre}
    if dbytes is not None:
        t_dec = ms["dec"] / K / 1e3
        dec_gbs = dbytes["total"] / t_dec / 1e9
        line["decode"] = {
            "workload": dw.name, "ms_per_launch": t_dec * 1e3, "gbs_actually_moved": dec_gbs,
            "frac_of_hbm": dec_gbs / hbm, "hbm_peak_gbs": hbm,
            "bytes_actually_moved": dbytes["total"], "bytes_if_no_skip": dbytes["total_dense"],
            "skip_fraction": dc[0] / max(1, dc[1]), "skipped_tiles": dc[0],
            "visited_tiles": dc[1],
            "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": dec_gbs / hbm, "traffic": ncu_traffic("decode_split_kernel"),
                         "peak_source": f"{peak_kind} hbm_gbs"}}
        if ems is not None:
            line["decode"]["e2e_ms_per_step"] = ems["dec"] / K
        if not pre:  # decode-only runs report GB/s as the value
            line.update(value=world * dec_gbs, unit="GB/s", roofline=line["decode"]["roofline"])
    if ems is not None and pre:
        h2d = sum(int(t.numel() * t.element_size()) for rd in pre for t in hp[rd].values())
        d2h = sum(int(a.numel() * a.element_size() + b.numel() * b.element_size())
                  for a, b in ho.values())
        if hq_dec is not None:
            h2d += int(hq_dec.numel() * 2 + hl_dec.numel() * 4)
            d2h += int(ho_dec[0].numel() * 2 + ho_dec[1].numel() * 4)
        line["e2e"] = {"value": world * stats[head]["executed"] * K / (ems[head] / 1e3) / 1e12,
                       "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    line["clocks"] = clock_rec
    line["gpu_launches"] = launches_per_step * K
    if not args.no_cpu_baseline and world == 1 and pre:
        units = oracle_sample_units(w, heads=args.cpu_heads)
        threads = os.cpu_count() or 1
        r = time_oracle(w, pre[head]["host"], units, threads)
        line["cpu_baseline"] = {
            "value": r["executed_flops"] / r["seconds"] / 1e12, "unit": "TFLOP/s",
            "cores": threads, "kind": "oracle", "seconds": r["seconds"],
            "sample": (f"all {w.n_q} query tiles of {args.cpu_heads} of {w.Hq} query heads "
                       f"({args.cpu_heads / w.Hq:.3f} of {w.name}, {head} reading), "
                       f"executed FLOPs / wall time")}
    return line


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
    ap.add_argument("--prefill", default=synth.LLAMA8B_PREFILL_16K.name,
                    choices=sorted(synth.PREFILL_WORKLOADS))
    ap.add_argument("--decode", default=synth.DECODE_B64_32K.name,
                    choices=sorted(synth.DECODE_WORKLOADS))
    ap.add_argument("--tsf", type=float, default=None, help="override the prefill factor")
    ap.add_argument("--reading", default="lit", choices=list(synth.READINGS))
    ap.add_argument("--readings", default="lit,rms",
                    help="generator readings timed for prefill (the --reading one is the headline)")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="restrict the step (profiling of one kernel on a small device footprint)")
    ap.add_argument("--decode-batch", type=int, default=0, help="override the decode batch")
    ap.add_argument("--cpu-heads", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    w = synth.PREFILL_WORKLOADS[args.prefill]
    if args.tsf is not None:
        w = w.replace(tsf=args.tsf)
    rank, world, local_rank = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    run_gpu(args, w, rank, world, local_rank)


if __name__ == "__main__":
    main()

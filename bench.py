#!/usr/bin/env python
"""Benchmark of the NF4 + double-quant frozen linear layer with LoRA on B200.

Headline (one JSON line on rank 0): forward + backward TFLOP/s of one
LLaMA-65B-shaped decoder layer's seven projections (hidden 8192, FFN 22016),
16 x 512 = 8192 tokens, LoRA rank 64, alpha 16, weights NF4 + double-quant.
A step is, for each projection: the fused forward (dequant-GEMM + LoRA) and the
backward (dX through the fused dequant-GEMM, dA, dB).  The weights are
quantized once, before timing, as a model load does; the encode, standalone
dequant and decode-shaped GEMV are measured beside it under "secondary".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 (torchrun, one rank per GPU) every rank runs an independent replica
of the same per-GPU workload (weak scaling, no data-path collective); the
process group is used only for the barrier and the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused NF4+LoRA linear fwd+bwd TFLOP/s and dequant/GEMV GB/s vs B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_fused_traffic.json")


def _sources_digest(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def fused_traffic():
    """DRAM bytes (read + written) of the average k_fused launch of the headline
    step and the algorithmic bytes of the same launches, from the ncu counters
    recorded in profiles/k_fused_traffic.json -- or (None, None) when those
    counters were not taken on the fused kernel's current source."""
    try:
        with open(TRAFFIC_FILE) as f:
            doc = json.load(f)
        if doc["source_sha256"] != _sources_digest(doc["sources"]):
            return None, None
        n = sum(v["launches_per_step"] for v in doc["per_launch"].values())
        traffic = sum((v["read"] + v["write"]) * v["launches_per_step"] for v in doc["per_launch"].values())
        algo = sum(v["algorithmic"] * v["launches_per_step"] for v in doc["per_launch"].values())
        return traffic // n, algo // n
    except (OSError, KeyError, ValueError, ZeroDivisionError):
        return None, None


FUSED_SOURCES = ["bit_nf4_quantized_encode_b200/csrc/gemm.cu", "bit_nf4_quantized_encode_b200/csrc/nf4_device.cuh",
                 "bit_nf4_quantized_encode_b200/csrc/sm100_ptx.cuh"]


def write_traffic(csv_paths):
    """Rebuild profiles/k_fused_traffic.json from ncu CSV logs of the --case runs
    (one file per shape and direction, named ..._{fwd|bwd}_NxK.csv; the last
    k_fused launch in each file is the measured one)."""
    import csv
    import re
    wl = workloads.LLAMA65B
    counts = {}
    for p in wl.projections:
        for d in ("fwd", "bwd"):
            key = f"{d}_{p.n}x{p.k}"
            counts[key] = counts.get(key, 0) + 1
    per = {}
    for path in csv_paths:
        m = re.search(r"(fwd|bwd)_(\d+)x(\d+)", os.path.basename(path))
        if not m:
            raise SystemExit(f"cannot tell direction and shape from {path}")
        d, n, k = m.group(1), int(m.group(2)), int(m.group(3))
        vals = {}
        with open(path) as f:
            lines = [ln for ln in f if ln.startswith('"')]
        for row in csv.DictReader(lines):
            if "k_fused" not in row.get("Kernel Name", ""):
                continue
            unit = row.get("Metric Unit", "")
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}.get(unit, 1)
            vals.setdefault(row["ID"], {})[row["Metric Name"]] = float(row["Metric Value"].replace(",", "")) * scale
        last = vals[max(vals, key=int)]
        # activations in, packed weight, LoRA factor and its rank-r operand, bf16 output
        algo = (2 * wl.m * (k if d == "fwd" else n) + n * k // 2 + n * k // 64 + 4 * (n * k // 16384)
                + 2 * wl.r * (n if d == "fwd" else k) + 2 * wl.m * wl.r + 2 * wl.m * (n if d == "fwd" else k))
        per[f"{d}_{n}x{k}"] = {"read": int(last["dram__bytes_read.sum"]), "write": int(last["dram__bytes_write.sum"]),
                               "algorithmic": int(algo), "launches_per_step": counts[f"{d}_{n}x{k}"],
                               "duration_ns": int(last.get("gpu__time_duration.sum", 0))}
    doc = {"what": "DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one k_fused launch per shape "
                   "and direction, LLaMA-65B layer projections at 8192 tokens, LoRA r 64; bench.py reads it for "
                   "roofline.traffic while source_sha256 matches the listed sources",
           "kernel": "k_fused", "workload": wl.name, "sources": FUSED_SOURCES,
           "source_sha256": _sources_digest(FUSED_SOURCES),
           "command": "python bench.py --case fused_{fwd,bwd} --case-n N --case-k K --case-m 8192 --case-iters 1; "
                      "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                      "--clock-control none -k regex:k_fused --csv --log-file traffic_{fwd,bwd}_NxK.csv <same command>",
           "per_launch": per}
    missing = set(counts) - set(per)
    if missing:
        raise SystemExit(f"no capture for {sorted(missing)}")
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(doc, f, indent=1)
    print(f"wrote {TRAFFIC_FILE}")


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self._t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

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
        if self._t:
            self._t.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return rank, local, world, pg


def barrier(pg, device=None):
    if pg is not None:
        if device is not None:
            pg.barrier(device_ids=[device.index])
        else:
            pg.barrier()


def max_over_ranks(pg, value: float, device=None) -> float:
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device if device is not None else "cpu")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- our arm
def layer_flops(wl) -> tuple:
    total, fused = 0, 0
    for p in wl.projections:
        f = workloads.linear_flops(p.n, p.k, wl.m, wl.r)
        total += f["total"]
        # FLOPs executed inside the fused dequant-GEMM launches: dense + LoRA up-projection
        fused += (2 * wl.m * p.n * p.k + 2 * wl.m * wl.r * p.n) + (2 * wl.m * p.n * p.k + 2 * wl.m * wl.r * p.k)
    return total, fused


def prepare_layer(qb, torch, wl, device):
    """Generate, upload and quantize the layer (untimed: a model load)."""
    projs = []
    for i, p in enumerate(wl.projections):
        w = workloads.weight((p.n, p.k), proj=i)
        qt = qb.qlora_quantize_nf4_dq(w.to(device))
        del w
        X = workloads.activations(wl.m, p.k, i)
        dY = workloads.grad_output(wl.m, p.n, i)
        st = dict(p=p, qt=qt, X_host=X.pin_memory(), dY_host=dY.pin_memory(),
                  X=X.to(device), dY=dY.to(device),
                  A=workloads.lora_a(wl.r, p.k, i).to(device), B=workloads.lora_b(p.n, wl.r, i).to(device))
        fw, bw = qb.qlora_linear_workspace_size(p.n, p.k, wl.m, wl.r)
        st["ws_f"] = torch.empty(fw, dtype=torch.uint8, device=device)
        st["ws_b"] = torch.empty(bw, dtype=torch.uint8, device=device)
        st["Y"] = torch.empty(wl.m, p.n, dtype=torch.bfloat16, device=device)
        st["XA"] = torch.empty(wl.m, wl.r, dtype=torch.float32, device=device)
        st["dX"] = torch.empty(wl.m, p.k, dtype=torch.bfloat16, device=device)
        st["dA"] = torch.empty(wl.r, p.k, dtype=torch.float32, device=device)
        st["dB"] = torch.empty(p.n, wl.r, dtype=torch.float32, device=device)
        st["dA_host"] = torch.empty(wl.r, p.k, dtype=torch.float32).pin_memory()
        st["dB_host"] = torch.empty(p.n, wl.r, dtype=torch.float32).pin_memory()
        projs.append(st)
    torch.cuda.synchronize()
    return projs


def run_step(qb, wl, projs, events=None):
    s = wl.s
    for st in projs:
        if events is not None:
            e0, e1 = events.pop()
            qb.qlora_time_next_gemm(e0, e1)
        qb.qlora_linear_fwd(st["qt"], st["X"], st["A"], st["B"], s, save_xa=True, Y=st["Y"], XA=st["XA"],
                            workspace=st["ws_f"])
        if events is not None:
            e0, e1 = events.pop()
            qb.qlora_time_next_gemm(e0, e1)
        qb.qlora_linear_bwd(st["qt"], st["X"], st["dY"], st["A"], st["B"], s, XA=st["XA"], dX=st["dX"],
                            dA=st["dA"], dB=st["dB"], workspace=st["ws_b"])


def run_step_e2e(qb, wl, projs, copy_stream):
    """Same step through the public API with inputs copied from pinned host memory
    and the LoRA gradients read back.

    The uploads run on their own stream, one projection after another, and each
    projection's forward and backward start as soon as its own inputs have
    landed. An upload waits until the previous step has finished with that
    projection's device buffers, so consecutive steps pipeline as a training
    loop that prefetches its inputs would. Every byte is still copied inside the
    step it belongs to."""
    import torch
    s = wl.s
    compute = torch.cuda.current_stream()
    for st in projs:
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(st["free"])
            st["X"].copy_(st["X_host"], non_blocking=True)
            st["dY"].copy_(st["dY_host"], non_blocking=True)
            st["ready"].record(copy_stream)
    for st in projs:
        compute.wait_event(st["ready"])
        qb.qlora_linear_fwd(st["qt"], st["X"], st["A"], st["B"], s, save_xa=True, Y=st["Y"], XA=st["XA"],
                            workspace=st["ws_f"])
        qb.qlora_linear_bwd(st["qt"], st["X"], st["dY"], st["A"], st["B"], s, XA=st["XA"], dX=st["dX"],
                            dA=st["dA"], dB=st["dB"], workspace=st["ws_b"])
        st["free"].record(compute)
        st["dA_host"].copy_(st["dA"], non_blocking=True)
        st["dB_host"].copy_(st["dB"], non_blocking=True)


def secondary(qb, torch, device, peaks):
    """Encode / dequant (4096^2 with outliers) and decode GEMV (65B FFN) bandwidths."""
    out = {}
    hbm = peaks["hbm_gbs"]
    # codec: rotate 4 weight sets (4 x 42 MB > L2)
    sets = [workloads.weight((4096, 4096), proj=j, outliers=True).to(device) for j in range(4)]
    qts = [qb.qlora_quantize_nf4_dq(w) for w in sets]
    ws = torch.empty(qb.qlora_nf4_sizes(4096, 4096)["workspace"], dtype=torch.uint8, device=device)
    outs = [torch.empty(4096, 4096, dtype=torch.bfloat16, device=device) for _ in range(4)]
    sz = qb.qlora_nf4_sizes(4096, 4096)
    codec_bytes = 4096 * 4096 * 2 + sz["codes"] + sz["absmax_q"] + sz["absmax_c2"] + 4
    for name, fn in (("encode_4096x4096", lambda j: qb.qlora_quantize_nf4_dq(sets[j], out=qts[j], workspace=ws)),
                     ("dequant_4096x4096", lambda j: qb.qlora_dequantize(qts[j], out=outs[j]))):
        for j in range(8):
            fn(j % 4)
        torch.cuda.synchronize()
        # one CUDA graph of 20 back-to-back calls removes host launch gaps
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for j in range(20):
                    fn(j % 4)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(2):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / 40
        del g
        gbs = codec_bytes / t / 1e9
        out[name] = {"us": round(t * 1e6, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                     "bytes": codec_bytes}
    stored_bytes = sz["codes"] + sz["absmax_q"] + sz["absmax_c2"] + 4
    out["bits_per_param"] = round(8 * stored_bytes / (4096 * 4096), 6)
    del sets, qts, outs
    # GEMV: 22016x8192 and 8192x22016, 2 weight sets each (> L2), M in {1, 4, 16}
    for (n, k) in ((22016, 8192), (8192, 22016)):
        wsets = []
        for j in range(2):
            w = workloads.weight((n, k), proj=20 + j).to(device)
            wsets.append(qb.qlora_quantize_nf4_dq(w))
            del w
        A = workloads.lora_a(64, k, 30).to(device)
        B = workloads.lora_b(n, 64, 30).to(device)
        szg = qb.qlora_nf4_sizes(n, k)
        wbytes = szg["codes"] + szg["absmax_q"] + szg["absmax_c2"] + 4 + (A.numel() + B.numel()) * 2
        for m in (1, 4, 16):
            X = workloads.activations(m, k, 31).to(device)
            Y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
            wsz = torch.empty(qb.qlora_linear_workspace_size(n, k, m, 64)[0], dtype=torch.uint8, device=device)
            call = lambda j: qb.qlora_linear_fwd(wsets[j % 2], X, A, B, 0.25, save_xa=False, Y=Y, workspace=wsz)
            for j in range(6):
                call(j)
            torch.cuda.synchronize()
            # one CUDA graph of 20 back-to-back calls removes host launch gaps
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for j in range(20):
                        call(j)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(5):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1) / 1e3 / 100
            byts = wbytes + m * k * 2 + m * n * 2
            gbs = byts / t / 1e9
            out[f"gemv_{n}x{k}_m{m}"] = {"us": round(t * 1e6, 2), "GB/s": round(gbs, 1),
                                         "frac_hbm": round(gbs / hbm, 4), "bytes": byts}
            del g
        if n > k:
            # several adapters over the same weight, one per group of tokens (16 tokens)
            for n_ad in (4, 16):
                m = 16
                X = workloads.activations(m, k, 31).to(device)
                Y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
                A_st = torch.stack([workloads.lora_a(64, k, 60 + a) for a in range(n_ad)]).to(device)
                B_st = torch.stack([workloads.lora_b(n, 64, 60 + a) for a in range(n_ad)]).to(device)
                idx = (torch.arange(m, dtype=torch.int32) % n_ad).to(device)
                wsz = torch.empty(qb.qlora_linear_workspace_size(n, k, m, 64)[0], dtype=torch.uint8, device=device)
                call = lambda j: qb.qlora_linear_fwd_multi(wsets[j % 2], X, A_st, B_st, idx, 0.25, save_xa=False,
                                                           Y=Y, workspace=wsz)
                t = graph_time(torch, lambda: [call(j) for j in range(2)], 10, 5) / 2
                byts = (szg["codes"] + szg["absmax_q"] + szg["absmax_c2"] + 4 + n_ad * (A.numel() + B.numel()) * 2
                        + m * k * 2 + m * n * 2)
                gbs = byts / t / 1e9
                out[f"gemv_multi_{n}x{k}_m{m}_adapters{n_ad}"] = {"us": round(t * 1e6, 2), "GB/s": round(gbs, 1),
                                                                   "frac_hbm": round(gbs / hbm, 4), "bytes": byts}
        del wsets
    # the stored form without double quantization: fp32 block constants (0.5 bits
    # per weight); 4 weight sets rotated (4 x 42 MB > L2), as for the DQ form
    wp = [workloads.weight((4096, 4096), proj=j, outliers=True).to(device) for j in range(4)]
    qp = [qb.qlora_quantize_nf4_dq(x, double_quant=False) for x in wp]
    outp = [torch.empty(4096, 4096, dtype=torch.bfloat16, device=device) for _ in range(4)]
    szp = qb.qlora_nf4_sizes(4096, 4096, double_quant=False)
    wsp = torch.empty(szp["workspace"], dtype=torch.uint8, device=device)
    pbytes = 4096 * 4096 * 2 + szp["codes"] + szp["absmax_q"]
    for name, fn in (("encode_nodq_4096x4096",
                      lambda: [qb.qlora_quantize_nf4_dq(wp[j], out=qp[j], workspace=wsp) for j in range(4)]),
                     ("dequant_nodq_4096x4096", lambda: [qb.qlora_dequantize(qp[j], out=outp[j]) for j in range(4)])):
        t = graph_time(torch, fn, 5, 2) / 4
        out[name] = {"us": round(t * 1e6, 2), "GB/s": round(pbytes / t / 1e9, 1),
                     "frac_hbm": round(pbytes / t / 1e9 / hbm, 4), "bytes": pbytes}
    del wp, qp, outp
    out["bits_per_param_nodq"] = round(8 * (szp["codes"] + szp["absmax_q"]) / (4096 * 4096), 6)
    return out


def cpu_oracle_sample(wl, m_sample: int, projs_idx=None) -> dict:
    """The oracle (as it stands) on a bounded sample of a layer workload: the
    weights dequantized by the C oracle, then fwd + bwd of m_sample tokens in
    float64.  Returns the measured seconds of both parts (quantization, a model
    load, is timed apart) and the TFLOP/s of the sample."""
    import oracle
    t_quant = time.time()
    qts = []
    for i, p in enumerate(wl.projections):
        if projs_idx is not None and i not in projs_idx:
            continue
        w = workloads.weight((p.n, p.k), proj=i)
        qts.append((i, p, oracle.quantize(workloads.bf16_bits(w))))
        del w
    t_quant = time.time() - t_quant
    t_deq, t_mm, flops = 0.0, 0.0, 0
    for i, p, qt in qts:
        X = workloads.activations(wl.m, p.k, i)[:m_sample].float().numpy()
        dY = workloads.grad_output(wl.m, p.n, i)[:m_sample].float().numpy()
        A = workloads.lora_a(wl.r, p.k, i).float().numpy()
        B = workloads.lora_b(p.n, wl.r, i).float().numpy()
        t0 = time.time()
        Wd = oracle.dequant_tensor(qt)
        t1 = time.time()
        oracle.linear_fwd(Wd, X, A, B, wl.s)
        oracle.linear_bwd(Wd, X, dY, A, B, wl.s)
        t2 = time.time()
        t_deq += t1 - t0
        t_mm += t2 - t1
        flops += workloads.linear_flops(p.n, p.k, m_sample, wl.r)["total"]
    t = t_deq + t_mm
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "seconds": round(t, 2), "dequant_seconds": round(t_deq, 2), "matmul_seconds": round(t_mm, 3),
            "setup_quantize_seconds": round(t_quant, 2),
            "sample": f"{m_sample} of {wl.m} tokens of each of {len(qts)} projections of {wl.name}: "
                      f"C-oracle dequant of the full weights + float64 numpy fwd+bwd"}


def cpu_baseline(slice5: int = 512) -> dict:
    """The oracle as it stands, timed on this host's cores (OpenMP in the C codec,
    the BLAS threads in numpy), on the five workloads:
      1 (tiny layer), 2 (4096^2 codec) and 4 (65B FFN decode forward) in full;
      3 (LLaMA-7B 7 projections, 8192 tokens) in full;
      5 (LLaMA-65B layer) on a slice of `slice5` tokens of every projection,
        extrapolated to 8192 tokens as dequant + (8192 / slice) x the slice's
        matmuls -- labelled as such.
    The headline value is workload 5's extrapolated TFLOP/s."""
    import oracle
    out = {}
    # 1: quantize + forward + backward of the tiny layer
    wl = workloads.TINY
    p = wl.projections[0]
    w = workloads.bf16_bits(workloads.weight((p.n, p.k)))
    X, A = workloads.activations(wl.m, p.k).float().numpy(), workloads.lora_a(wl.r, p.k).float().numpy()
    B, dY = workloads.lora_b(p.n, wl.r).float().numpy(), workloads.grad_output(wl.m, p.n).float().numpy()
    t0 = time.time()
    for _ in range(10):
        Wd = oracle.dequant_tensor(oracle.quantize(w))
        oracle.linear_fwd(Wd, X, A, B, wl.s)
        oracle.linear_bwd(Wd, X, dY, A, B, wl.s)
    out["1_" + wl.name] = {"us_per_call": round((time.time() - t0) / 10 * 1e6, 1),
                           "what": "quantize + dequant + fwd + bwd, in full"}
    # 2: encode + double quant, then dequant, of the 4096^2 weight with outliers
    wbits = workloads.bf16_bits(workloads.weight((4096, 4096), proj=0, outliers=True))
    t0 = time.time()
    qt = oracle.quantize(wbits)
    t1 = time.time()
    oracle.dequant_tensor(qt)
    t2 = time.time()
    sz = oracle.storage_bytes(4096 * 4096)
    nbytes = 4096 * 4096 * 2 + sz["codes"] + sz["absmax_q"] + sz["absmax_c2"] + sz["mean"]
    out["2_" + workloads.CODEC_4096.name] = {"encode_GB/s": round(nbytes / (t1 - t0) / 1e9, 3),
                                             "dequant_GB/s": round(nbytes / (t2 - t1) / 1e9, 3),
                                             "what": "in full"}
    del wbits, qt
    # 4: decode-shaped forward on the 65B FFN weights (dequant + fwd per call)
    g = {}
    for j, pj in enumerate(workloads.GEMV65B.projections):
        qt = oracle.quantize(workloads.bf16_bits(workloads.weight((pj.n, pj.k), proj=20 + j)))
        szg = oracle.storage_bytes(pj.n * pj.k)
        A = workloads.lora_a(64, pj.k, 30).float().numpy()
        B = workloads.lora_b(pj.n, 64, 30).float().numpy()
        for m in workloads.GEMV65B.token_counts:
            X = workloads.activations(m, pj.k, 31).float().numpy()
            t0 = time.time()
            Wd = oracle.dequant_tensor(qt)
            oracle.linear_fwd(Wd, X, A, B, 0.25)
            t = time.time() - t0
            nb = (szg["codes"] + szg["absmax_q"] + szg["absmax_c2"] + szg["mean"] + (A.size + B.size) * 2
                  + m * pj.k * 2 + m * pj.n * 2)
            g[f"{pj.n}x{pj.k}_m{m}"] = round(nb / t / 1e9, 3)
        del qt
    out["4_" + workloads.GEMV65B.name] = {"GB/s": g, "what": "dequant + fwd per call, in full"}
    # 3: LLaMA-7B projections, all 8192 tokens
    r3 = cpu_oracle_sample(workloads.LLAMA7B, workloads.LLAMA7B.m)
    out["3_" + workloads.LLAMA7B.name] = {"TFLOP/s": round(r3["value"], 5), "seconds": r3["seconds"],
                                          "what": "dequant + fwd + bwd, all 8192 tokens (in full)"}
    # 5: the headline layer on a token slice, extrapolated
    wl5 = workloads.LLAMA65B
    r5 = cpu_oracle_sample(wl5, slice5)
    t_full = r5["dequant_seconds"] + r5["matmul_seconds"] * wl5.m / slice5
    flops5 = sum(workloads.linear_flops(p.n, p.k, wl5.m, wl5.r)["total"] for p in wl5.projections)
    value = flops5 / t_full / 1e12
    out["5_" + wl5.name] = {"TFLOP/s_extrapolated": round(value, 5), "slice_TFLOP/s": round(r5["value"], 5),
                            "seconds": r5["seconds"],
                            "what": f"{slice5}-token slice of every projection, extrapolated to {wl5.m} tokens"}
    return {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{wl5.name}: {slice5} of {wl5.m} tokens of all 7 projections (C-oracle dequant of the "
                      f"full weights + float64 numpy fwd+bwd), extrapolated to {wl5.m} tokens; the other "
                      f"workloads under 'workloads'",
            "workloads": out}


def time_layer(qb, torch, wl, projs, steps: int, pg=None, device=None, with_clocks=False):
    """Times `steps` steps of a layer workload (inputs resident in HBM) with CUDA
    events on the launching stream, every fused dequant-GEMM launch bracketed by
    its own pair of events.  Returns the step time (max over ranks), the fused
    launches' durations, the kernel-launch count and the clocks seen."""
    gemm_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(2 * len(projs) * steps)]
    for a, b in gemm_events:          # torch creates the CUDA event on first record
        a.record()
        b.record()
    ev_stack = list(reversed(gemm_events))
    clocks = ClockSampler(device.index) if with_clocks else None
    barrier(pg, device)
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    launches0 = qb.qlora_kernel_launches()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run_step(qb, wl, projs, events=ev_stack)
    e1.record()
    torch.cuda.synchronize()
    launches = qb.qlora_kernel_launches() - launches0
    barrier(pg, device)
    clk = clocks.stop() if clocks else None
    t_local = e0.elapsed_time(e1) / 1e3
    t = max_over_ranks(pg, t_local, device)
    gemm_ms = [a.elapsed_time(b) for a, b in gemm_events]
    return dict(t=t, t_local=t_local, gemm_ms=gemm_ms, launches=launches, clocks=clk)


def layer_summary(wl, timing, steps, peaks, world=1) -> dict:
    flops_step, flops_fused_step = layer_flops(wl)
    value = world * steps * flops_step / timing["t"] / 1e12
    fused_avg_s = sum(timing["gemm_ms"]) / len(timing["gemm_ms"]) / 1e3
    achieved = flops_fused_step / (2 * len(wl.projections)) / fused_avg_s / 1e12
    sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    return {"TFLOP/s": round(value, 2), "ms_per_step": round(timing["t"] / steps * 1e3, 3),
            "frac_sustained": round(value / sus, 4), "frac_burst": round(value / peaks["bf16_tflops"], 4),
            "k_fused_TFLOP/s": round(achieved, 1), "k_fused_frac_sustained": round(achieved / sus, 4),
            "k_fused_frac_burst": round(achieved / peaks["bf16_tflops"], 4),
            "k_fused_share": round(sum(timing["gemm_ms"]) / 1e3 / timing["t_local"], 4),
            "flops_per_step": flops_step, "steps": steps}


def tiny_layer_us(qb, torch, device) -> dict:
    """The tiny layer (256 x 256, 16 tokens, r 8): launch-bound, so reported in
    microseconds per call, graph-timed over 20 back-to-back calls each."""
    wl = workloads.TINY
    p = wl.projections[0]
    w = workloads.weight((p.n, p.k)).to(device)
    qt = qb.qlora_quantize_nf4_dq(w)
    X, dY = workloads.activations(wl.m, p.k).to(device), workloads.grad_output(wl.m, p.n).to(device)
    A, B = workloads.lora_a(wl.r, p.k).to(device), workloads.lora_b(p.n, wl.r).to(device)
    fw, bw = qb.qlora_linear_workspace_size(p.n, p.k, wl.m, wl.r)
    wsf = torch.empty(fw, dtype=torch.uint8, device=device)
    wsb = torch.empty(bw, dtype=torch.uint8, device=device)
    wsq = torch.empty(qb.qlora_nf4_sizes(p.n, p.k)["workspace"], dtype=torch.uint8, device=device)
    Y = torch.empty(wl.m, p.n, dtype=torch.bfloat16, device=device)
    XA = torch.empty(wl.m, wl.r, dtype=torch.float32, device=device)
    dX = torch.empty(wl.m, p.k, dtype=torch.bfloat16, device=device)
    dA = torch.empty(wl.r, p.k, dtype=torch.float32, device=device)
    dB = torch.empty(p.n, wl.r, dtype=torch.float32, device=device)
    ops = {
        "quantize": lambda: qb.qlora_quantize_nf4_dq(w, out=qt, workspace=wsq),
        "fwd": lambda: qb.qlora_linear_fwd(qt, X, A, B, wl.s, Y=Y, XA=XA, workspace=wsf),
        "bwd": lambda: qb.qlora_linear_bwd(qt, X, dY, A, B, wl.s, XA=XA, dX=dX, dA=dA, dB=dB, workspace=wsb),
    }
    out = {}
    for name, fn in ops.items():
        out[f"{name}_us"] = round(graph_time(torch, fn, 20, 5) * 1e6, 2)
    return out


def graph_time(torch, fn, calls: int, replays: int) -> float:
    """Seconds per call of `fn`, captured `calls` times in one CUDA graph and
    replayed `replays` times (no host launch gaps)."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(calls):
                fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / 1e3 / (calls * replays)


def bench_ours(args):
    import torch
    import bit_nf4_quantized_encode_b200 as qb
    rank, local, world, pg = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_kind = load_peaks()
    wl = workloads.LLAMA65B
    flops_step, flops_fused_step = layer_flops(wl)
    projs = prepare_layer(qb, torch, wl, device)

    for _ in range(args.warmup):
        run_step(qb, wl, projs)
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0, "device wait timed out during warm-up"

    # timed region: K steps, fused-GEMM launches bracketed by events for the roofline
    K = args.steps
    tm = time_layer(qb, torch, wl, projs, K, pg, device, with_clocks=True)
    t, t_local, gemm_ms, launches, clk = tm["t"], tm["t_local"], tm["gemm_ms"], tm["launches"], tm["clocks"]

    # end to end: host inputs -> device -> fwd+bwd -> gradients back to host
    Ke = max(2, min(K, 5))
    copy_stream = torch.cuda.Stream()
    for st in projs:
        st["ready"], st["free"] = torch.cuda.Event(), torch.cuda.Event()
        st["free"].record()
    run_step_e2e(qb, wl, projs, copy_stream)
    torch.cuda.synchronize()
    barrier(pg, device)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record()
    copy_stream.wait_event(x0)          # no upload starts before the timed region
    for _ in range(Ke):
        run_step_e2e(qb, wl, projs, copy_stream)
    x1.record()                         # after the last backward, which waited for every upload
    torch.cuda.synchronize()
    te = max_over_ranks(pg, x0.elapsed_time(x1) / 1e3, device)
    h2d = sum(st["X"].numel() * 2 + st["dY"].numel() * 2 for st in projs)
    d2h = sum(st["dA"].numel() * 4 + st["dB"].numel() * 4 for st in projs)
    assert qb.qlora_read_device_errors() == 0
    del projs

    # the other layer workload (LLaMA-7B, 7 projections, 8192 tokens) and the tiny layer
    others = {}
    if not args.skip_secondary:
        wl3 = workloads.LLAMA7B
        projs3 = prepare_layer(qb, torch, wl3, device)
        for _ in range(3):
            run_step(qb, wl3, projs3)
        K3 = max(5, K // 2)
        tm3 = time_layer(qb, torch, wl3, projs3, K3, pg, device)
        others["3_" + wl3.name] = layer_summary(wl3, tm3, K3, peaks, world)
        del projs3
        others["1_" + workloads.TINY.name] = tiny_layer_us(qb, torch, device)
        assert qb.qlora_read_device_errors() == 0
    if pg is not None:                 # every rank takes the same collective steps
        barrier(pg, device)
        pg.destroy_process_group()
    if rank != 0:
        return

    value = world * K * flops_step / t / 1e12
    peak_t = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    fused_avg_s = sum(gemm_ms) / len(gemm_ms) / 1e3
    fused_flops_launch = flops_fused_step / (2 * len(wl.projections))
    achieved = fused_flops_launch / fused_avg_s / 1e12
    traffic, algo_bytes = fused_traffic()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded PCG64 normals, bf16), NF4+DQ weights quantized on device before timing",
        "config": {"workload": wl.name, "projections": [f"{p.name} {p.n}x{p.k}" for p in wl.projections],
                   "tokens": wl.m, "lora_rank": wl.r, "lora_alpha": wl.alpha, "nf4_blocksize": 64,
                   "dq_blocksize": 256, "l2": "inputs larger than L2 (3.9 GB of activations per step)",
                   "parallelism": f"replicas x{world} (no collective)",
                   "flops_per_step": flops_step},
        "e2e": {"value": round(world * Ke * flops_step / te / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke},
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "kernel": "k_fused (dequant-GEMM fwd and bwd-dX)",
                     "achieved": round(achieved, 1), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_t, 4), "peak_kind": f"{peak_kind} sustained bf16",
                     "frac_of_burst_peak": round(achieved / peaks["bf16_tflops"], 4),
                     "burst_peak": peaks["bf16_tflops"],
                     "traffic": traffic,
                     "traffic_unit": "DRAM bytes per average launch (ncu counters, profiles/k_fused_traffic.json; "
                                     "null when taken on other source)",
                     "algorithmic_bytes": algo_bytes,
                     "traffic_over_algorithmic": round(traffic / algo_bytes, 3) if traffic and algo_bytes else None,
                     "avg_launch_ms": round(fused_avg_s * 1e3, 4),
                     "share_of_step": round(sum(gemm_ms) / 1e3 / t_local, 4)},
        "clocks": clk,
    }
    if others:
        line["workloads"] = others
    if not args.skip_secondary:
        line["secondary"] = secondary(qb, torch, device, peaks)
    if not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline(slice5=args.cpu_tokens)
    print(json.dumps(line), flush=True)


def bench_reference(args):
    """The oracle as the reference arm: each step a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workloads.LLAMA65B
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, m_sample=args.ref_tokens, projs_idx={0})
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = cpu_oracle_sample(wl, m_sample=args.ref_tokens, projs_idx={0})
        vals.append(last["value"])
        secs += last["seconds"]
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "tokens": wl.m, "lora_rank": wl.r},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": last["cores"],
                             "kind": "oracle", "sample": last["sample"]},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_case(args):
    """One operation on a small case, for profiler captures (prints timings, no JSON)."""
    import torch
    import bit_nf4_quantized_encode_b200 as qb
    device = torch.device("cuda", 0)
    n, k, m, r = args.case_n, args.case_k, args.case_m, 64
    w = workloads.weight((n, k), proj=0).to(device)
    qt = qb.qlora_quantize_nf4_dq(w)
    X = workloads.activations(m, k).to(device)
    dY = workloads.grad_output(m, n).to(device)
    A, B = workloads.lora_a(r, k).to(device), workloads.lora_b(n, r).to(device)
    fw, bw = qb.qlora_linear_workspace_size(n, k, m, r)
    wsf = torch.empty(fw, dtype=torch.uint8, device=device)
    wsb = torch.empty(bw, dtype=torch.uint8, device=device)
    Y = torch.empty(m, n, dtype=torch.bfloat16, device=device)
    XA = torch.empty(m, r, dtype=torch.float32, device=device)
    out = torch.empty(n, k, dtype=torch.bfloat16, device=device)
    wse = torch.empty(qb.qlora_nf4_sizes(n, k)["workspace"], dtype=torch.uint8, device=device)
    ops = {
        "fused_fwd": lambda: qb.qlora_linear_fwd(qt, X, A, B, 0.25, Y=Y, XA=XA, workspace=wsf),
        "fused_bwd": lambda: qb.qlora_linear_bwd(qt, X, dY, A, B, 0.25, XA=XA, workspace=wsb),
        "encode": lambda: qb.qlora_quantize_nf4_dq(w, out=qt, workspace=wse),
        "dequant": lambda: qb.qlora_dequantize(qt, out=out),
    }
    fn = ops[args.case]
    qb.qlora_linear_fwd(qt, X, A, B, 0.25, Y=Y, XA=XA, workspace=wsf)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.case_iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    assert qb.qlora_read_device_errors() == 0
    print(f"case {args.case} n={n} k={k} m={m}: {e0.elapsed_time(e1) / args.case_iters * 1e3:.1f} us/call")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-secondary", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=512,
                    help="token slice of the LLaMA-65B layer in the CPU-oracle baseline")
    ap.add_argument("--ref-tokens", type=int, default=16, help="token sample per reference-arm step")
    ap.add_argument("--case", choices=["fused_fwd", "fused_bwd", "encode", "dequant"],
                    help="run one operation on a small case (for profiler captures) and exit")
    ap.add_argument("--case-n", type=int, default=8192)
    ap.add_argument("--case-k", type=int, default=8192)
    ap.add_argument("--case-m", type=int, default=4096)
    ap.add_argument("--case-iters", type=int, default=3)
    ap.add_argument("--write-traffic", nargs="+", metavar="CSV",
                    help="rebuild profiles/k_fused_traffic.json from ncu CSV logs of the --case runs and exit")
    args = ap.parse_args()
    if args.write_traffic:
        write_traffic(args.write_traffic)
        return
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()

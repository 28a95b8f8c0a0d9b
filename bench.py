#!/usr/bin/env python3
"""ECF8 decode benchmark.

Default workload: the Llama-3-70B weight set in FP8 E4M3 -- 80 decoder
layers of seven projections (q/o 8192x8192, k/v 1024x8192, gate/up
28672x8192, down 8192x28672), weights symmetric alpha-stable alpha=1.8 scaled
to max|w| = 448, one codebook per tensor, 68,451,041,280 bytes of FP8 in all,
held compressed in HBM and decoded layer by layer into ONE reused output
buffer on one stream.  One step = the 80-layer loop: 80 batched decode
launches (each the whole hot path: table build, chunk walk, scan,
compaction, assembly, store), inputs resident in HBM.  The same JSON line
carries the Llama-3-8B layer (one batched launch per step) and the
256-expert MoE set (768 tensors, one batched launch) as extra fields.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Other workloads (--workload llama3_8b_layer, sweep_<a>_<max>, moe, ...) time
one batched launch per step.  Multi-GPU (torchrun): every rank decodes its
own copy of the weights (weak scaling; the decode has no exchange step),
time = max over ranks.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ecf8_synth as synth  # noqa: E402

METRIC = "ECF8 decode GB/s (FP8 out) and % of HBM roofline on 1 B200; compression ratio"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0  # HGX B200 HBM3e specification, for context beside the measured copy peak
L2_BYTES = 126 * 1024 * 1024
KERNEL_SRC = os.path.join(ROOT, "lossless_fp8_weight_b200", "csrc", "ecf8_decode.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.txt")


HEADLINE = "llama3_70b"


def workload_by_name(name: str) -> synth.Workload:
    if name == HEADLINE:
        return synth.llama3_70b_layer(0)
    if name == "llama3_8b_layer":
        return synth.llama3_8b_layer()
    if name == "single_1k":
        return synth.single_normal_1k()
    if name.startswith("sweep_"):  # sweep_<alpha>_<max>
        _, a, m = name.split("_")
        return synth.alpha_sweep_point(float(a), float(m))
    if name.startswith("moe"):
        k = int(name[3:] or 256)
        return synth.moe_experts(k)
    if name.startswith("llama3_70b_layer"):
        return synth.llama3_70b_layer(int(name[len("llama3_70b_layer"):] or 0))
    raise SystemExit(f"unknown workload {name}")


def entropy_bits(hist) -> float:
    h = np.asarray(hist, dtype=np.float64)
    p = h[h > 0] / h.sum()
    return float(-(p * np.log2(p)).sum())


def prepare(workload: synth.Workload, L):
    """Generate and encode every tensor on the host (not timed)."""
    blobs, xs, stats = [], [], []
    for t in workload.tensors:
        x = t.generate()
        hist = L.histogram(x)
        cb = L.build_codebook(hist)
        blob = L.encode(x, codebook=cb)
        info = L.blob_info(blob)
        lens = info.lengths.astype(np.float64)
        stats.append({"n": int(x.size), "blob": int(blob.size), "hist": hist,
                      "code_bits": int(info.code_bits), "le6": float(hist[lens <= 6].sum()) / x.size,
                      "max_len": int(info.max_len)})
        blobs.append(blob)
        xs.append(x)
    return blobs, xs, stats


def compression_summary(stats):
    n = sum(s["n"] for s in stats)
    blob = sum(s["blob"] for s in stats)
    hist = sum(s["hist"].astype(np.float64) for s in stats)
    return {
        "n_bytes": n,
        "compressed_bytes": blob,
        "ratio": round(n / blob, 4),
        "savings_pct": round(100 * (1 - blob / n), 2),
        "exponent_entropy_bits": round(entropy_bits(hist), 4),
        "mean_code_bits": round(sum(s["code_bits"] for s in stats) / n, 4),
        "codes_le6_bits_frac": round(sum(s["le6"] * s["n"] for s in stats) / n, 5),
        "max_code_bits": max(s["max_len"] for s in stats),
    }


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sha() -> str:
    with open(KERNEL_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload_name: str, blob_bytes_per_launch=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source and this workload.  When the summary records the
    compressed bytes of its captured launch, the read bytes are scaled to
    blob_bytes_per_launch (the timed launches' average)."""
    try:
        rec = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.strip()
        if rec.get("kernel_sha") != kernel_sha() or rec.get("workload") != workload_name:
            return None
        if blob_bytes_per_launch is not None and "dram_read_bytes" in rec and "blob_bytes" in rec:
            read = float(rec["dram_read_bytes"]) * blob_bytes_per_launch / float(rec["blob_bytes"])
            return round(read + float(rec["dram_write_bytes"]))
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons, power = [], [], set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def oracle_cpu_baseline(blobs, xs, budget_s: float = 12.0):
    """Time the bit-serial oracle decoding tensors of the workload on host
    threads (one tensor per thread) for a bounded sample."""
    import oracle
    cores = min(len(blobs), os.cpu_count() or 1)
    order = sorted(range(len(blobs)), key=lambda i: xs[i].size)
    # a bounded sample: smallest tensors first until the estimated work fits the budget
    est_rate = 12e6  # weights/s per core, for sizing only
    picked, work = [], 0.0
    for i in order:
        if picked and (work + xs[i].size / est_rate) / cores > budget_s:
            break
        picked.append(i)
        work += xs[i].size / est_rate
    outs = {i: np.empty(xs[i].size, np.uint8) for i in picked}
    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=cores) as ex:
        rcs = list(ex.map(lambda i: oracle.decode_into(blobs[i], outs[i]), picked))
    dt = time.perf_counter() - t0
    assert all(rc == 0 for rc in rcs)
    for i in picked:
        assert np.array_equal(outs[i], xs[i])
    n = sum(xs[i].size for i in picked)
    return {"value": round(n / dt / 1e9, 5), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(picked)} of {len(blobs)} tensors ({n} weights), one tensor per thread, "
                      f"{dt:.2f} s"}


def run_reference(args, workload):
    """The oracle as the reference arm: host cores, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    L = load_library(build_only=True)
    sample = int(args.ref_sample)
    blobs, xs = [], []
    for t in workload.tensors:
        x = t.generate(count=min(sample, t.n), scale=t.scale() if t.dist == "sas" else None)
        xs.append(x)
        blobs.append(L.encode(x))
    cores = min(len(blobs), os.cpu_count() or 1)
    outs = [np.empty(x.size, np.uint8) for x in xs]

    def step():
        with cf.ThreadPoolExecutor(max_workers=cores) as ex:
            rcs = list(ex.map(lambda i: oracle.decode_into(blobs[i], outs[i]), range(len(blobs))))
        assert all(rc == 0 for rc in rcs)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    for x, o in zip(xs, outs):
        assert np.array_equal(x, o)
    n = sum(x.size for x in xs) * args.steps
    value = n / dt / 1e9
    summ = compression_summary([{"n": x.size, "blob": b.size, "hist": L.histogram(x),
                                 "code_bits": int(L.blob_info(b).code_bits), "le6": 0.0,
                                 "max_len": int(L.blob_info(b).max_len)} for x, b in zip(xs, blobs)])
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8", "data": "synthetic",
        "config": {"workload": (f"llama3_70b_{args.layers}layers_reused_buffer" if args.workload == HEADLINE
                                else workload.name),
                   "tensors": len(workload.tensors), "sample_weights_per_tensor": sample,
                   "ratio_of_sample": summ["ratio"]},
        "cpu_baseline": {"value": round(value, 5), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {sample} weights of each of the {len(xs)} tensors"
                                   + (" of layer 0" if args.workload == HEADLINE else "")
                                   + ", one tensor per thread, per step"},
        "e2e": {"value": round(value, 5), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (timing is the
    slowest rank's); a no-op without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


# ---------------------------------------------------------------- per-config sweep

def _blake(a: np.ndarray) -> str:
    return hashlib.blake2b(memoryview(np.ascontiguousarray(a)), digest_size=16).hexdigest()


def _encode_specs(specs, L, keep=False):
    """Generate and encode tensors one by one; keep a hash of each source."""
    out = []
    for t in specs:
        x = t.generate()
        hist = L.histogram(x)
        blob = L.encode(x, codebook=L.build_codebook(hist))
        info = L.blob_info(blob)
        out.append({"name": t.name, "n": int(x.size), "blob": blob, "info": info, "hist": hist,
                    "hash": _blake(x), "x": x if keep else None,
                    "le6": float(hist[info.lengths.astype(np.int64) <= 6].sum()) / max(1, x.size)})
    return out


def _upload(torch, dev, blobs):
    offs, o = [], 0
    for b in blobs:
        offs.append(o)
        o += (b.size + 255) // 256 * 256
    d = torch.empty(max(o, 256), dtype=torch.uint8, device=dev)
    for b, off in zip(blobs, offs):
        d[off:off + b.size].copy_(torch.from_numpy(b))
    return d, offs


def _time_launches(torch, fn, steps, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _record(name, recs, ms_per_call, n_calls_bytes, peak, extra=None):
    n = sum(r["n"] for r in recs)
    blob = sum(int(r["blob"].size) for r in recs)
    hist = sum(r["hist"].astype(np.float64) for r in recs)
    code_bits = sum(int(r["info"].code_bits) for r in recs)
    alg = blob + n
    d = {"workload": name, "tensors": len(recs), "n_bytes": n, "compressed_bytes": blob,
         "ratio": round(n / blob, 4), "savings_pct": round(100 * (1 - blob / n), 2),
         "exponent_entropy_bits": round(entropy_bits(hist), 4), "mean_code_bits": round(code_bits / n, 4),
         "codes_le6_bits_frac": round(sum(r["le6"] * r["n"] for r in recs) / n, 5),
         "max_code_bits": max(int(r["info"].max_len) for r in recs),
         "ms_per_call": round(ms_per_call, 5), "gbps_fp8_out": round(n_calls_bytes / ms_per_call / 1e6, 2),
         "roofline_frac": round(alg / ms_per_call / 1e6 / peak, 4) if extra is None or "alg_bytes" not in extra
         else round(extra["alg_bytes"] / ms_per_call / 1e6 / peak, 4)}
    if extra:
        d.update({k: v for k, v in extra.items() if k != "alg_bytes"})
    print(json.dumps(d), flush=True)
    return d


def run_sweep(args):
    """Every workload: compression ratio, exponent entropy, decode GB/s and
    roofline fraction, each output checked byte for byte against its source."""
    import torch
    L = load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, _ = measured_hbm_peak()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    results = []
    names = args.sweep.split(",") if args.sweep != "all" else ["single_1k", "llama3_8b_layer", "sweep", "moe",
                                                                  "llama3_70b"]

    def check_outputs(recs, d_out, out_offs):
        assert int(status.item()) == 0, f"decode status {int(status.item())}"
        for r, o in zip(recs, out_offs):
            got = d_out[o:o + r["n"]].cpu().numpy()
            assert _blake(got) == r["hash"], f"{r['name']}: decoded bytes differ from the source"

    def batched(recs, steps, name, extra=None):
        d_blob, offs = _upload(torch, dev, [r["blob"] for r in recs])
        out_offs, o = [], 0
        for r in recs:
            out_offs.append(o)
            o += (r["n"] + 255) // 256 * 256
        d_out = torch.empty(o, dtype=torch.uint8, device=dev)
        ws = torch.empty(max(L.batched_workspace_size(len(recs)), 16), dtype=torch.uint8, device=dev)
        batch = L.make_batch([L.BatchItem(r["info"], int(d_blob.data_ptr()) + bo, int(d_out.data_ptr()) + oo)
                              for r, bo, oo in zip(recs, offs, out_offs)])
        fn = lambda: L.decode_batched(batch, workspace=ws, status=status)  # noqa: E731
        ms = _time_launches(torch, fn, steps, 3)
        check_outputs(recs, d_out, out_offs)
        n = sum(r["n"] for r in recs)
        res = _record(name, recs, ms, n, peak, extra)
        del d_blob, d_out
        torch.cuda.empty_cache()
        return res

    for nm in names:
        if nm == "single_1k":
            recs = _encode_specs(synth.single_normal_1k().tensors, L)
            d_blob, _ = _upload(torch, dev, [recs[0]["blob"]])
            d_out = torch.empty(recs[0]["n"], dtype=torch.uint8, device=dev)
            fn = lambda: L.decode(recs[0]["info"], d_blob, d_out, status=status)  # noqa: E731
            ms = _time_launches(torch, fn, args.steps, 3)
            check_outputs(recs, d_out, [0])
            results.append(_record("single_1024x1024_normal16", recs, ms, recs[0]["n"], peak,
                                   {"launch": "ecf8_decode", "l2": "fits in L2"}))
        elif nm == "llama3_8b_layer":
            recs = _encode_specs(synth.llama3_8b_layer().tensors, L)
            results.append(batched(recs, args.steps, "llama3_8b_layer_sas1.8", {"launch": "ecf8_decode_batched"}))
        elif nm == "sweep":
            for a in synth.SWEEP_ALPHAS:
                for m in synth.SWEEP_MAXES:
                    wl = synth.alpha_sweep_point(a, m)
                    recs = _encode_specs(wl.tensors, L)
                    d_blob, _ = _upload(torch, dev, [recs[0]["blob"]])
                    d_out = torch.empty(recs[0]["n"], dtype=torch.uint8, device=dev)
                    fn = lambda: L.decode(recs[0]["info"], d_blob, d_out, status=status)  # noqa: E731
                    ms = _time_launches(torch, fn, args.steps, 3)
                    check_outputs(recs, d_out, [0])
                    results.append(_record(wl.name, recs, ms, recs[0]["n"], peak,
                                           {"launch": "ecf8_decode", "alpha": a, "max_abs": m}))
                    del d_blob, d_out
        elif nm == "moe":
            wl = synth.moe_experts(args.moe_experts)
            recs = _encode_specs(wl.tensors, L)
            results.append(batched(recs, max(3, args.steps // 20), wl.name,
                                   {"launch": "ecf8_decode_batched (workspace)"}))
        elif nm == "llama3_70b":
            # layer 0 is generated; layers 1..79 are device copies of its blobs
            # (host generation of all 68.45e9 weights would take ~30 min), so the
            # loop walks ~54 GB of distinct resident compressed bytes
            recs = _encode_specs(synth.llama3_70b_layer(0).tensors, L)
            layers = args.layers
            d_blob, offs = _upload(torch, dev, [r["blob"] for r in recs])
            copies = [d_blob] + [d_blob.clone() for _ in range(layers - 1)]
            out_offs, o = [], 0
            for r in recs:
                out_offs.append(o)
                o += (r["n"] + 255) // 256 * 256
            d_out = torch.empty(o, dtype=torch.uint8, device=dev)  # one buffer reused by every layer
            batches = [L.make_batch([L.BatchItem(r["info"], int(c.data_ptr()) + bo, int(d_out.data_ptr()) + oo)
                                     for r, bo, oo in zip(recs, offs, out_offs)]) for c in copies]

            def all_layers():
                for b in batches:
                    L.decode_batched(b, status=status)

            ms = _time_launches(torch, all_layers, max(1, args.steps // 50), 1)
            check_outputs(recs, d_out, out_offs)
            n_layer = sum(r["n"] for r in recs)
            blob_layer = sum(int(r["blob"].size) for r in recs)
            res = _record(f"llama3_70b_{layers}layers_reused_buffer", recs, ms, n_layer * layers, peak,
                          {"launch": f"{layers} x ecf8_decode_batched into one reused buffer",
                           "resident_compressed_bytes": blob_layer * layers,
                           "alg_bytes": (blob_layer + n_layer) * layers,
                           "note": "layers 1..N-1 are device copies of layer 0's blobs"})
            results.append(res)
            del copies, d_blob, d_out
            torch.cuda.empty_cache()
        else:
            raise SystemExit(f"unknown sweep item {nm}")
    if args.sweep_out:
        with open(args.sweep_out, "w") as f:
            for r in results:
                f.write(json.dumps(r) + "\n")


# Llama-3-8B layer tensors as (out_features, in_features) for y = x W^T
_LAYER_SHAPES = {"q_proj": (4096, 4096), "k_proj": (1024, 4096), "v_proj": (1024, 4096), "o_proj": (4096, 4096),
                 "gate_proj": (14336, 4096), "up_proj": (14336, 4096), "down_proj": (4096, 14336)}


def run_pipeline(args):
    """Decode-on-use (ECF8 walkthrough §3.2.2; DFloat11 article §4): a stack
    of Llama-3-8B layers whose FP8 GEMMs (y = x W^T for all 7 projections, M
    tokens) read weights that a 2-slot pool decodes one layer ahead on a
    second stream.  Reports ms per layer for the GEMMs alone on resident
    weights, decode then GEMMs on one stream, and the pipeline at several
    decode grid caps, and checks every layer's GEMM outputs against the GEMMs
    over the source weights."""
    import torch
    L = load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    recs = _encode_specs(synth.llama3_8b_layer().tensors, L, keep=True)
    d_blob, offs = _upload(torch, dev, [r["blob"] for r in recs])
    blobs = [d_blob[o:o + r["blob"].size] for r, o in zip(recs, offs)]
    outs, o = [], 0
    for r in recs:
        outs.append(o)
        o += (r["n"] + 255) // 256 * 256
    slot_bytes = o
    n_layers, M = args.pipeline_layers, args.pipeline_tokens
    layers = [[L.PipelineTensor(r["info"], b, off) for r, b, off in zip(recs, blobs, outs)] for _ in range(n_layers)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    one = torch.ones((), dtype=torch.float32, device=dev)
    xs = {}
    for r in recs:
        k = _LAYER_SHAPES[r["name"]][1]
        if k not in xs:
            xs[k] = torch.from_numpy(synth.alpha_sweep_point(1.7, 448.0).tensors[0].generate(count=M * k)).to(
                dev).view(torch.float8_e4m3fn).view(M, k)

    def gemms(slot, ys=None):
        for r, off in zip(recs, outs):
            n_out, k = _LAYER_SHAPES[r["name"]]
            w = slot[off:off + r["n"]].view(torch.float8_e4m3fn).view(n_out, k)
            y = torch._scaled_mm(xs[k], w.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            if ys is not None:
                ys.append(y)

    # reference outputs: GEMMs over the source weights
    ref = torch.empty(slot_bytes, dtype=torch.uint8, device=dev)
    for r, off in zip(recs, outs):
        ref[off:off + r["n"]].copy_(torch.from_numpy(r["x"]))
    want = []
    gemms(ref, want)
    items = [L.BatchItem(r["info"], b, ref[off:off + r["n"]]) for r, b, off in zip(recs, blobs, outs)]
    batch = L.make_batch(items)
    reps = max(1, args.steps // 50)
    results = {}

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps / n_layers

    results["gemm_only"] = timed(lambda: [gemms(ref) for _ in range(n_layers)])
    results["decode_only"] = timed(lambda: [L.decode_batched(batch, status=status) for _ in range(n_layers)])

    def serial():
        for _ in range(n_layers):
            L.decode_batched(batch, status=status)
            gemms(ref)
    results["serial"] = timed(serial)
    assert int(status.item()) == 0

    # the decode stream at high priority: its CTAs take SMs ahead of queued GEMM CTAs
    compute, decode = torch.cuda.Stream(), torch.cuda.Stream(priority=-1)
    slots = [torch.empty(slot_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    by_ptr = {t.data_ptr(): t for t in slots}
    checked = False
    for cap in args.pipeline_ctas:
        P = L.Pipeline(layers, slots, slot_bytes, depth=1, max_ctas=cap, status=status, decode_stream=decode)

        def one_pass(check=None):
            for l in range(n_layers):
                slot = by_ptr[P.acquire(l, compute)]
                with torch.cuda.stream(compute):
                    gemms(slot, check[l] if check is not None else None)
                P.release(l, compute)

        if not checked:
            got = [[] for _ in range(n_layers)]
            one_pass(got)
            torch.cuda.synchronize()
            for g in got:
                assert all(torch.equal(a, b) for a, b in zip(g, want))
            checked = True
        one_pass()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(compute)
        for _ in range(reps):
            one_pass()
        e1.record(compute)
        torch.cuda.synchronize()
        results[f"pipelined_ctas{cap}"] = e0.elapsed_time(e1) / reps / n_layers
        P.close()
    assert int(status.item()) == 0
    best = min(v for k, v in results.items() if k.startswith("pipelined"))
    hidden = (results["serial"] - best) / max(1e-9, results["serial"] - results["gemm_only"])
    line = {"workload": f"pipeline_llama3_8b_x{n_layers}_tokens{M}", "metric": "ms per layer",
            "gemm": "torch._scaled_mm e4m3 x e4m3 -> bf16, 7 projections",
            "ms_per_layer": {k: round(v, 4) for k, v in results.items()},
            "decode_hidden_frac": round(hidden, 3), "gemm_outputs_equal_source": True}
    print(json.dumps(line), flush=True)
    if args.sweep_out:
        with open(args.sweep_out, "a") as f:
            f.write(json.dumps(line) + "\n")


def run_encode(args):
    """Encoder throughput on the Llama-3-8B layer: the GPU encoder (histogram
    kernel, host codebook, encode kernels) against the library's multithreaded
    host encoder, every GPU blob checked byte for byte against the host one."""
    import torch
    L = load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    specs = synth.llama3_8b_layer().tensors
    xs = [t.generate() for t in specs]
    d_xs = [torch.from_numpy(x).to(dev) for x in xs]
    n = sum(x.size for x in xs)
    host_blobs = []
    t0 = time.perf_counter()
    for x in xs:
        host_blobs.append(L.encode(x))
    host_s = time.perf_counter() - t0
    for x, d, hb in zip(xs, d_xs, host_blobs):
        assert np.array_equal(L.encode_device(d).cpu().numpy(), hb)
    reps = max(1, args.steps // 20)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        for d in d_xs:
            L.encode_device(d)
    e1.record()
    torch.cuda.synchronize()
    wall = (time.perf_counter() - t0) / reps
    dev_ms = e0.elapsed_time(e1) / reps
    line = {"workload": "encode_llama3_8b_layer_sas1.8", "n_bytes": n,
            "gpu_encode_gbps_fp8_in": round(n / (dev_ms / 1e3) / 1e9, 2),
            "gpu_encode_ms_per_layer": round(dev_ms, 4), "gpu_encode_wall_ms_per_layer": round(wall * 1e3, 3),
            "host_encode_gbps_fp8_in": round(n / host_s / 1e9, 3), "host_cores": os.cpu_count(),
            "note": "GPU time includes the histogram's device-to-host copy and the host codebook per tensor",
            "blobs_equal_host_encoder": True}
    print(json.dumps(line), flush=True)
    if args.sweep_out:
        with open(args.sweep_out, "a") as f:
            f.write(json.dumps(line) + "\n")


def run_bf16(args):
    """BF16 variant: decode throughput on the Llama-3-8B decoder layer in BF16
    (seven launches, one per projection, on one stream), every output checked
    against its source weights first."""
    import torch
    L = load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    specs = synth.llama3_8b_layer_bf16().tensors
    xs = [t.generate_bf16() for t in specs]
    blobs = [L.bf16_encode(x) for x in xs]
    infos = [L.bf16_blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).to(dev) for b in blobs]
    d_tables = [torch.from_numpy(L.bf16_table(i)).to(dev) for i in infos]
    d_outs = [torch.empty(i.n, dtype=torch.int16, device=dev) for i in infos]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one(k, layout="auto"):  # on the current stream (the capture stream inside a graph)
        L.bf16_decode(infos[k], d_blobs[k], d_tables[k], d_outs[k], status, layout=layout)

    def layer():  # the layer's seven tensors in one batched launch
        L.bf16_decode_batched([(infos[k], d_blobs[k], d_tables[k], d_outs[k]) for k in range(len(specs))], status)

    def layer_separate():
        for k in range(len(specs)):
            one(k)

    def graphed(fn, reps):
        """fn() reps times as one CUDA graph, so that host launch cost stays out of the timing."""
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        return g

    layer()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"decode status {int(status.item())}"
    for x, d in zip(xs, d_outs):
        if not np.array_equal(d.cpu().numpy().view(np.uint16), x):
            raise SystemExit("BF16 decode mismatch in the benchmark configuration")
    n = sum(int(i.n) for i in infos)
    blob = sum(int(b.size) for b in blobs)
    alg = blob + 2 * n + len(specs) * 32768
    peak, peak_kind = measured_hbm_peak()
    launches0 = L.launch_count()
    g_layer = graphed(layer, 1)
    launches = (L.launch_count() - launches0) // 2  # the warm call's and the capture's
    ms = _time_launches(torch, g_layer.replay, max(1, args.steps), args.warmup)
    ms_separate = _time_launches(torch, graphed(layer_separate, 1).replay, max(1, args.steps), args.warmup)
    per = []
    for k, spec in enumerate(specs):
        g_one = graphed(lambda: one(k), 10)
        mk = _time_launches(torch, g_one.replay, max(1, args.steps), args.warmup) / 10
        ak = int(blobs[k].size) + 2 * int(infos[k].n) + 32768
        per.append({"tensor": spec.name, "n": int(infos[k].n), "ms": round(mk, 5),
                    "gbps_bf16_out": round(2 * infos[k].n / mk / 1e6, 2),
                    "roofline_frac": round(ak / mk / 1e6 / peak, 4)})
    # one 58.7M-weight projection under every table layout that holds its code
    big = max(range(len(specs)), key=lambda k: infos[k].n)
    by_layout = {}
    for layout in ("wide", "narrow", "narrow_lane", "byte"):
        try:
            one(big, layout)
        except L.Ecf8Error:
            continue
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert np.array_equal(d_outs[big].cpu().numpy().view(np.uint16), xs[big])
        g_l = graphed(lambda: one(big, layout), 10)
        ml = _time_launches(torch, g_l.replay, max(1, args.steps), args.warmup) / 10
        al = int(blobs[big].size) + 2 * int(infos[big].n) + 32768
        by_layout[layout] = {"ms": round(ml, 5), "roofline_frac": round(al / ml / 1e6 / peak, 4)}
    line = {"workload": "bf16_llama3_8b_layer_normal0.02", "dtype": "bf16 bits (u16)", "n_weights": n,
            "compressed_bytes": blob, "ratio_vs_bf16": round(2 * n / blob, 4),
            "bits_per_weight": round(8 * blob / n, 4), "ms_per_layer": round(ms, 5),
            "gbps_bf16_out": round(2 * n / ms / 1e6, 2), "gpu_launches_per_layer": launches,
            "ms_per_layer_one_launch_per_tensor": round(ms_separate, 5),
            "roofline": {"bound": "hbm", "achieved": round(alg / ms / 1e6, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(alg / ms / 1e6 / peak, 4),
                         "frac_of_nominal": round(alg / ms / 1e6 / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes": alg, "peak_source": f"{peak_kind} hbm_gbs"},
            "timing": "CUDA graph of the layer's batched launch, replayed; per tensor: graph of 10 launches "
                      "(tensors whose blob + output fit in L2 run L2-warm there)",
            "l2": "inputs+outputs larger than L2 (no flush)", "per_tensor": per,
            "auto_layout": {spec.name: L.bf16_auto_layout(i) for spec, i in zip(specs, infos)},
            f"{specs[big].name}_by_layout": by_layout, "outputs_checked": True}
    print(json.dumps(line), flush=True)
    if args.sweep_out:
        with open(args.sweep_out, "a") as f:
            f.write(json.dumps(line) + "\n")


# ---------------------------------------------------------------- headline: the 70B set, 80 layers

_GPU_CHUNK = 1 << 25


def _sas_on_gpu(torch, dev, spec):
    """A tensor of the spec's law drawn on the GPU: symmetric alpha-stable by
    Chambers, Mallows and Stuck in float64 from torch's Philox generator
    (seeded from the spec's seed, chunk by chunk), scaled so that max|w| =
    spec.max_abs, cast to E4M3 (saturating clamp, nearest even).  The same law
    as the host generator, not the same numbers."""
    import math

    def chunk_values(c, m):
        g = torch.Generator(device=dev)
        g.manual_seed((spec.seed * 1_000_003 + c) & 0x7FFFFFFFFFFFFFFF)
        u1 = torch.rand(m, dtype=torch.float64, device=dev, generator=g)
        u2 = torch.rand(m, dtype=torch.float64, device=dev, generator=g)
        v = math.pi * (u1 - 0.5)
        w = (-torch.log1p(-u2)).clamp_min(1e-300)
        a = spec.alpha
        return torch.sin(a * v) / torch.cos(v).pow(1.0 / a) * (torch.cos(v - a * v) / w).pow((1.0 - a) / a)

    n = spec.n
    chunks = [(c, min(_GPU_CHUNK, n - c * _GPU_CHUNK)) for c in range((n + _GPU_CHUNK - 1) // _GPU_CHUNK)]
    mx = max(float(chunk_values(c, m).abs().max()) for c, m in chunks)
    scale = spec.max_abs / mx
    out = torch.empty(n, dtype=torch.uint8, device=dev)
    for c, m in chunks:
        x = (chunk_values(c, m) * scale).clamp(-448.0, 448.0).to(torch.float32)
        out[c * _GPU_CHUNK:c * _GPU_CHUNK + m].copy_(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return out


def _encode_set(L, torch, d_xs):
    """Histogram, codebook and GPU encoding of device tensors: [(info, d_blob)], hists, codebooks."""
    row, hists, cbs = [], [], []
    for d in d_xs:
        h = L.histogram_device(d)
        cb = L.build_codebook(h)
        blob = L.encode_device(d, codebook=cb, hist=h)
        row.append((L.blob_info_device(blob), blob))
        hists.append(h)
        cbs.append(cb)
    return row, hists, cbs


def _gen_on_device(torch, dev, specs, world, rank):
    """Generate the specs' tensors with the host generator (rank 0) and place
    them on every rank's GPU (a broadcast when there are several ranks);
    returns the device tensors and, on rank 0, the host arrays."""
    import torch.distributed as dist
    xs, d_xs = [], []
    for t in specs:
        if rank == 0:
            x = t.generate()
            xs.append(x)
            d = torch.from_numpy(x).to(dev)
        else:
            d = torch.empty(t.n, dtype=torch.uint8, device=dev)
        if world > 1:
            dist.broadcast(d, 0)
        d_xs.append(d)
    return d_xs, xs


def _sources(torch, dev, spec_sets, world, rank, host_first=True):
    """Device tensors for a list of tensor sets: the first set from the host
    generator (it is what the parity tests decode and what the CPU baseline
    times), the others drawn on the GPU.  Returns (list of device lists, host
    arrays of the first set)."""
    out, xs0 = [], []
    for k, specs in enumerate(spec_sets):
        if k == 0 and host_first:
            d_xs, xs0 = _gen_on_device(torch, dev, specs, world, rank)
        else:
            d_xs = [_sas_on_gpu(torch, dev, t) for t in specs]
        out.append(d_xs)
    return out, xs0


def _layout_outputs(torch, dev, infos):
    offs, o = [], 0
    for i in infos:
        offs.append(o)
        o += (int(i.n) + 255) // 256 * 256
    return torch.empty(max(o, 256), dtype=torch.uint8, device=dev), offs


def _batch_for(L, row, d_out, out_offs):
    return L.make_batch([L.BatchItem(info, blob, int(d_out.data_ptr()) + oo)
                         for (info, blob), oo in zip(row, out_offs)])


def _summary(row, hists, cbs):
    n = sum(int(i.n) for i, _ in row)
    blob = sum(int(b.numel()) for _, b in row)
    hist = sum(h.astype(np.float64) for h in hists)
    bits = sum(int(i.code_bits) for i, _ in row)
    le6 = sum(float(h[cb.lengths.astype(np.int64) <= 6].sum()) for h, cb in zip(hists, cbs))
    return {"n_bytes": n, "compressed_bytes": blob, "ratio": round(n / blob, 4),
            "savings_pct": round(100 * (1 - blob / n), 2), "exponent_entropy_bits": round(entropy_bits(hist), 4),
            "mean_code_bits": round(bits / n, 4), "codes_le6_bits_frac": round(le6 / n, 5),
            "max_code_bits": max(int(i.max_len) for i, _ in row)}


def _extra_config(L, torch, dev, spec_sets, steps, status, name, peak, note):
    """One batched launch over every tensor of the spec sets per step: decode
    GB/s (FP8 out) and roofline fraction, every output checked first."""
    sets, _ = _sources(torch, dev, spec_sets, 1, 0)
    d_xs = [d for ds in sets for d in ds]
    row, hists, cbs = _encode_set(L, torch, d_xs)
    d_out, out_offs = _layout_outputs(torch, dev, [i for i, _ in row])
    ws = torch.empty(max(L.batched_workspace_size(len(row)), 16), dtype=torch.uint8, device=dev)
    batch = _batch_for(L, row, d_out, out_offs)
    fn = lambda: L.decode_batched(batch, workspace=ws, status=status)  # noqa: E731
    fn()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"{name}: decode status {int(status.item())}"
    for k, d_x in enumerate(d_xs):
        if not torch.equal(d_out[out_offs[k]:out_offs[k] + d_x.numel()], d_x):
            raise SystemExit(f"{name}: decoded bytes differ from the source (tensor {k})")
    ms = _time_launches(torch, fn, steps, 3)
    summ = _summary(row, hists, cbs)
    alg = summ["compressed_bytes"] + summ["n_bytes"]
    res = {"workload": name, "tensors": len(row), "launches_per_step": 1, "ms_per_step": round(ms, 5),
           "gbps_fp8_out": round(summ["n_bytes"] / ms / 1e6, 2),
           "roofline_frac": round(alg / ms / 1e6 / peak, 4), "note": note, **summ}
    del row, d_out, ws, d_xs, sets
    torch.cuda.empty_cache()
    return res


def _extra_bf16(L, torch, dev, steps, status, peak):
    """The BF16 variant (DFloat11 article §3.3 batching): the seven Llama-3-8B
    projections in BF16 decoded by one batched launch per step, outputs
    checked first; roofline bytes = blobs read + BF16 written + tables read."""
    specs = synth.llama3_8b_layer_bf16().tensors
    xs = [t.generate_bf16() for t in specs]
    blobs = [L.bf16_encode(x) for x in xs]
    infos = [L.bf16_blob_info(b) for b in blobs]
    d_blobs = [torch.from_numpy(b).to(dev) for b in blobs]
    d_tables = [torch.from_numpy(L.bf16_table(i)).to(dev) for i in infos]
    d_outs = [torch.empty(int(i.n), dtype=torch.int16, device=dev) for i in infos]
    items = [(infos[k], d_blobs[k], d_tables[k], d_outs[k]) for k in range(len(specs))]
    fn = lambda: L.bf16_decode_batched(items, status)  # noqa: E731
    fn()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"BF16 decode status {int(status.item())}"
    for x, d in zip(xs, d_outs):
        if not np.array_equal(d.cpu().numpy().view(np.uint16), x):
            raise SystemExit("BF16 decode mismatch")
    launches0 = L.launch_count()
    ms = _time_launches(torch, fn, steps, 3)
    launches = (L.launch_count() - launches0) // (steps + 3)
    n = sum(int(i.n) for i in infos)
    blob = sum(int(b.size) for b in blobs)
    alg = blob + 2 * n + len(specs) * int(L._lib.ecf8_bf16_table_bytes())
    res = {"workload": "bf16_llama3_8b_layer_normal0.02", "tensors": len(specs), "launches_per_step": launches,
           "ms_per_step": round(ms, 5), "gbps_bf16_out": round(2 * n / ms / 1e6, 2),
           "roofline_frac": round(alg / ms / 1e6 / peak, 4), "ratio_vs_bf16": round(2 * n / blob, 4),
           "bits_per_weight": round(8 * blob / n, 4), "n_weights": n, "compressed_bytes": blob}
    del d_blobs, d_tables, d_outs
    torch.cuda.empty_cache()
    return res


def run_headline(args):
    """The 70B set: 80 layers compressed-resident, decoded layer by layer into
    one reused buffer (ECF8 walkthrough §3.2.2: a pool sized for the largest
    layer, reused), one step = the 80-layer loop."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    L = load_library()
    layers = args.layers
    specs = synth.llama3_70b_layer(0).tensors
    # layer 0 from the host generator (the parity tests' tensors), layers
    # 1..79 drawn on the GPU from their own seeds; every tensor encoded on the
    # GPU with its own codebook.  The sources (68 GB) stay on the device until
    # every layer's decode has been compared with them, then are dropped.
    layer_specs = [synth.llama3_70b_layer(l).tensors for l in range(layers)]
    sets, xs = _sources(torch, dev, layer_specs[:1], world, rank)
    rows, hists, cbs, srcs = [], [], [], []
    for l in range(layers):
        d_xs = sets[0] if l == 0 else [_sas_on_gpu(torch, dev, t) for t in layer_specs[l]]
        row, h, cb = _encode_set(L, torch, d_xs)
        rows.append(row)
        hists += h
        cbs += cb
        srcs.append(d_xs)
    infos0 = [i for i, _ in rows[0]]
    d_out, out_offs = _layout_outputs(torch, dev, infos0)  # one buffer, reused by every layer
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    batches = [_batch_for(L, row, d_out, out_offs) for row in rows]
    stream = torch.cuda.current_stream(dev)

    def step():
        for b in batches:
            L.decode_batched(b, status=status, stream=stream)

    # correctness of the timed configuration: every layer bit-exact against its source
    for l, b in enumerate(batches):
        L.decode_batched(b, status=status, stream=stream)
        for k in range(len(specs)):
            if not torch.equal(d_out[out_offs[k]:out_offs[k] + int(infos0[k].n)], srcs[l][k]):
                raise SystemExit(f"decode mismatch: layer {l} tensor {specs[k].name}")
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"decode status {int(status.item())}"
    d_xs0 = srcs[0]
    del srcs, sets
    torch.cuda.empty_cache()

    n_layer = sum(int(i.n) for i in infos0)
    blob_layer = sum(int(b.numel()) for b in (blob for _, blob in rows[0]))
    blob_total = sum(int(b.numel()) for row in rows for _, b in row)
    n_total = n_layer * layers

    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    t_end = time.perf_counter() + 1.0
    w = 0
    while w < args.warmup or time.perf_counter() < t_end:
        step()
        w += 1
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches0 = L.launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    launches = L.launch_count() - launches0
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    per_launch_ms = elapsed_ms / max(1, launches)
    elapsed_ms, per_launch_ms = max_over_ranks([elapsed_ms, per_launch_ms], dev)
    if world > 1:
        dist.barrier()
    assert int(status.item()) == 0

    # end to end through the same call, one layer per step: pinned host blobs
    # -> device, decode, device -> pinned host output
    h_blobs, blob_offs, o = [], [], 0
    for _, b in rows[0]:
        blob_offs.append(o)
        o += (int(b.numel()) + 255) // 256 * 256
    h_blob = torch.empty(o, dtype=torch.uint8, pin_memory=True)
    d_stage = torch.empty(o, dtype=torch.uint8, device=dev)
    for (_, b), bo in zip(rows[0], blob_offs):
        h_blob[bo:bo + b.numel()].copy_(b.cpu())
    h_out = torch.empty(d_out.numel(), dtype=torch.uint8, pin_memory=True)
    e2e_batch = L.make_batch([L.BatchItem(info, d_stage[bo:bo + info.blob_bytes], int(d_out.data_ptr()) + oo)
                              for info, bo, oo in zip(infos0, blob_offs, out_offs)])
    e2e_steps = max(1, args.e2e_steps)

    def e2e_step():
        d_stage.copy_(h_blob, non_blocking=True)
        L.decode_batched(e2e_batch, status=status, stream=stream)
        h_out.copy_(d_out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1)], dev)
    out_np = h_out.numpy()
    for k, d_x in enumerate(d_xs0):
        if not np.array_equal(out_np[out_offs[k]:out_offs[k] + d_x.numel()], d_x.cpu().numpy()):
            raise SystemExit("end-to-end decode mismatch")
    e2e_blob_bytes = sum(int(i.blob_bytes) for i in infos0)

    value = n_total * args.steps * world / (elapsed_ms / 1e3) / 1e9
    e2e_value = n_layer * e2e_steps * world / (e2e_ms / 1e3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    # one launch = one layer: its compressed bytes read + FP8 bytes written,
    # averaged over the 80 layers the timed launches decode
    alg_launch = blob_total / layers + n_layer
    achieved = alg_launch / (per_launch_ms / 1e3) / 1e9
    traffic = recorded_traffic("llama3_70b_layer", blob_total / layers)
    summ = _summary([r for row in rows for r in row], hists, cbs)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        h_blobs = [b.cpu().numpy() for _, b in rows[0]]
        cpu = oracle_cpu_baseline(h_blobs, xs)
        del h_blobs
    del rows, batches, d_stage, h_blob, h_out, d_xs0
    torch.cuda.empty_cache()

    extras = {}
    if world == 1 and not args.no_extras:
        extras["llama3_8b_layer"] = _extra_config(
            L, torch, dev, [synth.llama3_8b_layer().tensors], max(20, args.steps), status,
            "llama3_8b_layer_sas1.8", peak, "one batched launch of the 7 tensors (host generator)")
        moe = synth.moe_experts(args.moe_experts).tensors
        extras["moe_256x3"] = _extra_config(
            L, torch, dev, [moe[:3], moe[3:]], max(5, args.steps), status, f"moe_{args.moe_experts}x3_sas1.7",
            peak, "expert 0 from the host generator, experts 1.. drawn on the GPU from their own seeds; "
                  "one batched launch of all tensors (workspace)")
        extras["bf16_llama3_8b_layer"] = _extra_bf16(L, torch, dev, max(20, args.steps), status, peak)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": f"llama3_70b_{layers}layers_reused_buffer",
                       "description": "Llama-3-70B FP8 weight set: 80 layers x {q,o 8192x8192; k,v 1024x8192; "
                                      "gate,up 28672x8192; down 8192x28672}, SaS a=1.8, max|w|=448, one codebook "
                                      "per tensor, compressed-resident, decoded layer by layer into one reused "
                                      "buffer on one stream",
                       "layers": layers, "tensors": 7 * layers, "launches_per_step": layers,
                       "chunk_bytes": int(infos0[0].chunk_bytes), "group_chunks": int(infos0[0].group_chunks),
                       "resident_compressed_bytes": blob_total, "fp8_bytes_per_step": n_total,
                       "layer_inputs": "layer 0 from the host generator (the parity tests' tensors); layers 1.. "
                                       "drawn on the GPU from their own seeds (the same SaS law, torch Philox); "
                                       "all encoded on the GPU, one codebook per tensor",
                       "l2": "inputs+outputs larger than L2 (no flush)", **summ},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs", "nominal_peak": NOMINAL_HBM_GBS,
                         "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": round(alg_launch), "launch_ms": round(per_launch_ms, 5),
                         "launch": "one layer (7 tensors, one batched decode)"},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": e2e_blob_bytes,
                    "d2h_bytes_per_step": int(d_out.numel()), "steps": e2e_steps,
                    "step": "one layer: pinned host blobs -> device, decode, device -> pinned host"},
            "gpu_launches": int(launches),
            "clocks": clk,
            "extra": extras,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def load_library(build_only=False):
    from lossless_fp8_weight_b200 import _build
    _build.build()
    import lossless_fp8_weight_b200 as L
    return L


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-extras", action="store_true", help="headline: leave out the 8B-layer and MoE fields")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-sample", type=int, default=1 << 21)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", default=None, help="all, or a comma list of single_1k,llama3_8b_layer,sweep,moe,llama3_70b")
    ap.add_argument("--sweep-out", default=None)
    ap.add_argument("--moe-experts", type=int, default=256)
    ap.add_argument("--layers", type=int, default=80)
    ap.add_argument("--pipeline", action="store_true", help="decode-on-use pipeline beside FP8 GEMMs")
    ap.add_argument("--encode", action="store_true", help="GPU encoder against the host encoder")
    ap.add_argument("--bf16", action="store_true", help="BF16 variant decode on the Llama-3-8B layer in BF16")
    ap.add_argument("--pipeline-layers", type=int, default=8)
    ap.add_argument("--pipeline-tokens", type=int, default=2048)
    ap.add_argument("--pipeline-ctas", type=lambda v: [int(c) for c in v.split(",")], default=[148, 74, 37, 18])
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    workload = workload_by_name(args.workload)
    if args.impl == "reference":
        return run_reference(args, workload)
    if args.sweep:
        return run_sweep(args)
    if args.pipeline:
        return run_pipeline(args)
    if args.encode:
        return run_encode(args)
    if args.bf16:
        return run_bf16(args)
    if args.workload == HEADLINE:
        return run_headline(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    L = load_library()

    blobs, xs, stats = prepare(workload, L)
    infos = [L.blob_info(b) for b in blobs]
    n_total = sum(i.n for i in infos)
    blob_total = sum(int(b.size) for b in blobs)

    dev = torch.device("cuda", local)
    # all blobs in one allocation, each at a 256-byte boundary
    offs, o = [], 0
    for b in blobs:
        offs.append(o)
        o += (b.size + 255) // 256 * 256
    d_blobs = torch.empty(o, dtype=torch.uint8, device=dev)
    for b, off in zip(blobs, offs):
        d_blobs[off:off + b.size].copy_(torch.from_numpy(b))
    out_offs, o = [], 0
    for i in infos:
        out_offs.append(o)
        o += (i.n + 255) // 256 * 256
    d_out = torch.empty(o, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_bytes = max(L.batched_workspace_size(len(infos)), 16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    items = [L.BatchItem(i, int(d_blobs.data_ptr()) + bo, int(d_out.data_ptr()) + oo)
             for i, bo, oo in zip(infos, offs, out_offs)]
    batch = L.make_batch(items)
    stream = torch.cuda.current_stream(dev)

    def step():
        L.decode_batched(batch, workspace=ws, status=status, stream=stream)

    # correctness of the timed configuration: bit-exact against the source bytes
    step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"decode status {int(status.item())}"
    host_out = d_out.cpu().numpy()
    for x, oo in zip(xs, out_offs):
        if not np.array_equal(host_out[oo:oo + x.size], x):
            raise SystemExit("decode mismatch in the benchmark configuration")
    del host_out

    # warm-up (and a >= 1 s pre-roll under the clock sampler)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    t_end = time.perf_counter() + 1.0
    w = 0
    while w < args.warmup or time.perf_counter() < t_end:
        step()
        w += 1
        if w % 50 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches0 = L.launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    # no events between the steps: each decode launch lets the next one start
    # its prologue early (programmatic dependent launch), and an event in
    # between would serialise them
    t0.record(stream)
    for k in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    launches = L.launch_count() - launches0
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    per_launch_ms = elapsed_ms / max(1, launches)  # one decode launch per step
    elapsed_ms, per_launch_ms = max_over_ranks([elapsed_ms, per_launch_ms], dev)
    if world > 1:
        dist.barrier()
    assert int(status.item()) == 0

    # end to end through the same call: pinned host blob -> device, decode,
    # device -> pinned host output, every step
    h_blob = torch.empty(d_blobs.numel(), dtype=torch.uint8, pin_memory=True)
    for b, off in zip(blobs, offs):
        h_blob[off:off + b.size].copy_(torch.from_numpy(b))
    h_out = torch.empty(d_out.numel(), dtype=torch.uint8, pin_memory=True)
    e2e_steps = max(1, min(args.e2e_steps, args.steps))

    def e2e_step():
        d_blobs.copy_(h_blob, non_blocking=True)
        step()
        h_out.copy_(d_out, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)
    out_np = h_out.numpy()
    for x, oo in zip(xs, out_offs):
        assert np.array_equal(out_np[oo:oo + x.size], x)

    value = n_total * args.steps * world / (elapsed_ms / 1e3) / 1e9
    e2e_value = n_total * e2e_steps * world / (e2e_ms / 1e3) / 1e9
    peak, peak_kind = measured_hbm_peak()
    alg_bytes = blob_total + n_total  # compressed bytes read + FP8 bytes written
    achieved = alg_bytes / (per_launch_ms / 1e3) / 1e9
    traffic = recorded_traffic(workload.name)
    comp = compression_summary(stats)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_cpu_baseline(blobs, xs)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": workload.name, "description": workload.description,
                       "tensors": len(workload.tensors), "batched_launch": True,
                       "chunk_bytes": int(infos[0].chunk_bytes), "group_chunks": int(infos[0].group_chunks),
                       "l2": "inputs+outputs larger than L2 (no flush)"
                             if alg_bytes > L2_BYTES else "fits in L2 (no flush)",
                       **comp},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": f"{peak_kind} hbm_gbs", "nominal_peak": NOMINAL_HBM_GBS,
                         "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "launch_ms": round(per_launch_ms, 5)},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": "GB/s",
                    "h2d_bytes_per_step": int(blob_total), "d2h_bytes_per_step": int(n_total),
                    "steps": e2e_steps},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Throughput of tile-routed FP16/INT8 causal prefill attention on B200.

One step = the whole hot path on one batch of synthetic inputs resident in
HBM: blockwise INT8 quantisation of Q and of K, packing of the routing
words, and the fused attention kernel.  Reported:

  value       tokens/s of the step (all ranks; weak scaling: every rank runs
              its own replica of the workload, no collective on the data path)
  effective   4 * d * Hq * sum L(L+1)/2 FLOP per step / step time
  roofline    the attention kernel against the mixed FP16/INT8 tensor-core
              roofline t_roof = (QK_fp16 + PV) / P_fp16 + QK_int8 / P_int8
  e2e         the same metric through the public API with host buffers:
              pinned host -> device copies of Q, K, V and the routing bytes and
              the device -> host copy of the output inside the timed region,
              steps pipelined over copy-in, compute and copy-out streams
  cpu_baseline  the CPU oracle, timed on this host's cores on a bounded
              sample of the same workload (rank 0, one GPU only)

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm

L2 is flushed (a 256 MiB write) before every timed step, outside the
per-step CUDA events.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "prefill attn tokens/s & effective TFLOPS vs mixed FP16/INT8 roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = W.LLAMA32_3B_4K.name
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
INT8_OVER_FP16 = 2.0  # nominal dense INT8 / FP16 tensor ratio (4.5 / 2.25 P)


# DRAM bytes (read + write) of one attention launch from an ncu capture of
# this bench's own command, keyed by workload and by a hash of the kernel
# sources the capture ran; a changed kernel reports null until re-captured.
NCU_TRAFFIC = {
    ("llama32_3b_b8_L4096_int8_75", "2625fb088d1686fc"): 466_481_920 + 178_798_080,
}
KERNEL_SOURCES = ("prefill_blockwise_int8_b200/csrc/attn_prefill.cu",
                  "prefill_blockwise_int8_b200/csrc/ptx.cuh",
                  "prefill_blockwise_int8_b200/csrc/internal.h")


# the same for the two adaptive-routing kernels (sums + rank, per call)
ROUTE_SOURCES = ("prefill_blockwise_int8_b200/csrc/route_adaptive.cu",)
ROUTE_TRAFFIC = {
    ("llama32_3b_b8_L4096_int8_75", "5a599996a59ca2de"):
        268_482_816 + 7_033_344 + 6_314_752,
}


def kernel_source_hash(sources=KERNEL_SOURCES):
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_name):
    return NCU_TRAFFIC.get((workload_name, kernel_source_hash()))


def measured_route_traffic(workload_name):
    return ROUTE_TRAFFIC.get((workload_name, kernel_source_hash(ROUTE_SOURCES)))


def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks of the default process group (x
    itself without one): the job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tilemix", "reference"],
                    default="tilemix")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(W.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="CPU time budget of the --impl reference run")
    ap.add_argument("--quant-on-chip", action="store_true",
                    help="quantise Q and K tiles inside the attention kernel "
                         "(no separate quantiser launches)")
    ap.add_argument("--routing", choices=["given", "adaptive"], default="given",
                    help="given: the workload's routing bytes are an input and "
                         "are packed each step; adaptive: each step derives "
                         "the routing words from Q and K on the device at the "
                         "workload's INT8 coverage")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, inp, share, on_chip=False, adaptive=False,
                    permille=None):
    """The line's config; both arms (GPU and the CPU oracle) report the same
    keys for the same workload and options."""
    lens = inp["seqlens"]
    return {
        "workload": w.name,
        "batch": int(len(lens)),
        "seq_len": int(lens.max()) if w.seqlen == 0 else int(w.seqlen),
        "total_tokens": int(lens.sum()),
        "hq": w.hq, "hkv": w.hkv, "head_dim": w.d,
        "tile": f"{w.block_m}x{w.block_n}", "group": int(inp["group"]),
        "kv_format": w.kv_format,
        "int8_group_coverage": w.coverage,
        "int8_pair_share": round(share, 4),
        "quant_block": [w.quant_block_q, w.quant_block_k],
        "inputs": "N(0,1) fp16" + (", 4 outlier channels x20 per Q/K head"
                                    if w.outliers else ""),
        "parallelism": "replicas",
        "l2": "flushed (256 MiB write) before every timed step",
        "quantisation": "on chip" if on_chip else "quantise once",
        "routing": ("adaptive (on device, exact logit-sum statistic, "
                    f"{permille} permille INT8)" if adaptive
                    else "given routing bytes"),
    }


# ----------------------------------------------------------------------------
# CPU oracle legs
# ----------------------------------------------------------------------------

def oracle_sample_rate(inp, target_s, seed=7):
    """tokens/s of the oracle on uniformly drawn query rows (all heads, the
    full causal row each).  Returns (tokens/s, sample description, cores)."""
    import oracle
    args, kw = oracle.prepare(inp)
    total = int(inp["seqlens"].sum())
    rng = np.random.default_rng(seed)
    n = 16
    elapsed = 0.0
    done = 0
    while True:
        rows = np.sort(rng.choice(total, size=min(n, total), replace=False))
        t0 = time.perf_counter()
        oracle.attn_prefill(*args, rows=rows, **kw)
        dt = time.perf_counter() - t0
        elapsed += dt
        done += len(rows)
        if elapsed >= target_s or done >= total:
            break
        per_row = elapsed / done
        n = int(max(16, min(total, (target_s - elapsed) / per_row)))
    cores = os.cpu_count() or 1
    desc = (f"{done} query tokens drawn uniformly from {total} "
            f"(all {inp['workload'].hq} heads, full causal rows), "
            f"{elapsed:.1f} s on {cores} threads; oracle quantiser and "
            f"packer excluded")
    return done / elapsed, desc, cores


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = W.WORKLOADS[args.workload]
    inp = W.make(w)
    share = None
    import oracle
    oargs, kw = oracle.prepare(inp)
    total = int(inp["seqlens"].sum())
    budget = args.ref_seconds  # seconds for warmup + steps together
    per_step = budget / (args.steps + args.warmup)
    rng = np.random.default_rng(11)
    # calibrate rows per step
    rows = np.sort(rng.choice(total, size=16, replace=False))
    t0 = time.perf_counter()
    oracle.attn_prefill(*oargs, rows=rows, **kw)
    per_row = (time.perf_counter() - t0) / 16
    n = int(max(1, min(total, per_step / per_row)))
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(total, size=n, replace=False))
        t0 = time.perf_counter()
        oracle.attn_prefill(*oargs, rows=rows, **kw)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    value = n * len(times) / sum(times)
    cores = os.cpu_count() or 1
    fp16_pairs, int8_pairs = _pairs(inp, oracle.pack_mask(
        inp["route"], inp["cu_seqlens"], inp["max_seqlen"], w.block_m,
        w.block_n, inp["group"]))
    share = int8_pairs / (fp16_pairs + int8_pairs)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, inp, share),
        "cpu_baseline": {
            "value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"each step {n} query tokens drawn uniformly from {total}"
                      f" (all heads, full causal rows) on {cores} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _pairs(inp, mask_words):
    from prefill_blockwise_int8_b200.roofline import pair_counts
    w = inp["workload"]
    return pair_counts(inp["seqlens"], mask_words, w.block_m, w.block_n,
                       inp["group"], w.hq, w.hkv)


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.out = None

    def __enter__(self):
        import tempfile
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv",
                                               delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200", "-i",
                 str(self.dev)], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.out.flush()

    def summary(self):
        try:
            lines = open(self.out.name).read().strip().splitlines()
        except OSError:
            lines = []
        finally:
            try:
                os.unlink(self.out.name)
            except OSError:
                pass
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=datetime.timedelta(seconds=300))

    import prefill_blockwise_int8_b200 as tm

    w = W.WORKLOADS[args.workload]
    inp = W.make(w)
    lens, cu_np = inp["seqlens"], inp["cu_seqlens"]
    ms, g = inp["max_seqlen"], inp["group"]
    T = int(lens.sum())
    t_h = {k: torch.from_numpy(inp[k]) for k in ("q", "k", "v", "route")}
    cu_h = torch.from_numpy(cu_np)
    q = t_h["q"].to(dev)
    k = t_h["k"].to(dev)
    v = t_h["v"].to(dev)
    route = t_h["route"].to(dev)
    cu = cu_h.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    q8 = torch.empty((T, w.hq, w.d), dtype=torch.int8, device=dev)
    k8 = torch.empty((T, w.hkv, w.d), dtype=torch.int8, device=dev)
    sq = torch.empty((w.hq, len(lens), -(-ms // w.quant_block_q)),
                     dtype=torch.float32, device=dev)
    sk = torch.empty((w.hkv, len(lens), -(-ms // w.quant_block_k)),
                     dtype=torch.float32, device=dev)
    mask = torch.empty(route.shape[:3], dtype=torch.int64, device=dev)
    out = torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # INT8 KV cache: K8, V8 and their scales are the inputs (quantised once,
    # outside the timed region, by the same quantiser); a step quantises Q,
    # packs the words and runs attention.
    kv8 = w.kv_format == "int8"
    v8 = sv = None
    if kv8:
        v8 = torch.empty((T, w.hkv, w.d), dtype=torch.int8, device=dev)
        sv = torch.empty_like(sk)
        tm.tilemix_quantize_blockwise(k, cu, ms, w.quant_block_k, x8=k8,
                                      scale=sk, status=status)
        tm.tilemix_quantize_blockwise(v, cu, ms, w.quant_block_k, x8=v8,
                                      scale=sv, status=status)
        torch.cuda.synchronize(dev)
        t_h = {"q": t_h["q"], "route": t_h["route"], "k8": k8.cpu(),
               "k_scale": sk.cpu(), "v8": v8.cpu(), "v_scale": sv.cpu()}
        del k, v
        k = v = None
    on_chip = args.quant_on_chip and not kv8
    adaptive = args.routing == "adaptive"
    if adaptive and kv8:
        raise SystemExit("--routing adaptive needs fp16 K (not an INT8 KV cache)")
    launches_per_step = (2 if on_chip else 3) + \
        (1 if adaptive else 0)
    permille = int(round(w.coverage * 1000))
    ws = None
    if adaptive:
        ws = torch.empty(max(16, tm.tilemix_route_adaptive_workspace_bytes(
            len(lens), ms, w.hkv, w.d, w.block_m)), dtype=torch.uint8,
            device=dev)

    # device buffers of one step: inputs (and O) per set, so the pipelined
    # end-to-end run can copy the next step's inputs while this one computes
    set0 = dict(q=q, k=k, v=v, cu=cu, route=route, k8=k8, k_scale=sk, v8=v8,
                v_scale=sv, out=out)

    def step(attn_events=None, route_events=None, b=None, quant_events=None):
        b = set0 if b is None else b
        if not kv8 and not on_chip:  # Q and K in one launch
            if quant_events:
                quant_events[0].record(stream)
            tm.tilemix_quantize_blockwise_qk(
                b["q"], b["k"], b["cu"], ms, w.quant_block_q, w.quant_block_k,
                q8=q8, q_scale=sq, k8=b["k8"], k_scale=b["k_scale"],
                status=status)
            if quant_events:
                quant_events[1].record(stream)
        elif not on_chip:
            tm.tilemix_quantize_blockwise(b["q"], b["cu"], ms, w.quant_block_q,
                                          x8=q8, scale=sq, status=status)
        if route_events:
            route_events[0].record(stream)
        if adaptive:
            tm.tilemix_route_adaptive(b["q"], b["k"], b["cu"], ms, w.block_m,
                                      w.block_n, g, permille, workspace=ws,
                                      mask=mask, want_route=False,
                                      status=status)
        else:
            tm.tilemix_pack_mask(b["route"], b["cu"], ms, w.block_m, w.block_n,
                                 g, mask=mask, status=status)
        if route_events:
            route_events[1].record(stream)
        if attn_events:
            attn_events[0].record(stream)
        tm.tilemix_attn_prefill(
            b["q"], b["k"], b["v"], b["cu"], ms, q8=q8, q_scale=sq, k8=b["k8"],
            k_scale=b["k_scale"], v8=b["v8"], v_scale=b["v_scale"], mask=mask,
            block_m=w.block_m, block_n=w.block_n, group=g,
            quant_block_q=w.quant_block_q, quant_block_k=w.quant_block_k,
            kv_format=tm.KV_INT8 if kv8 else tm.KV_FP16,
            quant_on_chip=on_chip, out=b["out"], status=status)
        if attn_events:
            attn_events[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} during warmup")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)]
          for _ in range(args.steps)]
    smi_index = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [p.strip() for p in vis.split(",")]
        if local < len(parts):
            smi_index = parts[local]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(smi_index) as clocks:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step((ev[i][1], ev[i][2]), (ev[i][4], ev[i][5]),
                 quant_events=(ev[i][6], ev[i][7]))
            ev[i][3].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[3]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    route_ms = [e[4].elapsed_time(e[5]) for e in ev]
    quant_ms = ([e[6].elapsed_time(e[7]) for e in ev]
                if not kv8 and not on_chip else None)
    total_ms = max_over_ranks(sum(step_ms), dev)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} in timed region")
    ms_step = total_ms / args.steps
    value = world * T / (ms_step * 1e-3)

    # ---- e2e through the public API with host buffers ----
    # Every step copies its inputs from pinned host memory and its output
    # back.  The steps are pipelined the way a serving loop would run them:
    # host-to-device copies on one stream, compute on the launching stream,
    # device-to-host copies on a third, with two device buffer sets, so step
    # i + 1's inputs cross PCIe while step i computes and step i - 1's output
    # returns.  Time = first copy issued to last output landed, over n steps.
    e2e = None
    if not args.no_e2e:
        names = ["q", "cu"] + ([] if adaptive else ["route"]) + \
            (["k8", "k_scale", "v8", "v_scale"] if kv8 else ["k", "v"])
        host = dict(t_h)
        host["cu"] = cu_h
        pin = {n: host[n].pin_memory() for n in names}
        sets = [set0, dict(set0)]
        for n in names + ["out"]:
            sets[1][n] = torch.empty_like(set0[n])
        out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory()
                 for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in pin.values())
        d2h = out_h[0].numel() * out_h[0].element_size()
        s_in = torch.cuda.Stream(dev)
        s_out = torch.cuda.Stream(dev)

        def run_pipelined(n):
            ev_in = [torch.cuda.Event() for _ in range(n)]
            ev_comp = [torch.cuda.Event() for _ in range(n)]
            ev_out = [torch.cuda.Event() for _ in range(n)]
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            s_in.wait_event(t0)
            s_out.wait_event(t0)
            for i in range(n):
                bs = sets[i % 2]
                with torch.cuda.stream(s_in):
                    if i >= 2:   # step i - 2 has finished reading this set
                        s_in.wait_event(ev_comp[i - 2])
                    for nm in names:
                        bs[nm].copy_(pin[nm], non_blocking=True)
                    ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                if i >= 2:       # and its output has left this set
                    stream.wait_event(ev_out[i - 2])
                step(b=bs)
                ev_comp[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[i])
                    out_h[i % 2].copy_(bs["out"], non_blocking=True)
                    ev_out[i].record(s_out)
            stream.wait_event(ev_out[n - 1])
            t1.record(stream)
            torch.cuda.synchronize(dev)
            return t0.elapsed_time(t1)

        n_e2e = max(4, min(args.steps, 12))
        run_pipelined(3)   # warm-up
        if world > 1:
            dist.barrier()
        e_ms = max_over_ranks(run_pipelined(n_e2e), dev)
        if status.item() != 0:
            raise RuntimeError(f"device status {status.item()} in e2e run")
        # the output of the last step equals the device-timed run's
        if not torch.equal(out_h[(n_e2e - 1) % 2].to(dev), out):
            raise RuntimeError("e2e output differs from the device-timed step")
        e2e = {"value": world * T / (e_ms / n_e2e * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "pipelined": True,
               "l2": "each step's inputs (%.0f MB) exceed L2; no flush" %
                     (h2d / 1e6)}

    # ---- roofline of the attention kernel ----
    from prefill_blockwise_int8_b200 import roofline as R
    mask_np = mask.cpu().numpy().view(np.uint64)
    fp16_pairs, int8_pairs = R.pair_counts(lens, mask_np, w.block_m,
                                           w.block_n, g, w.hq, w.hkv)
    wk = R.work(lens, w.d, w.hq, fp16_pairs, int8_pairs)
    peaks, peak_src = load_peaks()
    p16 = float(peaks["bf16_tflops"]) * 1e12  # fp16 dense = bf16 dense rate
    p8 = p16 * INT8_OVER_FP16
    t_roof = R.roofline_seconds(wk, p16, p8)
    attn_s = statistics.mean(attn_ms) * 1e-3
    achieved = wk["effective"] / attn_s / 1e12
    peak_eff = wk["effective"] / t_roof / 1e12
    roof = {
        "bound": "tensor", "achieved": round(achieved, 2),
        "peak": round(peak_eff, 2), "unit": "TFLOP/s",
        "frac": round(achieved / peak_eff, 4),
        "traffic": measured_traffic(w.name),
        "kernel": "attn_fwd_kernel",
        "attn_ms": round(attn_s * 1e3, 4),
        "t_roof_ms": round(t_roof * 1e3, 4),
        "peak_basis": (f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s"
                       f" for FP16; INT8 = x{INT8_OVER_FP16:g} (nominal "
                       "4.5/2.25 P dense ratio); mixed by routed pair share "
                       f"{wk['int8_pair_share']:.4f}"),
        "algorithmic_flop_per_launch": wk["effective"],
        "hbm_bytes_min_per_launch": R.min_hbm_bytes(
            T, w.hq, w.hkv, w.d, wk["int8_pair_share"]),
    }

    route_roof = None
    if adaptive:
        # the sums pass reads Q and K once; the words written are negligible
        nbytes = T * (w.hq + w.hkv) * w.d * 2
        r_s = statistics.mean(route_ms) * 1e-3
        gbs = nbytes / r_s / 1e9
        route_roof = {"bound": "hbm", "achieved": round(gbs, 1),
                      "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                      "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
                      "bytes_per_launch": nbytes,
                      "traffic": measured_route_traffic(w.name),
                      "kernels": "sums_kernel + rank_kernel"}

    quant_roof = None
    if quant_ms:
        # Q and K read once as fp16, Q8 and K8 written once, fp32 scales
        nq = -(-ms // w.quant_block_q) * w.hq * len(lens)
        nk = -(-ms // w.quant_block_k) * w.hkv * len(lens)
        nbytes = T * (w.hq + w.hkv) * w.d * 3 + 4 * (nq + nk)
        q_s = statistics.mean(quant_ms) * 1e-3
        gbs = nbytes / q_s / 1e9
        quant_roof = {"bound": "hbm", "achieved": round(gbs, 1),
                      "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                      "frac": round(gbs / float(peaks["hbm_gbs"]), 4),
                      "bytes_per_launch": nbytes,
                      "ms": round(q_s * 1e3, 4),
                      "kernel": "quantize_kernel (Q and K, one launch)"}

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        rate, desc, cores = oracle_sample_rate(inp, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16+int8", "data": "synthetic",
        "config": workload_config(w, inp, wk["int8_pair_share"],
                                  on_chip=on_chip, adaptive=adaptive,
                                  permille=permille),
        "routing_ms": round(statistics.mean(route_ms), 4),
        "routing_roofline": route_roof,
        "quantiser_roofline": quant_roof,
        "effective_tflops": wk["effective"] / (ms_step * 1e-3) / 1e12 * world,
        "attn_effective_tflops": achieved,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())

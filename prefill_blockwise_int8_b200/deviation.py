"""Numerical-deviation study: how far tile-routed FP16/INT8 attention moves
from the all-FP16 result as INT8 coverage grows.

The TileMix paperlayer summary, appendix G Numerical Analysis (G.1, G.3),
measures MaxDiff / MeanDiff of the routed kernel against a fixed FP16
reference across INT8 coverage and precision layouts.  Here the fixed
reference is this library's own FP16 path (TILEMIX_FLAG_FP16_ONLY: every
legal tile FP16, same kernel, same schedule), so a difference isolates what
INT8 routing changes.  Inputs are synthetic (seeded N(0,1) with outlier
channels in Q and K, the same generator as the benchmark); routing masks
draw exactly round(c * N_legal) INT8 groups per KV head.

    python -m prefill_blockwise_int8_b200.deviation --seqlen 8192
    python -m prefill_blockwise_int8_b200.deviation --policies band,adaptive

With --policies it compares routing policies (the static templates and the
adaptive one) at equal per-row INT8 shares instead.  The accumulation axis
(appendix G.4 of the same summary: FP16 against FP32 accumulation) repeats
each coverage with O accumulated in fp16 (the study-only
TILEMIX_FLAG_PV_F16_ACC), still measured against the fp32-accumulated
all-FP16 reference.  Needs a GPU; prints one line per coverage (and policy
or accumulator) and returns the rows.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

DEFAULT_COVERAGES = (0.0, 0.05, 0.10, 0.25, 0.50, 0.75, 1.0)
# Routing policies at a per-row INT8 share: the static templates of this
# library and the on-device adaptive policy (exact block logit sums).
POLICIES = ("row_random", "band", "bigbird", "sptrans", "adaptive")


ACCUMULATORS = ("f32", "f16")


def run(seqlen: int = 8192, hq: int = 8, hkv: int = 2, d: int = 128,
        block_m: int = 128, block_n: int = 128, coverages=DEFAULT_COVERAGES,
        seed: int = 7, device: str = "cuda", accumulators=("f32",)):
    import torch

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import workloads as W
    import prefill_blockwise_int8_b200 as tm

    base = W.Workload(name="deviation", batch=1, hq=hq, hkv=hkv, d=d,
                      block_m=block_m, block_n=block_n, group=0,
                      seqlen=seqlen, outliers=True, mask_recipe="exact",
                      coverage=0.0, coverage_unit="kv_head", seed=seed,
                      mask_seed=seed + 1)
    inp = W.make(base)
    dev = torch.device(device)
    cu = torch.from_numpy(inp["cu_seqlens"]).to(dev)
    q, k, v = (torch.from_numpy(inp[x]).to(dev) for x in "qkv")
    ms, g = inp["max_seqlen"], inp["group"]
    q8, sq = tm.tilemix_quantize_blockwise(q, cu, ms, 128)
    k8, sk = tm.tilemix_quantize_blockwise(k, cu, ms, 128)
    ref = tm.tilemix_attn_prefill(q, k, v, cu, ms, fp16_only=True,
                                  block_m=block_m, block_n=block_n,
                                  group=g).float()
    rows = []
    for c in coverages:
        w = base.with_(coverage=float(c), mask_seed=seed + 1 + int(c * 1000))
        route = torch.from_numpy(W.route_bytes(w, inp["seqlens"])).to(dev)
        mask = tm.tilemix_pack_mask(route, cu, ms, block_m, block_n, g)
        for acc in accumulators:
            out = tm.tilemix_attn_prefill(
                q, k, v, cu, ms, q8=q8, q_scale=sq, k8=k8, k_scale=sk,
                mask=mask, block_m=block_m, block_n=block_n, group=g,
                pv_f16_acc=(acc == "f16")).float()
            diff = (out - ref).abs()
            rows.append(dict(coverage=float(c), accumulate=acc,
                             max_diff=float(diff.max()),
                             mean_diff=float(diff.mean())))
    return rows


def run_policies(seqlen: int = 8192, hq: int = 8, hkv: int = 2, d: int = 128,
                 block_m: int = 128, block_n: int = 128,
                 coverages=DEFAULT_COVERAGES, policies=POLICIES, seed: int = 7,
                 device: str = "cuda"):
    """MaxDiff / MeanDiff against the FP16-only path for each routing policy
    at each per-row INT8 share (the INT8 groups of every query-tile row are
    round(c * G) of its G legal groups under every policy, so the policies
    differ only in which groups they send to INT8)."""
    import torch

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import workloads as W
    import prefill_blockwise_int8_b200 as tm

    base = W.Workload(name="deviation", batch=1, hq=hq, hkv=hkv, d=d,
                      block_m=block_m, block_n=block_n, group=0,
                      seqlen=seqlen, outliers=True, mask_recipe="exact",
                      coverage=0.0, coverage_unit="kv_head", seed=seed,
                      mask_seed=seed + 1)
    inp = W.make(base)
    dev = torch.device(device)
    cu = torch.from_numpy(inp["cu_seqlens"]).to(dev)
    q, k, v = (torch.from_numpy(inp[x]).to(dev) for x in "qkv")
    ms, g = inp["max_seqlen"], inp["group"]
    q8, sq = tm.tilemix_quantize_blockwise(q, cu, ms, 128)
    k8, sk = tm.tilemix_quantize_blockwise(k, cu, ms, 128)
    ref = tm.tilemix_attn_prefill(q, k, v, cu, ms, fp16_only=True,
                                  block_m=block_m, block_n=block_n,
                                  group=g).float()
    rows = []
    for c in coverages:
        permille = int(round(c * 1000))
        for pol in policies:
            if pol == "adaptive":
                route = tm.tilemix_route_adaptive(q, k, cu, ms, block_m,
                                                  block_n, g, permille)
            else:
                route = tm.tilemix_route_template(pol, permille, cu, ms, hkv,
                                                  block_m, block_n, g,
                                                  seed=seed)
            mask = tm.tilemix_pack_mask(route, cu, ms, block_m, block_n, g)
            out = tm.tilemix_attn_prefill(
                q, k, v, cu, ms, q8=q8, q_scale=sq, k8=k8, k_scale=sk,
                mask=mask, block_m=block_m, block_n=block_n, group=g).float()
            diff = (out - ref).abs()
            rows.append(dict(coverage=float(c), policy=pol,
                             max_diff=float(diff.max()),
                             mean_diff=float(diff.mean())))
    return rows


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--seqlen", type=int, default=8192)
    ap.add_argument("--hq", type=int, default=8)
    ap.add_argument("--hkv", type=int, default=2)
    ap.add_argument("--block-n", type=int, default=128)
    ap.add_argument("--policies", default="",
                    help="comma list of " + ",".join(POLICIES) + ": compare "
                         "routing policies at per-row INT8 shares instead of "
                         "the per-KV-head random masks")
    ap.add_argument("--accumulate", default="f32",
                    help="comma list of " + ",".join(ACCUMULATORS) + ": the "
                         "P V accumulator(s) to measure (f16 is study only)")
    args = ap.parse_args(argv)
    if args.policies:
        pols = tuple(p for p in args.policies.split(",") if p)
        rows = run_policies(seqlen=args.seqlen, hq=args.hq, hkv=args.hkv,
                            block_n=args.block_n, policies=pols)
        print(f"{'INT8 coverage':>14} {'policy':>11} {'MaxDiff':>10} "
              f"{'MeanDiff':>10}")
        for r in rows:
            print(f"{r['coverage']:>14.2f} {r['policy']:>11} "
                  f"{r['max_diff']:>10.3e} {r['mean_diff']:>10.3e}")
        return rows
    accs = tuple(a for a in args.accumulate.split(",") if a)
    bad = [a for a in accs if a not in ACCUMULATORS]
    if bad:
        raise SystemExit(f"unknown accumulator(s) {bad}")
    rows = run(seqlen=args.seqlen, hq=args.hq, hkv=args.hkv,
               block_n=args.block_n, accumulators=accs)
    print(f"{'INT8 coverage':>14} {'P V acc':>8} {'MaxDiff':>10} "
          f"{'MeanDiff':>10}")
    for r in rows:
        print(f"{r['coverage']:>14.2f} {r['accumulate']:>8} "
              f"{r['max_diff']:>10.3e} {r['mean_diff']:>10.3e}")
    return rows


if __name__ == "__main__":
    main()

"""Numerical-deviation study on the GPU: the routed kernel with no INT8
group equals the FP16-only path exactly, and the deviation from it grows
with INT8 coverage (paperlayer summary, appendix G.1: deviation rises with
INT8 coverage; the 0% configuration stays at the FP16 reference)."""
import pytest

pytestmark = pytest.mark.gpu

pytest.importorskip("torch")


def test_deviation_grows_with_coverage():
    from prefill_blockwise_int8_b200 import deviation
    rows = deviation.run(seqlen=4096, hq=4, hkv=2,
                         coverages=(0.0, 0.25, 0.5, 1.0))
    by = {r["coverage"]: r for r in rows}
    assert by[0.0]["max_diff"] == 0.0
    means = [by[c]["mean_diff"] for c in (0.25, 0.5, 1.0)]
    assert 0.0 < means[0] < means[1] < means[2]


def test_policies_agree_at_the_ends_of_the_coverage_range():
    # no INT8 group: every policy is the FP16 path; every group INT8: every
    # policy gives the same mask, so the same output
    from prefill_blockwise_int8_b200 import deviation
    rows = deviation.run_policies(seqlen=2048, hq=4, hkv=2,
                                  coverages=(0.0, 0.5, 1.0))
    at = {(r["coverage"], r["policy"]): r for r in rows}
    for pol in deviation.POLICIES:
        assert at[(0.0, pol)]["max_diff"] == 0.0
        assert at[(1.0, pol)]["mean_diff"] == at[(1.0, "band")]["mean_diff"]
        assert at[(0.5, pol)]["mean_diff"] > 0.0


def test_f16_accumulator_axis():
    # Study only (appendix G.4 of the paperlayer summary: FP16 against FP32
    # accumulation): with O accumulated in fp16 the output moves away from
    # the fp32-accumulated FP16 reference even with no INT8 group; the mode
    # is deterministic and finite on these inputs.  It is not held to the
    # output tolerance, so no bound on the size of the deviation is asserted.
    import math
    from prefill_blockwise_int8_b200 import deviation
    kw = dict(seqlen=2048, hq=4, hkv=2, coverages=(0.0, 0.5),
              accumulators=deviation.ACCUMULATORS)
    rows = deviation.run(**kw)
    again = deviation.run(**kw)
    at = {(r["coverage"], r["accumulate"]): r for r in rows}
    assert at[(0.0, "f32")]["max_diff"] == 0.0
    assert at[(0.0, "f16")]["max_diff"] > 0.0
    for r in rows:
        assert math.isfinite(r["max_diff"]) and math.isfinite(r["mean_diff"])
    assert rows == again


def test_deviation_statistics_match_the_oracle():
    # MaxDiff / MeanDiff of the routed output against the FP16-only output
    # (appendix G.1's statistics), once from the GPU path and once from the
    # oracle on the same small seeded inputs (50% INT8 groups, outlier
    # channels, two ragged sequences).  Each GPU output lies within the
    # output tolerance of its oracle output, so the two MaxDiffs agree
    # within twice that tolerance; the MeanDiffs must agree to 10%, which a
    # mis-scaled or mis-routed INT8 path would not meet.
    import numpy as np
    import workloads as W
    from _gpu_path import MAX_ABS, run_gpu, run_oracle
    lens = np.array([300, 700], dtype=np.int32)
    w = W.Workload(name="deviation_small", batch=2, hq=4, hkv=2, d=128,
                   block_m=128, block_n=64, group=1, seqlen=0, outliers=True,
                   mask_recipe="bernoulli", coverage=0.5, seed=11, mask_seed=12,
                   coverage_unit="kv_head")
    q, k, v = W.qkv(w.with_(seqlen=1), lens)
    inp = dict(workload=w, seqlens=lens, cu_seqlens=W.cu_seqlens(lens),
               max_seqlen=int(lens.max()), group=1, q=q, k=k, v=v,
               route=W.route_bytes(w, lens))
    g_r = run_gpu(inp)["out"].astype(np.float64)
    g_f = run_gpu(inp, fp16_only=True)["out"].astype(np.float64)
    o_r = run_oracle(inp)[0]
    o_f = run_oracle(inp, fp16_only=True)[0]
    gd, od = np.abs(g_r - g_f), np.abs(o_r - o_f)
    assert od.mean() > 1e-4  # INT8 routing moves the oracle's output
    assert abs(gd.max() - od.max()) <= 2 * MAX_ABS
    assert abs(gd.mean() - od.mean()) <= 0.1 * od.mean()

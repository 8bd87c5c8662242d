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

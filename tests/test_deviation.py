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

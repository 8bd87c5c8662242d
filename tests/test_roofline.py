"""Host-side work accounting behind the bench's roofline: routed pair counts
against the oracle's own count, the effective-FLOP closed form, the mixed
roofline time, and the compulsory HBM bytes."""
import numpy as np
import pytest

import oracle
import workloads as W
from prefill_blockwise_int8_b200 import roofline as R


def _varlen_inputs():
    w = W.Workload(name="acct", batch=3, hq=6, hkv=2, d=32, block_m=64,
                   block_n=64, group=2, seqlen=0, outliers=False,
                   mask_recipe="bernoulli", coverage=0.5, seed=3,
                   mask_seed=4, coverage_unit="kv_head")
    lens = np.array([300, 1, 517], np.int32)
    q, k, v = W.qkv(w.with_(seqlen=1), lens)
    return dict(workload=w, seqlens=lens, cu_seqlens=W.cu_seqlens(lens),
                max_seqlen=int(lens.max()), group=2, q=q, k=k, v=v,
                route=W.route_bytes(w, lens))


def test_tile_pairs_brute_force():
    for L, bm, bn in [(1, 64, 64), (200, 64, 64), (130, 128, 64), (77, 64, 128)]:
        for m in range(-(-L // bm)):
            for n in range(-(-L // bn)):
                want = sum(1 for i in range(m * bm, min((m + 1) * bm, L))
                           for j in range(n * bn, min((n + 1) * bn, L)) if j <= i)
                assert R._tile_pairs(L, m, n, bm, bn) == want


def test_pair_counts_equal_the_oracle_count():
    inp = _varlen_inputs()
    w = inp["workload"]
    args, kw = oracle.prepare(inp)
    (_, counts) = oracle.attn_prefill(*args, rows=np.array([0]),
                                      want_pair_counts=True, **kw)
    words = oracle.pack_mask(inp["route"], inp["cu_seqlens"],
                             inp["max_seqlen"], w.block_m, w.block_n, 2)
    fp16, int8 = R.pair_counts(inp["seqlens"], words, w.block_m, w.block_n,
                               2, w.hq, w.hkv)
    assert (fp16, int8) == (int(counts[0]), int(counts[1]))
    assert fp16 > 0 and int8 > 0
    # all-FP16 mode counts every legal pair as FP16
    f_only, i_only = R.pair_counts(inp["seqlens"], words, w.block_m,
                                   w.block_n, 2, w.hq, w.hkv, fp16_only=True)
    assert i_only == 0 and f_only == fp16 + int8


def test_work_and_roofline_closed_forms():
    lens, d, hq = [4096] * 8, 128, 24
    legal = hq * sum(L * (L + 1) // 2 for L in lens)
    wk = R.work(lens, d, hq, legal // 4, legal - legal // 4)
    assert wk["effective"] == 4 * d * hq * sum(L * (L + 1) // 2 for L in lens)
    assert wk["qk_fp16"] + wk["qk_int8"] == wk["pv"]
    t = R.roofline_seconds(wk, 1.0e15, 2.0e15)
    assert t == pytest.approx((wk["qk_fp16"] + wk["pv"]) / 1e15 +
                              wk["qk_int8"] / 2e15, rel=1e-15)
    # all FP16: both halves at the FP16 rate; all INT8 saves a quarter
    all16 = R.work(lens, d, hq, legal, 0)
    all8 = R.work(lens, d, hq, 0, legal)
    assert R.roofline_seconds(all8, 1e15, 2e15) == pytest.approx(
        0.75 * R.roofline_seconds(all16, 1e15, 2e15), rel=1e-12)
    with pytest.raises(AssertionError):   # counts must cover every legal pair
        R.work(lens, d, hq, legal, 1)


def test_min_hbm_bytes():
    T, hq, hkv, d = 32768, 24, 8, 128
    fp16 = 2 * d * T
    # mixed: both Q formats and both K formats, V and O once
    assert R.min_hbm_bytes(T, hq, hkv, d, 0.77) == \
        hq * (fp16 + d * T) + hkv * (fp16 + d * T) + hkv * fp16 + hq * fp16
    assert R.min_hbm_bytes(T, hq, hkv, d, 0.0) == 2 * hq * fp16 + 2 * hkv * fp16
    assert R.min_hbm_bytes(T, hq, hkv, d, 1.0) == \
        hq * d * T + hkv * d * T + hkv * fp16 + hq * fp16

"""The seeded synthetic workloads match their stated recipes: legal-group
counts, forced FP16 groups and INT8 shares of the LLaMA-3.2-3B batch, the
INT8 KV cache and the 32K sweep, exact per-unit coverage, outlier channels,
and varlen lengths.  The generators draw numbers only; nothing here is
method arithmetic."""
import numpy as np

import oracle
import workloads as W
from prefill_blockwise_int8_b200 import roofline as R


def _counts(w):
    lens = W.seqlens(w)
    g = W.group_size(w, lens)
    route = W.route_bytes(w, lens)
    tm = W.tm_max(int(lens.max()), w.block_m)
    out = []
    for b in range(w.batch):
        n_legal = forced = 0
        for m in range(tm):
            ng, part = W.legal_groups(int(lens[b]), m, w.block_m, w.block_n, g)
            n_legal += ng
            forced += (len(part | {0}) if ng else 0)
        for hk in range(w.hkv):
            out.append((n_legal, forced, int(route[b, hk].sum())))
    return lens, g, route, out


def test_llama32_3b_batch_recipe():
    w = W.LLAMA32_3B_4K
    lens, g, route, counts = _counts(w)
    assert g == 1 and (lens == 4096).all()
    # per (sequence, KV head): 1056 legal groups, 95 forced FP16 (group 0 and
    # every group with a partially masked tile), 264 FP16 in all, 792 INT8
    assert set(counts) == {(1056, 95, 792)}
    words = oracle.pack_mask(route, W.cu_seqlens(lens), 4096, 128, 64, 1)
    fp16, int8 = R.pair_counts(lens, words, 128, 64, 1, w.hq, w.hkv)
    assert round(int8 / (fp16 + int8), 4) == 0.7732


def test_int8_kv_cache_recipe():
    w = W.INT8KV_16K
    _, g, _, counts = _counts(w)
    assert g == 2
    n_legal, forced, int8 = counts[0]
    assert (n_legal, forced) == (4160, 254)
    assert all(c == counts[0] for c in counts)
    assert int8 == n_legal - int(np.floor(0.25 * n_legal + 0.5))


def test_sweep_exact_coverage_per_kv_head():
    for pct in (0, 25, 50, 75, 100):
        w = W.WORKLOADS[f"sweep_L32768_h32x8_int8_{pct}"]
        _, g, _, counts = _counts(w)
        assert g == 4
        for n_legal, _, int8 in counts:
            assert n_legal == 8320
            assert int8 == int(np.floor(pct / 100 * n_legal + 0.5))


def test_outlier_channels_and_varlen_lengths():
    w = W.TINY.with_(seqlen=512, hq=2, hkv=1, d=64, outliers=True, seed=5)
    q, k, v = W.qkv(w)
    for x in (q, k):
        for h in range(x.shape[1]):
            rms = np.sqrt((x[:, h].astype(np.float64) ** 2).mean(axis=0))
            big = np.flatnonzero(rms > 8)
            assert len(big) == 4                      # four scaled channels
            assert (rms[big] > 15).all() and (rms[rms <= 8] < 1.5).all()
    assert np.sqrt((v.astype(np.float64) ** 2).mean()) < 1.5   # V unscaled
    lens = W.seqlens(W.VARLEN16)
    assert len(lens) == 16 and lens.min() >= 512 and lens.max() <= 8192
    assert W.group_size(W.VARLEN16, lens) == -(-(-(-int(lens.max()) // 64)) // 64)

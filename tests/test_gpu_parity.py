"""GPU parity: every CUDA step against the CPU oracle on the same seeded
inputs, through the C ABI.

* quantiser: Q8/K8 codes and fp32 scales byte-exact;
* packer: routing words bit-exact (junk in illegal groups cleared);
* attention: INT32 score tiles of INT8-routed groups bit-exact; fp16 output
  within max-abs 3e-3 and relative L2 2e-3 of the fp64 oracle; LSE within
  1e-3; at sizes that span several tiles with ragged tails, and at the full
  workload sizes on sampled rows.
"""
import json
import os

import numpy as np
import pytest

import oracle
import workloads as W
from _gpu_path import (LSE_ABS, compare, dev_tensor, run_gpu, run_oracle,
                       sample_rows)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def tm():
    import prefill_blockwise_int8_b200 as m
    return m


def small(L, *, hq=4, hkv=2, d=128, bm=128, bn=64, g=1, recipe="diag_first",
          cov=0.75, seed=5, outliers=True, qb=128, kb=128, kv="fp16"):
    lens = [L] if isinstance(L, int) else list(L)
    w = W.Workload(name="small", batch=len(lens), hq=hq, hkv=hkv, d=d,
                   block_m=bm, block_n=bn, group=g, seqlen=0, outliers=outliers,
                   mask_recipe=recipe, coverage=cov, seed=seed,
                   mask_seed=seed + 100, quant_block_q=qb, quant_block_k=kb,
                   coverage_unit="kv_head", kv_format=kv)
    lens = np.array(lens, dtype=np.int32)
    # the fixed-length generator stream, drawn for T = sum(lens) tokens
    q, k, v = W.qkv(w.with_(seqlen=1), lens)
    return dict(workload=w, seqlens=lens, cu_seqlens=W.cu_seqlens(lens),
                max_seqlen=int(max(lens.max(), 1)), group=g, q=q, k=k, v=v,
                route=W.route_bytes(w, lens))


# ----------------------------------------------------------------------------
# quantiser and packer
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
def test_quantize_bitexact_varlen(tm, d, block):
    lens = np.array([1, 127, 128, 129, 300, 0, 1000], dtype=np.int32)
    cu = W.cu_seqlens(lens)
    rng = np.random.default_rng(d + block)
    x = (rng.standard_normal((lens.sum(), 3, d)) * 4).astype(np.float16)
    x[cu[3]:cu[3] + 5, 2, 7] = 300.0   # an outlier
    x[cu[2]:cu[3], 1, :] = 0           # an all-zero block
    ref8, refs = oracle.quantize_blockwise(x, cu, int(lens.max()), block)
    g8, gs = tm.tilemix_quantize_blockwise(dev_tensor(x), dev_tensor(cu),
                                           int(lens.max()), block)
    torch.cuda.synchronize()
    assert np.array_equal(g8.cpu().numpy(), ref8)
    assert np.array_equal(gs.cpu().numpy().view(np.uint32), refs.view(np.uint32))


@pytest.mark.parametrize("qb,kb", [(128, 128), (64, 128), (128, 32)])
def test_quantize_qk_one_launch_bitexact(tm, qb, kb):
    """Q and K in one launch: byte-exact to the oracle for each tensor (and
    so to two single launches), with different heads and block sizes."""
    lens = np.array([1, 127, 128, 129, 300, 0, 1000], dtype=np.int32)
    cu = W.cu_seqlens(lens)
    rng = np.random.default_rng(qb + 3 * kb)
    q = (rng.standard_normal((lens.sum(), 6, 128)) * 4).astype(np.float16)
    k = (rng.standard_normal((lens.sum(), 2, 128)) * 4).astype(np.float16)
    k[cu[4]:cu[4] + 2, 1, 3] = -500.0  # an outlier
    q[cu[2]:cu[3], 4, :] = 0           # an all-zero block
    ms = int(lens.max())
    rq8, rqs = oracle.quantize_blockwise(q, cu, ms, qb)
    rk8, rks = oracle.quantize_blockwise(k, cu, ms, kb)
    q8, qs, k8, ks = tm.tilemix_quantize_blockwise_qk(
        dev_tensor(q), dev_tensor(k), dev_tensor(cu), ms, qb, kb)
    torch.cuda.synchronize()
    assert np.array_equal(q8.cpu().numpy(), rq8)
    assert np.array_equal(k8.cpu().numpy(), rk8)
    assert np.array_equal(qs.cpu().numpy().view(np.uint32), rqs.view(np.uint32))
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), rks.view(np.uint32))


def test_quantize_qk_full_size_equals_single_launches(tm):
    """At the LLaMA-3.2-3B prefill shape the one-launch codes and scales
    equal those of one launch per tensor (which the test above and the
    single-tensor tests pin to the oracle)."""
    w = W.LLAMA32_3B_4K
    inp = W.make(w)
    cu = dev_tensor(inp["cu_seqlens"])
    q, k = dev_tensor(inp["q"]), dev_tensor(inp["k"])
    ms = inp["max_seqlen"]
    q8a, qsa = tm.tilemix_quantize_blockwise(q, cu, ms, w.quant_block_q)
    k8a, ksa = tm.tilemix_quantize_blockwise(k, cu, ms, w.quant_block_k)
    q8b, qsb, k8b, ksb = tm.tilemix_quantize_blockwise_qk(
        q, k, cu, ms, w.quant_block_q, w.quant_block_k)
    torch.cuda.synchronize()
    assert torch.equal(q8a, q8b) and torch.equal(k8a, k8b)
    assert torch.equal(qsa.view(torch.int32), qsb.view(torch.int32))
    assert torch.equal(ksa.view(torch.int32), ksb.view(torch.int32))


def test_quantize_golden_ties(tm):
    here = os.path.dirname(__file__)
    cases = json.load(open(os.path.join(here, "golden",
                                        "quantize_examples.json")))["cases"]
    for c in cases:
        x = np.array(c["x"], dtype=np.float16)
        L, d = x.shape
        xp = np.zeros((L, 1, 8), dtype=np.float16)  # head_dim multiple of 8
        xp[:, 0, :d] = x
        g8, gs = tm.tilemix_quantize_blockwise(
            dev_tensor(xp), dev_tensor(np.array([0, L], np.int32)), L, L)
        torch.cuda.synchronize()
        assert gs.item() == np.float32(c["scale"]), c["name"]
        assert np.array_equal(g8.cpu().numpy()[:, 0, :d], np.array(c["q"])), c["name"]


def test_pack_bitexact_all_workloads(tm):
    for w in [W.TINY, W.LLAMA32_3B_4K, W.VARLEN16, W.INT8KV_16K,
              W.sweep_32k(75)]:
        lens = W.seqlens(w)
        cu = W.cu_seqlens(lens)
        g = W.group_size(w, lens)
        route = W.route_bytes(w, lens, junk_in_illegal=True)
        ref = oracle.pack_mask(route, cu, int(lens.max()), w.block_m,
                               w.block_n, g)
        got = tm.tilemix_pack_mask(dev_tensor(route), dev_tensor(cu),
                                   int(lens.max()), w.block_m, w.block_n, g)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy().view(np.uint64), ref), w.name


# ----------------------------------------------------------------------------
# attention, small sizes, every output element
# ----------------------------------------------------------------------------

def test_tiny_workload_full(tm):
    inp = W.make(W.TINY)
    got = run_gpu(inp, want_lse=True, want_dump=True)
    assert got["status"] == 0
    (ref, lse), kw = run_oracle(inp, want_lse=True)
    assert np.array_equal(got["q8"], kw["q8"])
    assert np.array_equal(got["mask"], kw["mask"])
    compare(got["out"], ref)
    assert np.abs(got["lse"] - lse).max() <= LSE_ABS
    dump = oracle.qk_dump(inp["cu_seqlens"], 256, kw["q8"], kw["k8"],
                          kw["mask"], hq=2, hkv=1, d=64, block_m=64,
                          block_n=64, group=1, fill=-1)
    assert np.array_equal(got["dump"], dump)
    assert (dump != -1).any()


CASES = {
    # name: (lens, kwargs of small())
    "d128_bn64_ragged": ([1000], dict()),
    "d128_bn128_two_seqs": ([700, 300], dict(bn=128, hkv=1, recipe="exact", cov=0.5)),
    "d64_bn128_g2": ([1100, 257], dict(d=64, bn=128, g=2, recipe="exact", cov=0.5)),
    "d64_bm64_dual": ([700], dict(d=64, bm=64, bn=64, recipe="bernoulli", cov=0.5)),
    "d128_bm64_dual": ([513, 64, 200], dict(bm=64, bn=64, recipe="bernoulli", cov=0.5)),
    "mha": ([333], dict(hq=3, hkv=3, recipe="exact", cov=0.5)),
    "gqa7": ([520], dict(hq=7, hkv=1, recipe="exact", cov=0.5)),
    "all_int8": ([600], dict(recipe="exact", cov=1.0)),
    "all_fp16_mask": ([600], dict(recipe="exact", cov=0.0)),
    "no_outliers": ([400, 1], dict(outliers=False, recipe="bernoulli", cov=0.5)),
    "qblock64_kblock64": ([450], dict(qb=64, kb=64, recipe="exact", cov=0.5)),
    "kblock256_bn128": ([700], dict(bn=128, kb=256, qb=256, recipe="exact", cov=0.5)),
    "seq_len_one": ([1], dict()),
    "tiny_seqs_and_empty": ([1, 2, 0, 3, 130], dict(recipe="bernoulli", cov=0.5)),
    "exactly_64_groups": ([4096], dict(hq=2, hkv=1, recipe="exact", cov=0.5)),
    "exactly_64_groups_g2": ([8192], dict(hq=1, hkv=1, bn=64, g=2, recipe="exact", cov=0.5)),
    # INT8 KV cache: K8 / V8 + block scales are the inputs
    "kv8_d128_bn128": ([700, 129], dict(bn=128, kv="int8", recipe="exact", cov=0.5)),
    "kv8_d128_bn64_kblock64": ([450], dict(kb=64, kv="int8", recipe="exact", cov=0.5)),
    "kv8_d64_mha": ([333], dict(d=64, hq=3, hkv=3, bn=128, kv="int8", recipe="exact", cov=0.5)),
    "kv8_dual": ([300], dict(bm=64, bn=64, kv="int8", recipe="bernoulli", cov=0.5)),
    "kv8_all_int8": ([400], dict(kv="int8", recipe="exact", cov=1.0)),
    "kv8_all_fp16": ([400], dict(kv="int8", recipe="exact", cov=0.0)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_small_cases(tm, name):
    lens, kw = CASES[name]
    inp = small(lens, **kw)
    got = run_gpu(inp, want_lse=True)
    assert got["status"] == 0
    work = sum(int(L) * int(L) for L in lens) * inp["workload"].hq
    # every row while the oracle stays within a few seconds, else a sample
    rows = None if work <= 8_000_000 else sample_rows(
        inp["seqlens"], inp["cu_seqlens"], per_seq=64,
        block=inp["workload"].block_m)
    (ref, lse), okw = run_oracle(inp, want_lse=True, rows=rows)
    assert np.array_equal(got["q8"], okw["q8"])
    assert np.array_equal(got["k8"], okw["k8"])
    compare(got["out"], ref, rows=rows)
    sel = slice(None) if rows is None else rows
    assert np.abs(got["lse"][:, sel] - lse[:, sel]).max() <= LSE_ABS


def test_fp16_only_flag(tm):
    inp = small([900], recipe="exact", cov=1.0)
    got = run_gpu(inp, fp16_only=True)
    ref, _ = run_oracle(inp, fp16_only=True)
    compare(got["out"], ref)
    # the flag ignores the mask: all-INT8 words must not change the result
    ref_int8, _ = run_oracle(inp)
    assert np.abs(ref_int8 - ref).max() > 1e-3


def test_explicit_head_map(tm):
    inp = small([640], hq=4, hkv=2, recipe="exact", cov=0.5)
    hm = [1, 0, 1, 0]
    got = run_gpu(inp, head_map=hm)
    ref, _ = run_oracle(inp, head_map=hm)
    compare(got["out"], ref)


def _mask_past_route_row(dump, lens, bm, bn, fill=-1):
    """Blank the keys past the last query of each routing row: every row of
    the routing row masks them, and the kernel may skip them in 64-key
    steps (the C ABI documents this)."""
    out = dump.copy()
    for b, L in enumerate(lens):
        for m in range(out.shape[2]):
            last = min((m + 1) * bm, int(L)) - 1
            for n in range(out.shape[3]):
                first_dead = max(0, last + 1 - n * bn)
                if first_dead < bn:
                    out[b, :, m, n, :, first_dead:] = fill
    return out


@pytest.mark.parametrize("bm,bn,g", [(128, 128, 1), (128, 64, 1), (64, 64, 2)])
def test_int8_tiles_bitexact_dump(tm, bm, bn, g):
    inp = small([700, 300], bm=bm, bn=bn, g=g, hkv=1, recipe="exact", cov=0.5)
    got = run_gpu(inp, want_dump=True)
    _, kw = run_oracle(inp, rows=np.array([0]))
    dump = oracle.qk_dump(inp["cu_seqlens"], 700, kw["q8"], kw["k8"],
                          kw["mask"], hq=4, hkv=1, d=128, block_m=bm,
                          block_n=bn, group=g, fill=-1)
    lens = inp["seqlens"]
    assert np.array_equal(_mask_past_route_row(got["dump"], lens, bm, bn),
                          _mask_past_route_row(dump, lens, bm, bn))
    assert (_mask_past_route_row(dump, lens, bm, bn) != -1).any()


@pytest.mark.parametrize("bm,bn,g", [(128, 64, 1), (64, 64, 2)])
def test_visited_tiles_are_exactly_the_legal_set(tm, bm, bn, g):
    # every group INT8 and junk bits set in every illegal group: the INT32
    # dump (filled with -1 first) is written for every legal tile and for
    # nothing above the diagonal or past a sequence end
    inp = small([700, 300, 129], bm=bm, bn=bn, g=g, hkv=1, recipe="exact",
                cov=1.0)
    w = inp["workload"]
    junk = W.route_bytes(w, inp["seqlens"], junk_in_illegal=True)
    got = run_gpu(inp, route=junk, want_dump=True)
    assert got["status"] == 0
    _, kw = run_oracle(inp, rows=np.array([0]))
    dump = oracle.qk_dump(inp["cu_seqlens"], 700, kw["q8"], kw["k8"],
                          kw["mask"], hq=4, hkv=1, d=128, block_m=bm,
                          block_n=bn, group=g, fill=-1)
    lens = inp["seqlens"]
    ref = _mask_past_route_row(dump, lens, bm, bn)
    assert np.array_equal(_mask_past_route_row(got["dump"], lens, bm, bn), ref)
    # nearly every entry of a legal tile holds a dot product (an exact -1 is
    # possible but rare), so the check above covers the whole legal set
    legal_pairs = 4 * sum(L * (L + 1) // 2 for L in lens.tolist())
    assert (ref != -1).sum() >= 0.99 * legal_pairs


def test_expired_wait_reports_timeout_and_the_context_survives(tm):
    # the test-only flag withholds every CTA's first V tile: the MMA
    # issuer's bounded wait expires (about 2 s), the kernel reports
    # TILEMIX_ERR_TIMEOUT and exits cleanly; later calls work as before
    inp = small([300, 129], recipe="exact", cov=0.5)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    got = run_gpu(inp, expire_wait=True)
    t1.record()
    torch.cuda.synchronize()
    assert got["status"] == 4            # TILEMIX_ERR_TIMEOUT
    assert t0.elapsed_time(t1) < 30e3    # bounded: no wait outlives its limit
    again = run_gpu(inp)
    assert again["status"] == 0
    ref, _ = run_oracle(inp)
    compare(again["out"], ref)


def test_garbage_bits_in_illegal_groups_change_nothing(tm):
    inp = small([777, 200], bm=128, bn=64, recipe="exact", cov=0.5)
    clean = run_gpu(inp)["out"]
    w = inp["workload"]
    junk = W.route_bytes(w, inp["seqlens"], junk_in_illegal=True)
    dirty = run_gpu(inp, route=junk)["out"]
    assert np.array_equal(clean, dirty)


def test_deterministic_and_stream(tm):
    inp = small([1000], recipe="exact", cov=0.5)
    a = run_gpu(inp)["out"]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_gpu(inp, stream=s)["out"]
    assert np.array_equal(a, b)


def test_coverage_changes_result_monotonically(tm):
    # more INT8 coverage moves the output further from the all-FP16 result
    inp = small([1024], recipe="exact", cov=0.0)
    base = run_gpu(inp, fp16_only=True)["out"]
    devs = []
    for cov in (0.0, 0.5, 1.0):
        inp2 = small([1024], recipe="exact", cov=cov)
        devs.append(np.abs(run_gpu(inp2)["out"] - base).mean())
    assert devs[0] == 0.0
    assert devs[0] < devs[1] < devs[2]


# ----------------------------------------------------------------------------
# device-detected errors
# ----------------------------------------------------------------------------

def test_bad_cu_seqlens_sets_status(tm):
    inp = small([300, 200])
    cu = np.array([0, 400, 500], np.int32)   # length 400 > max_seqlen 300
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = dev_tensor(inp["q"])
    k = dev_tensor(inp["k"])
    v = dev_tensor(inp["v"])
    tm.tilemix_attn_prefill(q, k, v, dev_tensor(cu), 300, fp16_only=True,
                            block_m=128, block_n=64, status=status)
    torch.cuda.synchronize()
    assert status.item() == 5


def test_head_map_out_of_range_sets_status(tm):
    inp = small([300])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tm.tilemix_attn_prefill(
        dev_tensor(inp["q"]), dev_tensor(inp["k"]), dev_tensor(inp["v"]),
        dev_tensor(inp["cu_seqlens"]), 300, fp16_only=True, block_m=128,
        block_n=64, head_map=dev_tensor(np.array([0, 1, 2, 0], np.int32)),
        status=status)
    torch.cuda.synchronize()
    assert status.item() == 5


def test_int8_kv_cache_fp16_only_flag(tm):
    inp = small([260], kv="int8", recipe="exact", cov=0.5)
    got = run_gpu(inp, fp16_only=True)
    assert got["status"] == 0
    ref, _ = run_oracle(inp, fp16_only=True)
    compare(got["out"], ref)


def test_int8_kv_cache_needs_its_buffers(tm):
    inp = small([128])
    with pytest.raises(tm.TilemixError):
        tm.tilemix_attn_prefill(dev_tensor(inp["q"]), None, None,
                                dev_tensor(inp["cu_seqlens"]), 128,
                                k8=dev_tensor(np.zeros((128, 2, 128), np.int8)),
                                kv_format=tm.KV_INT8)


# ----------------------------------------------------------------------------
# full workload sizes, sampled rows
# ----------------------------------------------------------------------------

def test_full_size_every_row_llama32_3b(tm):
    # the bench workload (8 x 4096 tokens, 24 / 8 heads, 75% INT8): every
    # output element against the oracle, and every LSE
    w = W.LLAMA32_3B_4K
    inp = W.make(w)
    got = run_gpu(inp, want_lse=True)
    assert got["status"] == 0
    (ref, lse), kw = run_oracle(inp, want_lse=True)
    assert np.array_equal(got["q8"], kw["q8"])
    assert np.array_equal(got["k8"], kw["k8"])
    assert np.array_equal(got["sq"].view(np.uint32), kw["q_scale"].view(np.uint32))
    assert np.array_equal(got["sk"].view(np.uint32), kw["k_scale"].view(np.uint32))
    assert np.array_equal(got["mask"], kw["mask"])
    compare(got["out"], ref)
    assert np.abs(got["lse"] - lse).max() <= LSE_ABS


@pytest.mark.parametrize("wname", [
    W.VARLEN16.name, W.INT8KV_16K.name, W.sweep_32k(0).name,
    W.sweep_32k(25).name, W.sweep_32k(50).name, W.sweep_32k(75).name,
    W.sweep_32k(100).name])
def test_full_size_sampled_rows(tm, wname):
    # 512 random query rows per sequence (all heads, whole causal rows) plus
    # the first and last rows of the first, middle and last query tiles
    w = W.WORKLOADS[wname]
    inp = W.make(w)
    got = run_gpu(inp, want_lse=True)
    assert got["status"] == 0
    rows = sample_rows(inp["seqlens"], inp["cu_seqlens"], per_seq=512,
                       block=w.block_m)
    (ref, lse), kw = run_oracle(inp, rows=rows, want_lse=True)
    assert np.array_equal(got["q8"], kw["q8"])
    assert np.array_equal(got["sq"].view(np.uint32), kw["q_scale"].view(np.uint32))
    assert np.array_equal(got["mask"], kw["mask"])
    compare(got["out"], ref, rows=rows)
    assert np.abs(got["lse"][:, rows] - lse[:, rows]).max() <= LSE_ABS


# ----------------------------------------------------------------------------
# routing templates: byte-exact against the oracle, then through attention
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", sorted(oracle.LAYOUTS))
def test_route_template_bitexact(tm, layout):
    shapes = [([700, 300, 1, 0, 1500], 2, 128, 64, 1),
              ([4096] * 8, 8, 128, 64, 1),
              ([8192], 2, 128, 128, 1),
              ([20000], 1, 64, 64, 5)]
    for lens, hkv, bm, bn, g in shapes:
        lens = np.array(lens, np.int32)
        cu = W.cu_seqlens(lens)
        ms = int(max(lens.max(), 1))
        for permille in (0, 250, 500, 750, 1000):
            got = tm.tilemix_route_template(layout, permille, dev_tensor(cu),
                                            ms, hkv, bm, bn, g, seed=77)
            torch.cuda.synchronize()
            ref = oracle.route_template(layout, permille, 77, cu, ms, hkv, bm,
                                        bn, g)
            assert np.array_equal(got.cpu().numpy(), ref), (lens, permille)


def test_route_template_hash_known_answers(tm):
    # the device's splitmix64 against the generator's published outputs for
    # seed 1234567 (tests/golden): with seed = 1234567 - 256 gamma, row 4 of
    # 64 x 64 tiles hashes exactly the published states 1..5, and row-random
    # keeps the groups with the largest high halves FP16
    here = os.path.dirname(__file__)
    g = json.load(open(os.path.join(here, "golden",
                                    "splitmix64_known_answers.json")))
    gamma = int(g["gamma"], 16)
    seed = (g["seed"] - 256 * gamma) % (1 << 64)
    hi = [int(v) >> 32 for v in g["outputs"]]
    by_rank = sorted(range(5), key=lambda j: (-hi[j], j))
    cu = dev_tensor(np.array([0, 320], np.int32))
    for permille in (0, 200, 400, 600, 800, 1000):
        k_int8 = (permille * 5 + 500) // 1000
        want = np.ones(5, np.uint8)
        want[by_rank[:5 - k_int8]] = 0
        got = tm.tilemix_route_template("row_random", permille, cu, 320, 1,
                                        64, 64, 1, seed=seed)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy()[0, 0, 4, :5], want), permille


def test_route_template_through_attention(tm):
    inp = small([900, 333], bn=64)
    w = inp["workload"]
    route = tm.tilemix_route_template(
        "bigbird", 750, dev_tensor(inp["cu_seqlens"]), inp["max_seqlen"],
        w.hkv, w.block_m, w.block_n, inp["group"], seed=5).cpu().numpy()
    got = run_gpu(inp, route=route)
    assert got["status"] == 0
    ref, _ = run_oracle(inp, route=route)
    compare(got["out"], ref)


# ----------------------------------------------------------------------------
# adaptive routing: route bytes and routing words byte-exact against the
# oracle's exact-integer statistic, then through attention
# ----------------------------------------------------------------------------

ADAPTIVE_CASES = {
    # lens, hq, hkv, d, block_m, block_n, g, head_map, value recipe
    "ragged_d128_bn64": ([700, 300, 1, 0, 1500], 4, 2, 128, 128, 64, 1, None, "outliers"),
    "d64_bm64_g2": ([1000, 77], 6, 2, 64, 64, 64, 2, None, "normal"),
    "d96_head_map": ([513], 6, 2, 96, 128, 128, 1, [1, 0, 0, 1, 1, 0], "normal"),
    "ties_small_ints": ([640, 130], 2, 1, 32, 64, 64, 1, None, "ternary"),
    "g5_long": ([20000], 2, 1, 64, 128, 64, 5, None, "normal"),
    # a KV head no query head maps to: all statistics 0, ties everywhere
    "head_map_idle_kv_head": ([300, 129], 2, 3, 64, 64, 64, 1, [2, 0], "normal"),
}


def adaptive_inputs(lens, hq, hkv, d, recipe, seed=21):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    if recipe == "ternary":   # many exactly equal statistics: tie-breaking
        q = rng.integers(0, 2, (T, hq, d)).astype(np.float16)
        k = rng.integers(-1, 2, (T, hkv, d)).astype(np.float16)
        k[:, :, 1:] = 0
    else:
        q = rng.standard_normal((T, hq, d)).astype(np.float16)
        k = rng.standard_normal((T, hkv, d)).astype(np.float16)
        if recipe == "outliers":
            q[:, :, 5] *= 40
            k[:, :, 5] *= 40
    return q, k


@pytest.mark.parametrize("name", sorted(ADAPTIVE_CASES))
def test_route_adaptive_bitexact(tm, name):
    lens, hq, hkv, d, bm, bn, g, hmap, recipe = ADAPTIVE_CASES[name]
    lens = np.array(lens, np.int32)
    cu = W.cu_seqlens(lens)
    ms = int(max(lens.max(), 1))
    q, k = adaptive_inputs(lens, hq, hkv, d, recipe)
    qd, kd, cud = dev_tensor(q), dev_tensor(k), dev_tensor(cu)
    hm = None if hmap is None else dev_tensor(np.array(hmap, np.int32))
    tmr = -(-ms // bm)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for permille in (0, 250, 750, 1000):
        mask = torch.full((len(lens), hkv, tmr), -1, dtype=torch.int64,
                          device="cuda")
        route, mask = tm.tilemix_route_adaptive(
            qd, kd, cud, ms, bm, bn, g, permille, head_map=hm, mask=mask,
            status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ref = oracle.route_adaptive(q, k, cu, ms, bm, bn, g, permille,
                                    head_map=hmap)
        assert np.array_equal(route.cpu().numpy(), ref), permille
        words = oracle.pack_mask(ref, cu, ms, bm, bn, g)
        assert np.array_equal(mask.cpu().numpy().view(np.uint64), words)


def test_route_adaptive_full_size_sampled(tm):
    # LLaMA-3.2-3B prefill shape: 8 x 4096 tokens, 24 / 8 heads, d 128,
    # 128 x 64 tiles; the oracle checks two whole sequences
    lens = np.full(8, 4096, np.int32)
    cu = W.cu_seqlens(lens)
    q, k = adaptive_inputs(lens, 24, 8, 128, "outliers", seed=4)
    route = tm.tilemix_route_adaptive(dev_tensor(q), dev_tensor(k),
                                      dev_tensor(cu), 4096, 128, 64, 1, 750)
    torch.cuda.synchronize()
    got = route.cpu().numpy()
    for b in (0, 7):
        sl = slice(int(cu[b]), int(cu[b + 1]))
        ref = oracle.route_adaptive(q[sl], k[sl], np.array([0, 4096], np.int32),
                                    4096, 128, 64, 1, 750)
        assert np.array_equal(got[b], ref[0]), b


def test_route_adaptive_bad_seqlens_reported(tm):
    q, k = adaptive_inputs([100], 2, 1, 64, "normal")
    cu = np.array([0, 100], np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # a sequence longer than max_seqlen: reported, its rows route nothing
    route = tm.tilemix_route_adaptive(dev_tensor(q), dev_tensor(k),
                                      dev_tensor(cu), 64, 64, 64, 1, 500,
                                      status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5     # TILEMIX_ERR_BAD_SEQLENS
    assert not route.cpu().numpy().any()


def test_route_adaptive_bad_head_map_reported(tm):
    # a head_map entry outside [0, hkv): reported, and no row is ranked on
    # the sums that left that head out (every byte and word written 0)
    q, k = adaptive_inputs([300, 129], 4, 2, 64, "normal")
    cu = np.array([0, 300, 429], np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mask = torch.full((2, 2, 5), -1, dtype=torch.int64, device="cuda")
    route = torch.full((2, 2, 5, 64), 9, dtype=torch.uint8, device="cuda")
    tm.tilemix_route_adaptive(dev_tensor(q), dev_tensor(k), dev_tensor(cu),
                              300, 64, 64, 1, 500,
                              head_map=dev_tensor(np.array([0, 1, 2, 0], np.int32)),
                              route=route, mask=mask, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5     # TILEMIX_ERR_BAD_SEQLENS
    assert not route.cpu().numpy().any()
    assert not mask.cpu().numpy().any()


def test_route_adaptive_through_attention(tm):
    inp = small([900, 333], bn=64)
    w = inp["workload"]
    route = tm.tilemix_route_adaptive(
        dev_tensor(inp["q"]), dev_tensor(inp["k"]), dev_tensor(inp["cu_seqlens"]),
        inp["max_seqlen"], w.block_m, w.block_n, inp["group"], 750).cpu().numpy()
    ref_route = oracle.route_adaptive(inp["q"], inp["k"], inp["cu_seqlens"],
                                      inp["max_seqlen"], w.block_m, w.block_n,
                                      inp["group"], 750)
    assert np.array_equal(route, ref_route)
    got = run_gpu(inp, route=route)
    assert got["status"] == 0
    ref, _ = run_oracle(inp, route=route)
    compare(got["out"], ref)


# ----------------------------------------------------------------------------
# on-chip quantisation: identical to quantise-once, element for element
# ----------------------------------------------------------------------------

ON_CHIP_CASES = {
    "d128_bn64_two_seqs": ([700, 300, 1], dict()),
    "d128_bn128_g2": ([1500], dict(bn=128, g=2, recipe="exact", cov=0.5)),
    "d64_bm64_dual": ([400], dict(d=64, bm=64, bn=64, recipe="bernoulli", cov=0.5)),
    "gqa7_all_int8": ([520], dict(hq=7, hkv=1, recipe="exact", cov=1.0)),
}


@pytest.mark.parametrize("name", sorted(ON_CHIP_CASES))
def test_quant_on_chip_equals_quantise_once(tm, name):
    # the INT8 tiles made on chip hold exactly the quantise-once integers
    # (INT32 dumps identical); both modes' outputs and LSE are within the
    # tolerance of the oracle (the two modes run different kernels, so their
    # float rounding may differ)
    lens, kw = ON_CHIP_CASES[name]
    inp = small(lens, **kw)
    once = run_gpu(inp, want_lse=True, want_dump=True)
    chip = run_gpu(inp, want_lse=True, want_dump=True, on_chip=True)
    assert once["status"] == 0 and chip["status"] == 0
    assert np.array_equal(chip["dump"], once["dump"])
    (ref, lse), _ = run_oracle(inp, want_lse=True)
    compare(chip["out"], ref)
    compare(once["out"], ref)
    assert np.abs(chip["lse"] - lse).max() <= LSE_ABS
    assert np.abs(once["lse"] - lse).max() <= LSE_ABS


def test_quant_on_chip_full_size_sampled_rows(tm):
    w = W.LLAMA32_3B_4K
    inp = W.make(w)
    got = run_gpu(inp, on_chip=True)
    assert got["status"] == 0
    rows = sample_rows(inp["seqlens"], inp["cu_seqlens"], per_seq=16,
                       block=w.block_m)
    ref, _ = run_oracle(inp, rows=rows)
    compare(got["out"], ref, rows=rows)


def test_quant_on_chip_host_checks(tm):
    inp = small([256])
    q = dev_tensor(inp["q"])
    with pytest.raises(tm.TilemixError):  # 64-token K blocks are not tiles
        tm.tilemix_attn_prefill(q, dev_tensor(inp["k"]), dev_tensor(inp["v"]),
                                dev_tensor(inp["cu_seqlens"]), 256,
                                mask=torch.zeros((1, 2, 2), dtype=torch.int64,
                                                 device="cuda"),
                                block_m=128, block_n=64, quant_block_k=64,
                                quant_on_chip=True)

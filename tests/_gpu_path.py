"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on generator inputs, run the oracle on the same inputs, compare."""
import numpy as np

import oracle
import workloads as W

# Output tolerances (fp16 output of an fp32-accumulated kernel against the
# fp64 oracle): max |gpu - ref| <= 3e-3 and ||gpu - ref||_2 / ||ref||_2 <=
# 2e-3.  Error budget: half an fp16 ulp of the output (<= 9.8e-4 for
# |o| < 4), fp16 rounding of P (relative 2^-11 per weight, <= 4.9e-4 * |v|),
# exp2 (ex2.approx 2 ulp; the FMA-pipe cubic 7.5e-5 relative), fp32 score
# arithmetic (~1e-6 relative); with the INT8 KV cache, V = v8 * sv rounded to
# fp16 on chip (relative 2^-10 per value).
MAX_ABS = 3e-3
REL_L2 = 2e-3
LSE_ABS = 1e-3


def torch_mod():
    import torch
    return torch


def dev_tensor(a):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_gpu(inp, *, fp16_only=False, want_lse=False, want_dump=False,
            head_map=None, stream=None, route=None, on_chip=False,
            expire_wait=False):
    """Quantise Q and K, pack the routing words and run attention on the GPU.
    Returns numpy copies of everything the path produced."""
    torch = torch_mod()
    import prefill_blockwise_int8_b200 as tm
    w = inp["workload"]
    ms = inp["max_seqlen"]
    g = inp["group"]
    cu = dev_tensor(inp["cu_seqlens"])
    q, k, v = dev_tensor(inp["q"]), dev_tensor(inp["k"]), dev_tensor(inp["v"])
    t, hq, d = q.shape
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q8, sq = tm.tilemix_quantize_blockwise(q, cu, ms, w.quant_block_q,
                                           status=status, stream=stream)
    k8, sk = tm.tilemix_quantize_blockwise(k, cu, ms, w.quant_block_k,
                                           status=status, stream=stream)
    kv8 = w.kv_format == "int8"
    v8 = sv = None
    if kv8:  # the INT8 KV cache: K and V arrive quantised, fp16 K/V unused
        v8, sv = tm.tilemix_quantize_blockwise(v, cu, ms, w.quant_block_k,
                                               status=status, stream=stream)
        k = v = None
    r = dev_tensor(inp["route"] if route is None else route)
    mask = tm.tilemix_pack_mask(r, cu, ms, w.block_m, w.block_n, g,
                                status=status, stream=stream)
    lse = torch.zeros((hq, t), dtype=torch.float32, device="cuda") \
        if want_lse else None
    dump = None
    if want_dump:
        tmr = -(-ms // w.block_m)
        tn = -(-ms // w.block_n)
        dump = torch.full((len(inp["seqlens"]), hq, tmr, tn, w.block_m,
                           w.block_n), -1, dtype=torch.int32, device="cuda")
    hm = dev_tensor(np.asarray(head_map, np.int32)) if head_map is not None \
        else None
    out = tm.tilemix_attn_prefill(
        q, k, v, cu, ms, q8=None if on_chip else q8,
        q_scale=None if on_chip else sq, k8=None if on_chip else k8,
        k_scale=None if on_chip else sk, v8=v8, quant_on_chip=on_chip,
        v_scale=sv, mask=mask, block_m=w.block_m, block_n=w.block_n, group=g,
        quant_block_q=w.quant_block_q, quant_block_k=w.quant_block_k,
        head_map=hm, fp16_only=fp16_only, lse=lse, qk_dump=dump,
        kv_format=tm.KV_INT8 if kv8 else tm.KV_FP16, status=status,
        test_expire_wait=expire_wait, stream=stream)
    torch.cuda.synchronize()
    res = dict(status=int(status.item()),
               out=out.float().cpu().numpy().astype(np.float64),
               q8=q8.cpu().numpy(), sq=sq.cpu().numpy(), k8=k8.cpu().numpy(),
               sk=sk.cpu().numpy(),
               mask=mask.cpu().numpy().view(np.uint64))
    if want_lse:
        res["lse"] = lse.cpu().numpy().astype(np.float64)
    if want_dump:
        res["dump"] = dump.cpu().numpy()
    return res


def run_oracle(inp, *, fp16_only=False, rows=None, want_lse=False,
               head_map=None, route=None):
    if route is not None:
        inp = dict(inp, route=route)
    args, kw = oracle.prepare(inp, fp16_only=fp16_only)
    if head_map is not None:
        kw["head_map"] = np.asarray(head_map, np.int32)
    res = oracle.attn_prefill(*args, rows=rows, want_lse=want_lse, **kw)
    return res, kw


def compare(got, ref, rows=None, max_abs=MAX_ABS, rel_l2=REL_L2):
    if rows is not None:
        got, ref = got[rows], ref[rows]
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert np.isfinite(got).all(), "non-finite GPU output"
    assert mx <= max_abs, f"max abs err {mx:.3e} > {max_abs}"
    assert rl2 <= rel_l2, f"rel L2 err {rl2:.3e} > {rel_l2}"
    return mx, rl2


def sample_rows(lens, cu, per_seq=48, seed=0, block=128):
    """Token indices to check at full size: the first and last rows of the
    first, middle and last query tiles of each sequence plus random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b, L in enumerate(lens):
        L = int(L)
        if L == 0:
            continue
        s = int(cu[b])
        tiles = -(-L // block)
        for tt in {0, tiles // 2, tiles - 1}:
            for r in (tt * block, tt * block + 1, min(L, (tt + 1) * block) - 1):
                if 0 <= r < L:
                    rows.add(s + r)
        rows.add(s + L - 1)
        for r in rng.integers(0, L, size=per_seq):
            rows.add(s + int(r))
    return np.array(sorted(rows), dtype=np.int64)

"""CPU oracle for tile-routed FP16/INT8 causal prefill attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The product path (``prefill_blockwise_int8_b200``) never
imports it and shares no code with it.

The attention, quantiser and packer arithmetic lives in
``tilemix_oracle.c`` (plain C, fp64, exact integer dots); this module
compiles it with gcc and marshals numpy arrays.  Each C function cites the
passage of the TileMix pages it restates.  The routing templates and the
adaptive routing statistic are plain Python below, in exact integers.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, dense textbook attention in fp64, library attention, brute
force on tiny inputs, hand-worked quantiser examples in ``tests/golden``).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from pathlib import Path

import numpy as np

_DIR = Path(__file__).resolve().parent
_SRC = _DIR / "tilemix_oracle.c"
_LIB_PATH = _DIR / "libtilemix_oracle.so"
_lib = None


def compile_library(src: Path, out: Path) -> Path:
    """gcc a C source of the oracle into a shared library (no fast-math, no
    FMA contraction)."""
    tmp = Path(out).with_suffix(f".{os.getpid()}.tmp")
    subprocess.check_call([
        "gcc", "-O3", "-std=c11", "-fPIC", "-shared", "-pthread",
        "-ffp-contract=off", "-fno-fast-math", "-D_GNU_SOURCE",
        str(src), "-o", str(tmp), "-lm"])
    os.replace(tmp, out)
    return Path(out)


def build(force: bool = False) -> Path:
    """Compile the oracle (if its library is missing or older)."""
    if force or not _LIB_PATH.exists() or \
            _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        compile_library(_SRC, _LIB_PATH)
    return _LIB_PATH


class _AttnArgs(C.Structure):
    _fields_ = [
        ("batch", C.c_int), ("max_seqlen", C.c_int), ("hq", C.c_int),
        ("hkv", C.c_int), ("d", C.c_int),
        ("cu_seqlens", C.c_void_p), ("head_map", C.c_void_p),
        ("q", C.c_void_p), ("q8", C.c_void_p), ("q_scale", C.c_void_p),
        ("kv_int8", C.c_int),
        ("k", C.c_void_p), ("k8", C.c_void_p), ("k_scale", C.c_void_p),
        ("v", C.c_void_p), ("v8", C.c_void_p), ("v_scale", C.c_void_p),
        ("mask", C.c_void_p), ("block_m", C.c_int), ("block_n", C.c_int),
        ("group", C.c_int), ("fp16_only", C.c_int),
        ("quant_block_q", C.c_int), ("quant_block_k", C.c_int),
        ("softmax_scale", C.c_double),
        ("out", C.c_void_p), ("lse", C.c_void_p),
        ("rows", C.c_void_p), ("n_rows", C.c_int64),
        ("nthreads", C.c_int), ("pair_counts", C.c_void_p),
    ]


def _load():
    global _lib
    if _lib is None:
        # TILEMIX_ORACLE_LIB: a library built from a copy of the source (the
        # mutation test plants mistakes in such copies); default: build().
        override = os.environ.get("TILEMIX_ORACLE_LIB")
        lib = C.CDLL(override if override else str(build()))
        lib.oracle_quantize_blockwise.restype = C.c_int
        lib.oracle_quantize_blockwise.argtypes = [
            C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int,
            C.c_int, C.c_void_p, C.c_void_p]
        lib.oracle_pack_mask.restype = C.c_int
        lib.oracle_pack_mask.argtypes = [
            C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int,
            C.c_int, C.c_int, C.c_void_p]
        lib.oracle_attn.restype = C.c_int
        lib.oracle_attn.argtypes = [C.POINTER(_AttnArgs)]
        lib.oracle_qk_dump.restype = C.c_int
        lib.oracle_qk_dump.argtypes = [C.POINTER(_AttnArgs), C.c_void_p]
        lib.oracle_half_to_double.restype = C.c_double
        lib.oracle_half_to_double.argtypes = [C.c_uint16]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def half_to_double(bits: int) -> float:
    return _load().oracle_half_to_double(bits)


def quantize_blockwise(x: np.ndarray, cu_seqlens: np.ndarray, max_seqlen: int,
                       block: int = 128):
    """x: float16 [T, H, d] -> (int8 [T, H, d], float32 [H, B, nblk])."""
    x = _c(x, np.float16)
    cu = _c(cu_seqlens, np.int32)
    t, heads, d = x.shape
    batch = len(cu) - 1
    nblk = -(-max_seqlen // block)
    x8 = np.zeros((t, heads, d), dtype=np.int8)
    scale = np.zeros((heads, batch, nblk), dtype=np.float32)
    rc = _load().oracle_quantize_blockwise(
        _ptr(x), _ptr(cu), batch, max_seqlen, heads, d, block, _ptr(x8),
        _ptr(scale))
    if rc:
        raise OracleError(f"oracle_quantize_blockwise failed ({rc})")
    return x8, scale


def pack_mask(route: np.ndarray, cu_seqlens: np.ndarray, max_seqlen: int,
              block_m: int, block_n: int, group: int) -> np.ndarray:
    """route: uint8 [B, Hkv, Tm_max, 64] -> uint64 [B, Hkv, Tm_max]."""
    route = _c(route, np.uint8)
    cu = _c(cu_seqlens, np.int32)
    batch, hkv, tm, ng = route.shape
    if ng != 64 or tm != -(-max_seqlen // block_m):
        raise OracleError("route must be [batch, hkv, ceil(max_seqlen/BM), 64]")
    mask = np.zeros((batch, hkv, tm), dtype=np.uint64)
    rc = _load().oracle_pack_mask(_ptr(route), _ptr(cu), batch, max_seqlen,
                                  hkv, block_m, block_n, group, _ptr(mask))
    if rc:
        raise OracleError(f"oracle_pack_mask failed ({rc})")
    return mask


def _args(cu_seqlens, max_seqlen, q, k=None, v=None, *, q8=None, q_scale=None,
          k8=None, k_scale=None, v8=None, v_scale=None, mask=None,
          block_m=128, block_n=128, group=1, head_map=None, fp16_only=False,
          quant_block_q=128, quant_block_k=128, softmax_scale=None,
          kv_int8=False, hkv=None):
    keep = []

    def hold(a, dt):
        a = _c(a, dt)
        keep.append(a)
        return a

    cu = hold(cu_seqlens, np.int32)
    q = hold(q, np.float16)
    t, hq, d = q.shape
    if hkv is None:
        hkv = (k8 if kv_int8 else k).shape[1]
    a = _AttnArgs()
    a.batch, a.max_seqlen, a.hq, a.hkv, a.d = len(cu) - 1, max_seqlen, hq, hkv, d
    a.cu_seqlens = _ptr(cu)
    a.head_map = _ptr(hold(head_map, np.int32)) if head_map is not None else None
    a.q = _ptr(q)
    a.q8 = _ptr(hold(q8, np.int8)) if q8 is not None else None
    a.q_scale = _ptr(hold(q_scale, np.float32)) if q_scale is not None else None
    a.kv_int8 = int(kv_int8)
    a.k = _ptr(hold(k, np.float16)) if k is not None else None
    a.k8 = _ptr(hold(k8, np.int8)) if k8 is not None else None
    a.k_scale = _ptr(hold(k_scale, np.float32)) if k_scale is not None else None
    a.v = _ptr(hold(v, np.float16)) if v is not None else None
    a.v8 = _ptr(hold(v8, np.int8)) if v8 is not None else None
    a.v_scale = _ptr(hold(v_scale, np.float32)) if v_scale is not None else None
    a.mask = _ptr(hold(mask, np.uint64)) if mask is not None else None
    a.block_m, a.block_n, a.group = block_m, block_n, group
    a.fp16_only = int(fp16_only)
    a.quant_block_q, a.quant_block_k = quant_block_q, quant_block_k
    a.softmax_scale = (1.0 / np.sqrt(d)) if not softmax_scale else softmax_scale
    return a, keep, (t, hq, d)


def attn_prefill(cu_seqlens, max_seqlen, q, k=None, v=None, *, rows=None,
                 nthreads=0, want_lse=False, want_pair_counts=False, **kw):
    """Causal tile-routed attention in fp64.

    Returns out float64 [T, hq, d] (rows not listed in `rows` stay 0), and
    optionally lse float64 [hq, T] and pair counts (fp16, int8)."""
    a, keep, (t, hq, d) = _args(cu_seqlens, max_seqlen, q, k, v, **kw)
    out = np.zeros((t, hq, d), dtype=np.float64)
    lse = np.zeros((hq, t), dtype=np.float64) if want_lse else None
    counts = np.zeros(2, dtype=np.int64) if want_pair_counts else None
    a.out, a.lse = _ptr(out), _ptr(lse)
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        keep.append(rows)
        a.rows, a.n_rows = _ptr(rows), len(rows)
    a.nthreads = nthreads
    a.pair_counts = _ptr(counts)
    rc = _load().oracle_attn(C.byref(a))
    if rc:
        raise OracleError(f"oracle_attn failed ({rc})")
    res = [out]
    if want_lse:
        res.append(lse)
    if want_pair_counts:
        res.append(counts)
    return res[0] if len(res) == 1 else tuple(res)


def qk_dump(cu_seqlens, max_seqlen, q8, k8, mask, *, hq, hkv, d, block_m,
            block_n, group, head_map=None, fill=0):
    """INT32 accumulators of every INT8-routed legal tile,
    int32 [B, hq, Tm_max, Tn_max, BM, BN]; untouched entries hold `fill`."""
    t = q8.shape[0]
    dummy_q = np.zeros((t, hq, d), dtype=np.float16)
    a, keep, _ = _args(cu_seqlens, max_seqlen, dummy_q, None, None, q8=q8,
                       k8=k8, k_scale=np.ones(1, np.float32),
                       q_scale=np.ones(1, np.float32), mask=mask,
                       block_m=block_m, block_n=block_n, group=group,
                       head_map=head_map, hkv=hkv)
    tm = -(-max_seqlen // block_m)
    tn = -(-max_seqlen // block_n)
    dump = np.full((len(cu_seqlens) - 1, hq, tm, tn, block_m, block_n), fill,
                   dtype=np.int32)
    rc = _load().oracle_qk_dump(C.byref(a), _ptr(dump))
    if rc:
        raise OracleError(f"oracle_qk_dump failed ({rc})")
    return dump


def prepare(inputs: dict, fp16_only: bool = False):
    """Run the oracle's own quantiser and packer on generator output and
    return the keyword arguments of `attn_prefill` for that workload."""
    w = inputs["workload"]
    cu, ms = inputs["cu_seqlens"], inputs["max_seqlen"]
    q8, sq = quantize_blockwise(inputs["q"], cu, ms, w.quant_block_q)
    k8, sk = quantize_blockwise(inputs["k"], cu, ms, w.quant_block_k)
    mask = pack_mask(inputs["route"], cu, ms, w.block_m, w.block_n,
                     inputs["group"])
    kw = dict(q8=q8, q_scale=sq, k8=k8, k_scale=sk, mask=mask,
              block_m=w.block_m, block_n=w.block_n, group=inputs["group"],
              quant_block_q=w.quant_block_q, quant_block_k=w.quant_block_k,
              fp16_only=fp16_only)
    if w.kv_format == "int8":
        v8, sv = quantize_blockwise(inputs["v"], cu, ms, w.quant_block_k)
        kw.update(kv_int8=True, v8=v8, v_scale=sv)
        args = (cu, ms, inputs["q"], None, None)
    else:
        args = (cu, ms, inputs["q"], inputs["k"], inputs["v"])
    return args, kw


# ----------------------------------------------------------------------------
# Static routing templates (paperlayer summary, appendix B Precision Layouts:
# All FP16 / All INT8 references, Band, Global, Row-Random, Aligned Sparse,
# BigBird and SpTrans at an INT8 coverage of the legal tile groups).  The
# pages give the names only; this restates the reading documented with the
# C declaration of tilemix_route_template: per query-tile row, the
# G - round(c G) groups with the highest (priority, hash) key stay FP16.
# ----------------------------------------------------------------------------

LAYOUTS = {"all_fp16": 0, "all_int8": 1, "band": 2, "global": 3,
           "row_random": 4, "aligned": 5, "bigbird": 6, "sptrans": 7}
_M64 = (1 << 64) - 1


def splitmix64(z: int) -> int:
    """The output function of the splitmix64 generator (Steele, Lea and
    Flood, OOPSLA 2014): two xor-shift-multiply rounds and a final xor."""
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _priority(layout: int, j: int, d: int) -> int:
    if layout == LAYOUTS["band"]:
        return 63 - d
    if layout == LAYOUTS["global"]:
        return 63 - j
    if layout == LAYOUTS["aligned"]:
        return 1 if j % 4 == 0 else 0
    if layout == LAYOUTS["bigbird"]:
        return 1 if (j == 0 or d <= 1) else 0
    if layout == LAYOUTS["sptrans"]:
        return 2 if d <= 1 else (1 if j % 4 == 3 else 0)
    return 0


def route_template(layout, int8_permille: int, seed: int, cu_seqlens,
                   max_seqlen: int, hkv: int, block_m: int, block_n: int,
                   group: int) -> np.ndarray:
    """uint8 [batch, hkv, ceil(max_seqlen / block_m), 64], 1 = INT8."""
    code = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(cu)
    tm = -(-max_seqlen // block_m)
    out = np.zeros((len(lens), hkv, tm, 64), dtype=np.uint8)
    for b, L in enumerate(lens.tolist()):
        for m in range(tm):
            if m * block_m >= L:
                continue
            G = ((min((m + 1) * block_m, L) - 1) // block_n) // group + 1
            k_int8 = (int8_permille * G + 500) // 1000
            if code == LAYOUTS["all_fp16"]:
                k_int8 = 0
            if code == LAYOUTS["all_int8"]:
                k_int8 = G
            k_fp16 = G - k_int8
            for hk in range(hkv):
                keys = []
                for j in range(G):
                    c = ((b * hkv + hk) * tm + m) * 64 + j
                    h = splitmix64(seed + (c + 1) * 0x9E3779B97F4A7C15) >> 32
                    keys.append((_priority(code, j, G - 1 - j) << 32) | h)
                # FP16: the k_fp16 largest keys, ties to the smaller index
                order = sorted(range(G), key=lambda i: (-keys[i], i))
                for j in order[k_fp16:]:
                    out[b, hk, m, j] = 1
    return out


def fp16_fixed(x) -> np.ndarray:
    """Exact integer value of fp16 numbers times 2^24 (int64): every finite
    fp16 value is an integer multiple of 2^-24 below 2^16 in magnitude."""
    return (np.asarray(x, dtype=np.float16).astype(np.float64)
            * 2.0 ** 24).astype(np.int64)


def route_adaptive_statistic(q, k, cu_seqlens, max_seqlen: int, block_m: int,
                             block_n: int, group: int, head_map=None):
    """Adaptive-routing statistic I[b][hk][m] = list over the row's G legal
    groups j of (sum of the row's queries over hk's heads) . (sum of group j's
    keys), in exact integers (fp16 values scaled by 2^24).

    Reading of the TileMix pages' remark that the kernel interface takes
    adaptive routing policies (paperlayer summary, Limitations) and of the
    heavy-hitter analysis (appendix G.5): the statistic equals 2^48 times the
    sum of all raw logits between the row's queries and the group's keys."""
    q = np.asarray(q, dtype=np.float16)
    k = np.asarray(k, dtype=np.float16)
    _, hq, _ = q.shape
    hkv = k.shape[1]
    hmap = [h // (hq // hkv) for h in range(hq)] if head_map is None \
        else [int(x) for x in head_map]
    cu = [int(x) for x in cu_seqlens]
    tm = -(-max_seqlen // block_m)
    xq, xk = fp16_fixed(q), fp16_fixed(k)
    kpg = group * block_n
    stats = []
    for b in range(len(cu) - 1):
        start, L = cu[b], cu[b + 1] - cu[b]
        per_b = []
        for hk in range(hkv):
            heads = [h for h in range(hq) if hmap[h] == hk]
            per_h = []
            for m in range(tm):
                if m * block_m >= L:
                    per_h.append([])
                    continue
                r0, r1 = start + m * block_m, start + min((m + 1) * block_m, L)
                G = ((min((m + 1) * block_m, L) - 1) // block_n) // group + 1
                sq = xq[r0:r1][:, heads, :].sum(axis=(0, 1)).astype(object) \
                    if heads else np.zeros(q.shape[2], dtype=object)
                row = []
                for j in range(G):
                    k0, k1 = start + j * kpg, start + min((j + 1) * kpg, L)
                    sk = xk[k0:k1, hk, :].sum(axis=0).astype(object)
                    row.append(int(np.dot(sq, sk)))
                per_h.append(row)
            per_b.append(per_h)
        stats.append(per_b)
    return stats


def route_adaptive(q, k, cu_seqlens, max_seqlen: int, block_m: int,
                   block_n: int, group: int, int8_permille: int,
                   head_map=None) -> np.ndarray:
    """uint8 [batch, hkv, ceil(max_seqlen / block_m), 64], 1 = INT8: per
    legal row, the G - k_int8 groups with the largest statistic stay FP16
    (ties to the smaller group index), k_int8 = round-half-up of
    permille * G / 1000 as for the routing templates."""
    stats = route_adaptive_statistic(q, k, cu_seqlens, max_seqlen, block_m,
                                     block_n, group, head_map)
    hkv = np.asarray(k).shape[1]
    tm = -(-max_seqlen // block_m)
    out = np.zeros((len(stats), hkv, tm, 64), dtype=np.uint8)
    for b, per_b in enumerate(stats):
        for hk, per_h in enumerate(per_b):
            for m, imp in enumerate(per_h):
                G = len(imp)
                k_fp16 = G - (int8_permille * G + 500) // 1000
                order = sorted(range(G), key=lambda j: (-imp[j], j))
                for j in order[k_fp16:]:
                    out[b, hk, m, j] = 1
    return out

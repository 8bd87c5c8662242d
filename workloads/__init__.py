"""Seeded synthetic inputs for tile-routed FP16/INT8 prefill attention.

This module is shared by the CUDA path (tests, bench) and by the CPU oracle.
It holds none of the method's arithmetic: it only draws numbers.  What it
produces per workload:

* sequence lengths (fixed, or drawn for a variable-length batch),
* Q [T, Hq, d], K [T, Hkv, d], V [T, Hkv, d] as IEEE fp16 (numpy ``float16``),
  drawn N(0, 1) in float32 and cast with round-to-nearest-even; Q and K may
  carry 4 outlier channels per head scaled by 20,
* routing bytes ``route[b, hk, m, j]`` (1 = INT8, 0 = FP16), one byte per
  (sequence, KV head, query-tile row, key-tile group), with j < 64.

To hit an exact INT8 coverage the mask recipes must know which tile groups
are *legal* (hold at least one causal (i, j) pair).  ``legal_groups`` below
is a small, self-contained restatement of that rule used only to draw
masks; the kernel and the oracle each apply legality on their own.

Random stream order (numpy ``Generator(PCG64(seed))``), per workload:
  1. varlen only: ``seqlens = integers(lo, hi, endpoint=True, size=batch)``
  2. ``Q, K, V = standard_normal((T, H, d), float32)`` in that order
  3. outliers: for each Q head, then each K head,
     ``choice(d, 4, replace=False)`` channels multiplied by 20
The mask uses its own stream ``Generator(PCG64(mask_seed))``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

ROUTE_GROUPS = 64  # one 64-bit routing word per query-tile row


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    d: int
    block_m: int
    block_n: int
    group: int                 # g: key tiles per routing bit; 0 = derive from max length
    seqlen: int = 0            # fixed length per sequence (0 = varlen)
    varlen_lo: int = 0
    varlen_hi: int = 0
    outliers: bool = False
    kv_format: str = "fp16"    # "fp16" | "int8" (K and V arrive quantised)
    mask_recipe: str = "bernoulli"   # "bernoulli" | "diag_first" | "exact"
    coverage: float = 0.5      # INT8 share of legal groups (or Bernoulli p)
    coverage_unit: str = "kv_head"   # for "exact": "kv_head" | "sequence"
    seed: int = 0
    mask_seed: int = 1000
    quant_block_q: int = 128
    quant_block_k: int = 128

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workload shapes.  Names say what they are.
TINY = Workload(
    name="tiny_L256_h2x1_d64", batch=1, hq=2, hkv=1, d=64, block_m=64,
    block_n=64, group=1, seqlen=256, outliers=False, mask_recipe="bernoulli",
    coverage=0.5, seed=0, mask_seed=1000)

LLAMA32_3B_4K = Workload(
    name="llama32_3b_b8_L4096_int8_75", batch=8, hq=24, hkv=8, d=128,
    block_m=128, block_n=64, group=1, seqlen=4096, outliers=True,
    mask_recipe="diag_first", coverage=0.75, seed=1, mask_seed=1001)

VARLEN16 = Workload(
    name="varlen16_512_8192_h28x4_int8_50", batch=16, hq=28, hkv=4, d=128,
    block_m=128, block_n=64, group=0, varlen_lo=512, varlen_hi=8192,
    outliers=True, mask_recipe="exact", coverage=0.5, coverage_unit="sequence",
    seed=2, mask_seed=1002)

INT8KV_16K = Workload(
    name="int8kv_b2_L16384_mha32_int8_75", batch=2, hq=32, hkv=32, d=128,
    block_m=128, block_n=128, group=2, seqlen=16384, outliers=True,
    kv_format="int8", mask_recipe="diag_first", coverage=0.75, seed=3,
    mask_seed=1003)


def sweep_32k(coverage_pct: int) -> Workload:
    """Long-context sweep point; the data seed is shared by all points and
    only the mask stream changes with the coverage."""
    k = {0: 0, 25: 1, 50: 2, 75: 3, 100: 4}[coverage_pct]
    return Workload(
        name=f"sweep_L32768_h32x8_int8_{coverage_pct}", batch=1, hq=32, hkv=8,
        d=128, block_m=128, block_n=128, group=4, seqlen=32768, outliers=True,
        mask_recipe="exact", coverage=coverage_pct / 100.0,
        coverage_unit="kv_head", seed=40, mask_seed=40 + k)


WORKLOADS = {w.name: w for w in
             [TINY, LLAMA32_3B_4K, VARLEN16, INT8KV_16K]
             + [sweep_32k(c) for c in (0, 25, 50, 75, 100)]}


# ----------------------------------------------------------------------------
# sequence lengths and tile counts
# ----------------------------------------------------------------------------

def seqlens(w: Workload) -> np.ndarray:
    if w.seqlen > 0:
        return np.full(w.batch, w.seqlen, dtype=np.int32)
    rng = np.random.Generator(np.random.PCG64(w.seed))
    return rng.integers(w.varlen_lo, w.varlen_hi, endpoint=True,
                        size=w.batch).astype(np.int32)


def cu_seqlens(lens: np.ndarray) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens, dtype=np.int64)
    return cu


def group_size(w: Workload, lens: np.ndarray) -> int:
    """g, or the smallest g with ceil(ceil(max L / BN) / g) <= 64."""
    if w.group > 0:
        return w.group
    tn = -(-int(lens.max()) // w.block_n)
    return max(1, -(-tn // ROUTE_GROUPS))


def tm_max(max_seqlen: int, block_m: int) -> int:
    return -(-max_seqlen // block_m)


# ----------------------------------------------------------------------------
# Q / K / V
# ----------------------------------------------------------------------------

def qkv(w: Workload, lens: np.ndarray | None = None):
    """Return (q, k, v) as float16 arrays [T, H, d]."""
    if lens is None:
        lens = seqlens(w)
    rng = np.random.Generator(np.random.PCG64(w.seed))
    if w.seqlen == 0:  # consume the same draws as seqlens()
        rng.integers(w.varlen_lo, w.varlen_hi, endpoint=True, size=w.batch)
    t = int(lens.sum())
    q = rng.standard_normal((t, w.hq, w.d), dtype=np.float32)
    k = rng.standard_normal((t, w.hkv, w.d), dtype=np.float32)
    v = rng.standard_normal((t, w.hkv, w.d), dtype=np.float32)
    if w.outliers:
        for h in range(w.hq):
            ch = rng.choice(w.d, 4, replace=False)
            q[:, h, ch] *= 20.0
        for h in range(w.hkv):
            ch = rng.choice(w.d, 4, replace=False)
            k[:, h, ch] *= 20.0
    return q.astype(np.float16), k.astype(np.float16), v.astype(np.float16)


# ----------------------------------------------------------------------------
# routing bytes
# ----------------------------------------------------------------------------

def legal_groups(length: int, m: int, block_m: int, block_n: int, g: int):
    """(number of legal groups, set of groups holding a partially masked
    tile) for query-tile row m of a causal sequence of `length` tokens.
    Used only to draw masks with an exact coverage."""
    if m * block_m >= length:
        return 0, set()
    first_row = m * block_m
    last_row = min((m + 1) * block_m, length) - 1
    n_last = last_row // block_n
    partial = set()
    for n in range(n_last + 1):
        last_key = n * block_n + block_n - 1
        if last_key > first_row or last_key >= length:
            partial.add(n // g)
    return n_last // g + 1, partial


def _round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


def route_bytes(w: Workload, lens: np.ndarray | None = None,
                junk_in_illegal: bool = False) -> np.ndarray:
    """uint8 [batch, hkv, Tm_max, 64]; 1 = INT8, 0 = FP16.

    Recipes:
      bernoulli  - every legal group INT8 with probability `coverage`;
      diag_first - per (sequence, KV head): FP16 on group 0 and on every group
                   holding a partially masked tile, then more FP16 groups drawn
                   uniformly without replacement until the FP16 count is
                   round((1 - coverage) * N_legal); the rest INT8;
      exact      - per unit (sequence, or (sequence, KV head)): exactly
                   round(coverage * N_legal) INT8 groups drawn uniformly.
    """
    if lens is None:
        lens = seqlens(w)
    g = group_size(w, lens)
    tm = tm_max(int(lens.max()), w.block_m)
    rng = np.random.Generator(np.random.PCG64(w.mask_seed))
    route = np.zeros((w.batch, w.hkv, tm, ROUTE_GROUPS), dtype=np.uint8)
    legal = np.zeros_like(route, dtype=bool)
    forced = np.zeros_like(route, dtype=bool)
    for b in range(w.batch):
        for m in range(tm):
            ng, part = legal_groups(int(lens[b]), m, w.block_m, w.block_n, g)
            if ng > ROUTE_GROUPS:
                raise ValueError("more than 64 legal groups in a row; raise g")
            legal[b, :, m, :ng] = True
            if ng:
                forced[b, :, m, 0] = True
                for j in part:
                    forced[b, :, m, j] = True

    if w.mask_recipe == "bernoulli":
        for b in range(w.batch):
            for hk in range(w.hkv):
                for m in range(tm):
                    for j in range(ROUTE_GROUPS):
                        if legal[b, hk, m, j]:
                            route[b, hk, m, j] = rng.random() < w.coverage
    elif w.mask_recipe == "diag_first":
        for b in range(w.batch):
            for hk in range(w.hkv):
                lg = legal[b, hk]
                n_legal = int(lg.sum())
                target_fp16 = _round_half_up((1.0 - w.coverage) * n_legal)
                free = np.flatnonzero((lg & ~forced[b, hk]).ravel())
                extra = max(0, target_fp16 - int((lg & forced[b, hk]).sum()))
                pick = rng.choice(len(free), size=min(extra, len(free)),
                                  replace=False)
                fp16 = (lg & forced[b, hk]).ravel().copy()
                fp16[free[pick]] = True
                r = (lg.ravel() & ~fp16).astype(np.uint8)
                route[b, hk] = r.reshape(lg.shape)
    elif w.mask_recipe == "exact":
        units = ([(b, None) for b in range(w.batch)]
                 if w.coverage_unit == "sequence"
                 else [(b, hk) for b in range(w.batch) for hk in range(w.hkv)])
        for b, hk in units:
            sl = (b,) if hk is None else (b, hk)
            lg = legal[sl]
            idx = np.flatnonzero(lg.ravel())
            n_int8 = _round_half_up(w.coverage * len(idx))
            pick = rng.choice(len(idx), size=n_int8, replace=False)
            r = np.zeros(lg.size, dtype=np.uint8)
            r[idx[pick]] = 1
            route[sl] = r.reshape(lg.shape)
    else:
        raise ValueError(f"unknown mask recipe {w.mask_recipe!r}")

    if junk_in_illegal:
        junk = rng.integers(0, 256, size=route.shape, dtype=np.uint8)
        route = np.where(legal, route, junk).astype(np.uint8)
    return route


def make(w: Workload, junk_in_illegal: bool = False):
    """Everything a call needs, as numpy arrays, plus the derived sizes."""
    lens = seqlens(w)
    q, k, v = qkv(w, lens)
    return dict(
        workload=w, seqlens=lens, cu_seqlens=cu_seqlens(lens),
        max_seqlen=int(lens.max()), group=group_size(w, lens),
        q=q, k=k, v=v, route=route_bytes(w, lens, junk_in_illegal))

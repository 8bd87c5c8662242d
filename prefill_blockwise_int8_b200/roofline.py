"""Work accounting for the tile-routed attention path (host side, numpy).

Algorithmic work of one call, counted over legal (causal) pairs only:
  QK_x = 2 * d * Hq * (#legal pairs whose tile group routes to x),
  PV   = 2 * d * Hq * (#legal pairs),
  effective FLOP = QK_fp16 + QK_int8 + PV = 4 * d * Hq * sum_b L_b (L_b + 1) / 2.
The mixed tensor-core roofline time is
  t_roof = (QK_fp16 + PV) / P_fp16 + QK_int8 / P_int8,
weighted by the routed pair share, which differs slightly from the nominal
group coverage at tile and sequence boundaries (appendix B of the TileMix
paperlayer summary notes the same deviation).
"""
from __future__ import annotations

import numpy as np


def _tile_pairs(L: int, m: int, n: int, bm: int, bn: int) -> int:
    """Legal causal pairs (i, j), j <= i < L, inside score tile (m, n)."""
    i0, i1 = m * bm, min((m + 1) * bm, L)   # rows [i0, i1)
    j0, j1 = n * bn, min((n + 1) * bn, L)   # keys [j0, j1)
    if i0 >= i1 or j0 >= j1:
        return 0
    i = np.arange(i0, i1)
    return int(np.clip(np.minimum(i, j1 - 1) - j0 + 1, 0, None).sum())


def pair_counts(seqlens, mask_words, block_m: int, block_n: int, group: int,
                hq: int, hkv: int, head_map=None, fp16_only: bool = False):
    """(fp16 pairs, int8 pairs) summed over every query head.

    mask_words: uint64 [batch, hkv, ceil(max_len / block_m)]."""
    words = np.asarray(mask_words).view(np.uint64)
    if head_map is None:
        head_map = [h // (hq // hkv) for h in range(hq)]
    heads_of = np.bincount(np.asarray(head_map), minlength=hkv)
    fp16 = int8 = 0
    cache = {}
    for b, L in enumerate(np.asarray(seqlens).tolist()):
        tm = -(-L // block_m)
        for m in range(tm):
            last = min((m + 1) * block_m, L) - 1
            for n in range(last // block_n + 1):
                key = (L, m, n)
                if key not in cache:
                    cache[key] = _tile_pairs(L, m, n, block_m, block_n)
                pairs = cache[key]
                for hk in range(hkv):
                    if heads_of[hk] == 0:
                        continue
                    bit = 0 if fp16_only else \
                        int((int(words[b, hk, m]) >> (n // group)) & 1)
                    if bit:
                        int8 += pairs * int(heads_of[hk])
                    else:
                        fp16 += pairs * int(heads_of[hk])
    return fp16, int8


def work(seqlens, d: int, hq: int, fp16_pairs: int, int8_pairs: int):
    """FLOP / integer-op counts of one call."""
    legal = fp16_pairs + int8_pairs
    assert legal == hq * sum(int(L) * (int(L) + 1) // 2 for L in seqlens)
    return dict(qk_fp16=2 * d * fp16_pairs, qk_int8=2 * d * int8_pairs,
                pv=2 * d * legal, effective=4 * d * legal,
                int8_pair_share=int8_pairs / legal if legal else 0.0)


def roofline_seconds(w: dict, peak_fp16_flops: float, peak_int8_ops: float):
    return (w["qk_fp16"] + w["pv"]) / peak_fp16_flops + \
        w["qk_int8"] / peak_int8_ops


def min_hbm_bytes(total_tokens: int, hq: int, hkv: int, d: int,
                  int8_pair_share: float) -> int:
    """Compulsory HBM bytes of the attention kernel: Q (fp16 and/or Q8),
    K (fp16 and/or K8) and V read once, O written once."""
    fp16 = 2 * d * total_tokens
    i8 = d * total_tokens
    q = hq * (fp16 + i8) if 0 < int8_pair_share < 1 else \
        hq * (i8 if int8_pair_share == 1 else fp16)
    k = hkv * (fp16 + i8) if 0 < int8_pair_share < 1 else \
        hkv * (i8 if int8_pair_share == 1 else fp16)
    return q + k + hkv * fp16 + hq * fp16

"""The oracle's pins catch plausible mistakes.

A copy of the oracle's C source with one planted mistake (a dropped term, a
wrong sign or bit, a transposed operand, an off-by-one, a wrong constant) is
compiled to a temporary library, and the pins of test_oracle_pins.py run
against it in a subprocess; every planted mistake must fail at least one
pin.  An unmutated copy compiled the same way must pass them all, so a
failure means a pin caught the mistake, not a broken harness.  Mistakes in
the Python half (routing statistic) are planted by patching, in process.
Nothing here touches the oracle itself or any GPU.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tilemix_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# name: (text in tilemix_oracle.c, replacement)
MUTATIONS = {
    "int8_path_drops_k_scale": (
        "s[j] = a->softmax_scale * ((double)acc * sq * sk);",
        "s[j] = a->softmax_scale * ((double)acc * sq);"),
    "routing_bit_inverted": (
        "return (int)((word >> (n / a->group)) & 1u);",
        "return (int)(((~word) >> (n / a->group)) & 1u);"),
    "routing_ignores_group": (
        "return (int)((word >> (n / a->group)) & 1u);",
        "return (int)((word >> n) & 1u);"),
    "fp16_scores_use_q_for_k": (
        "(double)half_bits_to_float(a->k[koff + c]);",
        "(double)half_bits_to_float(a->q[koff + c]);"),
    "weights_not_normalised": (
        "double w = s[j] / l;",
        "double w = s[j];"),
    "kv_heads_interleaved": (
        "return h / (a->hq / a->hkv);",
        "return h % a->hkv;"),
    "quant_scale_over_128": (
        "float s = amax / 127.0f; /* one IEEE fp32 division */",
        "float s = amax / 128.0f;"),
    "quant_rounds_half_away": (
        "float rq = rintf(ratio); /* round half to even */",
        "float rq = roundf(ratio);"),
    "packer_keeps_one_illegal_group": (
        "return (int)(last_row / block_n); /* keys j <= last_row are legal */",
        "return (int)(last_row / block_n) + 1;"),
}


def _run_pins(tmp_path, source):
    src = tmp_path / "tilemix_oracle.c"
    src.write_text(source)
    lib = oracle.compile_library(src, tmp_path / "liboracle_copy.so")
    env = dict(os.environ, TILEMIX_ORACLE_LIB=str(lib))
    return subprocess.run(
        [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
         "-m", "not gpu", PINS],
        env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)


def test_unmutated_copy_passes_every_pin(tmp_path):
    r = _run_pins(tmp_path, open(SRC).read())
    assert r.returncode == 0, r.stdout[-3000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(tmp_path, name):
    old, new = MUTATIONS[name]
    source = open(SRC).read()
    assert source.count(old) == 1, name
    r = _run_pins(tmp_path, source.replace(old, new))
    assert r.returncode == 1, (name, r.stdout[-3000:])   # 1: tests failed
    assert " failed" in r.stdout, name


def test_python_half_mistakes_fail_a_pin(monkeypatch):
    import test_oracle_pins as pins
    good_fixed = oracle.fp16_fixed
    # the integer scaling off by a factor of two
    monkeypatch.setattr(oracle, "fp16_fixed", lambda x: good_fixed(x) * 2)
    with pytest.raises(AssertionError):
        pins.test_adaptive_statistic_is_the_brute_force_logit_sum()
    monkeypatch.setattr(oracle, "fp16_fixed", good_fixed)
    # FP16 sent to the smallest statistics instead of the largest
    good_stat = oracle.route_adaptive_statistic
    monkeypatch.setattr(
        oracle, "route_adaptive_statistic",
        lambda *a, **k: [[[[-x for x in row] for row in per_h]
                          for per_h in per_b] for per_b in good_stat(*a, **k)])
    with pytest.raises(AssertionError):
        pins.test_adaptive_keeps_the_heaviest_groups_fp16()
    monkeypatch.setattr(oracle, "route_adaptive_statistic", good_stat)
    # ties to the larger group index: scale every statistic by 128 and add
    # the index, which keeps every strict order and flips every tie
    monkeypatch.setattr(
        oracle, "route_adaptive_statistic",
        lambda *a, **k: [[[[128 * x + j for j, x in enumerate(row)]
                           for row in per_h] for per_h in per_b]
                         for per_b in good_stat(*a, **k)])
    with pytest.raises(AssertionError):
        pins.test_adaptive_ties_go_to_the_smaller_group()

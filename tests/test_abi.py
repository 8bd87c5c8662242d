"""C-ABI checks that need no GPU: the library loads, exports every function
include/tilemix.h declares, the Python struct mirrors the C layout, and the
host-side argument checks reject bad calls before any launch."""
import ctypes as C
import os
import re
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tilemix.h")

tm = pytest.importorskip("prefill_blockwise_int8_b200")

OK, INVALID, UNSUPPORTED, NO_DEVICE = 0, 1, 2, 6
FAKE = 0x10000  # 64 KiB: 16-byte aligned, never dereferenced on the host


def _device_visible():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # no torch: no device either
        return False


# A call that passes every host check would launch a kernel on the fake
# pointers, so it is only made where no device exists (it then stops at the
# device check); a reject stops before any launch and runs everywhere.
DEVICE_VISIBLE = _device_visible()


def accepted(fn, *args):
    if DEVICE_VISIBLE:
        return True
    rc = fn(*args)
    return rc in (NO_DEVICE, OK)


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tilemix_[a-z0-9_]+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert set(names) == set(tm.EXPORTED_SYMBOLS)
    for n in names:
        assert hasattr(tm.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", str(tm.library_path())],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (tilemix_\w+)", out))
    assert set(names) <= exported


def test_version_and_status_strings():
    assert tm.tilemix_version() >> 16 == 1
    for code in range(7):
        assert tm.tilemix_status_string(code)
    assert tm.tilemix_status_string(99) == "unknown status"


def test_params_struct_layout_matches_c():
    fields = [f for f, _ in tm.AttnParams._fields_]
    prog = ["#include <stdio.h>", "#include <stddef.h>", '#include "tilemix.h"',
            "int main(void) {",
            'printf("size %zu\\n", sizeof(tilemix_attn_params));']
    for f in fields:
        prog.append(f'printf("{f} %zu\\n", offsetof(tilemix_attn_params, {f}));')
    prog.append("return 0; }")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(c, "w").write("\n".join(prog))
        subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I",
                        os.path.join(ROOT, "include"), c, "-o", exe],
                       check=True)
        out = subprocess.run([exe], capture_output=True, text=True,
                             check=True).stdout
    got = dict(line.split() for line in out.strip().splitlines())
    assert int(got["size"]) == C.sizeof(tm.AttnParams)
    for f in fields:
        assert int(got[f]) == getattr(tm.AttnParams, f).offset, f


def good_params(**kw):
    p = tm.AttnParams()
    p.struct_size = C.sizeof(tm.AttnParams)
    p.kv_format = tm.KV_FP16
    p.q = p.k = p.v = p.out = p.q8 = p.k8 = FAKE
    p.q_scale = p.k_scale = p.cu_seqlens = p.mask = FAKE
    p.batch, p.max_seqlen, p.total_tokens = 2, 4096, 8192
    p.hq, p.hkv, p.head_dim = 24, 8, 128
    p.block_m, p.block_n, p.group = 128, 64, 1
    p.causal = 1
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def call(p):
    return tm.lib.tilemix_attn_prefill(C.byref(p), None)


def test_attn_host_checks_accept_a_valid_call():
    # valid arguments get past every host check; with no GPU in this
    # process the call then stops at the device check
    assert accepted(call, good_params()), tm.tilemix_last_error()


@pytest.mark.parametrize("field,value,expect", [
    ("struct_size", 8, INVALID),
    ("causal", 0, UNSUPPORTED),
    ("head_dim", 96, UNSUPPORTED),
    ("block_n", 32, UNSUPPORTED),
    ("block_m", 256, UNSUPPORTED),
    ("kv_format", 7, INVALID),
    ("group", 0, INVALID),
    ("hkv", 5, INVALID),              # 24 % 5 != 0 and no head_map
    ("max_seqlen", 64 * 64 + 1, INVALID),   # 65 key tiles of 64 with g = 1
    ("q", 0, INVALID),
    ("out", FAKE + 8, INVALID),       # misaligned for TMA
    ("mask", 0, INVALID),             # routed mode needs the words
    ("quant_block_k", 96, UNSUPPORTED),     # not a multiple of block_n
    ("flags", 0x80, INVALID),
    ("flags", 0x10, INVALID),         # the first undefined bit
])
def test_attn_host_checks_reject(field, value, expect):
    assert call(good_params(**{field: value})) == expect
    assert tm.tilemix_last_error()


def test_attn_block_m64_needs_block_n64():
    assert call(good_params(block_m=64, block_n=128)) == UNSUPPORTED


def test_attn_fp16_only_needs_no_int8_operands():
    p = good_params(flags=tm.FLAG_FP16_ONLY, mask=0, q8=0, k8=0, q_scale=0,
                    k_scale=0)
    assert accepted(call, p)


def test_flag_values_match_the_header():
    text = open(os.path.join(ROOT, "include", "tilemix.h")).read()
    flags = dict(re.findall(r"#define TILEMIX_FLAG_(\w+) (\d+)u", text))
    assert flags, "no TILEMIX_FLAG_ defines found"
    for name, value in flags.items():
        assert getattr(tm, "FLAG_" + name) == int(value), name


def test_attn_study_flag_is_accepted():
    # TILEMIX_FLAG_PV_F16_ACC (study only) passes the host checks, alone
    # and with the FP16-only reference mode
    assert tm.FLAG_PV_F16_ACC == 8
    assert accepted(call, good_params(flags=tm.FLAG_PV_F16_ACC))
    p = good_params(flags=tm.FLAG_PV_F16_ACC | tm.FLAG_FP16_ONLY, mask=0,
                    q8=0, k8=0, q_scale=0, k_scale=0)
    assert accepted(call, p)


def test_group_lifts_the_64_bit_limit():
    p = good_params(max_seqlen=64 * 64 * 2, total_tokens=64 * 64 * 4, group=2)
    assert accepted(call, p)


def test_quantize_and_pack_host_checks():
    q = tm.lib.tilemix_quantize_blockwise
    assert q(None, FAKE, 1, 128, 128, 2, 64, 128, FAKE, FAKE, None, None) == INVALID
    assert q(FAKE, FAKE, 1, 128, 128, 2, 60, 128, FAKE, FAKE, None, None) == INVALID
    assert q(FAKE, FAKE, 1, 128, 128, 2, 256, 256, FAKE, FAKE, None, None) == INVALID
    assert q(FAKE + 4, FAKE, 1, 128, 128, 2, 64, 128, FAKE, FAKE, None, None) == INVALID
    assert accepted(q, FAKE, FAKE, 1, 128, 128, 2, 64, 128, FAKE, FAKE, None, None)
    assert q(FAKE, FAKE, 0, 0, 0, 2, 64, 128, FAKE, FAKE, None, None) == OK
    pk = tm.lib.tilemix_pack_mask
    assert pk(FAKE, FAKE, 1, 64 * 65, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert accepted(pk, FAKE, FAKE, 1, 64 * 65, 1, 64, 64, 2, FAKE, None, None)
    assert pk(FAKE + 8, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert pk(None, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID


def test_quantize_qk_host_checks():
    # (q, k, cu, batch, max_seqlen, T, hq, hkv, d, block_q, block_k,
    #  q8, q_scale, k8, k_scale, status, stream)
    qk = tm.lib.tilemix_quantize_blockwise_qk
    good = [FAKE, FAKE, FAKE, 1, 128, 128, 6, 2, 128, 128, 128,
            FAKE, FAKE, FAKE, FAKE, None, None]

    def call(**over):
        a = list(good)
        names = ["q", "k", "cu", "batch", "ms", "T", "hq", "hkv", "d", "bq",
                 "bk", "q8", "qs", "k8", "ks", "status", "stream"]
        for nm, v in over.items():
            a[names.index(nm)] = v
        return qk(*a)

    assert call(k=None) == INVALID
    assert call(k8=None) == INVALID
    assert call(q=FAKE + 8) == INVALID          # not 16-byte aligned
    assert call(ks=FAKE + 2) == INVALID         # not 4-byte aligned
    assert call(hkv=0) == INVALID
    assert call(d=60) == INVALID
    assert call(bk=300) == INVALID
    assert call(d=256, bq=256) == INVALID       # block * d > 32768
    assert call(hq=65535, hkv=1) == UNSUPPORTED
    assert call(batch=0, ms=0) == OK            # nothing to do, nothing launched
    assert accepted(qk, *good)


def test_route_template_host_checks():
    rt = tm.lib.tilemix_route_template
    # layout, int8_permille, seed, cu, batch, max_seqlen, hkv, bm, bn, g, route
    assert accepted(rt, 2, 750, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None)
    assert rt(8, 750, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(-1, 750, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(2, 1001, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(2, -1, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(2, 750, 1, FAKE, 1, 64 * 65, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(2, 750, 1, FAKE, 1, 128, 1, 64, 64, 1, FAKE + 8, None, None) == INVALID
    assert rt(2, 750, 1, None, 1, 128, 1, 64, 64, 1, FAKE, None, None) == INVALID
    assert rt(2, 750, 1, FAKE, 0, 0, 1, 64, 64, 1, FAKE, None, None) == OK


def test_route_adaptive_host_checks():
    ra = tm.lib.tilemix_route_adaptive
    ws = tm.tilemix_route_adaptive_workspace_bytes(1, 128, 2, 128, 64)
    assert ws == 8 * 128 * 1 * 2 * (2 + 64)
    assert tm.tilemix_route_adaptive_workspace_bytes(-1, 128, 2, 128, 64) == 0

    def args(**kw):
        a = dict(q=FAKE, k=FAKE, cu=FAKE, batch=1, max_seqlen=128,
                 total_tokens=128, hq=4, hkv=2, d=128, head_map=None, bm=64,
                 bn=64, g=1, permille=750, ws=FAKE, ws_bytes=ws, route=FAKE,
                 mask=None, status=None, stream=None)
        a.update(kw)
        return list(a.values())

    assert accepted(ra, *args())
    assert accepted(ra, *args(route=None, mask=FAKE))
    assert ra(*args(ws_bytes=ws - 1)) == INVALID
    assert ra(*args(ws=None)) == INVALID
    assert ra(*args(route=None, mask=None)) == INVALID
    assert ra(*args(mask=FAKE + 4)) == INVALID
    assert ra(*args(q=FAKE + 8)) == INVALID
    assert ra(*args(permille=1001)) == INVALID
    assert ra(*args(hkv=3)) == INVALID            # 4 % 3 and no head_map
    assert ra(*args(max_seqlen=64 * 65)) == INVALID
    assert ra(*args(d=60)) == UNSUPPORTED
    assert ra(*args(d=264)) == UNSUPPORTED
    assert ra(*args(bn=1 << 15)) == UNSUPPORTED    # limbs could leave int32
    assert ra(*args(hq=512, hkv=2, bm=128)) == UNSUPPORTED   # rows * d >= 2^22
    assert ra(*args(batch=0, max_seqlen=0, ws=None, ws_bytes=0)) == OK


def test_every_compute_entry_point_cites_its_passage():
    # each declaration of a call that launches work is preceded by a comment
    # naming the passage of the pages it implements (or saying it has none)
    src = open(HEADER).read()
    utility = {"tilemix_status_string", "tilemix_last_error", "tilemix_version",
               "tilemix_route_adaptive_workspace_bytes"}
    for name in declared_functions():
        if name in utility:
            continue
        decl = re.search(r"\n[a-z_ ]+\*?\s*" + name + r"\s*\(", src)
        assert decl, name
        comment = src[:decl.start()].rsplit("*/", 1)[0].rsplit("/*", 1)[1]
        assert "Pages:" in comment or "No counterpart" in comment, name


def test_binding_refuses_host_tensors_no_cpu_fallback():
    torch = pytest.importorskip("torch")
    x = torch.zeros((4, 2, 64), dtype=torch.float16)
    k = torch.zeros((4, 1, 64), dtype=torch.float16)
    cu = torch.tensor([0, 4], dtype=torch.int32)
    route = torch.zeros((1, 1, 1, 64), dtype=torch.uint8)
    calls = [
        lambda: tm.tilemix_quantize_blockwise(x, cu, 4, 128),
        lambda: tm.tilemix_quantize_blockwise_qk(x, k, cu, 4, 128, 128),
        lambda: tm.tilemix_pack_mask(route, cu, 4, 64, 64, 1),
        lambda: tm.tilemix_route_template("band", 500, cu, 4, 1, 64, 64, 1),
        lambda: tm.tilemix_route_adaptive(x, k, cu, 4, 64, 64, 1, 500),
        lambda: tm.tilemix_attn_prefill(x, k, k, cu, 4, fp16_only=True,
                                        block_m=64, block_n=64),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()


def test_missing_library_fails_loudly():
    stand_in = tm._Missing(OSError("not built"))
    with pytest.raises(ImportError, match="build"):
        stand_in.tilemix_attn_prefill


def test_import_maps_no_library():
    # the package and its host-side helpers import without mapping
    # libtilemix.so; the library loads on the first call into it
    code = ("import prefill_blockwise_int8_b200 as tm, "
            "prefill_blockwise_int8_b200.roofline\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libtilemix.so' not in maps, 'mapped at import'\n"
            "tm.lib.tilemix_version\n"
            "assert 'libtilemix.so' in open('/proc/self/maps').read()\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT,
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

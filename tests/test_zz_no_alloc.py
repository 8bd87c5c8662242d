"""tilemix_route_adaptive_noalloc: adaptive routing with the library's
static device scratch instead of a caller workspace.  The C call allocates
nothing; it must give the same bytes and words as the workspace call and as
the oracle, leave device memory untouched from call to call, run inside a
CUDA graph capture, and refuse a request larger than the static scratch.

Named to be collected last; it needs nothing the other tests leave behind.
"""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
tm = pytest.importorskip("prefill_blockwise_int8_b200")

INVALID = 1
FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below stops on the host


def test_static_scratch_size_matches_the_header():
    src = open(os.path.join(ROOT, "include", "tilemix.h")).read()
    m = re.search(r"#define\s+TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "macro missing"
    assert int(m.group(1)) << int(m.group(2)) == tm.ROUTE_ADAPTIVE_STATIC_BYTES
    assert "tilemix_route_adaptive_noalloc" in tm.EXPORTED_SYMBOLS
    assert hasattr(tm.lib, "tilemix_route_adaptive_noalloc")


def test_oversize_request_is_refused_on_the_host():
    # 64 sequences of 8192 tokens, 8 KV heads, d 128, 128-row tiles:
    # 8 * 128 * 64 * 8 * (64 + 64) bytes = 64 MiB of scratch > 32 MiB
    need = tm.tilemix_route_adaptive_workspace_bytes(64, 8192, 8, 128, 128)
    assert need > tm.ROUTE_ADAPTIVE_STATIC_BYTES
    rc = tm.lib.tilemix_route_adaptive_noalloc(
        FAKE, FAKE, FAKE, 64, 8192, 64 * 8192, 24, 8, 128, None, 128, 128, 1,
        750, FAKE, None, None, None)
    assert rc == INVALID
    assert "static scratch" in tm.tilemix_last_error()
    # the usual host checks run first, as for the workspace call
    rc = tm.lib.tilemix_route_adaptive_noalloc(
        FAKE, FAKE, FAKE, 1, 128, 128, 4, 2, 128, None, 64, 64, 1, 1001, FAKE,
        None, None, None)
    assert rc == INVALID


def _case(seed=31):
    lens = np.array([700, 300, 1, 0, 1500], np.int32)
    rng = np.random.default_rng(seed)
    T = int(lens.sum())
    q = rng.standard_normal((T, 6, 128)).astype(np.float16)
    k = rng.standard_normal((T, 2, 128)).astype(np.float16)
    q[:, :, 3] *= 30
    k[:, :, 3] *= 30
    return lens, W.cu_seqlens(lens), q, k


@pytest.mark.gpu
def test_noalloc_matches_workspace_call_and_oracle():
    torch = pytest.importorskip("torch")
    lens, cu, q, k = _case()
    ms, bm, bn, g = int(lens.max()), 128, 64, 1
    qd, kd, cud = (torch.from_numpy(x).cuda() for x in (q, k, cu))
    tmr = -(-ms // bm)
    for permille in (0, 500, 750, 1000):
        route = torch.full((len(lens), 2, tmr, 64), 7, dtype=torch.uint8, device="cuda")
        mask = torch.full((len(lens), 2, tmr), -1, dtype=torch.int64, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        tm.tilemix_route_adaptive_noalloc(qd, kd, cud, ms, bm, bn, g, permille,
                                          route=route, mask=mask, status=status)
        ref_route, ref_mask = tm.tilemix_route_adaptive(
            qd, kd, cud, ms, bm, bn, g, permille,
            mask=torch.empty_like(mask))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(route, ref_route)
        assert torch.equal(mask, ref_mask)
        want = oracle.route_adaptive(q, k, cu, ms, bm, bn, g, permille)
        assert np.array_equal(route.cpu().numpy(), want), permille


@pytest.mark.gpu
def test_noalloc_allocates_nothing_and_captures_in_a_graph():
    torch = pytest.importorskip("torch")
    lens, cu, q, k = _case(seed=32)
    ms, bm, bn, g = int(lens.max()), 128, 64, 1
    qd, kd, cud = (torch.from_numpy(x).cuda() for x in (q, k, cu))
    tmr = -(-ms // bm)
    mask = torch.empty((len(lens), 2, tmr), dtype=torch.int64, device="cuda")
    # the first call loads the module (and its static scratch) on this device
    tm.tilemix_route_adaptive_noalloc(qd, kd, cud, ms, bm, bn, g, 500,
                                      route=None, mask=mask)
    torch.cuda.synchronize()
    eager = mask.clone()
    free0, _ = torch.cuda.mem_get_info()
    used0 = torch.cuda.memory_allocated()
    for _ in range(5):
        tm.tilemix_route_adaptive_noalloc(qd, kd, cud, ms, bm, bn, g, 500,
                                          route=None, mask=mask)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == used0
    assert torch.equal(mask, eager)

    # a capture fails on any allocation; replaying it must reproduce the words
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    mask.zero_()
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=side):
        tm.tilemix_route_adaptive_noalloc(qd, kd, cud, ms, bm, bn, g, 500,
                                          route=None, mask=mask)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(mask, eager)
    del graph

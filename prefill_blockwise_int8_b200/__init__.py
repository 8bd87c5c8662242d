"""Tile-routed FP16/INT8 causal prefill attention on B200 (sm_100a).

Thin Python binding of the C ABI in ``include/tilemix.h`` (``libtilemix.so``,
built in-tree by ``python -m prefill_blockwise_int8_b200.build``).  This
module only marshals arguments: it takes torch tensors that already live on
the GPU, passes their device pointers and the current CUDA stream, and
raises ``TilemixError`` when a call returns a non-OK status.  Every step of
the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and importing this package fails loudly when the library
is missing.

Entry points (same names as the C ABI):
  tilemix_quantize_blockwise(x, cu_seqlens, max_seqlen, block=128)
      -> (x8, scale)
  tilemix_quantize_blockwise_qk(q, k, cu_seqlens, max_seqlen) (one launch)
      -> (q8, q_scale, k8, k_scale)
  tilemix_pack_mask(route, cu_seqlens, max_seqlen, block_m, block_n, group)
      -> mask
  tilemix_attn_prefill(q, k, v, cu_seqlens, max_seqlen, ...) -> out
"""
from __future__ import annotations

import ctypes as C
from pathlib import Path

__all__ = [
    "TilemixError", "lib", "library_path", "EXPORTED_SYMBOLS",
    "tilemix_quantize_blockwise", "tilemix_quantize_blockwise_qk",
    "tilemix_pack_mask", "tilemix_attn_prefill",
    "tilemix_route_template", "tilemix_route_adaptive",
    "tilemix_route_adaptive_workspace_bytes", "tilemix_route_adaptive_noalloc",
    "ROUTE_ADAPTIVE_STATIC_BYTES", "tilemix_status_string",
    "tilemix_last_error", "tilemix_version", "KV_FP16", "KV_INT8", "FLAG_FP16_ONLY",
    "FLAG_QUANT_ON_CHIP", "FLAG_TEST_EXPIRE_WAIT", "FLAG_PV_F16_ACC", "STATUS",
    "LAYOUTS",
]

_LIB_PATH = Path(__file__).resolve().parent / "libtilemix.so"

KV_FP16, KV_INT8 = 0, 1
FLAG_FP16_ONLY = 1
FLAG_QUANT_ON_CHIP = 2
FLAG_TEST_EXPIRE_WAIT = 4  # test only: makes a bounded device wait expire
FLAG_PV_F16_ACC = 8  # study only: O accumulated in fp16 (no tolerance)
STATUS = {0: "TILEMIX_OK", 1: "TILEMIX_ERR_INVALID_ARG",
          2: "TILEMIX_ERR_UNSUPPORTED", 3: "TILEMIX_ERR_CUDA",
          4: "TILEMIX_ERR_TIMEOUT", 5: "TILEMIX_ERR_BAD_SEQLENS",
          6: "TILEMIX_ERR_NO_DEVICE"}

# Routing-template layouts (TILEMIX_LAYOUT_*).
LAYOUTS = {"all_fp16": 0, "all_int8": 1, "band": 2, "global": 3,
           "row_random": 4, "aligned": 5, "bigbird": 6, "sptrans": 7}

# Every function include/tilemix.h declares.
EXPORTED_SYMBOLS = (
    "tilemix_quantize_blockwise", "tilemix_quantize_blockwise_qk",
    "tilemix_pack_mask", "tilemix_attn_prefill",
    "tilemix_route_template", "tilemix_route_adaptive_workspace_bytes",
    "tilemix_route_adaptive", "tilemix_route_adaptive_noalloc",
    "tilemix_status_string", "tilemix_last_error", "tilemix_version",
)

# TILEMIX_ROUTE_ADAPTIVE_STATIC_BYTES: the static scratch of
# tilemix_route_adaptive_noalloc on each device.
ROUTE_ADAPTIVE_STATIC_BYTES = 32 << 20


class TilemixError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")
        self.status = status


class AttnParams(C.Structure):
    """Mirror of tilemix_attn_params (include/tilemix.h)."""
    _fields_ = [
        ("struct_size", C.c_uint32), ("kv_format", C.c_int),
        ("flags", C.c_uint32),
        ("q", C.c_void_p), ("q8", C.c_void_p), ("q_scale", C.c_void_p),
        ("k", C.c_void_p), ("k8", C.c_void_p), ("k_scale", C.c_void_p),
        ("v", C.c_void_p), ("v8", C.c_void_p), ("v_scale", C.c_void_p),
        ("cu_seqlens", C.c_void_p), ("batch", C.c_int),
        ("max_seqlen", C.c_int), ("total_tokens", C.c_int),
        ("hq", C.c_int), ("hkv", C.c_int), ("head_dim", C.c_int),
        ("head_map", C.c_void_p),
        ("mask", C.c_void_p), ("block_m", C.c_int), ("block_n", C.c_int),
        ("group", C.c_int),
        ("quant_block_q", C.c_int), ("quant_block_k", C.c_int),
        ("softmax_scale", C.c_float), ("causal", C.c_int),
        ("out", C.c_void_p), ("lse", C.c_void_p), ("qk_dump", C.c_void_p),
        ("status", C.c_void_p),
    ]


def library_path() -> Path:
    return _LIB_PATH


def _load() -> C.CDLL:
    if not _LIB_PATH.exists():
        raise ImportError(
            f"{_LIB_PATH} is missing: build the CUDA library with "
            "`python -m prefill_blockwise_int8_b200.build` (nvcc, sm_100a)")
    lib = C.CDLL(str(_LIB_PATH))
    vp, i32 = C.c_void_p, C.c_int
    lib.tilemix_quantize_blockwise.restype = i32
    lib.tilemix_quantize_blockwise.argtypes = [
        vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
    lib.tilemix_quantize_blockwise_qk.restype = i32
    lib.tilemix_quantize_blockwise_qk.argtypes = [
        vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp,
        vp, vp]
    lib.tilemix_pack_mask.restype = i32
    lib.tilemix_pack_mask.argtypes = [
        vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    lib.tilemix_route_template.restype = i32
    lib.tilemix_route_template.argtypes = [
        i32, i32, C.c_uint64, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp]
    lib.tilemix_route_adaptive_workspace_bytes.restype = C.c_size_t
    lib.tilemix_route_adaptive_workspace_bytes.argtypes = [i32] * 5
    lib.tilemix_route_adaptive.restype = i32
    lib.tilemix_route_adaptive.argtypes = [
        vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, i32, i32, i32, vp,
        C.c_size_t, vp, vp, vp, vp]
    lib.tilemix_route_adaptive_noalloc.restype = i32
    lib.tilemix_route_adaptive_noalloc.argtypes = [
        vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, i32, i32, i32, i32, vp,
        vp, vp, vp]
    lib.tilemix_attn_prefill.restype = i32
    lib.tilemix_attn_prefill.argtypes = [C.POINTER(AttnParams), vp]
    lib.tilemix_status_string.restype = C.c_char_p
    lib.tilemix_status_string.argtypes = [i32]
    lib.tilemix_last_error.restype = C.c_char_p
    lib.tilemix_last_error.argtypes = []
    lib.tilemix_version.restype = C.c_uint32
    lib.tilemix_version.argtypes = []
    return lib


class _Missing:
    """Stands in for the library when it is missing or older than the
    sources (so the package imports for a build); any use raises."""

    def __init__(self, err: Exception):
        self._err = err

    def __getattr__(self, name):
        raise ImportError(f"libtilemix.so unusable ({self._err}); build it "
                          "with `python -m prefill_blockwise_int8_b200.build`")


class _Lazy:
    """The library, mapped into the process on the first attribute access
    (importing the package, or its host-side helpers such as ``roofline``,
    maps nothing).  A missing or unusable library raises at that access."""

    def __init__(self):
        self._lib = None

    def __getattr__(self, name):
        if self._lib is None:
            try:
                self._lib = _load()
            except (OSError, AttributeError, ImportError) as e:
                self._lib = _Missing(e)
        return getattr(self._lib, name)


lib = _Lazy()


def reload_library():
    """Load libtilemix.so now (again, after a build); raises if unusable."""
    lib._lib = _load()
    return lib


def tilemix_status_string(status: int) -> str:
    return lib.tilemix_status_string(status).decode()


def tilemix_last_error() -> str:
    return lib.tilemix_last_error().decode()


def tilemix_version() -> int:
    return int(lib.tilemix_version())


# ----------------------------------------------------------------------------
# torch marshalling
# ----------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _check(rc: int, where: str):
    if rc != 0:
        raise TilemixError(rc, where, tilemix_last_error())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dev(t, name, dtype=None):
    torch = _torch()
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def tilemix_quantize_blockwise(x, cu_seqlens, max_seqlen: int, block: int = 128,
                               *, x8=None, scale=None, status=None,
                               stream=None):
    """Blockwise symmetric INT8 quantisation of fp16 x [T, H, d].

    Returns (x8 int8 [T, H, d], scale fp32 [H, batch, ceil(max_seqlen/block)])."""
    torch = _torch()
    _dev(x, "x", torch.float16)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    t, heads, d = x.shape
    batch = cu_seqlens.numel() - 1
    nblk = -(-max_seqlen // block)
    if x8 is None:
        x8 = torch.empty((t, heads, d), dtype=torch.int8, device=x.device)
    if scale is None:
        scale = torch.empty((heads, batch, nblk), dtype=torch.float32,
                            device=x.device)
    _dev(x8, "x8", torch.int8)
    _dev(scale, "scale", torch.float32)
    _check(lib.tilemix_quantize_blockwise(
        _ptr(x), _ptr(cu_seqlens), batch, max_seqlen, t, heads, d, block,
        _ptr(x8), _ptr(scale), _ptr(status), _stream(stream)),
        "tilemix_quantize_blockwise")
    return x8, scale


def tilemix_quantize_blockwise_qk(q, k, cu_seqlens, max_seqlen: int,
                                  block_q: int = 128, block_k: int = 128, *,
                                  q8=None, q_scale=None, k8=None, k_scale=None,
                                  status=None, stream=None):
    """Q and K quantised in one launch: returns (q8, q_scale, k8, k_scale),
    equal to two tilemix_quantize_blockwise calls."""
    torch = _torch()
    _dev(q, "q", torch.float16)
    _dev(k, "k", torch.float16)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    t, hq, d = q.shape
    tk, hkv, dk = k.shape
    if (tk, dk) != (t, d):
        raise ValueError("q and k must share tokens and head_dim")
    batch = cu_seqlens.numel() - 1
    if q8 is None:
        q8 = torch.empty((t, hq, d), dtype=torch.int8, device=q.device)
    if k8 is None:
        k8 = torch.empty((t, hkv, d), dtype=torch.int8, device=q.device)
    if q_scale is None:
        q_scale = torch.empty((hq, batch, -(-max_seqlen // block_q)),
                              dtype=torch.float32, device=q.device)
    if k_scale is None:
        k_scale = torch.empty((hkv, batch, -(-max_seqlen // block_k)),
                              dtype=torch.float32, device=q.device)
    for tns, nm, dt in ((q8, "q8", torch.int8), (k8, "k8", torch.int8),
                        (q_scale, "q_scale", torch.float32),
                        (k_scale, "k_scale", torch.float32)):
        _dev(tns, nm, dt)
    _check(lib.tilemix_quantize_blockwise_qk(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), batch, max_seqlen, t, hq, hkv, d,
        block_q, block_k, _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale),
        _ptr(status), _stream(stream)), "tilemix_quantize_blockwise_qk")
    return q8, q_scale, k8, k_scale


def tilemix_pack_mask(route, cu_seqlens, max_seqlen: int, block_m: int,
                      block_n: int, group: int, *, mask=None, status=None,
                      stream=None):
    """uint8 route [B, Hkv, ceil(max_seqlen/block_m), 64] -> uint64 words
    [B, Hkv, ceil(max_seqlen/block_m)] (returned as torch.int64 storage)."""
    torch = _torch()
    _dev(route, "route", torch.uint8)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    batch, hkv, tm, ng = route.shape
    if ng != 64:
        raise ValueError("route last dimension must be 64")
    if mask is None:
        mask = torch.empty((batch, hkv, tm), dtype=torch.int64,
                           device=route.device)
    _dev(mask, "mask")
    _check(lib.tilemix_pack_mask(
        _ptr(route), _ptr(cu_seqlens), batch, max_seqlen, hkv, block_m,
        block_n, group, _ptr(mask), _ptr(status), _stream(stream)),
        "tilemix_pack_mask")
    return mask


def tilemix_route_template(layout, int8_permille: int, cu_seqlens,
                           max_seqlen: int, hkv: int, block_m: int,
                           block_n: int, group: int, *, seed: int = 0,
                           route=None, status=None, stream=None):
    """Route bytes [B, Hkv, ceil(max_seqlen/block_m), 64] (uint8, 1 = INT8)
    of a named layout ("band", "bigbird", ... or a TILEMIX_LAYOUT_* value)
    with an INT8 share of int8_permille / 1000 of each row's legal groups."""
    torch = _torch()
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    code = LAYOUTS[layout] if isinstance(layout, str) else int(layout)
    batch = cu_seqlens.numel() - 1
    tm = -(-max_seqlen // block_m)
    if route is None:
        route = torch.empty((batch, hkv, tm, 64), dtype=torch.uint8,
                            device=cu_seqlens.device)
    _dev(route, "route", torch.uint8)
    _check(lib.tilemix_route_template(
        code, int8_permille, seed & 0xFFFFFFFFFFFFFFFF, _ptr(cu_seqlens), batch,
        max_seqlen, hkv, block_m, block_n, group, _ptr(route), _ptr(status),
        _stream(stream)), "tilemix_route_template")
    return route


def tilemix_route_adaptive_workspace_bytes(batch: int, max_seqlen: int,
                                           hkv: int, head_dim: int,
                                           block_m: int) -> int:
    """Bytes of device scratch tilemix_route_adaptive needs."""
    return int(lib.tilemix_route_adaptive_workspace_bytes(
        batch, max_seqlen, hkv, head_dim, block_m))


def tilemix_route_adaptive(q, k, cu_seqlens, max_seqlen: int, block_m: int,
                           block_n: int, group: int, int8_permille: int, *,
                           head_map=None, workspace=None, route=None,
                           mask=None, want_route: bool = True, status=None,
                           stream=None):
    """Route bytes [B, Hkv, ceil(max_seqlen/block_m), 64] (uint8, 1 = INT8)
    chosen from the data: per query-tile row, the groups whose summed raw
    logits with the row are largest stay FP16.  q fp16 [T, hq, d], k fp16
    [T, hkv, d].  `workspace` (uint8 CUDA tensor) is allocated here when not
    given.  Returns the route bytes, or (route, mask) when `mask` (uint64
    words [B, Hkv, Tm], int64 CUDA tensor) is given; want_route=False skips
    the bytes (route is then None)."""
    torch = _torch()
    _dev(q, "q", torch.float16)
    _dev(k, "k", torch.float16)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    _dev(head_map, "head_map", torch.int32)
    t, hq, d = q.shape
    hkv = k.shape[1]
    batch = cu_seqlens.numel() - 1
    tm = -(-max_seqlen // block_m)
    need = tilemix_route_adaptive_workspace_bytes(batch, max_seqlen, hkv, d,
                                                  block_m)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8,
                                device=q.device)
    _dev(workspace, "workspace")
    if route is None and want_route:
        route = torch.empty((batch, hkv, tm, 64), dtype=torch.uint8,
                            device=q.device)
    _dev(route, "route", torch.uint8)
    _dev(mask, "mask", torch.int64)
    _check(lib.tilemix_route_adaptive(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), batch, max_seqlen, t, hq, hkv, d,
        _ptr(head_map), block_m, block_n, group, int8_permille,
        _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(route), _ptr(mask), _ptr(status), _stream(stream)),
        "tilemix_route_adaptive")
    return route if mask is None else (route, mask)


def tilemix_route_adaptive_noalloc(q, k, cu_seqlens, max_seqlen: int,
                                   block_m: int, block_n: int, group: int,
                                   int8_permille: int, *, route, mask=None,
                                   head_map=None, status=None, stream=None):
    """tilemix_route_adaptive with the library's static device scratch: the
    C call allocates nothing (outputs are the caller's: `route` uint8
    [B, Hkv, Tm, 64] and/or `mask` int64 [B, Hkv, Tm], either may be None).
    Calls that can overlap on the device share that scratch and must be
    ordered (one stream, or events)."""
    torch = _torch()
    _dev(q, "q", torch.float16)
    _dev(k, "k", torch.float16)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    _dev(head_map, "head_map", torch.int32)
    _dev(route, "route", torch.uint8)
    _dev(mask, "mask", torch.int64)
    t, hq, d = q.shape
    _check(lib.tilemix_route_adaptive_noalloc(
        _ptr(q), _ptr(k), _ptr(cu_seqlens), cu_seqlens.numel() - 1, max_seqlen,
        t, hq, k.shape[1], d, _ptr(head_map), block_m, block_n, group,
        int8_permille, _ptr(route), _ptr(mask), _ptr(status), _stream(stream)),
        "tilemix_route_adaptive_noalloc")
    return route, mask


def tilemix_attn_prefill(q, k, v, cu_seqlens, max_seqlen: int, *, q8=None,
                         q_scale=None, k8=None, k_scale=None, v8=None,
                         v_scale=None, mask=None, block_m: int = 128,
                         block_n: int = 128, group: int = 1,
                         quant_block_q: int = 128, quant_block_k: int = 128,
                         softmax_scale: float = 0.0, head_map=None,
                         fp16_only: bool = False, kv_format: int = KV_FP16,
                         quant_on_chip: bool = False,
                         test_expire_wait: bool = False,
                         pv_f16_acc: bool = False, out=None, lse=None,
                         qk_dump=None, status=None, stream=None):
    """Causal tile-routed attention.  q fp16 [T, hq, d]; k, v fp16
    [T, hkv, d] (or k8/v8 int8 + scales with kv_format=KV_INT8).
    Returns out fp16 [T, hq, d]."""
    torch = _torch()
    _dev(q, "q", torch.float16)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    t, hq, d = q.shape
    kv_src = k8 if kv_format == KV_INT8 else k
    if kv_src is None:
        raise ValueError("k (or k8 for KV_INT8) is required")
    hkv = kv_src.shape[1]
    for name, tt, dt in (("k", k, torch.float16), ("v", v, torch.float16),
                         ("q8", q8, torch.int8), ("k8", k8, torch.int8),
                         ("v8", v8, torch.int8),
                         ("q_scale", q_scale, torch.float32),
                         ("k_scale", k_scale, torch.float32),
                         ("v_scale", v_scale, torch.float32),
                         ("head_map", head_map, torch.int32),
                         ("lse", lse, torch.float32),
                         ("qk_dump", qk_dump, torch.int32)):
        _dev(tt, name, dt)
    _dev(mask, "mask")
    if out is None:
        out = torch.empty_like(q)
    _dev(out, "out", torch.float16)
    p = AttnParams()
    p.struct_size = C.sizeof(AttnParams)
    p.kv_format = kv_format
    p.flags = (FLAG_FP16_ONLY if fp16_only else 0) | \
        (FLAG_QUANT_ON_CHIP if quant_on_chip else 0) | \
        (FLAG_TEST_EXPIRE_WAIT if test_expire_wait else 0) | \
        (FLAG_PV_F16_ACC if pv_f16_acc else 0)
    p.q, p.q8, p.q_scale = _ptr(q), _ptr(q8), _ptr(q_scale)
    p.k, p.k8, p.k_scale = _ptr(k), _ptr(k8), _ptr(k_scale)
    p.v, p.v8, p.v_scale = _ptr(v), _ptr(v8), _ptr(v_scale)
    p.cu_seqlens = _ptr(cu_seqlens)
    p.batch = cu_seqlens.numel() - 1
    p.max_seqlen = max_seqlen
    p.total_tokens = t
    p.hq, p.hkv, p.head_dim = hq, hkv, d
    p.head_map = _ptr(head_map)
    p.mask = _ptr(mask)
    p.block_m, p.block_n, p.group = block_m, block_n, group
    p.quant_block_q, p.quant_block_k = quant_block_q, quant_block_k
    p.softmax_scale = softmax_scale
    p.causal = 1
    p.out, p.lse, p.qk_dump, p.status = (_ptr(out), _ptr(lse), _ptr(qk_dump),
                                         _ptr(status))
    _check(lib.tilemix_attn_prefill(C.byref(p), _stream(stream)),
           "tilemix_attn_prefill")
    return out

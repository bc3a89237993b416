"""Zebra3D multi-view global attention for B200 (sm_100a).

Python binding of the C ABI in include/zebra.h (libzebra.so). Every function
here only marshals arguments: tensors become device pointers and strides,
torch's current CUDA stream is passed along, and a nonzero status raises
ZebraError. All computation runs in the library's CUDA kernels; there is no
fallback. Function names match the C entry points.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "Geom", "Layout", "ZebraError", "lib", "geom",
    "zebra_keep_count", "zebra_tile_pool", "zebra_tile_select", "zebra_sparse_attn",
    "zebra_linear_attn", "zebra_hybrid_layer", "zebra_workspace_bytes", "zebra_last_error",
    "zebra_sync_status", "zebra_launch_count", "zebra_version", "workspace", "zebra_profile_enable",
    "zebra_profile_report", "zebra_linear_attn_noalloc", "zebra_affine_moments", "zebra_affine_solve",
    "affine_moments_buffer", "zebra_debug_inject", "zebra_affine_residual", "zebra_allocate_layers",
    "zebra_coverage", "zebra_coverage_workspace_bytes",
    "ZEBRA_OK", "ZEBRA_ERR_INVALID_ARG", "ZEBRA_ERR_UNSUPPORTED", "ZEBRA_ERR_WORKSPACE", "ZEBRA_ERR_CUDA",
    "ZEBRA_ERR_TIMEOUT", "ZEBRA_ERR_NUMERIC", "ZEBRA_AFFINE_GROUP_DOUBLES", "ZEBRA_F32", "ZEBRA_BF16", "ZEBRA_LAYER_LINEAR", "ZEBRA_LAYER_SPARSE",
    "ZEBRA_LAYER_DENSE", "ZEBRA_OP_SELECT", "ZEBRA_OP_SPARSE", "ZEBRA_OP_LINEAR", "ZEBRA_OP_HYBRID_LINEAR",
    "ZEBRA_OP_HYBRID_SPARSE", "ZEBRA_OP_HYBRID_DENSE", "ZEBRA_OP_AFFINE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzebra.so")

(ZEBRA_OK, ZEBRA_ERR_INVALID_ARG, ZEBRA_ERR_UNSUPPORTED, ZEBRA_ERR_WORKSPACE, ZEBRA_ERR_CUDA, ZEBRA_ERR_TIMEOUT,
 ZEBRA_ERR_NUMERIC) = range(7)
ZEBRA_F32, ZEBRA_BF16 = 0, 1
ZEBRA_LAYER_LINEAR, ZEBRA_LAYER_SPARSE, ZEBRA_LAYER_DENSE = 0, 1, 2
(ZEBRA_OP_SELECT, ZEBRA_OP_SPARSE, ZEBRA_OP_LINEAR, ZEBRA_OP_HYBRID_LINEAR, ZEBRA_OP_HYBRID_SPARSE,
 ZEBRA_OP_HYBRID_DENSE, ZEBRA_OP_AFFINE) = range(7)
ZEBRA_AFFINE_GROUP_DOUBLES = 8322


class Geom(ctypes.Structure):
    _fields_ = [("views", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("n_special", ctypes.c_int32), ("tile", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32)]

    @property
    def tiles_per_view(self):
        return ((self.grid_h + 7) // 8) * ((self.grid_w + 7) // 8)

    @property
    def n_tiles(self):
        return self.views * self.tiles_per_view

    @property
    def n_tokens(self):
        return self.views * (self.n_special + self.grid_h * self.grid_w)

    @property
    def mask_words(self):
        return (self.n_tiles + 31) // 32


class Layout(ctypes.Structure):
    _fields_ = [("tok_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64)]


class ZebraError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"zebra error {code}: {msg}")
        self.code = code


def geom(views, grid_h, grid_w, heads, n_special=5, tile=8, head_dim=64) -> Geom:
    return Geom(views, grid_h, grid_w, n_special, tile, heads, head_dim)


_lib = None
_P = ctypes.c_void_p
_G = ctypes.POINTER(Geom)
_L = ctypes.POINTER(Layout)


def lib() -> ctypes.CDLL:
    """The loaded libzebra.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m linear_global_attention_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "zebra_keep_count": (ctypes.c_int32, [ctypes.c_double, ctypes.c_int32]),
            "zebra_tile_pool": (ctypes.c_int, [_G, ctypes.c_int, _P, _L, _P, _P, _P, _P]),
            "zebra_tile_select": (ctypes.c_int, [_G, _P, _P, ctypes.c_double, _P, _P, _P, _P, ctypes.c_size_t, _P]),
            "zebra_sparse_attn": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _P, _L, ctypes.c_double, _P, _P, _P,
                                                 ctypes.c_size_t, _P]),
            "zebra_linear_attn": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _P, _L, _P, _P, ctypes.c_float,
                                                 ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
            "zebra_hybrid_layer": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _P, _P, _P, ctypes.c_double,
                                                  ctypes.c_float, ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
            "zebra_workspace_bytes": (ctypes.c_size_t, [_G, ctypes.c_int, ctypes.c_int, ctypes.c_double]),
            "zebra_last_error": (ctypes.c_char_p, []),
            "zebra_sync_status": (ctypes.c_int, [_P]),
            "zebra_launch_count": (ctypes.c_uint64, []),
            "zebra_version": (ctypes.c_char_p, []),
            "zebra_linear_attn_noalloc": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _P, _L, _P, _P, ctypes.c_float,
                                                         ctypes.c_float, _P, _P]),
            "zebra_affine_moments": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _L, ctypes.c_int, _P, _P,
                                                    ctypes.c_size_t, _P]),
            "zebra_affine_solve": (ctypes.c_int, [_G, _P, ctypes.c_int, ctypes.c_double, _P, _P, _P]),
            "zebra_affine_residual": (ctypes.c_int, [_G, _P, ctypes.c_int, _P, _P, _P, _P]),
            "zebra_coverage": (ctypes.c_int, [_G, ctypes.c_int, _P, _P, _L, _P, _P, ctypes.c_int32, _P, _P, _P,
                                              ctypes.c_size_t, _P]),
            "zebra_coverage_workspace_bytes": (ctypes.c_size_t, [_G, ctypes.c_int32]),
            "zebra_allocate_layers": (ctypes.c_int32, [_P, ctypes.c_int32, ctypes.c_double, _P]),
            "zebra_profile_enable": (ctypes.c_int, [ctypes.c_int]),
            "zebra_debug_inject": (ctypes.c_int, [ctypes.c_int32, ctypes.c_uint64]),
            "zebra_profile_report": (ctypes.c_longlong, [ctypes.c_char_p, ctypes.c_size_t]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc: int):
    if rc != ZEBRA_OK:
        raise ZebraError(rc, zebra_last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype(t):
    import torch
    if t.dtype == torch.bfloat16:
        return ZEBRA_BF16
    if t.dtype == torch.float32:
        return ZEBRA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _layout(x, *others):
    """Strides of a [N, H, 64] view (channels contiguous); q, k and v must share them."""
    if x.dim() != 3 or x.shape[-1] != 64 or x.stride(-1) != 1:
        raise ValueError("expected a [N, H, 64] tensor with contiguous channels")
    for o in others:
        if o.stride() != x.stride() or o.shape != x.shape or o.dtype != x.dtype:
            raise ValueError("q, k and v must share shape, dtype and strides")
    return Layout(x.stride(0), x.stride(1))


def zebra_last_error() -> str:
    return lib().zebra_last_error().decode()


def zebra_version() -> str:
    return lib().zebra_version().decode()


def zebra_launch_count() -> int:
    return int(lib().zebra_launch_count())


def zebra_keep_count(y: float, n_tiles: int) -> int:
    return int(lib().zebra_keep_count(y, n_tiles))


def zebra_workspace_bytes(g: Geom, op: int, dtype: int = ZEBRA_BF16, y: float = 0.0) -> int:
    n = lib().zebra_workspace_bytes(ctypes.byref(g), op, dtype, y)
    if n == 0:
        raise ZebraError(ZEBRA_ERR_INVALID_ARG, zebra_last_error())
    return int(n)


def workspace(g: Geom, op: int, dtype: int = ZEBRA_BF16, y: float = 0.0, device="cuda"):
    """A device byte buffer of zebra_workspace_bytes() bytes (allocated by torch)."""
    import torch
    return torch.empty(zebra_workspace_bytes(g, op, dtype, y), dtype=torch.uint8, device=device)


def zebra_sync_status(stream=None) -> int:
    return int(lib().zebra_sync_status(_stream(stream)))


def zebra_debug_inject(block: int, wait_ns: int = 0):
    """Error-path test hook of the sparse kernel (see include/zebra.h); (-1, 0) turns it off."""
    _check(lib().zebra_debug_inject(int(block), int(wait_ns)))


def zebra_tile_pool(g: Geom, x, x_mean, x_packed=None, tile_counts=None, stream=None):
    lay = _layout(x)
    _check(lib().zebra_tile_pool(ctypes.byref(g), _dtype(x), _ptr(x), ctypes.byref(lay), _ptr(x_mean),
                                 _ptr(x_packed), _ptr(tile_counts), _stream(stream)))


def zebra_tile_select(g: Geom, q_mean, k_mean, y: float, mask, near_tie=None, ws=None, stream=None) -> int:
    k_out = ctypes.c_int32(0)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().zebra_tile_select(ctypes.byref(g), _ptr(q_mean), _ptr(k_mean), y, _ptr(mask), _ptr(near_tie),
                                   ctypes.byref(k_out), _ptr(ws), nbytes, _stream(stream)))
    return k_out.value


def zebra_sparse_attn(g: Geom, q, k, v, y: float, out, ws, mask=None, stream=None):
    lay = _layout(q, k, v)
    _check(lib().zebra_sparse_attn(ctypes.byref(g), _dtype(q), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(lay), y,
                                   _ptr(mask), _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)))


def zebra_linear_attn(g: Geom, q, k, v, A, b, out, ws, rope_base=100.0, eps=1e-6, stream=None):
    lay = _layout(q, k, v)
    _check(lib().zebra_linear_attn(ctypes.byref(g), _dtype(q), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(lay),
                                   _ptr(A), _ptr(b), rope_base, eps, _ptr(out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)))


def zebra_linear_attn_noalloc(g: Geom, q, k, v, A, b, out, rope_base=100.0, eps=1e-6, stream=None):
    """zebra_linear_attn with its scratch in the library's built-in device array (no workspace)."""
    lay = _layout(q, k, v)
    _check(lib().zebra_linear_attn_noalloc(ctypes.byref(g), _dtype(q), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(lay),
                                           _ptr(A), _ptr(b), rope_base, eps, _ptr(out), _stream(stream)))


def affine_moments_buffer(g: Geom, per_head: bool = False, device="cuda"):
    """Zeroed float64 moments of one affine fit (1 group pooled, H groups per head)."""
    import torch
    groups = g.heads if per_head else 1
    return torch.zeros(groups * ZEBRA_AFFINE_GROUP_DOUBLES, dtype=torch.float64, device=device)


def zebra_affine_moments(g: Geom, x, y, moments, ws, per_head: bool = False, stream=None):
    """Adds the moments of samples x (linear output) -> y (teacher output), both [N, H, 64], to `moments`."""
    lay = _layout(x, y)
    _check(lib().zebra_affine_moments(ctypes.byref(g), _dtype(x), _ptr(x), _ptr(y), ctypes.byref(lay),
                                      1 if per_head else 0, _ptr(moments), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)))


def zebra_affine_solve(g: Geom, moments, lam: float, A, b, per_head: bool = False, stream=None):
    """A [H, 64, 64], b [H, 64] (float32) of the centred ridge fit of `moments`."""
    _check(lib().zebra_affine_solve(ctypes.byref(g), _ptr(moments), 1 if per_head else 0, float(lam), _ptr(A),
                                    _ptr(b), _stream(stream)))


def zebra_affine_residual(g: Geom, moments, A, b, err, per_head: bool = False, stream=None):
    """err (float64, one per group): mean |A x + b - y|^2 of each group's samples, from `moments`."""
    _check(lib().zebra_affine_residual(ctypes.byref(g), _ptr(moments), 1 if per_head else 0, _ptr(A), _ptr(b),
                                       _ptr(err), _stream(stream)))


def zebra_coverage_workspace_bytes(g: Geom, n_query_tiles: int) -> int:
    n = lib().zebra_coverage_workspace_bytes(ctypes.byref(g), int(n_query_tiles))
    if n == 0:
        raise ZebraError(ZEBRA_ERR_INVALID_ARG, zebra_last_error())
    return int(n)


def zebra_coverage(g: Geom, q, k, mask, query_tiles, selected_mass, special_mass, ws, stream=None):
    """Dense softmax mass of the sampled tiles' rows on their selected key tiles and on the special keys.
    query_tiles: host sequence of tile indices; outputs [n, H, 64] float32."""
    import numpy as np
    lay = _layout(q, k)
    t = np.ascontiguousarray(np.asarray(query_tiles, dtype=np.int32))
    _check(lib().zebra_coverage(ctypes.byref(g), _dtype(q), _ptr(q), _ptr(k), ctypes.byref(lay), _ptr(mask),
                                t.ctypes.data_as(ctypes.c_void_p), len(t), _ptr(selected_mass), _ptr(special_mass),
                                _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def zebra_allocate_layers(errors, linear_fraction: float):
    """Host call: 0/1 int32 array, 1 for the round(x * L) layers of lowest error (ties in index order)."""
    import numpy as np
    e = np.ascontiguousarray(np.asarray(errors, dtype=np.float64))
    out = np.zeros(len(e), dtype=np.int32)
    n = lib().zebra_allocate_layers(e.ctypes.data_as(ctypes.c_void_p), len(e), float(linear_fraction),
                                    out.ctypes.data_as(ctypes.c_void_p))
    if n < 0:
        raise ZebraError(ZEBRA_ERR_INVALID_ARG, "bad arguments to zebra_allocate_layers")
    return out


def zebra_hybrid_layer(g: Geom, kind: int, x, w_qkv, w_o, A, b, y, x_out, ws, rope_base=100.0, eps=1e-6,
                       stream=None):
    _check(lib().zebra_hybrid_layer(ctypes.byref(g), kind, _ptr(x), _ptr(w_qkv), _ptr(w_o), _ptr(A), _ptr(b), y,
                                    rope_base, eps, _ptr(x_out), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)))


def zebra_profile_enable(on: bool = True):
    _check(lib().zebra_profile_enable(1 if on else 0))


def zebra_profile_report() -> dict:
    """{"kernels": {name: (records, total_ms)}, "launches": {name: kernel launches},
    "logits": {"sparse_rows": n, "special_rows": n}}.

    A record is one bracketed interval: one kernel launch, or for the sparse
    attention kernel the launches of one call (its work goes out in rounds of
    one resident wave).
    """
    n = lib().zebra_profile_report(None, 0)
    buf = ctypes.create_string_buffer(int(n) + 1)
    lib().zebra_profile_report(buf, len(buf))
    rep = {"kernels": {}, "launches": {}, "logits": {}}
    for line in buf.value.decode().splitlines():
        parts = line.split()
        if parts[0] == "kernel":
            rep["kernels"][parts[1]] = (int(parts[2]), float(parts[3]))
            rep["launches"][parts[1]] = int(parts[4])
        elif parts[0] == "logits":
            rep["logits"][parts[1]] = int(parts[2])
    return rep

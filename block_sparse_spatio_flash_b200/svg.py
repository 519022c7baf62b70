"""Thin ctypes binding of libsvgattn (include/svg.h). Argument marshalling only.

Every function has the name of the C entry point it calls and raises ``SvgError`` when the
entry point returns a negative code. Tensors are torch tensors already on the GPU; the
library receives their raw device pointers and the current CUDA stream. Importing this
module loads the CUDA library and fails loudly when it has not been built: there is no CPU
or fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

# SVG_CHECKED=1 loads the checked build (device-side bounds checks, svg_checks_failed).
_LIB_NAME = "libsvgattn_checked.so" if os.environ.get("SVG_CHECKED") == "1" else "libsvgattn.so"
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", _LIB_NAME)
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing; build it with `python -m block_sparse_spatio_flash_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

SVG_OK = 0
SVG_ERR_ARG = -1
SVG_ERR_UNSUPPORTED = -2
SVG_ERR_CUDA = -3
SVG_ERR_TIMEOUT = -4
SVG_ERR_WORKSPACE = -5
SVG_ROUTE_SPATIAL, SVG_ROUTE_TEMPORAL = 0, 1
SVG_MASK_EXACT, SVG_MASK_ROUNDED = 0, 1
SVG_LAYOUT_SINK_PREFIX, SVG_LAYOUT_FULL_SPACE_MAJOR = 0, 1
SVG_MODE_SPLIT, SVG_MODE_NAIVE = 0, 1

LIB_PATH = _LIB_PATH


class svg_geom(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32)]


class svg_mask(ctypes.Structure):
    _fields_ = [("frame_window", ctypes.c_int32), ("spatial_band", ctypes.c_int32),
                ("sink_frames", ctypes.c_int32), ("variant", ctypes.c_int32), ("layout", ctypes.c_int32)]


class svg_tile(ctypes.Structure):
    _fields_ = [("bq", ctypes.c_int32), ("bk", ctypes.c_int32)]


class svg_tilemap_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("total_bytes", "cls", "cnt", "row_ptr", "cols", "pair_ptr",
                                               "pair_ent", "pair_cnt", "pair_order", "pair_grp")] + \
               [(n, ctypes.c_int32) for n in ("nq", "nk", "npairs")]


class svg_launch_opts(ctypes.Structure):
    _fields_ = [("order", ctypes.c_int32), ("d_cta_trace", ctypes.c_void_p), ("trace_ctas", ctypes.c_int32)]


SVG_ORDER_HEAD_MAJOR, SVG_ORDER_WORK = 0, 1


class svg_tilemap_summary_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in ("retained_exact", "retained_map", "n_full", "n_boundary",
                                               "n_empty", "visited_area", "pair_entries", "pair_half_tiles")]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_u8p = ctypes.POINTER(ctypes.c_uint8)
_sig = {
    "svg_version": (ctypes.c_int, []),
    "svg_checked_build": (ctypes.c_int, []),
    "svg_checks_failed": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _i32]),
    "svg_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "svg_last_cuda_error": (ctypes.c_char_p, []),
    "svg_tilemap_bytes": (_sz, [svg_geom, svg_tile]),
    "svg_tilemap_get_layout": (ctypes.c_int, [svg_geom, svg_tile, ctypes.POINTER(svg_tilemap_layout)]),
    "svg_build_tilemap": (ctypes.c_int, [svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp]),
    "svg_tilemap_summary": (ctypes.c_int, [_vp, ctypes.POINTER(svg_tilemap_summary_t), _vp]),
    "svg_permute": (ctypes.c_int, [_vp, _vp, _i32, _i64, _i32, _u8p, svg_geom, svg_mask, _i32, _vp]),
    "svg_attention_scratch_bytes": (_sz, []),
    "svg_attention_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p, _vp,
                                         _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp, _vp]),
    "svg_dense_attention_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _i32,
                                               _vp, _sz, _vp, _vp]),
    "svg_read_status": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_int32), _vp]),
    "svg_route_work_bytes": (_sz, [_i32, _i64, _i32, _i32]),
    "svg_route_heads": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, svg_geom, svg_mask, _vp, _i32,
                                       _vp, _sz, _vp, _vp, _vp]),
    "svg_attention_fwd_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p,
                                                 _vp, _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _vp]),
    "svg_attention_fwd_fused": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p, _vp,
                                               _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp, _vp]),
    "svg_attention_fwd_qk8": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p, _vp,
                                             _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp, _vp]),
    "svg_attention_fwd_ex": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p, _vp,
                                            _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp,
                                            ctypes.POINTER(svg_launch_opts), _vp]),
    "svg_test_attention_fwd_stall": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p,
                                                    _vp, _vp, svg_geom, svg_mask, svg_tile, _i32, _vp, _sz, _vp, _vp]),
    "svg_attention_host_buffer_bytes": (_sz, [_i64, _i32, _i32]),
    "svg_attention_fwd_host": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i32, _i64, _i32, ctypes.c_float, _u8p, _vp, _vp,
                                              svg_geom, svg_mask, svg_tile, _i32, _i32, _vp, _sz]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


class SvgError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        detail = f"; last CUDA error: {svg_last_cuda_error()}" if code == SVG_ERR_CUDA else ""
        super().__init__(f"{where}: {svg_error_string(code)} (code {code}){detail}")


def _check(code: int, where: str) -> int:
    if code < 0:
        raise SvgError(code, where)
    return code


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _routes(routes: Sequence[int]):
    arr = (ctypes.c_uint8 * len(routes))(*[int(r) for r in routes])
    return arr


def make_geom(frames, grid_h, grid_w) -> svg_geom:
    return svg_geom(frames, grid_h, grid_w)


def make_mask(frame_window, spatial_band, sink_frames=1, variant=SVG_MASK_EXACT,
              layout=SVG_LAYOUT_SINK_PREFIX) -> svg_mask:
    return svg_mask(frame_window, spatial_band, sink_frames, variant, layout)


def make_tile(bq, bk) -> svg_tile:
    return svg_tile(bq, bk)


# ------------------------------------------------------------------------------ entry points
def svg_version() -> int:
    return _lib.svg_version()


def svg_checked_build() -> bool:
    return bool(_lib.svg_checked_build())


def svg_checks_failed(reset: bool = True) -> int:
    """Failed device-side bounds checks since the last reset (checked build; 0 otherwise)."""
    n = ctypes.c_uint32(0)
    _check(_lib.svg_checks_failed(ctypes.byref(n), 1 if reset else 0), "svg_checks_failed")
    return int(n.value)


def svg_error_string(code: int) -> str:
    return _lib.svg_error_string(code).decode()


def svg_last_cuda_error() -> str:
    return _lib.svg_last_cuda_error().decode()


def svg_tilemap_bytes(geom: svg_geom, tile: svg_tile) -> int:
    return int(_lib.svg_tilemap_bytes(geom, tile))


def svg_tilemap_get_layout(geom: svg_geom, tile: svg_tile) -> svg_tilemap_layout:
    out = svg_tilemap_layout()
    _check(_lib.svg_tilemap_get_layout(geom, tile, ctypes.byref(out)), "svg_tilemap_get_layout")
    return out


def svg_build_tilemap(geom: svg_geom, mask: svg_mask, tile: svg_tile, route: int, ws: torch.Tensor,
                      stream=None) -> None:
    _check(_lib.svg_build_tilemap(geom, mask, tile, route, _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "svg_build_tilemap")


def svg_tilemap_summary(ws: torch.Tensor, stream=None) -> svg_tilemap_summary_t:
    out = svg_tilemap_summary_t()
    _check(_lib.svg_tilemap_summary(_ptr(ws), ctypes.byref(out), _stream(stream)), "svg_tilemap_summary")
    return out


def svg_permute(x: torch.Tensor, out: torch.Tensor, routes: Sequence[int], geom: svg_geom, mask: svg_mask,
                inverse: bool = False, stream=None) -> torch.Tensor:
    heads, tokens, d = x.shape
    _check(_lib.svg_permute(_ptr(x), _ptr(out), heads, tokens, d, _routes(routes), geom, mask,
                            1 if inverse else 0, _stream(stream)), "svg_permute")
    return out


def svg_attention_scratch_bytes() -> int:
    return int(_lib.svg_attention_scratch_bytes())


def svg_attention_fwd(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile, mode=SVG_MODE_SPLIT,
                      scratch=None, lse=None, scale: float = 0.0, status=None, stream=None) -> torch.Tensor:
    heads, tokens, d = q.shape
    _check(_lib.svg_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                  _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile, mode,
                                  _ptr(scratch), scratch.numel() * scratch.element_size(), _ptr(status),
                                  _stream(stream)), "svg_attention_fwd")
    return o


def svg_attention_fwd_fused(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile, mode=SVG_MODE_SPLIT,
                            scratch=None, lse=None, scale: float = 0.0, status=None, stream=None) -> torch.Tensor:
    """svg_attention_fwd on ORIGINAL-order q/k/v/o/lse for every head (permutation fused)."""
    heads, tokens, d = q.shape
    _check(_lib.svg_attention_fwd_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                        _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile, mode,
                                        _ptr(scratch), scratch.numel() * scratch.element_size(), _ptr(status),
                                        _stream(stream)), "svg_attention_fwd_fused")
    return o


def svg_attention_fwd_qk8(q8, k8, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile, mode=SVG_MODE_SPLIT,
                          scratch=None, lse=None, scale: float = 0.0, status=None, stream=None) -> torch.Tensor:
    """svg_attention_fwd with e4m3 Q and K (torch.float8_e4m3fn or uint8 [H, N, 128]); v / o bf16."""
    heads, tokens, d = v.shape
    _check(_lib.svg_attention_fwd_qk8(_ptr(q8), _ptr(k8), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                      _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile, mode,
                                      _ptr(scratch), scratch.numel() * scratch.element_size(), _ptr(status),
                                      _stream(stream)), "svg_attention_fwd_qk8")
    return o


def svg_attention_fwd_ex(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile, mode=SVG_MODE_SPLIT,
                         scratch=None, lse=None, scale: float = 0.0, status=None, order=SVG_ORDER_HEAD_MAJOR,
                         cta_trace=None, stream=None) -> torch.Tensor:
    """svg_attention_fwd with a scheduling order and an optional per-CTA trace (device int64 tensor
    [n, 4]: start ns, end ns, items, half-tiles per CTA)."""
    heads, tokens, d = q.shape
    opts = svg_launch_opts(order, None if cta_trace is None else cta_trace.data_ptr(),
                           0 if cta_trace is None else cta_trace.shape[0])
    if cta_trace is not None:
        _ptr(cta_trace)
    _check(_lib.svg_attention_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                     _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile, mode,
                                     _ptr(scratch), scratch.numel() * scratch.element_size(), _ptr(status),
                                     ctypes.byref(opts), _stream(stream)), "svg_attention_fwd_ex")
    return o


def svg_test_attention_fwd_stall(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile,
                                 mode=SVG_MODE_SPLIT, scratch=None, lse=None, scale: float = 0.0, status=None,
                                 stream=None) -> torch.Tensor:
    """Test hook: svg_attention_fwd whose launch waits on a barrier nothing completes and ends with
    SVG_ERR_TIMEOUT in its status word after the wait limit."""
    heads, tokens, d = q.shape
    _check(_lib.svg_test_attention_fwd_stall(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                             _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile,
                                             mode, _ptr(scratch), scratch.numel() * scratch.element_size(),
                                             _ptr(status), _stream(stream)), "svg_test_attention_fwd_stall")
    return o


def svg_dense_attention_fwd(q, k, v, o, bk=128, scratch=None, lse=None, scale: float = 0.0, status=None,
                            stream=None) -> torch.Tensor:
    heads, tokens, d = q.shape
    _check(_lib.svg_dense_attention_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                        bk, _ptr(scratch), scratch.numel() * scratch.element_size(), _ptr(status),
                                        _stream(stream)), "svg_dense_attention_fwd")
    return o


def svg_attention_fwd_noalloc(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile,
                              mode=SVG_MODE_SPLIT, lse=None, scale: float = 0.0, status=None,
                              stream=None) -> torch.Tensor:
    """svg_attention_fwd without a scratch argument: the library's static device scratch is
    used instead (shared by every call on the device; overlapping calls race)."""
    heads, tokens, d = q.shape
    _check(_lib.svg_attention_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), heads, tokens, d, scale,
                                          _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile,
                                          mode, _ptr(status), _stream(stream)), "svg_attention_fwd_noalloc")
    return o


def _hptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("expected a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def svg_attention_host_buffer_bytes(tokens: int, d: int, chunk_heads: int) -> int:
    return int(_lib.svg_attention_host_buffer_bytes(tokens, d, chunk_heads))


def svg_attention_fwd_host(q, k, v, o, routes, ws_spatial, ws_temporal, geom, mask, tile, buf, chunk_heads=1,
                           mode=SVG_MODE_SPLIT, scale: float = 0.0) -> torch.Tensor:
    """End to end on host tensors (q/k/v/o: CPU [H, N, d] bf16, original order; pinned memory
    overlaps the copies with compute). buf: device uint8 tensor of
    svg_attention_host_buffer_bytes(N, d, min(chunk_heads, H)) bytes. Synchronous."""
    heads, tokens, d = q.shape
    _check(_lib.svg_attention_fwd_host(_hptr(q), _hptr(k), _hptr(v), _hptr(o), heads, tokens, d, scale,
                                       _routes(routes), _ptr(ws_spatial), _ptr(ws_temporal), geom, mask, tile, mode,
                                       chunk_heads, _ptr(buf), buf.numel() * buf.element_size()),
           "svg_attention_fwd_host")
    return o


def svg_route_work_bytes(heads: int, tokens: int, d: int, n_rows: int) -> int:
    return int(_lib.svg_route_work_bytes(heads, tokens, d, n_rows))


def svg_route_heads(q, k, v, geom, mask, rows, route, err=None, work=None, scale: float = 0.0,
                    stream=None) -> torch.Tensor:
    """Route every head to the spatial or temporal mask from sampled rows (device tensors:
    q/k/v [H, N, d] bf16 original order, rows int32, route uint8 [H], err float32 [H, 2])."""
    heads, tokens, d = q.shape
    if work is None:
        work = torch.empty(svg_route_work_bytes(heads, tokens, d, rows.numel()), dtype=torch.uint8, device=q.device)
    _check(_lib.svg_route_heads(_ptr(q), _ptr(k), _ptr(v), heads, tokens, d, scale, geom, mask, _ptr(rows),
                                rows.numel(), _ptr(work), work.numel() * work.element_size(), _ptr(route),
                                _ptr(err), _stream(stream)), "svg_route_heads")
    return route


def svg_read_status(scratch_or_status: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(_lib.svg_read_status(_ptr(scratch_or_status), ctypes.byref(v), _stream(stream)), "svg_read_status")
    return int(v.value)


# ------------------------------------------------------------------------------ small helpers
def alloc_workspace(geom: svg_geom, tile: svg_tile, device="cuda") -> torch.Tensor:
    """A device buffer for one tile map (uint8, 256-byte aligned by the caching allocator)."""
    n = svg_tilemap_bytes(geom, tile)
    if n == 0:
        raise SvgError(SVG_ERR_ARG, "svg_tilemap_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_scratch(device="cuda") -> torch.Tensor:
    return torch.empty(svg_attention_scratch_bytes(), dtype=torch.uint8, device=device)


def tilemap_arrays(ws: torch.Tensor, geom: svg_geom, tile: svg_tile) -> dict:
    """Views of the arrays inside a built tile-map workspace (device tensors)."""
    L = svg_tilemap_get_layout(geom, tile)
    nq, nk, np_ = L.nq, L.nk, L.npairs

    def u32(off, n):
        return ws[off: off + 4 * n].view(torch.int32)

    return {
        "cls": ws[L.cls: L.cls + nq * nk].view(nq, nk),
        "cnt": u32(L.cnt, nq * nk).view(nq, nk),
        "row_ptr": u32(L.row_ptr, nq + 1),
        "cols": u32(L.cols, nq * nk),
        "pair_ptr": u32(L.pair_ptr, np_ + 1),
        "pair_ent": u32(L.pair_ent, np_ * nk),
        "pair_cnt": u32(L.pair_cnt, 2 * np_).view(np_, 2),
        "pair_order": u32(L.pair_order, np_),
        "pair_grp": u32(L.pair_grp, 2 * np_).view(np_, 2),
        "nq": nq, "nk": nk, "npairs": np_,
    }

"""Host-only checks of the C ABI: the library loads, exports every entry point that
include/svg.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svg.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(svg_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def svg():
    from block_sparse_spatio_flash_b200 import build
    build.build()
    from block_sparse_spatio_flash_b200 import svg as mod
    return mod


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("svg_build_tilemap", "svg_permute", "svg_attention_fwd", "svg_dense_attention_fwd",
              "svg_tilemap_bytes", "svg_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol(svg):
    lib = ctypes.CDLL(svg.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_has_no_torch_dependency(svg):
    import subprocess
    out = subprocess.run(["ldd", svg.LIB_PATH], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out


def test_error_strings(svg):
    for code in (0, -1, -2, -3, -4, -5):
        assert svg.svg_error_string(code)
    assert "unknown" in svg.svg_error_string(-99)
    assert svg.svg_version() >= 10000


def test_tilemap_layout_sizes(svg):
    g = svg.make_geom(21, 45, 80)
    for bq, bk in [(128, 128), (256, 64), (512, 128), (64, 64)]:
        t = svg.make_tile(bq, bk)
        L = svg.svg_tilemap_get_layout(g, t)
        n = 21 * 45 * 80
        assert L.nq == -(-n // bq) and L.nk == -(-n // bk) and L.npairs == -(-n // 256)
        assert L.total_bytes == svg.svg_tilemap_bytes(g, t)
        offs = [L.cls, L.cnt, L.row_ptr, L.cols, L.pair_ptr, L.pair_ent, L.pair_cnt, L.pair_order, L.pair_grp]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert L.cnt - L.cls >= L.nq * L.nk and L.pair_ent - L.pair_ptr >= 4 * (L.npairs + 1)
        assert L.pair_grp >= L.pair_order + 4 * L.npairs and L.total_bytes >= L.pair_grp + 8 * L.npairs


def test_bad_tile_and_geometry_rejected(svg):
    g = svg.make_geom(4, 8, 16)
    assert svg.svg_tilemap_bytes(g, svg.make_tile(96, 64)) == 0
    assert svg.svg_tilemap_bytes(svg.make_geom(0, 8, 16), svg.make_tile(64, 64)) == 0
    lib = ctypes.CDLL(svg.LIB_PATH)
    m = svg.make_mask(1, 16)
    # bad route / mask / tile / workspace: rejected before any device work
    assert lib.svg_build_tilemap(g, m, svg.make_tile(64, 64), 2, ctypes.c_void_p(256), 1 << 30, None) == -1
    assert lib.svg_build_tilemap(g, svg.make_mask(-1, 16), svg.make_tile(64, 64), 0,
                                 ctypes.c_void_p(256), 1 << 30, None) == -1
    assert lib.svg_build_tilemap(g, svg.make_mask(1, 16, sink_frames=5), svg.make_tile(64, 64), 0,
                                 ctypes.c_void_p(256), 1 << 30, None) == -1
    assert lib.svg_build_tilemap(g, m, svg.make_tile(64, 32), 0, ctypes.c_void_p(256), 1 << 30, None) == -2
    assert lib.svg_build_tilemap(g, m, svg.make_tile(64, 64), 0, None, 1 << 30, None) == -5
    assert lib.svg_build_tilemap(g, m, svg.make_tile(64, 64), 0, ctypes.c_void_p(256), 16, None) == -5
    assert lib.svg_build_tilemap(g, m, svg.make_tile(64, 64), 0, ctypes.c_void_p(257), 1 << 30, None) == -5


def test_attention_argument_checks(svg):
    lib = ctypes.CDLL(svg.LIB_PATH)
    g, m, t = svg.make_geom(4, 8, 16), svg.make_mask(1, 16), svg.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    p = ctypes.c_void_p(1 << 20)
    f = lib.svg_attention_fwd
    f.argtypes = svg._sig["svg_attention_fwd"][1]
    # null tensors, misaligned tensors, bad head count, bad d
    assert f(None, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -1
    assert f(ctypes.c_void_p((1 << 20) + 2), p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256,
             None, None) == -1
    assert f(p, p, p, p, None, 0, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -1
    assert f(p, p, p, p, None, 2, 512, 96, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -2
    # scratch missing or too small
    assert f(p, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, None, 256, None, None) == -1
    assert f(p, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 8, None, None) == -1
    d = lib.svg_dense_attention_fwd
    d.argtypes = svg._sig["svg_dense_attention_fwd"][1]
    assert d(p, p, p, None, None, 2, 512, 64, 0.0, 128, p, 256, None, None) == -1
    assert d(p, p, p, p, None, 2, 512, 64, 0.0, 32, p, 256, None, None) == -2


def test_permute_argument_checks(svg):
    lib = ctypes.CDLL(svg.LIB_PATH)
    f = lib.svg_permute
    f.argtypes = svg._sig["svg_permute"][1]
    g, m = svg.make_geom(4, 8, 16), svg.make_mask(1, 16)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 30)
    assert f(a, b, 2, 511, 64, routes, g, m, 0, None) == -1           # tokens != frames*h*w
    assert f(a, a, 2, 512, 64, routes, g, m, 0, None) == -1           # in == out
    assert f(a, b, 2, 512, 48, routes, g, m, 0, None) == -2           # d
    assert f(a, b, 2, 512, 64, routes, g, m, 2, None) == -1           # inverse flag
    bad = (ctypes.c_uint8 * 2)(0, 7)
    assert f(a, b, 2, 512, 64, bad, g, m, 0, None) == -1              # route value


def test_route_argument_checks(svg):
    """Head routing: workspace size and argument rejections, all before any device work."""
    lib = ctypes.CDLL(svg.LIB_PATH)
    g, m = svg.make_geom(4, 8, 16), svg.make_mask(1, 16)
    wb = svg.svg_route_work_bytes
    assert wb(2, 512, 64, 0) == 0 and wb(0, 512, 64, 8) == 0 and wb(2, 512, 96, 8) == 0
    # status block + per-row errors (rounded to 256 bytes) + one chunk state of 3 x (d + 2) floats per row
    assert wb(2, 512, 64, 8) == 256 + 256 + 2 * 8 * 1 * 3 * 66 * 4
    # 75,600 keys: 37 chunks of 2,048 would exceed the cap of 32
    assert wb(10, 75600, 128, 64) == 256 + (10 * 64 * 3 * 4 + 255) // 256 * 256 + 10 * 64 * 32 * 3 * 130 * 4
    f = lib.svg_route_heads
    f.argtypes = svg._sig["svg_route_heads"][1]
    p, rt = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)
    ok_bytes = wb(2, 512, 64, 8)
    assert f(None, p, p, 2, 512, 64, 0.0, g, m, p, 8, p, ok_bytes, rt, None, None) == -1       # null q
    assert f(p, p, p, 2, 512, 64, 0.0, g, m, None, 8, p, ok_bytes, rt, None, None) == -1       # null rows
    assert f(p, p, p, 2, 512, 64, 0.0, g, m, p, 8, p, ok_bytes, None, None, None) == -1        # null route
    assert f(ctypes.c_void_p((1 << 20) + 8), p, p, 2, 512, 64, 0.0, g, m, p, 8, p, ok_bytes, rt, None,
             None) == -1                                                                    # misaligned q
    assert f(p, p, p, 2, 512, 64, 0.0, g, m, p, 8, ctypes.c_void_p((1 << 20) + 64), ok_bytes, rt, None,
             None) == -1                                                                    # misaligned work
    assert f(p, p, p, 2, 511, 64, 0.0, g, m, p, 8, p, ok_bytes, rt, None, None) == -1         # tokens mismatch
    assert f(p, p, p, 2, 512, 64, 0.0, g, m, p, 0, p, ok_bytes, rt, None, None) == -1         # no rows
    assert f(p, p, p, 2, 512, 96, 0.0, g, m, p, 8, p, ok_bytes, rt, None, None) == -2         # d
    assert f(p, p, p, 2, 512, 64, 0.0, g, m, p, 8, p, ok_bytes - 4, rt, None, None) == -5     # workspace


def test_host_entry_argument_checks(svg):
    """Host-buffer entry point: buffer size rule and rejections before any device work."""
    lib = ctypes.CDLL(svg.LIB_PATH)
    hb = svg.svg_attention_host_buffer_bytes
    one = (512 * 64 * 2 + 255) // 256 * 256
    assert hb(512, 64, 1) == 3 * 7 * one + 256 + 256
    assert hb(512, 96, 1) == 0 and hb(512, 64, 0) == 0 and hb(0, 64, 1) == 0
    f = lib.svg_attention_fwd_host
    f.argtypes = svg._sig["svg_attention_fwd_host"][1]
    g, m, t = svg.make_geom(4, 8, 16), svg.make_mask(1, 16), svg.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    hbuf = ctypes.create_string_buffer(16)
    h = ctypes.cast(hbuf, ctypes.c_void_p)
    dbuf = ctypes.c_void_p(1 << 20)
    need = hb(512, 64, 2)
    assert f(None, h, h, h, 2, 512, 64, 0.0, routes, dbuf, dbuf, g, m, t, 0, 2, dbuf, need) == -1   # null q
    assert f(h, h, h, h, 2, 512, 64, 0.0, routes, dbuf, dbuf, g, m, t, 0, 0, dbuf, need) == -1      # chunk 0
    assert f(h, h, h, h, 2, 511, 64, 0.0, routes, dbuf, dbuf, g, m, t, 0, 2, dbuf, need) == -1      # tokens
    assert f(h, h, h, h, 2, 512, 64, 0.0, routes, dbuf, dbuf, g, m, t, 0, 2,
             ctypes.c_void_p((1 << 20) + 16), need) == -1                                          # alignment
    assert f(h, h, h, h, 2, 512, 96, 0.0, routes, dbuf, dbuf, g, m, t, 0, 2, dbuf, need) == -2      # d
    assert f(h, h, h, h, 2, 512, 64, 0.0, routes, dbuf, dbuf, g, m, t, 7, 2, dbuf, need) == -1      # mode
    assert f(h, h, h, h, 2, 512, 64, 0.0, routes, dbuf, dbuf, g, m, t, 0, 2, dbuf, need - 1) == -5  # buffer
    bad = (ctypes.c_uint8 * 2)(0, 3)
    assert f(h, h, h, h, 2, 512, 64, 0.0, bad, dbuf, dbuf, g, m, t, 0, 2, dbuf, need) == -1         # route


def test_qk8_argument_checks(svg):
    lib = ctypes.CDLL(svg.LIB_PATH)
    f = lib.svg_attention_fwd_qk8
    f.argtypes = svg._sig["svg_attention_fwd_qk8"][1]
    g, m, t = svg.make_geom(4, 8, 16), svg.make_mask(1, 16), svg.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    p = ctypes.c_void_p(1 << 20)
    assert f(p, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -2   # d = 64
    assert f(None, p, p, p, None, 2, 512, 128, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -1  # null q8


def test_fused_rejects_more_rows_than_a_tma_coordinate_holds(svg):
    """The fused-order call gathers rows of a [heads * tokens, d] view with signed 32-bit row
    coordinates: heads * tokens above 2^31 - 1 is rejected before any device work."""
    lib = ctypes.CDLL(svg.LIB_PATH)
    f = lib.svg_attention_fwd_fused
    f.argtypes = svg._sig["svg_attention_fwd_fused"][1]
    g, m, t = svg.make_geom(32, 256, 256), svg.make_mask(1, 16), svg.make_tile(128, 128)
    tokens = 32 * 256 * 256  # 2^21
    p = ctypes.c_void_p(1 << 20)
    routes = (ctypes.c_uint8 * 1024)(*([1] * 1024))
    assert f(p, p, p, p, None, 1024, tokens, 128, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -2


def test_stall_test_entry_checks_arguments_like_the_regular_call(svg):
    lib = ctypes.CDLL(svg.LIB_PATH)
    f = lib.svg_test_attention_fwd_stall
    f.argtypes = svg._sig["svg_test_attention_fwd_stall"][1]
    g, m, t = svg.make_geom(4, 8, 16), svg.make_mask(1, 16), svg.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    p = ctypes.c_void_p(1 << 20)
    assert f(None, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -1
    assert f(p, p, p, p, None, 2, 512, 96, 0.0, routes, p, p, g, m, t, 0, p, 256, None, None) == -2


def test_extended_entry_argument_checks(svg):
    """svg_attention_fwd_ex: a missing options struct, an unknown order and a trace buffer without
    entries or misaligned are rejected before any device work."""
    lib = ctypes.CDLL(svg.LIB_PATH)
    f = lib.svg_attention_fwd_ex
    f.argtypes = svg._sig["svg_attention_fwd_ex"][1]
    g, m, t = svg.make_geom(4, 8, 16), svg.make_mask(1, 16), svg.make_tile(64, 64)
    routes = (ctypes.c_uint8 * 2)(0, 1)
    p = ctypes.c_void_p(1 << 20)
    args = (p, p, p, p, None, 2, 512, 64, 0.0, routes, p, p, g, m, t, 0, p, 256, None)
    assert f(*args, None, None) == -1
    assert f(*args, ctypes.byref(svg.svg_launch_opts(7, None, 0)), None) == -1
    assert f(*args, ctypes.byref(svg.svg_launch_opts(svg.SVG_ORDER_WORK, (1 << 20), 0)), None) == -1
    assert f(*args, ctypes.byref(svg.svg_launch_opts(svg.SVG_ORDER_WORK, (1 << 20) + 4, 148)), None) == -1

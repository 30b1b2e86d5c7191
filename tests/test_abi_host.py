"""Host-side checks of the C-ABI library: it loads, exports every entry point
the header declares, computes packed sizes in closed form, and rejects bad
arguments before touching a GPU.  No kernel runs here."""
import ctypes
import json
import os
import re

import pytest

from gemm_w4a16_b200 import build as lib_build
from gemm_w4a16_b200 import w4a16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a16.h")
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def L():
    lib_build.build()
    return w4a16.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a16_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 8
    assert set(names) == set(w4a16.EXPORTED)
    for n in names:
        assert hasattr(L, n), n


def test_debug_library_exports_the_same_symbols(L):
    """The index-check build (libw4a16_debug.so) is the same API."""
    import ctypes

    assert os.path.exists(w4a16.DEBUG_LIB_PATH)
    D = ctypes.CDLL(w4a16.DEBUG_LIB_PATH)
    for n in declared_functions():
        assert hasattr(D, n), n


def test_library_switch_restores_the_main_library(L):
    """w4a16.library(DEBUG_LIB_PATH) routes the binding through the
    index-check build inside the block (same host-side answers) and back to
    libw4a16.so after it."""
    main_path = w4a16.LIB_PATH
    sizes = w4a16.packed_sizes(12288, 4096)
    path = w4a16.select_path(12288, 4096, 16)
    with w4a16.library(w4a16.DEBUG_LIB_PATH):
        assert w4a16.lib()._name == w4a16.DEBUG_LIB_PATH
        assert w4a16.packed_sizes(12288, 4096) == sizes
        assert w4a16.select_path(12288, 4096, 16) == path
        assert w4a16.status_string(w4a16.ERR_BOUNDS)
    assert w4a16.LIB_PATH == main_path
    assert w4a16.lib()._name == main_path


def test_status_strings(L):
    for code in range(7):
        assert w4a16.status_string(code)
    assert w4a16.status_string(99) == "unknown status"


def test_packed_sizes_closed_form(L):
    for M, K in [(256, 256), (12288, 4096), (4096, 11008), (128256, 4096), (200, 384), (1, 128)]:
        wq, s, z = w4a16.packed_sizes(M, K)
        mp = -(-M // 128) * 128
        assert wq == mp * K // 2
        assert s == mp * (K // 128) * 2
        assert z == mp * (K // 128) // 2


def test_pages_footprint_facts(L):
    """Section 3.1 of the PerfXLLM page: int4 is 1/4 of fp16 and scale+zero
    add about 1 %; 7B parameters in fp16 take about 14 GB."""
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    G = facts["group_size"]["value"]
    M, K = facts["gemm_sweep_M"]["value"], facts["gemm_sweep_K"]["value"]
    assert G == 128 and (M, K) == (12288, 4096)
    wq, s, z = w4a16.packed_sizes(M, K, G)
    fp16 = M * K * 2
    assert wq / fp16 == facts["int4_vs_fp16_ratio"]["value"]
    overhead = (s + z) / fp16
    assert abs(overhead - facts["scale_zero_overhead_fraction"]["value"]) < 0.001
    assert abs(overhead - 2.5 / 256) < 1e-12
    assert abs(facts["fp16_7b_bytes"]["params"] * 2 - facts["fp16_7b_bytes"]["value"]) < 0.05e9


def test_rejects_bad_arguments_without_launching(L):
    bad = ctypes.c_void_p(0x1001)      # never dereferenced: checks fail first
    good = ctypes.c_void_p(0x10000)
    null = ctypes.c_void_p(0)
    g = L.w4a16_gemm_ex
    args = lambda **kw: [kw.get("wq", good), good, good, kw.get("x", good), kw.get("y", good),
                         kw.get("M", 256), kw.get("K", 256), kw.get("N", 1),
                         kw.get("group", 128), kw.get("path", 0), null]
    assert g(*args(wq=null)) == w4a16.ERR_INVALID_ARG
    assert g(*args(y=null)) == w4a16.ERR_INVALID_ARG
    assert g(*args(M=0)) == w4a16.ERR_INVALID_ARG
    assert g(*args(N=0)) == w4a16.ERR_INVALID_ARG
    assert g(*args(N=-3)) == w4a16.ERR_INVALID_ARG
    assert g(*args(K=-128)) == w4a16.ERR_INVALID_ARG
    assert g(*args(path=7)) == w4a16.ERR_INVALID_ARG
    assert g(*args(group=64)) == w4a16.ERR_UNSUPPORTED
    assert g(*args(K=200)) == w4a16.ERR_UNSUPPORTED
    assert g(*args(x=bad)) == w4a16.ERR_MISALIGNED
    assert g(*args(wq=bad)) == w4a16.ERR_MISALIGNED
    assert L.w4a16_gemm(good, good, good, good, bad, 256, 256, 1, 128, null) == w4a16.ERR_MISALIGNED
    assert L.w4a16_dequant_debug(good, good, good, null, 256, 256, 128, null) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_dequant_debug(good, good, good, bad, 256, 256, 128, null) == w4a16.ERR_MISALIGNED
    q3 = L.w4a16_gemm_qkv
    assert q3(good, good, good, good, null, 128, 64, 64, 256, 1, 128, good, null, good, null) == \
        w4a16.ERR_INVALID_ARG
    assert q3(good, good, good, good, null, 0, 64, 64, 256, 1, 128, good, good, good, null) == \
        w4a16.ERR_INVALID_ARG
    assert q3(good, good, good, good, null, 128, 64, 64, 200, 1, 128, good, good, good, null) == \
        w4a16.ERR_UNSUPPORTED
    assert q3(good, good, good, good, null, 128, 64, 64, 256, 1, 128, good, bad, good, null) == \
        w4a16.ERR_MISALIGNED
    assert q3(good, good, good, good, ctypes.c_void_p(0x10001), 128, 64, 64, 256, 1, 128, good, good, good,
              null) == w4a16.ERR_MISALIGNED
    assert L.w4a16_quantize(null, 256, 256, 128, good, good, good, null) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_quantize(good, 256, 200, 128, good, good, good, null) == w4a16.ERR_UNSUPPORTED
    assert L.w4a16_quantize(good, 256, 256, 64, good, good, good, null) == w4a16.ERR_UNSUPPORTED
    assert L.w4a16_quantize(good, 0, 256, 128, good, good, good, null) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_quantize(bad, 256, 256, 128, good, good, good, null) == w4a16.ERR_MISALIGNED
    assert L.w4a16_quantize(good, 256, 256, 128, bad, good, good, null) == w4a16.ERR_MISALIGNED
    assert L.w4a16_pack(good, good, good, 256, 256, 100, good, good, good, null) == w4a16.ERR_UNSUPPORTED
    assert L.w4a16_pack(good, good, null, 256, 256, 128, good, good, good, null) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_pack(good, good, good, 256, 256, 128, bad, good, good, null) == w4a16.ERR_MISALIGNED
    sz = ctypes.c_size_t()
    assert L.w4a16_packed_sizes(256, 256, 128, None, ctypes.byref(sz), ctypes.byref(sz)) == \
        w4a16.ERR_INVALID_ARG
    assert L.w4a16_device_status(null, None) == w4a16.ERR_INVALID_ARG
    L.w4a16_selftest_wait_timeout.argtypes = [ctypes.c_longlong, ctypes.c_void_p]
    assert L.w4a16_selftest_wait_timeout(-1, null) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_selftest_wait_timeout(1 << 40, null) == w4a16.ERR_INVALID_ARG


def test_add_rmsnorm_rejects_bad_arguments_without_launching(L):
    """Each call breaks one rule and must fail on the host (none may reach a
    launch: the addresses are not memory).  N = 2, K = 64: 256 bytes a row
    block; the fake buffers sit 64 KB apart."""
    p = lambda a: ctypes.c_void_p(a)
    h, d, g, r, x, null = 0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0
    f = L.w4a16_add_rmsnorm

    def call(h=h, d=d, g=g, eps=1e-6, N=2, K=64, r=r, x=x):
        return f(p(h), p(d), p(g), eps, N, K, p(r), p(x), p(null))

    assert call(h=null) == w4a16.ERR_INVALID_ARG
    assert call(g=null) == w4a16.ERR_INVALID_ARG
    assert call(x=null) == w4a16.ERR_INVALID_ARG
    assert call(N=0) == w4a16.ERR_INVALID_ARG
    assert call(K=0) == w4a16.ERR_INVALID_ARG
    assert call(eps=-1.0) == w4a16.ERR_INVALID_ARG
    assert call(eps=float("nan")) == w4a16.ERR_INVALID_ARG
    assert call(eps=float("inf")) == w4a16.ERR_INVALID_ARG
    assert call(K=60) == w4a16.ERR_UNSUPPORTED
    assert call(K=65536 + 8) == w4a16.ERR_UNSUPPORTED
    for name in ("h", "d", "g", "r", "x"):
        assert call(**{name: {"h": h, "d": d, "g": g, "r": r, "x": x}[name] + 8}) == w4a16.ERR_MISALIGNED
    assert call(x=h + 128) == w4a16.ERR_INVALID_ARG          # X inside h
    assert call(x=d + 240) == w4a16.ERR_INVALID_ARG          # X overlaps d's last bytes
    assert call(x=g) == w4a16.ERR_INVALID_ARG                # X on gamma
    assert call(x=r + 16) == w4a16.ERR_INVALID_ARG           # X inside r_out
    assert call(r=h + 16) == w4a16.ERR_INVALID_ARG           # r_out partly over h
    assert call(r=d - 16) == w4a16.ERR_INVALID_ARG           # r_out partly over d
    assert call(r=g) == w4a16.ERR_INVALID_ARG                # r_out on gamma


def test_overlapping_buffers_rejected_without_launching(L):
    """Outputs may not overlap inputs or each other.  M = K = 256, N = 2:
    packed codes 32 KB, scales 1 KB, zeros 256 B, X and Y 1 KB; every fake
    buffer sits 1 MB from the next, so the one overlap planted per call is the
    only one (and no call reaches a launch)."""
    p = lambda a: ctypes.c_void_p(a)
    wq, sc, zp, x, y, bias, yq, yk, yv = (k << 20 for k in range(1, 10))
    null = p(0)
    ex = lambda Y: L.w4a16_gemm_ex(p(wq), p(sc), p(zp), p(x), p(Y), 256, 256, 2, 128, 0, null)
    assert ex(x) == w4a16.ERR_INVALID_ARG                    # Y on X
    assert ex(wq + 0x1000) == w4a16.ERR_INVALID_ARG          # Y inside the packed codes
    assert ex(zp + 0x80) == w4a16.ERR_INVALID_ARG            # Y over the zeros
    assert L.w4a16_gemm(p(wq), p(sc), p(zp), p(x), p(sc + 0x100), 256, 256, 2, 128, null) == \
        w4a16.ERR_INVALID_ARG                                # Y over the scales

    def qkv(Yq=yq, Yk=yk, Yv=yv, B=bias):                    # Mq = 128, Mk = Mv = 64
        return L.w4a16_gemm_qkv(p(wq), p(sc), p(zp), p(x), p(B), 128, 64, 64, 256, 2, 128,
                                p(Yq), p(Yk), p(Yv), null)

    assert qkv(Yk=yq + 256) == w4a16.ERR_INVALID_ARG         # Yk inside Yq (512 B)
    assert qkv(Yv=x + 16) == w4a16.ERR_INVALID_ARG           # Yv over X
    assert qkv(Yq=bias + 256) == w4a16.ERR_INVALID_ARG       # Yq over the bias (512 B)
    assert qkv(Yv=wq + 0x2000) == w4a16.ERR_INVALID_ARG      # Yv inside the packed codes
    # quantiser: W 128 KB, q 64 KB, scales 1 KB, zeros 512 B
    assert L.w4a16_quantize(p(wq), 256, 256, 128, p(wq + 0x10000), p(sc), p(zp), null) == \
        w4a16.ERR_INVALID_ARG                                # q inside W
    assert L.w4a16_quantize(p(wq), 256, 256, 128, p(x), p(x + 0x1000), p(zp), null) == \
        w4a16.ERR_INVALID_ARG                                # scales inside q
    # pack: inputs q 64 KB, scales 1 KB, zeros 512 B; outputs 32 KB, 1 KB, 256 B
    assert L.w4a16_pack(p(x), p(sc), p(zp), 256, 256, 128, p(x + 0x100), p(yq), p(yk), null) == \
        w4a16.ERR_INVALID_ARG                                # packed codes over q
    assert L.w4a16_pack(p(x), p(sc), p(zp), 256, 256, 128, p(yq), p(yq + 0x400), p(yk), null) == \
        w4a16.ERR_INVALID_ARG                                # packed scales inside packed codes
    assert L.w4a16_dequant_debug(p(wq), p(sc), p(zp), p(sc), 256, 256, 128, null) == \
        w4a16.ERR_INVALID_ARG                                # W_out on the scales


def test_select_path_is_monotone_in_n(L):
    assert w4a16.select_path(0, 4096, 1) == -1
    assert w4a16.select_path(4096, 100, 1) == -1
    assert w4a16.select_path(12288, 4096, 1) == w4a16.PATH_GEMV
    paths = [w4a16.select_path(12288, 4096, n) for n in (1, 2, 4, 8, 16, 64, 256, 4096)]
    first_tc = paths.index(w4a16.PATH_TC) if w4a16.PATH_TC in paths else len(paths)
    assert all(p == w4a16.PATH_GEMV for p in paths[:first_tc])
    assert all(p == w4a16.PATH_TC for p in paths[first_tc:])


def test_workspace_size_closed_form(L):
    """Workspace of the split decode path: one counter per (row block, lane
    quarter), rounded up to 256 bytes, then per CTA two fp32 partials of
    128 rows x N tokens; G = min(SMs, units) CTAs.  Zero where the automatic
    path needs a workspace (N > 64)."""
    for M, K in [(12288, 4096), (4096, 11008), (200, 384), (128256, 4096)]:
        nb, U = -(-M // 128), -(-M // 128) * (K // 128)
        cnt = -(-nb * 16 // 256) * 256
        one = w4a16.workspace_size(M, K, 1)
        G = (one - cnt) // 1024
        assert (one - cnt) % 1024 == 0 and 1 <= G <= U
        for N in (2, 7, 16, 17, 64):
            assert w4a16.workspace_size(M, K, N) == cnt + G * 2 * N * 128 * 4
        assert w4a16.workspace_size(M, K, 65) == 0
    n = ctypes.c_size_t()
    assert L.w4a16_gemm_workspace_size(256, 256, 1, 128, None) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_gemm_workspace_size(256, 256, 0, 128, ctypes.byref(n)) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_gemm_workspace_size(256, 200, 1, 128, ctypes.byref(n)) == w4a16.ERR_UNSUPPORTED
    assert L.w4a16_gemm_workspace_size(256, 256, 1, 64, ctypes.byref(n)) == w4a16.ERR_UNSUPPORTED


def test_select_path_with_workspace(L):
    """A workspace does not change the automatic choice: the decode kernel up
    to GEMV_MAX_TOKENS, the tile kernel above."""
    for N in (1, 2, 5, w4a16.GEMV_MAX_TOKENS):
        assert w4a16.select_path_ws(12288, 4096, N) == w4a16.PATH_GEMV
        assert w4a16.select_path(12288, 4096, N) == w4a16.PATH_GEMV
    for N in (w4a16.GEMV_MAX_TOKENS + 1, 64, 4096):
        assert w4a16.select_path_ws(12288, 4096, N) == w4a16.PATH_TC
    # Up to 8192 rows (64 row blocks) two decode launches beat the tile kernel.
    for M in (4096, 6144, 8192):
        assert w4a16.select_path(M, 4096, 2 * w4a16.GEMV_MAX_TOKENS) == w4a16.PATH_GEMV
        assert w4a16.select_path(M, 4096, 2 * w4a16.GEMV_MAX_TOKENS + 1) == w4a16.PATH_TC
    assert w4a16.select_path(8320, 4096, 2 * w4a16.GEMV_MAX_TOKENS) == w4a16.PATH_TC
    assert w4a16.select_path_ws(12288, 100, 1) == -1


def test_workspace_entry_points_reject_bad_arguments_without_launching(L):
    """Each call breaks one rule and fails on the host.  M = K = 256, N = 2;
    fake buffers 1 MB apart; the workspace need is a few KB."""
    p = lambda a: ctypes.c_void_p(a)
    wq, sc, zp, x, y, ws, yq, yk, yv = (k << 20 for k in range(1, 10))
    null = p(0)
    need = w4a16.workspace_size(256, 256, 2)
    GT = w4a16.PATH_GEMV_TC

    def call(path=GT, W=ws, nbytes=need, flags=0, Y=y, N=2):
        return L.w4a16_gemm_ws(p(wq), p(sc), p(zp), p(x), p(Y), 256, 256, N, 128, path, p(W), nbytes,
                               flags, null)

    assert call(W=0, nbytes=0) == w4a16.ERR_INVALID_ARG          # forced split path, no workspace
    assert call(nbytes=need - 1) == w4a16.ERR_INVALID_ARG        # too small
    assert call(W=0, nbytes=64) == w4a16.ERR_INVALID_ARG         # size without a buffer
    assert call(flags=4) == w4a16.ERR_INVALID_ARG                # unknown flag
    assert call(path=4) == w4a16.ERR_INVALID_ARG
    assert call(W=ws + 8) == w4a16.ERR_MISALIGNED
    assert call(W=y - 16) == w4a16.ERR_INVALID_ARG               # workspace runs into Y
    assert call(W=x + 256) == w4a16.ERR_INVALID_ARG              # workspace on X
    assert call(W=wq + 0x100) == w4a16.ERR_INVALID_ARG           # workspace inside the codes
    assert call(N=65, nbytes=1 << 24) == w4a16.ERR_UNSUPPORTED   # more tokens than the kernel takes
    assert L.w4a16_gemm_ex(p(wq), p(sc), p(zp), p(x), p(y), 256, 256, 2, 128, GT, null) == \
        w4a16.ERR_INVALID_ARG                                    # no workspace on this entry point

    def qkv(W=ws, nbytes=need, Yv=yv, flags=0):
        return L.w4a16_gemm_qkv_ws(p(wq), p(sc), p(zp), p(x), null, 128, 64, 64, 256, 2, 128, p(yq), p(yk),
                                   p(Yv), p(W), nbytes, flags, null)

    assert qkv(W=yk + 128) == w4a16.ERR_INVALID_ARG              # workspace over Yk
    assert qkv(Yv=ws + 64) == w4a16.ERR_INVALID_ARG              # Yv inside the workspace
    assert qkv(flags=2) == w4a16.ERR_INVALID_ARG
    assert qkv(W=ws + 8) == w4a16.ERR_MISALIGNED


def test_gate_up_entry_points_reject_bad_arguments_without_launching(L):
    """Mi = 128 (weight 256 x 256), N = 2; fake buffers 1 MB apart."""
    p = lambda a: ctypes.c_void_p(a)
    wq, sc, zp, x, h, ws, q = (k << 20 for k in range(1, 8))
    null = p(0)
    pk = L.w4a16_pack_gate_up
    assert pk(p(q), p(sc), p(zp), 0, 256, 128, p(wq), p(ws), p(h), null) == w4a16.ERR_INVALID_ARG
    assert pk(p(q), p(sc), p(zp), 128, 200, 128, p(wq), p(ws), p(h), null) == w4a16.ERR_UNSUPPORTED
    assert pk(p(q), p(sc), p(zp), 128, 256, 128, p(wq + 8), p(ws), p(h), null) == w4a16.ERR_MISALIGNED
    assert pk(p(q), p(sc), p(zp), 128, 256, 128, p(q + 0x100), p(ws), p(h), null) == w4a16.ERR_INVALID_ARG
    g = L.w4a16_gemm_gate_up
    assert g(p(wq), p(sc), p(zp), p(x), null, 128, 256, 2, 128, null) == w4a16.ERR_INVALID_ARG
    assert g(p(wq), p(sc), p(zp), p(x), p(h), 0, 256, 2, 128, null) == w4a16.ERR_INVALID_ARG
    assert g(p(wq), p(sc), p(zp), p(x), p(h), 128, 256, 2, 64, null) == w4a16.ERR_UNSUPPORTED
    assert g(p(wq), p(sc), p(zp), p(x), p(h + 8), 128, 256, 2, 128, null) == w4a16.ERR_MISALIGNED
    assert g(p(wq), p(sc), p(zp), p(x), p(x + 64), 128, 256, 2, 128, null) == w4a16.ERR_INVALID_ARG
    assert g(p(wq), p(sc), p(zp), p(x), p(wq + 0x100), 128, 256, 2, 128, null) == w4a16.ERR_INVALID_ARG
    gw = L.w4a16_gemm_gate_up_ws
    need = w4a16.workspace_size(256, 256, 2)
    GT = w4a16.PATH_GEMV_TC
    assert gw(p(wq), p(sc), p(zp), p(x), p(h), 128, 256, 2, 128, GT, null, 0, 0, null) == w4a16.ERR_INVALID_ARG
    assert gw(p(wq), p(sc), p(zp), p(x), p(h), 128, 256, 2, 128, GT, p(ws), need - 1, 0, null) == \
        w4a16.ERR_INVALID_ARG
    assert gw(p(wq), p(sc), p(zp), p(x), p(h), 128, 256, 2, 128, GT, p(h + 64), need, 0, null) == \
        w4a16.ERR_INVALID_ARG                                    # workspace over H
    assert gw(p(wq), p(sc), p(zp), p(x), p(h), 128, 256, 2, 128, 9, p(ws), need, 0, null) == \
        w4a16.ERR_INVALID_ARG

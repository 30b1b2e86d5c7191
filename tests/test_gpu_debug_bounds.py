"""The index-check build, libw4a16_debug.so (-DW4A16_DEBUG_BOUNDS): the
decode kernel checks every access to the packed weights, the activations,
its shared-memory slices and its outputs against their extents and records a
failure in the device status word (W4A16_ERR_BOUNDS) instead of making the
access.  On valid launches every check passes: the status stays OK and the
results match the oracle, on ragged row blocks, K splits over clusters, the
4-way row split in one and in several waves, one and two 8-token blocks,
early weights, and the fused QKV, gate/up and normalising forms.  (No test
drives a check to fail: that would take an out-of-bounds launch.)"""
from __future__ import annotations

import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from gpu_util import assert_close, pack_problem, to_f64  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    import torch  # noqa: F401

    from gemm_w4a16_b200 import build, w4a16

    build.build()
    assert os.path.exists(w4a16.DEBUG_LIB_PATH), "libw4a16_debug.so was not built"
    with w4a16.library(w4a16.DEBUG_LIB_PATH):
        assert w4a16.lib()._name == w4a16.DEBUG_LIB_PATH
        yield


def _check_status():
    from gemm_w4a16_b200 import w4a16

    assert w4a16.device_status() == w4a16.OK


@pytest.mark.parametrize("M,K,N", [(200, 384, 1), (1500, 2048, 1), (1500, 2048, 5), (1000, 2048, 12),
                                   (4200, 2048, 16), (12288, 4096, 1), (4096, 11008, 1), (22016, 4096, 1),
                                   (4096, 4096, 16)])
@pytest.mark.parametrize("flags", [0, 1], ids=["plain", "early"])
def test_decode_checks_pass(M, K, N, flags):
    import oracle
    from gemm_w4a16_b200 import synth, w4a16

    p = synth.make_problem(M, K, N, seed=M + K + N)
    w, x = pack_problem(p)
    ws = w4a16.Workspace(x.device, w4a16.workspace_size(M, K, N))
    y = w4a16.gemm_ws(w, x, path=w4a16.PATH_GEMV, workspace=ws,
                      flags=w4a16.FLAG_EARLY_WEIGHTS if flags else 0)
    _check_status()
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x)
    assert_close(to_f64(y), ref, f"debug build M={M} K={K} N={N}")


@pytest.mark.parametrize("N", [1, 3, 12])
def test_fused_forms_checks_pass(N):
    import torch

    import oracle
    from gemm_w4a16_b200 import synth, w4a16

    # QKV split + bias.
    splits = (200, 72, 72)
    M, K = sum(splits), 384
    p = synth.make_problem(M, K, N, seed=50 + N)
    w, x = pack_problem(p)
    bias = torch.randn(M, device=x.device).half()
    outs = w4a16.gemm_qkv(w, x, splits, bias=bias)
    _check_status()
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x) + bias.double().cpu().numpy()[None, :]
    y = torch.cat(outs, dim=1)
    assert_close(to_f64(y), ref, f"debug build QKV N={N}")
    # SiLU(gate) * up.
    Mi = 100
    pg = synth.make_problem(2 * Mi, K, N, seed=60 + N)
    q, z, s, xg = (torch.from_numpy(pg.q).cuda(), torch.from_numpy(pg.zeros).cuda(),
                   torch.from_numpy(pg.scales.view(np.float16)).cuda(),
                   torch.from_numpy(pg.x.view(np.float16)).cuda())
    wg = w4a16.pack_gate_up(q, s, z)
    h = w4a16.gemm_gate_up(wg, xg)
    _check_status()
    assert_close(to_f64(h), oracle.gate_up(pg.q, pg.zeros, pg.scales, pg.x, Mi), f"debug build gate/up N={N}")


def test_normalising_prologue_checks_pass():
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    splits = (256, 128, 128)
    M, K, N = sum(splits), 1024, 4
    p = synth.make_problem(M, K, N, seed=77)
    w, _ = pack_problem(p)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    h = torch.randn((N, K), device="cuda", generator=gen).half()
    d = torch.randn((N, K), device="cuda", generator=gen).half()
    gamma = (1.0 + 0.1 * torch.randn(K, device="cuda", generator=gen)).half()
    r1 = torch.empty_like(h)
    outs = w4a16.add_rmsnorm_gemm_qkv(h, gamma, w, splits, d=d, r_out=r1)
    _check_status()
    r2, X = w4a16.add_rmsnorm(h, gamma, d=d, r_out=torch.empty_like(h))
    ref = w4a16.gemm_qkv(w, X, splits)
    _check_status()
    assert torch.equal(r1, r2)
    for a, b in zip(outs, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))

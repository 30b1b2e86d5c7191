"""GPU parity of the fused gate/up projection (w4a16_pack_gate_up +
w4a16_gemm_gate_up[_ws]) against the oracle's gate_up, on every kernel.

H[n][i] = silu(g) * u is compared with the oracle's fp64 value within the
tensor bar of tests/gpu_util.py (the GPU rounds H once from fp32 g, u and
silu; the oracle works in fp64).  Small and decode-size cases compare every
element; N = 4096 compares sampled channels (from every 64-channel block of
the packed weight its first, last and one random channel)."""
import numpy as np
import pytest

import oracle
from gemm_w4a16_b200 import synth
from gemm_w4a16_b200 import w4a16
from tests.gpu_util import assert_close, device_problem, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

GEMV, TC, GT = w4a16.PATH_GEMV, w4a16.PATH_TC, w4a16.PATH_GEMV_TC
NAMES = {GEMV: "gemv", TC: "tc", GT: "gemv_tc", w4a16.PATH_AUTO: "auto"}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gemm_w4a16_b200 import build

    build.build()
    yield
    torch.cuda.synchronize()
    assert w4a16.device_status() == w4a16.OK


def _packed(p):
    q, s, z, x = device_problem(p)
    return w4a16.pack_gate_up(q, s, z), x


def _run(w, x, path, H=None):
    if path == w4a16.PATH_AUTO:
        H = w4a16.gemm_gate_up(w, x, H=H)
    else:
        H = w4a16.gemm_gate_up_ws(w, x, H=H, path=path)
    torch.cuda.synchronize()
    return H


def _channels(Mi, seed):
    rng = np.random.default_rng(seed)
    ch = [0, 1, 15, 16, Mi // 2, Mi - 2, Mi - 1]
    for c0 in range(0, Mi, 64):
        c1 = min(Mi, c0 + 64)
        ch += [c0, c1 - 1, int(rng.integers(c0, c1))]
    return np.unique(np.asarray([c for c in ch if 0 <= c < Mi], dtype=np.int64))


def test_pack_order_matches_the_documented_interleave():
    """dequant_debug of the gate/up packing: packed row 32 q + j of block b is
    the gate row of channel 64 b + 16 q + j, row 32 q + 16 + j its up row,
    bit for bit against the oracle's dequantisation of the canonical rows."""
    Mi, K = 200, 384
    p = synth.make_problem(2 * Mi, K, 1, seed=11)
    w, _ = _packed(p)
    Wp = w4a16.dequant_debug(w4a16.PackedWeight(w.wq, w.scales, w.zeros, 128 * ((Mi + 63) // 64), K))
    got = Wp.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.dequant(p.q, p.zeros, p.scales)
    for r in range(got.shape[0]):
        b, rr = divmod(r, 128)
        i = b * 64 + (rr // 32) * 16 + (rr % 16)
        if i >= Mi:
            assert not got[r].any(), r
        else:
            src = i if rr % 32 < 16 else Mi + i
            assert np.array_equal(got[r], ref[src]), r


@pytest.mark.parametrize("path", [GEMV, TC, GT, w4a16.PATH_AUTO], ids=lambda p: NAMES[p])
@pytest.mark.parametrize("Mi,K,N", [(128, 256, 1), (200, 384, 2), (37, 128, 3), (1000, 1024, 5),
                                    (64, 512, 16), (1000, 1024, 11), (4104, 2048, 9)])
def test_gate_up_small_full(Mi, K, N, path):
    p = synth.make_problem(2 * Mi, K, N, seed=Mi + K + N)
    w, x = _packed(p)
    H = torch.full((N, Mi), float("nan"), dtype=torch.float16, device="cuda")
    _run(w, x, path, H)
    ref = oracle.gate_up(p.q, p.zeros, p.scales, p.x, Mi)
    assert_close(to_f64(H), ref, f"gate_up Mi={Mi} K={K} N={N} path={NAMES[path]}")


@pytest.mark.parametrize("path,N", [(GEMV, 1), (GEMV, 2), (GT, 1), (GT, 2), (GT, 16), (TC, 16),
                                    (w4a16.PATH_AUTO, 1)],
                         ids=["gemv-1", "gemv-2", "gemv_tc-1", "gemv_tc-2", "gemv_tc-16", "tc-16", "auto-1"])
def test_gate_up_llama7b_full(path, N):
    """The LLaMA-7B feed-forward shape (Mi = 11008, K = 4096), every element,
    NaN-prefilled output."""
    Mi, K = 11008, 4096
    p = synth.make_problem(2 * Mi, K, N, seed=N + 3)
    w, x = _packed(p)
    H = torch.full((N, Mi), float("nan"), dtype=torch.float16, device="cuda")
    _run(w, x, path, H)
    ref = oracle.gate_up(p.q, p.zeros, p.scales, p.x, Mi)
    assert_close(to_f64(H), ref, f"gate_up LLaMA-7B N={N} path={NAMES[path]}")


def test_gate_up_llama7b_prefill_sampled():
    Mi, K, N = 11008, 4096, 4096
    p = synth.make_problem(2 * Mi, K, N, seed=17, outlier_frac=0.01)
    w, x = _packed(p)
    H = torch.full((N, Mi), float("nan"), dtype=torch.float16, device="cuda")
    _run(w, x, w4a16.PATH_AUTO, H)
    assert torch.isfinite(H.float()).all()
    ch = _channels(Mi, 17)
    rows = np.concatenate([ch, Mi + ch])
    acc = oracle.gemm_rows(p.q, p.zeros, p.scales, p.x, rows)
    ref = oracle.silu_mul(acc, len(ch))
    got = to_f64(H[:, torch.from_numpy(ch).cuda()])
    assert_close(got, ref, "gate_up prefill (sampled channels)")

"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle.

Small cases compare every element; full-size workloads compare sampled output
rows, which the oracle computes one by one.  Bars: bit-exact for the
dequantised weights and for exactly representable special cases; otherwise
max |Y - Y_ref| <= 2e-3 max |Y_ref| and relative L2 <= 5e-4 (tests/gpu_util.py).
"""
import numpy as np
import pytest

import oracle
from gemm_w4a16_b200 import synth
from gemm_w4a16_b200 import w4a16
from tests.gpu_util import assert_close, pack_problem, sample_rows, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

PATHS = [w4a16.PATH_GEMV, w4a16.PATH_TC]
PATH_NAMES = {w4a16.PATH_AUTO: "auto", w4a16.PATH_GEMV: "gemv", w4a16.PATH_TC: "tc"}

LLAMA7B = [(12288, 4096), (4096, 4096), (22016, 4096), (4096, 11008)]
LLAMA3 = [(6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336), (128256, 4096)]
SWEEP_N = [1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gemm_w4a16_b200 import build

    build.build()
    yield
    torch.cuda.synchronize()
    assert w4a16.device_status() == w4a16.OK


def run(w, x, path):
    y = w4a16.gemm_ex(w, x, path=path)
    torch.cuda.synchronize()
    return y


def full_case(M, K, N, path, seed=0, outlier_frac=0.0):
    p = synth.make_problem(M, K, N, seed=seed, outlier_frac=outlier_frac)
    w, x = pack_problem(p)
    y = to_f64(run(w, x, path))
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x)
    return assert_close(y, ref, f"M={M} K={K} N={N} path={PATH_NAMES[path]}")


def sampled_case(M, K, N, path, seed=0, outlier_frac=0.0, nrows=64):
    p = synth.make_problem(M, K, N, seed=seed, outlier_frac=outlier_frac)
    w, x = pack_problem(p)
    y = run(w, x, path)
    rows = sample_rows(M, nrows, seed=seed + N)
    ys = to_f64(y[:, torch.from_numpy(rows).to(y.device)])
    ref = oracle.gemm_rows(p.q, p.zeros, p.scales, p.x, rows)
    return assert_close(ys, ref, f"M={M} K={K} N={N} path={PATH_NAMES[path]} (sampled)")


# ---------------------------------------------------------------- dequant --

@pytest.mark.parametrize("M,K", [(256, 256), (200, 384), (1, 128), (12288, 4096),
                                 (4096, 11008), (22016, 4096), (4096, 14336)])
def test_dequant_bit_exact(M, K):
    p = synth.make_problem(M, K, 1, seed=1)
    w, _ = pack_problem(p)
    W = w4a16.dequant_debug(w)
    torch.cuda.synchronize()
    got = W.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.dequant(p.q, p.zeros, p.scales)
    assert np.array_equal(got, ref)


def test_dequant_bit_exact_lm_head_rows():
    M, K = 128256, 4096
    p = synth.make_problem(M, K, 1, seed=2)
    w, _ = pack_problem(p)
    W = w4a16.dequant_debug(w)
    rows = sample_rows(M, 256, seed=2)
    got = W[torch.from_numpy(rows).to(W.device)].view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.dequant(p.q[rows], p.zeros[rows], p.scales[rows])
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ small, full --

@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
@pytest.mark.parametrize("N", [1, 8])
def test_tiny_config(N, path):
    full_case(256, 256, N, path)


@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
@pytest.mark.parametrize("M,K,N", [(200, 384, 1), (200, 384, 3), (1, 128, 1), (33, 256, 5),
                                   (129, 640, 7), (300, 1024, 17), (130, 512, 40),
                                   (640, 1280, 130), (96, 128, 2)])
def test_ragged_shapes(M, K, N, path):
    full_case(M, K, N, path, seed=M + K + N)


@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
def test_outlier_channels_small(path):
    full_case(384, 1024, 33, path, seed=5, outlier_frac=0.01)


# ------------------------------------------------------ exact special cases --

@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
def test_q_equal_z_gives_zero(path):
    p = synth.make_problem(256, 512, 16, seed=3)
    g = np.arange(512) // 128
    p.q = np.ascontiguousarray(p.zeros[:, g])
    w, x = pack_problem(p)
    y = run(w, x, path)
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
def test_unit_scale_integer_inputs_bit_exact(path):
    """s = 1, z = 8, X in {-1, 0, 1}, K = 256: |Y| <= 2048, exact in fp32 and
    fp16, so the GPU must equal the integer result bit for bit."""
    rng = np.random.default_rng(4)
    M, K, N = 384, 256, 24
    p = synth.make_problem(M, K, N, seed=4)
    p.zeros[:] = 8
    p.scales[:] = 0x3C00
    xi = rng.integers(-1, 2, (N, K))
    p.x = xi.astype(np.float16).view(np.uint16)
    w, x = pack_problem(p)
    y = run(w, x, path).float().cpu().numpy()
    ref = xi.astype(np.int64) @ (p.q.astype(np.int64) - 8).T
    assert np.array_equal(y, ref.astype(np.float32))


# ---------------------------------------------------------- invariances ----

@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
def test_deterministic(path):
    p = synth.make_problem(4096, 4096, 64, seed=6)
    w, x = pack_problem(p)
    a = run(w, x, path).clone()
    b = run(w, x, path)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_gemv_equals_column_of_multi_token_product():
    p = synth.make_problem(1024, 2048, 8, seed=7)
    w, x = pack_problem(p)
    y = run(w, x, w4a16.PATH_GEMV)
    for j in range(8):
        yj = run(w, x[j:j + 1].contiguous(), w4a16.PATH_GEMV)
        assert torch.equal(yj[0].view(torch.int16), y[j].view(torch.int16))


def test_output_guard_bands_untouched():
    M, K, N = 200, 384, 5
    p = synth.make_problem(M, K, N, seed=8)
    w, x = pack_problem(p)
    pad = 64
    buf = torch.full((N * M + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    for path in PATHS:
        buf.fill_(12345)
        y = buf[pad:pad + N * M].view(torch.float16).view(N, M)
        w4a16.gemm_ex(w, x, Y=y, path=path)
        torch.cuda.synchronize()
        assert torch.all(buf[:pad] == 12345) and torch.all(buf[-pad:] == 12345)
        ref = oracle.gemm(p.q, p.zeros, p.scales, p.x)
        assert_close(to_f64(y), ref, f"guarded path={PATH_NAMES[path]}")


# ------------------------------------------------- full-size workloads ----

@pytest.mark.parametrize("M,K", LLAMA7B)
def test_llama7b_decode_n1(M, K):
    sampled_case(M, K, 1, w4a16.PATH_AUTO)


@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
@pytest.mark.parametrize("N", SWEEP_N)
def test_qkv_n_sweep(N, path):
    sampled_case(12288, 4096, N, path, nrows=48 if N >= 1024 else 64)


@pytest.mark.parametrize("M,K,N", [(12288, 4096, 4096), (4096, 11008, 2048)])
def test_prefill_with_outlier_channels(M, K, N):
    sampled_case(M, K, N, w4a16.PATH_AUTO, outlier_frac=0.01, nrows=32)


@pytest.mark.parametrize("N", [1, 16, 64])
@pytest.mark.parametrize("M,K", LLAMA3)
def test_llama3_batched_decode(M, K, N):
    sampled_case(M, K, N, w4a16.PATH_AUTO)


# --------------------------------------------------------- group quantiser ----

def _quantize_inputs(M, K, seed):
    """fp16 weights ~ N(0, 0.05) with special groups: all zero, constant,
    one-signed, a single large outlier."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, 0.05, size=(M, K))
    if K >= 512 and M >= 4:
        w[0, 0:128] = 0.0
        w[1, 128:256] = 0.37
        w[2, 256:384] = np.abs(w[2, 256:384]) + 0.01
        w[3, 384:512] = -np.abs(w[3, 384:512])
        w[M - 1, K - 7] = 6.5
    return w.astype(np.float16)


@pytest.mark.parametrize("M,K", [(256, 256), (200, 384), (1, 128), (37, 1024), (4096, 4096),
                                 (12288, 4096)])
def test_quantize_bit_exact(M, K):
    """Codes, scales and zeros equal the oracle's bit for bit (same fp32
    decisions on both sides)."""
    w = _quantize_inputs(M, K, seed=M + K)
    q_ref, s_ref, z_ref = oracle.quantize(w.view(np.uint16))
    q, s, z = w4a16.quantize(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint16), s_ref)
    assert np.array_equal(z.cpu().numpy(), z_ref)


def test_quantize_pack_gemm_pipeline():
    """fp16 W -> w4a16_quantize -> w4a16_pack -> w4a16_gemm against the oracle
    layer on the oracle's own quantisation of the same W."""
    M, K, N = 384, 1024, 5
    w = _quantize_inputs(M, K, seed=21)
    x = np.random.default_rng(22).normal(0, 1, size=(N, K)).astype(np.float16)
    q, s, z = w4a16.quantize(torch.from_numpy(w).cuda())
    packed = w4a16.pack(q, s, z)
    for path in (w4a16.PATH_GEMV, w4a16.PATH_TC):
        y = w4a16.gemm_ex(packed, torch.from_numpy(x).cuda(), path=path)
        q_ref, s_ref, z_ref = oracle.quantize(w.view(np.uint16))
        ref = oracle.gemm(q_ref, z_ref, s_ref, x.view(np.uint16))
        assert_close(to_f64(y), ref, f"quantize+pack+gemm path={PATH_NAMES[path]}")


# ------------------------------------------------- fused QKV split + bias ----

@pytest.mark.parametrize("splits,K,N", [((200, 72, 72), 384, 1), ((200, 72, 72), 384, 2),
                                        ((200, 72, 72), 384, 5), ((128, 64, 64), 256, 130),
                                        ((4096, 1024, 1024), 4096, 1), ((4096, 1024, 1024), 4096, 16)])
def test_gemm_qkv_split_and_bias(splits, K, N):
    """Three outputs = the plain product's column ranges bit for bit without
    bias; with an fp16 bias, within tolerance of the oracle's fp64 product
    plus bias."""
    M = sum(splits)
    p = synth.make_problem(M, K, N, seed=M + K + N)
    w, x = pack_problem(p)
    y = run(w, x, w4a16.PATH_AUTO)
    outs = w4a16.gemm_qkv(w, x, splits)
    c = np.cumsum((0,) + tuple(splits))
    for i, o in enumerate(outs):
        assert torch.equal(o.view(torch.int16), y[:, c[i]:c[i + 1]].contiguous().view(torch.int16))
    bias = (np.random.default_rng(M).normal(0, 1, size=M)).astype(np.float16)
    # Caller-owned outputs, filled with NaN first: every element is written.
    outs = tuple(torch.full((N, m), float("nan"), dtype=torch.float16, device="cuda") for m in splits)
    w4a16.gemm_qkv(w, x, splits, bias=torch.from_numpy(bias).cuda(), out=outs)
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x) + bias.astype(np.float64)[None, :]
    for i, o in enumerate(outs):
        assert_close(to_f64(o), ref[:, c[i]:c[i + 1]], f"qkv split {i} N={N}")

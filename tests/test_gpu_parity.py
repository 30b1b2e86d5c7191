"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle.

Small cases and every full-size workload with N <= 64 compare every element;
the larger-N workloads (N >= 128, prefill) compare sampled output rows -- from
every 128-row tile its first, last and one random row, plus random rows --
which the oracle computes one by one.  Bars: bit-exact for the
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


@pytest.mark.parametrize("N", list(range(1, 18)))
def test_gemv_every_token_count(N):
    """Every token count of one 8-token decode launch (1..8, the eight
    columns of its MMA tile), then two launches (9..16) and a third (17), on
    a weight taller than 4096 rows with a ragged row block."""
    full_case(4200, 2048, N, w4a16.PATH_GEMV, seed=300 + N)


@pytest.mark.parametrize("N", list(range(9, 34)))
def test_gemv_two_block_launches(N):
    """Weights of at most 4096 rows take 9..16 tokens in one launch of two
    8-token MMA column blocks sharing the dequantised weights: every count
    9..16, then two launches (17..32) and a third (33), on a ragged row block
    with a K split across a cluster."""
    full_case(1000, 2048, N, w4a16.PATH_GEMV, seed=400 + N)


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
    full_case(M, K, 1, w4a16.PATH_AUTO, seed=M + K)


@pytest.mark.parametrize("path", PATHS, ids=lambda p: PATH_NAMES[p])
@pytest.mark.parametrize("N", SWEEP_N)
def test_qkv_n_sweep(N, path):
    if N <= 64:
        full_case(12288, 4096, N, path)
    else:
        sampled_case(12288, 4096, N, path, nrows=48 if N >= 1024 else 64)


@pytest.mark.parametrize("M,K,N", [(12288, 4096, 4096), (4096, 11008, 2048)])
def test_prefill_with_outlier_channels(M, K, N):
    sampled_case(M, K, N, w4a16.PATH_AUTO, outlier_frac=0.01, nrows=32)


@pytest.mark.parametrize("N", [1, 16, 64])
@pytest.mark.parametrize("M,K", LLAMA3)
def test_llama3_batched_decode(M, K, N):
    full_case(M, K, N, w4a16.PATH_AUTO, seed=M + N)


@pytest.mark.parametrize("path,N", [(w4a16.PATH_GEMV, 1), (w4a16.PATH_TC, 16), (w4a16.PATH_TC, 4096)],
                         ids=["gemv-n1", "tc-n16", "tc-n4096"])
def test_output_guard_bands_full_size(path, N):
    """The fused QKV shape written into the middle of a larger buffer: the
    bytes around Y stay untouched (every row tile and token of the output)."""
    M, K, pad = 12288, 4096, 4096
    p = synth.make_problem(M, K, N, seed=77 + N)
    w, x = pack_problem(p)
    buf = torch.full((N * M + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + N * M].view(torch.float16).view(N, M)
    w4a16.gemm_ex(w, x, Y=y, path=path)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 12345) and torch.all(buf[-pad:] == 12345)
    assert torch.isfinite(y.float()).all()
    if N <= 64:
        assert_close(to_f64(y), oracle.gemm(p.q, p.zeros, p.scales, p.x), f"guarded full size N={N}")


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
                                        ((200, 72, 72), 384, 5), ((200, 72, 72), 384, 12),
                                        ((128, 64, 64), 256, 130),
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


# ------------------------------------------ residual add + RMS normalisation ----

NORM_EPS = 1e-6


def _norm_inputs(N, K, seed, outliers=0):
    """h, d ~ N(0, 1) fp16 (the residual stream and the block output added to
    it), gamma ~ N(1, 0.1); `outliers` fixed channels of h scaled by 50 in
    fp32 before the fp16 rounding."""
    rng = np.random.default_rng(seed)
    h = rng.normal(0, 1, (N, K))
    if outliers:
        h[:, rng.choice(K, size=outliers, replace=False)] *= 50.0
    d = rng.normal(0, 1, (N, K))
    gamma = rng.normal(1, 0.1, K)
    return h.astype(np.float16), d.astype(np.float16), gamma.astype(np.float16)


def _assert_norm_close(X, x_ref, what):
    """Per element |X - x| <= 2^-10 |x| + 2^-24: one fp16 rounding (2^-11
    relative, 2^-25 absolute for subnormals) on top of fp32 arithmetic whose
    relative error stays below 1e-5 (a sum of non-negative squares over at
    most 256 sequential terms per thread plus 8 reduction steps, then the
    mean, the root and two products), and the C9 tensor bar."""
    y = to_f64(X)
    bound = np.abs(x_ref) * 2.0 ** -10 + 2.0 ** -24
    bad = np.abs(y - x_ref) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond the bound"
    assert_close(y, x_ref, what)


@pytest.mark.parametrize("N,K", [(1, 8), (1, 4096), (3, 4096), (7, 24), (5, 5120), (2, 65536),
                                 (64, 8192), (33, 11008)])
def test_add_rmsnorm_matches_oracle(N, K):
    h, d, gamma = _norm_inputs(N, K, seed=N + K)
    th, td, tg = (torch.from_numpy(a).cuda() for a in (h, d, gamma))
    r = torch.empty_like(th)
    _, X = w4a16.add_rmsnorm(th, tg, eps=NORM_EPS, d=td, r_out=r)
    _, X2 = w4a16.add_rmsnorm(th, tg, eps=NORM_EPS, d=td)
    torch.cuda.synchronize()
    r_ref, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS, d=d.view(np.uint16))
    assert np.array_equal(r.cpu().numpy().view(np.uint16), r_ref)
    _assert_norm_close(X, x_ref, f"add_rmsnorm N={N} K={K}")
    assert torch.equal(X.view(torch.int16), X2.view(torch.int16))      # deterministic


def test_add_rmsnorm_without_d_and_in_place():
    N, K = 6, 4096
    h, d, gamma = _norm_inputs(N, K, seed=11)
    tg = torch.from_numpy(gamma).cuda()
    # No d: X from h alone, nothing else written.
    _, X = w4a16.add_rmsnorm(torch.from_numpy(h).cuda(), tg, eps=NORM_EPS)
    _, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS)
    _assert_norm_close(X, x_ref, "add_rmsnorm without d")
    r_ref, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS, d=d.view(np.uint16))
    # The residual updated in place, over h and over d.
    for target in ("h", "d"):
        th, td = torch.from_numpy(h).cuda(), torch.from_numpy(d).cuda()
        dst = th if target == "h" else td
        _, X = w4a16.add_rmsnorm(th, tg, eps=NORM_EPS, d=td, r_out=dst)
        torch.cuda.synchronize()
        assert np.array_equal(dst.cpu().numpy().view(np.uint16), r_ref), target
        _assert_norm_close(X, x_ref, f"add_rmsnorm in place over {target}")


def test_add_rmsnorm_zero_rows_outliers_and_guard_bands():
    N, K, pad = 16, 4096, 64
    h, d, gamma = _norm_inputs(N, K, seed=12, outliers=40)
    h[3] = 0
    d[3] = 0
    th, td, tg = (torch.from_numpy(a).cuda() for a in (h, d, gamma))
    buf = torch.full((N * K + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    X = buf[pad:pad + N * K].view(torch.float16).view(N, K)
    w4a16.add_rmsnorm(th, tg, eps=NORM_EPS, d=td, X=X)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 12345) and torch.all(buf[-pad:] == 12345)
    assert torch.count_nonzero(X[3]).item() == 0
    _, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS, d=d.view(np.uint16))
    _assert_norm_close(X, x_ref, "add_rmsnorm with outlier channels")


def test_add_rmsnorm_full_size_sampled_rows():
    """16384 token rows of LLaMA-7B width (4096), the benchmarked size; sampled
    rows against the oracle (each row is normalised on its own)."""
    N, K = 16384, 4096
    h, d, gamma = _norm_inputs(N, K, seed=13, outliers=40)
    th, td, tg = (torch.from_numpy(a).cuda() for a in (h, d, gamma))
    r = torch.empty_like(th)
    _, X = w4a16.add_rmsnorm(th, tg, eps=NORM_EPS, d=td, r_out=r)
    torch.cuda.synchronize()
    rows = sample_rows(N, 256, seed=13)
    r_ref, x_ref = oracle.add_rmsnorm(h[rows].view(np.uint16), gamma.view(np.uint16), NORM_EPS,
                                      d=d[rows].view(np.uint16))
    ti = torch.from_numpy(rows).cuda()
    assert np.array_equal(r[ti].cpu().numpy().view(np.uint16), r_ref)
    _assert_norm_close(X[ti], x_ref, "add_rmsnorm full size (sampled rows)")


def test_add_rmsnorm_then_fused_qkv():
    """The layer's first two steps chained on the GPU: X from the residual add
    and normalisation, then the fused QKV projection; against the oracle's
    chain, whose X is rounded to fp16 by the oracle itself."""
    N, K, splits = 5, 4096, (4096, 1024, 1024)
    M = sum(splits)
    h, d, gamma = _norm_inputs(N, K, seed=14)
    p = synth.make_problem(M, K, N, seed=14)
    w, _ = pack_problem(p)
    _, X = w4a16.add_rmsnorm(*(torch.from_numpy(a).cuda() for a in (h, gamma)), eps=NORM_EPS,
                             d=torch.from_numpy(d).cuda())
    outs = w4a16.gemm_qkv(w, X, splits)
    _, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS, d=d.view(np.uint16))
    y_ref = oracle.gemm(p.q, p.zeros, p.scales, oracle.fp16_from_double(x_ref))
    c = np.cumsum((0,) + splits)
    for i, o in enumerate(outs):
        assert_close(to_f64(o), y_ref[:, c[i]:c[i + 1]], f"add_rmsnorm -> qkv split {i}")


# ---------------------------- residual add + RMS norm as the QKV prologue ----

@pytest.mark.parametrize("N,K,splits,with_d,with_bias", [
    (1, 4096, (4096, 1024, 1024), True, False),     # LLaMA-7B-shaped GQA projection, one token
    (1, 4096, (4096, 4096, 4096), True, True),      # LLaMA-7B QKV with a bias
    (2, 4096, (4096, 1024, 1024), False, False),    # no d: r = h
    (8, 4096, (4096, 1024, 1024), True, True),      # a full decode launch of 8 tokens
    (3, 1152, (200, 72, 72), True, True),           # ragged K and projection borders inside tiles
    (5, 11008, (1024, 256, 256), True, False),      # a long row: sum of squares over 11008 channels
])
def test_add_rmsnorm_fused_into_qkv(N, K, splits, with_d, with_bias):
    """One launch (w4a16_add_rmsnorm_gemm_qkv) against the two-launch chain
    (w4a16_add_rmsnorm, then w4a16_gemm_qkv): the same bits for Yq, Yk, Yv and
    r, since the prologue repeats the norm kernel's arithmetic in its order;
    and against the oracle's chain within C9, every element.  Outputs
    NaN-prefilled."""
    M = sum(splits)
    h, d, gamma = _norm_inputs(N, K, seed=N + K, outliers=8)
    p = synth.make_problem(M, K, N, seed=N + K)
    w, _ = pack_problem(p)
    ht, gt = torch.from_numpy(h).cuda(), torch.from_numpy(gamma).cuda()
    dt = torch.from_numpy(d).cuda() if with_d else None
    bias = (np.random.default_rng(M).normal(0, 1, size=M)).astype(np.float16) if with_bias else None
    bt = torch.from_numpy(bias).cuda() if with_bias else None
    r_chain, X = w4a16.add_rmsnorm(ht, gt, eps=NORM_EPS, d=dt, r_out=torch.empty_like(ht))
    chain = w4a16.gemm_qkv(w, X, splits, bias=bt)
    outs = tuple(torch.full((N, m), float("nan"), dtype=torch.float16, device="cuda") for m in splits)
    r_fused = torch.full_like(ht, float("nan"))
    fused = w4a16.add_rmsnorm_gemm_qkv(ht, gt, w, splits, eps=NORM_EPS, d=dt, r_out=r_fused, bias=bt, out=outs)
    torch.cuda.synchronize()
    for a, b in zip(fused, chain):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(r_fused.view(torch.int16), r_chain.view(torch.int16))
    _, x_ref = oracle.add_rmsnorm(h.view(np.uint16), gamma.view(np.uint16), NORM_EPS,
                                  d=d.view(np.uint16) if with_d else None)
    y_ref = oracle.gemm(p.q, p.zeros, p.scales, oracle.fp16_from_double(x_ref))
    if with_bias:
        y_ref = y_ref + bias.astype(np.float64)[None, :]
    c = np.cumsum((0,) + tuple(splits))
    for i, o in enumerate(fused):
        assert_close(to_f64(o), y_ref[:, c[i]:c[i + 1]], f"add_rmsnorm + qkv fused, split {i}, N={N}")


def test_add_rmsnorm_fused_into_qkv_early_weights_in_a_chain():
    """Under programmatic launch the prologue reads h and d only after the
    previous kernel (here the norm kernel writing h in place) completed."""
    N, K, splits = 1, 4096, (4096, 1024, 1024)
    M = sum(splits)
    h, d, gamma = _norm_inputs(N, K, seed=21)
    p = synth.make_problem(M, K, N, seed=21)
    w, _ = pack_problem(p)
    ht, dt, gt = (torch.from_numpy(a).cuda() for a in (h, d, gamma))
    h2 = ht.clone()
    d2 = torch.from_numpy(_norm_inputs(N, K, seed=22)[1]).cuda()
    # Reference: r1 = h + d (in place), then the fused call on (r1, d2).
    ref_in = ht.clone()
    w4a16.add_rmsnorm(ref_in, gt, eps=NORM_EPS, d=dt, r_out=ref_in)
    ref = w4a16.add_rmsnorm_gemm_qkv(ref_in, gt, w, splits, eps=NORM_EPS, d=d2)
    torch.cuda.synchronize()
    w4a16.add_rmsnorm(h2, gt, eps=NORM_EPS, d=dt, r_out=h2)
    got = w4a16.add_rmsnorm_gemm_qkv(h2, gt, w, splits, eps=NORM_EPS, d=d2, flags=w4a16.FLAG_EARLY_WEIGHTS)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_add_rmsnorm_fused_into_qkv_rejects_without_launching():
    L = w4a16.lib()
    N, K, splits = 2, 256, (128, 64, 64)
    p = synth.make_problem(sum(splits), K, N, seed=3)
    w, _ = pack_problem(p)
    h = torch.zeros((16, K), dtype=torch.float16, device="cuda")
    g = torch.ones(K, dtype=torch.float16, device="cuda")
    ys = [torch.empty((16, m), dtype=torch.float16, device="cuda") for m in splits]
    s = torch.cuda.current_stream().cuda_stream

    def call(N=2, r_out=None, eps=1e-6, flags=0, h_ptr=None):
        return L.w4a16_add_rmsnorm_gemm_qkv(h.data_ptr() if h_ptr is None else h_ptr, None, g.data_ptr(), eps,
                                            r_out, w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), None,
                                            *splits, K, N, 128, ys[0].data_ptr(), ys[1].data_ptr(),
                                            ys[2].data_ptr(), flags, s)
    assert call(N=9) == w4a16.ERR_UNSUPPORTED              # more tokens than one decode launch
    assert call(r_out=h.data_ptr()) == w4a16.ERR_INVALID_ARG   # in place over h
    assert call(eps=-1.0) == w4a16.ERR_INVALID_ARG
    assert call(flags=2) == w4a16.ERR_INVALID_ARG
    assert call(h_ptr=h.data_ptr() + 8) == w4a16.ERR_MISALIGNED
    assert call(r_out=ys[0].data_ptr()) == w4a16.ERR_INVALID_ARG   # r over Yq

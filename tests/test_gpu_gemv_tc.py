"""GPU parity of the split tensor-core decode path (W4A16_PATH_GEMV_TC, the
workspace entry points) against the CPU oracle, through the C ABI.

Full-size LLaMA shapes compare every output element: at N <= 16 the oracle
computes a whole projection in seconds.  Bars as in tests/gpu_util.py; exact
special cases bit for bit.  Also: the split-block reduction (blocks shared by
several CTAs, CTAs spanning several blocks, fewer units than SMs), the
workspace left zero-filled after each call, determinism, guard bands,
NaN-prefilled outputs, the fused QKV form, and programmatic dependent launch
on a chain of dependent calls.
"""
import numpy as np
import pytest

import oracle
from gemm_w4a16_b200 import synth
from gemm_w4a16_b200 import w4a16
from tests.gpu_util import assert_close, pack_problem, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

GT = w4a16.PATH_GEMV_TC
LLAMA7B = [(12288, 4096), (4096, 4096), (22016, 4096), (4096, 11008)]
LLAMA3 = [(6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336), (128256, 4096)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gemm_w4a16_b200 import build

    build.build()
    yield
    torch.cuda.synchronize()
    assert w4a16.device_status() == w4a16.OK


def run(w, x, ws=None, flags=0):
    y = w4a16.gemm_ws(w, x, path=GT, workspace=ws, flags=flags)
    torch.cuda.synchronize()
    return y


def full_case(M, K, N, seed=0, outlier_frac=0.0, ws=None):
    p = synth.make_problem(M, K, N, seed=seed, outlier_frac=outlier_frac)
    w, x = pack_problem(p)
    y = to_f64(run(w, x, ws))
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x)
    return assert_close(y, ref, f"M={M} K={K} N={N} path=gemv_tc")


def test_auto_choice_with_workspace():
    assert w4a16.select_path_ws(12288, 4096, 1) == w4a16.PATH_GEMV
    assert w4a16.select_path_ws(12288, 4096, 16) == w4a16.PATH_TC
    assert w4a16.workspace_size(12288, 4096, 17) > 0      # a forced split path up to 64 tokens
    assert w4a16.workspace_size(12288, 4096, 65) == 0
    assert w4a16.workspace_size(12288, 4096, 1) > 0


# ------------------------------------------------------------ small, full --

@pytest.mark.parametrize("N", [1, 8])
def test_tiny_config(N):
    full_case(256, 256, N)


@pytest.mark.parametrize("M,K,N", [(200, 384, 1), (200, 384, 3), (1, 128, 1), (33, 256, 5),
                                   (129, 640, 7), (96, 128, 2), (300, 1024, 16), (1000, 1152, 9),
                                   (128, 8192, 1), (2048, 128, 4)])
def test_ragged_and_few_unit_shapes(M, K, N):
    """Fewer units than SMs (one unit per CTA), one row block over many CTAs
    (K = 8192: 64 groups), one group per block (K = 128: no block split)."""
    full_case(M, K, N, seed=M + K + N)


@pytest.mark.parametrize("N", list(range(1, 17)) + [17, 24, 31, 32, 33, 40, 48, 63, 64])
def test_every_token_count(N):
    """Every N of the 16-token configuration, then the 32- and 64-token ones
    around their edges."""
    full_case(1536, 2048, N, seed=100 + N)


def test_outlier_channels_small():
    full_case(384, 1024, 13, seed=5, outlier_frac=0.01)


def test_q_equal_z_gives_zero():
    p = synth.make_problem(1280, 2048, 16, seed=3)
    g = np.arange(2048) // 128
    p.q = np.ascontiguousarray(p.zeros[:, g])
    w, x = pack_problem(p)
    y = run(w, x)
    assert torch.count_nonzero(y).item() == 0


def test_unit_scale_integer_inputs_bit_exact():
    """s = 1, z = 8, X in {-1, 0, 1}: |Y| <= 8 K = 2048 at K = 256 (exact in
    fp32 and fp16), on a shape whose blocks are split between CTAs."""
    rng = np.random.default_rng(4)
    M, K, N = 3 * 1280, 256, 11
    p = synth.make_problem(M, K, N, seed=4)
    p.zeros[:] = 8
    p.scales[:] = 0x3C00
    xi = rng.integers(-1, 2, (N, K))
    p.x = xi.astype(np.float16).view(np.uint16)
    w, x = pack_problem(p)
    y = run(w, x).float().cpu().numpy()
    ref = xi.astype(np.int64) @ (p.q.astype(np.int64) - 8).T
    assert np.array_equal(y, ref.astype(np.float32))


# --------------------------------------------- full-size, every element ----

@pytest.mark.parametrize("M,K", LLAMA7B)
def test_llama7b_decode_n1_full(M, K):
    full_case(M, K, 1, seed=M + K)


@pytest.mark.parametrize("N", [2, 4, 8, 16, 32, 64])
def test_qkv_few_tokens_full(N):
    full_case(12288, 4096, N, seed=N)


@pytest.mark.parametrize("N", [1, 16, 64])
@pytest.mark.parametrize("M,K", LLAMA3)
def test_llama3_batched_decode_full(M, K, N):
    full_case(M, K, N, seed=M + N)


# ------------------------------------------------ workspace and invariants ----

def test_workspace_left_zero_and_calls_repeat_bit_exactly():
    """Two calls in a row on one workspace give the same bits, and the
    counters (the workspace's first bytes) are zero after each call."""
    M, K, N = 4096, 4096, 3
    p = synth.make_problem(M, K, N, seed=6)
    w, x = pack_problem(p)
    ws = w4a16.Workspace(x.device, w4a16.workspace_size(M, K, N))
    ncnt = ((M + 127) // 128) * 4 * 4
    a = run(w, x, ws).clone()
    assert torch.count_nonzero(ws.buf[:ncnt]).item() == 0
    b = run(w, x, ws)
    assert torch.count_nonzero(ws.buf[:ncnt]).item() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert_close(to_f64(b), oracle.gemm(p.q, p.zeros, p.scales, p.x), "repeat")


def test_output_guard_bands_and_nan_prefill():
    M, K, N, pad = 4000, 1536, 5, 64
    p = synth.make_problem(M, K, N, seed=8)
    w, x = pack_problem(p)
    buf = torch.full((N * M + 2 * pad,), 12345, dtype=torch.int16, device="cuda")
    y = buf[pad:pad + N * M].view(torch.float16).view(N, M)
    y.fill_(float("nan"))
    w4a16.gemm_ws(w, x, Y=y, path=GT)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 12345) and torch.all(buf[-pad:] == 12345)
    assert_close(to_f64(y), oracle.gemm(p.q, p.zeros, p.scales, p.x), "guarded gemv_tc")


def test_every_path_through_the_workspace_entry_point():
    """w4a16_gemm_ws with each forced path on the same inputs: each within
    the bar of the oracle."""
    M, K, N = 2560, 4096, 2
    p = synth.make_problem(M, K, N, seed=9)
    w, x = pack_problem(p)
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x)
    for path in (w4a16.PATH_AUTO, w4a16.PATH_GEMV, w4a16.PATH_TC, GT):
        y = w4a16.gemm_ws(w, x, path=path)
        torch.cuda.synchronize()
        assert_close(to_f64(y), ref, f"path {path}")


def test_argument_checks():
    M, K, N = 256, 256, 2
    p = synth.make_problem(M, K, N, seed=10)
    w, x = pack_problem(p)
    y = torch.empty((N, M), dtype=torch.float16, device="cuda")
    L = w4a16.lib()
    s = torch.cuda.current_stream().cuda_stream
    need = w4a16.workspace_size(M, K, N)
    ws = torch.zeros(need + 256, dtype=torch.uint8, device="cuda")
    args = (w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), x.data_ptr(), y.data_ptr(), M, K, N, 128)
    # The forced split path without a workspace, or with one too small.
    assert L.w4a16_gemm_ws(*args, GT, None, 0, 0, s) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_gemm_ws(*args, GT, ws.data_ptr(), need - 1, 0, s) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_gemm_ex(*args, GT, s) == w4a16.ERR_INVALID_ARG
    # Unknown flags, a misaligned workspace, a workspace over the output.
    assert L.w4a16_gemm_ws(*args, GT, ws.data_ptr(), need, 2, s) == w4a16.ERR_INVALID_ARG
    assert L.w4a16_gemm_ws(*args, GT, ws.data_ptr() + 8, need, 0, s) == w4a16.ERR_MISALIGNED
    assert L.w4a16_gemm_ws(*args[:4], ws.data_ptr(), M, K, N, 128, GT, ws.data_ptr(), need, 0,
                           s) == w4a16.ERR_INVALID_ARG
    # More tokens than the split kernel takes.
    x65 = torch.zeros((65, K), dtype=torch.float16, device="cuda")
    y65 = torch.empty((65, M), dtype=torch.float16, device="cuda")
    assert L.w4a16_gemm_ws(w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), x65.data_ptr(),
                           y65.data_ptr(), M, K, 65, 128, GT, ws.data_ptr(), ws.numel(), 0,
                           s) == w4a16.ERR_UNSUPPORTED
    # Null workspace: AUTO falls back to the workspace-free choice.
    assert L.w4a16_gemm_ws(*args, w4a16.PATH_AUTO, None, 0, 0, s) == w4a16.OK
    torch.cuda.synchronize()


# ------------------------------------------------------- fused QKV form ----

@pytest.mark.parametrize("splits,K,N", [((200, 72, 72), 384, 1), ((4096, 1024, 1024), 4096, 1),
                                        ((4096, 1024, 1024), 4096, 16), ((4096, 4096, 4096), 4096, 3)])
def test_gemm_qkv_ws_split_and_bias(splits, K, N):
    M = sum(splits)
    p = synth.make_problem(M, K, N, seed=M + K + N)
    w, x = pack_problem(p)
    y = w4a16.gemm_ws(w, x)          # the automatic path, as gemm_qkv_ws takes
    outs = w4a16.gemm_qkv_ws(w, x, splits)
    c = np.cumsum((0,) + tuple(splits))
    for i, o in enumerate(outs):
        assert torch.equal(o.view(torch.int16), y[:, c[i]:c[i + 1]].contiguous().view(torch.int16))
    bias = (np.random.default_rng(M).normal(0, 1, size=M)).astype(np.float16)
    outs = tuple(torch.full((N, m), float("nan"), dtype=torch.float16, device="cuda") for m in splits)
    w4a16.gemm_qkv_ws(w, x, splits, bias=torch.from_numpy(bias).cuda(), out=outs)
    torch.cuda.synchronize()
    ref = oracle.gemm(p.q, p.zeros, p.scales, p.x) + bias.astype(np.float64)[None, :]
    for i, o in enumerate(outs):
        assert_close(to_f64(o), ref[:, c[i]:c[i + 1]], f"qkv split {i} N={N}")


# ---------------------------------------- programmatic dependent launch ----

def _chain(weights, x0, flags, graph):
    """y_{i+1} = W_i . y_i, each call reading the previous call's output."""
    ws = w4a16.Workspace(x0.device, max(w4a16.workspace_size(w.M, w.K, x0.shape[0]) for w in weights))
    ys = [x0] + [torch.empty((x0.shape[0], w.M), dtype=torch.float16, device=x0.device) for w in weights]

    def body():
        for i, w in enumerate(weights):
            w4a16.gemm_ws(w, ys[i], Y=ys[i + 1], path=GT, workspace=ws, flags=flags)

    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            body()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body()
        for y in ys[1:]:
            y.fill_(float("nan"))
        g.replay()
        g.replay()
    else:
        body()
    torch.cuda.synchronize()
    return [y.clone() for y in ys[1:]]


@pytest.mark.parametrize("graph", [False, True])
def test_early_weights_on_dependent_chain(graph):
    """Eight chained square projections: with early weight streaming each
    call still reads its X only after the previous call completed, so the
    results equal the plain launches bit for bit (a call that read its X
    early would see the NaN the outputs were filled with, or stale values).
    The first step is checked against the oracle."""
    K, N, depth = 2048, 2, 8
    rng = np.random.default_rng(31)
    probs = [synth.make_problem(K, K, N, seed=40 + i) for i in range(depth)]
    weights = [pack_problem(p)[0] for p in probs]
    # Small activations keep the chain in fp16 range (a gain of about 3.5 per step).
    x0_host = (rng.normal(0, 1, (N, K)) * 0.01).astype(np.float16)
    x0 = torch.from_numpy(x0_host).cuda()
    plain = _chain(weights, x0, 0, graph=False)
    early = _chain(weights, x0, w4a16.FLAG_EARLY_WEIGHTS, graph=graph)
    for a, b in zip(plain, early):
        assert torch.isfinite(b.float()).all()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ref = oracle.gemm(probs[0].q, probs[0].zeros, probs[0].scales, x0_host.view(np.uint16))
    assert_close(to_f64(plain[0]), ref, "chain step 0")

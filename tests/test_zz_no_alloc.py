"""w4a16_gemm_noalloc (the split decode kernel on a fixed device array, for
callers that cannot allocate device memory) against w4a16_gemm_ws on the same
kernel with a caller workspace, through the C ABI.  Two calls in a row each
time: the array keeps the last call's contents, so the second call checks
that every call starts from cleared counters.  Collected last, so it also
runs after every other test in one process."""

import pytest

from gemm_w4a16_b200 import synth
from gemm_w4a16_b200 import w4a16
from tests.gpu_util import assert_close, pack_problem, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

GT = w4a16.PATH_GEMV_TC


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gemm_w4a16_b200 import build

    build.build()
    yield
    torch.cuda.synchronize()
    assert w4a16.device_status() == w4a16.OK


def _noalloc(w, x, y, flags=0):
    L = w4a16.lib()
    s = torch.cuda.current_stream().cuda_stream
    return L.w4a16_gemm_noalloc(w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), x.data_ptr(),
                                y.data_ptr(), w.M, w.K, x.shape[0], 128, flags, s)


@pytest.mark.parametrize("M,K,N", [(12288, 4096, 1), (4096, 11008, 4), (200, 384, 3), (22016, 4096, 16)])
def test_noalloc_matches_workspace_entry_point(M, K, N):
    p = synth.make_problem(M, K, N, seed=M + N)
    w, x = pack_problem(p)
    ws = w4a16.Workspace(x.device, w4a16.workspace_size(M, K, N))
    ref = to_f64(w4a16.gemm_ws(w, x, path=GT, workspace=ws))
    for flags in (0, w4a16.FLAG_EARLY_WEIGHTS):
        for _ in range(2):
            y = torch.full((N, M), float("nan"), dtype=torch.float16, device=x.device)
            assert _noalloc(w, x, y, flags) == w4a16.OK
            torch.cuda.synchronize()
            assert_close(to_f64(y), ref, f"noalloc M={M} K={K} N={N} flags={flags}")


def test_noalloc_rejects_sizes_beyond_its_array():
    """The array holds 4 MiB: N = 64 on a 148-SM device needs about 9.7 MB of
    partials; N = 65 is beyond the kernel.  Both fail on the host."""
    M, K = 4096, 4096
    p = synth.make_problem(128, 256, 1, seed=1)
    w, _ = pack_problem(p)
    L = w4a16.lib()
    big = w4a16.workspace_size(M, K, 64)
    x = torch.zeros((64, K), dtype=torch.float16, device="cuda")
    y = torch.empty((64, M), dtype=torch.float16, device="cuda")
    if big > (4 << 20):
        assert L.w4a16_gemm_noalloc(w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), x.data_ptr(),
                                    y.data_ptr(), M, K, 64, 128, 0, None) == w4a16.ERR_UNSUPPORTED
    x65 = torch.zeros((65, K), dtype=torch.float16, device="cuda")
    y65 = torch.empty((65, M), dtype=torch.float16, device="cuda")
    assert L.w4a16_gemm_noalloc(w.wq.data_ptr(), w.scales.data_ptr(), w.zeros.data_ptr(), x65.data_ptr(),
                                y65.data_ptr(), M, K, 65, 128, 0, None) == w4a16.ERR_UNSUPPORTED
    assert L.w4a16_gemm_noalloc(None, w.scales.data_ptr(), w.zeros.data_ptr(), x.data_ptr(), y.data_ptr(),
                                M, K, 1, 128, 0, None) == w4a16.ERR_INVALID_ARG

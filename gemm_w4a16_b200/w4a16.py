"""ctypes binding of libw4a16 (include/w4a16.h), same entry-point names.

Argument marshalling only: every step of the layer runs in the CUDA library.
PyTorch supplies device memory and the current stream.  If the library is
missing the calls raise; there is no fallback of any kind.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libw4a16.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libw4a16_debug.so")   # the index-check build (-DW4A16_DEBUG_BOUNDS)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(7)
PATH_AUTO, PATH_GEMV, PATH_TC, PATH_GEMV_TC = 0, 1, 2, 3
FLAG_EARLY_WEIGHTS = 1
GEMV_TC_MAX_TOKENS = 64      # forced W4A16_PATH_GEMV_TC
GEMV_MAX_TOKENS = 8          # tokens of one decode-kernel launch; AUTO takes it up to here
GROUP = 128

EXPORTED = (
    "w4a16_status_string", "w4a16_packed_sizes", "w4a16_pack", "w4a16_gemm",
    "w4a16_gemm_ex", "w4a16_select_path", "w4a16_dequant_debug",
    "w4a16_device_status", "w4a16_selftest_wait_timeout", "w4a16_quantize", "w4a16_gemm_qkv",
    "w4a16_add_rmsnorm", "w4a16_gemm_workspace_size", "w4a16_gemm_ws", "w4a16_gemm_qkv_ws",
    "w4a16_select_path_ws", "w4a16_pack_gate_up", "w4a16_gemm_gate_up", "w4a16_gemm_gate_up_ws",
    "w4a16_gemm_noalloc", "w4a16_add_rmsnorm_gemm_qkv",
)

_lib = None
_lock = threading.Lock()
_vp = ctypes.c_void_p
_i = ctypes.c_int
_szp = ctypes.POINTER(ctypes.c_size_t)
_sz = ctypes.c_size_t
_u = ctypes.c_uint


class W4A16Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib():
    """Load libw4a16.so; raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with gemm_w4a16_b200/build.py "
                    "(there is no fallback implementation)")
            L = ctypes.CDLL(LIB_PATH)
            L.w4a16_status_string.argtypes = [_i]
            L.w4a16_status_string.restype = ctypes.c_char_p
            L.w4a16_packed_sizes.argtypes = [_i, _i, _i, _szp, _szp, _szp]
            L.w4a16_packed_sizes.restype = _i
            L.w4a16_quantize.argtypes = [_vp, _i, _i, _i, _vp, _vp, _vp, _vp]
            L.w4a16_quantize.restype = _i
            L.w4a16_add_rmsnorm.argtypes = [_vp, _vp, _vp, ctypes.c_float, _i, _i, _vp, _vp, _vp]
            L.w4a16_add_rmsnorm.restype = _i
            L.w4a16_pack.argtypes = [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp]
            L.w4a16_pack.restype = _i
            L.w4a16_gemm.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
            L.w4a16_gemm.restype = _i
            L.w4a16_gemm_qkv.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]
            L.w4a16_add_rmsnorm_gemm_qkv.argtypes = [_vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp, _vp,
                                                     _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _u, _vp]
            L.w4a16_add_rmsnorm_gemm_qkv.restype = _i
            L.w4a16_gemm_qkv.restype = _i
            L.w4a16_gemm_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
            L.w4a16_gemm_ex.restype = _i
            L.w4a16_select_path.argtypes = [_i, _i, _i]
            L.w4a16_select_path.restype = _i
            L.w4a16_select_path_ws.argtypes = [_i, _i, _i]
            L.w4a16_select_path_ws.restype = _i
            L.w4a16_gemm_workspace_size.argtypes = [_i, _i, _i, _i, _szp]
            L.w4a16_gemm_workspace_size.restype = _i
            L.w4a16_gemm_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp]
            L.w4a16_gemm_noalloc.restype = _i
            L.w4a16_gemm_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _u, _vp]
            L.w4a16_gemm_ws.restype = _i
            L.w4a16_gemm_qkv_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                            _vp, _sz, _u, _vp]
            L.w4a16_gemm_qkv_ws.restype = _i
            L.w4a16_pack_gate_up.argtypes = [_vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp]
            L.w4a16_pack_gate_up.restype = _i
            L.w4a16_gemm_gate_up.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]
            L.w4a16_gemm_gate_up.restype = _i
            L.w4a16_gemm_gate_up_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _u, _vp]
            L.w4a16_gemm_gate_up_ws.restype = _i
            L.w4a16_dequant_debug.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _vp]
            L.w4a16_dequant_debug.restype = _i
            L.w4a16_device_status.argtypes = [_vp, ctypes.POINTER(_i)]
            L.w4a16_device_status.restype = _i
            L.w4a16_selftest_wait_timeout.argtypes = [ctypes.c_longlong, _vp]
            L.w4a16_selftest_wait_timeout.restype = _i
            _lib = L
    return _lib


@contextlib.contextmanager
def library(path: str):
    """Route every call made in the block through the library at `path`
    (DEBUG_LIB_PATH: the same API with the decode kernel's index checks),
    then go back to the previous one."""
    global LIB_PATH, _lib
    with _lock:
        saved = (LIB_PATH, _lib)
        LIB_PATH, _lib = path, None
    try:
        yield
    finally:
        with _lock:
            LIB_PATH, _lib = saved


def status_string(status: int) -> str:
    return lib().w4a16_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise W4A16Error(status, where)


def _stream_ptr(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None else _vp(0)


def packed_sizes(M: int, K: int, group: int = GROUP):
    """(wq_bytes, scales_bytes, zeros_bytes) of the packed layout."""
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().w4a16_packed_sizes(M, K, group, ctypes.byref(a), ctypes.byref(b),
                                    ctypes.byref(c)), "w4a16_packed_sizes")
    return a.value, b.value, c.value


def select_path(M: int, K: int, N: int) -> int:
    return int(lib().w4a16_select_path(M, K, N))


def select_path_ws(M: int, K: int, N: int) -> int:
    """The path w4a16_gemm_ws takes when given a workspace."""
    return int(lib().w4a16_select_path_ws(M, K, N))


def workspace_size(M: int, K: int, N: int, group: int = GROUP) -> int:
    """Bytes of workspace the workspace entry points need for these sizes on
    the current device (automatic choice or forced split decode path; 0 for
    N > 64)."""
    n = ctypes.c_size_t()
    _check(lib().w4a16_gemm_workspace_size(M, K, N, group, ctypes.byref(n)), "w4a16_gemm_workspace_size")
    return n.value


class Workspace:
    """A device buffer for the workspace entry points (zero-filled when made;
    each split-path call clears the counters it uses), so one buffer
    serves any number of calls in one stream; `ensure` grows it (outside
    CUDA-graph capture) to the size a call needs."""

    def __init__(self, device=None, nbytes: int = 0):
        import torch

        self.device = torch.device("cuda") if device is None else torch.device(device)
        self.buf = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def ensure(self, nbytes: int) -> "Workspace":
        import torch

        if nbytes > self.buf.numel():
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return self

    def clear(self) -> None:
        """Zero-fill again (needed only after a call that timed out)."""
        self.buf.zero_()


_default_ws = {}


def default_workspace(device, stream) -> Workspace:
    """One workspace per (device, stream): calls in one stream never overlap."""
    key = (device.index, stream.cuda_stream)
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(device)
    return ws


@dataclass
class PackedWeight:
    """The three packed device buffers of one M x K weight."""

    wq: "object"       # torch.uint8 [wq_bytes]
    scales: "object"   # torch.uint8 [scales_bytes] (fp16 values)
    zeros: "object"    # torch.uint8 [zeros_bytes]
    M: int
    K: int
    group: int = GROUP
    mi: int = 0        # > 0: packed in the gate/up row order (w4a16_pack_gate_up), M = 2 mi

    @property
    def nbytes(self) -> int:
        return self.wq.numel() + self.scales.numel() + self.zeros.numel()


def empty_packed(M: int, K: int, device, group: int = GROUP) -> PackedWeight:
    import torch

    a, b, c = packed_sizes(M, K, group)
    mk = lambda n: torch.empty(n, dtype=torch.uint8, device=device)
    return PackedWeight(mk(a), mk(b), mk(c), M, K, group)


def quantize(W, group: int = GROUP, stream=None):
    """fp16 W [M, K] (device) -> canonical (q uint8 [M, K], scales fp16
    [M, K/G], zeros uint8 [M, K/G]) via w4a16_quantize."""
    import torch

    if W.dtype != torch.float16 or not W.is_cuda or not W.is_contiguous() or W.dim() != 2:
        raise ValueError("W must be a contiguous CUDA fp16 [M, K] tensor")
    M, K = W.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=W.device)
    scales = torch.empty((M, K // group), dtype=torch.float16, device=W.device)
    zeros = torch.empty((M, K // group), dtype=torch.uint8, device=W.device)
    _check(lib().w4a16_quantize(_ptr(W), M, K, group, _ptr(q), _ptr(scales), _ptr(zeros),
                                _stream_ptr(stream)), "w4a16_quantize")
    return q, scales, zeros


def add_rmsnorm(h, gamma, eps: float = 1e-6, d=None, r_out=None, X=None, stream=None):
    """Residual add + RMS normalisation via w4a16_add_rmsnorm: r = h + d
    (fp16, written to r_out when given; r_out may be h or d) and
    X = r * gamma / sqrt(eps + mean(r^2)) per token row.  h, d, r_out, X:
    contiguous CUDA fp16 [N, K]; gamma [K].  Returns (r_out, X)."""
    import torch

    def _ok(t, shape):
        return (t.dtype == torch.float16 and t.is_cuda and t.is_contiguous()
                and tuple(t.shape) == tuple(shape))

    if h.dim() != 2 or not _ok(h, h.shape):
        raise ValueError("h must be a contiguous CUDA fp16 [N, K] tensor")
    N, K = h.shape
    if not _ok(gamma, (K,)):
        raise ValueError("gamma must be a contiguous CUDA fp16 tensor of K values")
    for name, t in (("d", d), ("r_out", r_out), ("X", X)):
        if t is not None and not _ok(t, (N, K)):
            raise ValueError(f"{name} must be a contiguous CUDA fp16 [N, K] tensor")
    if X is None:
        X = torch.empty((N, K), dtype=torch.float16, device=h.device)
    _check(lib().w4a16_add_rmsnorm(_ptr(h), _ptr(d), _ptr(gamma), float(eps), N, K, _ptr(r_out), _ptr(X),
                                   _stream_ptr(stream)), "w4a16_add_rmsnorm")
    return r_out, X


def pack(q, scales, zeros, group: int = GROUP, out: PackedWeight | None = None,
         stream=None) -> PackedWeight:
    """Canonical device tensors (q uint8 [M,K], scales fp16 [M,K/G], zeros
    uint8 [M,K/G]) -> packed buffers, via w4a16_pack."""
    M, K = q.shape
    for t in (q, scales, zeros):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("pack expects contiguous CUDA tensors")
    if out is None:
        out = empty_packed(M, K, q.device, group)
    _check(lib().w4a16_pack(_ptr(q), _ptr(scales), _ptr(zeros), M, K, group,
                            _ptr(out.wq), _ptr(out.scales), _ptr(out.zeros),
                            _stream_ptr(stream)), "w4a16_pack")
    return out


def pack_gate_up(q, scales, zeros, group: int = GROUP, out: PackedWeight | None = None,
                 stream=None) -> PackedWeight:
    """Canonical device tensors of a [2 Mi, K] weight whose rows are the gate
    projection then the up projection -> packed buffers in the gate/up row
    order, via w4a16_pack_gate_up."""
    M, K = q.shape
    if M % 2:
        raise ValueError("the gate/up weight has 2 Mi rows")
    for t in (q, scales, zeros):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("pack_gate_up expects contiguous CUDA tensors")
    if out is None:
        out = empty_packed(M, K, q.device, group)
    out.mi = M // 2
    _check(lib().w4a16_pack_gate_up(_ptr(q), _ptr(scales), _ptr(zeros), M // 2, K, group,
                                    _ptr(out.wq), _ptr(out.scales), _ptr(out.zeros),
                                    _stream_ptr(stream)), "w4a16_pack_gate_up")
    return out


def _gate_up_args(w: PackedWeight, X, H):
    import torch

    if not w.mi:
        raise ValueError("the weight must be packed with pack_gate_up")
    N, K = X.shape
    if K != w.K or X.dtype != torch.float16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA fp16 [N, K] tensor")
    if H is None:
        H = torch.empty((N, w.mi), dtype=torch.float16, device=X.device)
    elif H.dtype != torch.float16 or not H.is_cuda or not H.is_contiguous() or tuple(H.shape) != (N, w.mi):
        raise ValueError("H must be a contiguous CUDA fp16 [N, Mi] tensor")
    return N, K, H


def gemm_gate_up(w: PackedWeight, X, H=None, stream=None):
    """H [N, Mi] = silu(X . W_gate^T) * (X . W_up^T), fp16, via w4a16_gemm_gate_up."""
    N, K, H = _gate_up_args(w, X, H)
    _check(lib().w4a16_gemm_gate_up(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(H), w.mi, K, N,
                                    w.group, _stream_ptr(stream)), "w4a16_gemm_gate_up")
    return H


def gemm_gate_up_ws(w: PackedWeight, X, H=None, path: int = PATH_AUTO, workspace: Workspace | None = None,
                    flags: int = 0, stream=None):
    """gemm_gate_up through w4a16_gemm_gate_up_ws (forced path, workspace)."""
    import torch

    N, K, H = _gate_up_args(w, X, H)
    st = torch.cuda.current_stream(X.device) if stream is None else stream
    ws = workspace if workspace is not None else default_workspace(X.device, st)
    need = workspace_size(w.M, K, N, w.group) if path in (PATH_AUTO, PATH_GEMV_TC) else 0
    ws.ensure(need)
    _check(lib().w4a16_gemm_gate_up_ws(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(H), w.mi, K, N,
                                       w.group, path, _ptr(ws.buf), ws.nbytes, int(flags),
                                       _vp(st.cuda_stream)), "w4a16_gemm_gate_up_ws")
    return H


def gemm_ex(w: PackedWeight, X, Y=None, path: int = PATH_AUTO, stream=None):
    """Y [N, M] fp16 = X [N, K] fp16 . dequant(W)^T via w4a16_gemm_ex."""
    import torch

    N, K = X.shape
    if K != w.K or X.dtype != torch.float16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA fp16 [N, K] tensor")
    if Y is None:
        Y = torch.empty((N, w.M), dtype=torch.float16, device=X.device)
    _check(lib().w4a16_gemm_ex(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X),
                               _ptr(Y), w.M, K, N, w.group, path, _stream_ptr(stream)),
           "w4a16_gemm_ex")
    return Y


def _qkv_outs(w: PackedWeight, X, splits, bias, out):
    """Checked (Yq, Yk, Yv) for the fused QKV form: `out`, or new tensors."""
    import torch

    N, K = X.shape
    Mq, Mk, Mv = (int(v) for v in splits)
    if Mq + Mk + Mv != w.M:
        raise ValueError("splits must add up to the weight's rows")
    if K != w.K or X.dtype != torch.float16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA fp16 [N, K] tensor")
    if bias is not None and (bias.dtype != torch.float16 or not bias.is_cuda or bias.numel() != w.M
                             or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous CUDA fp16 tensor of M values")
    if out is None:
        return [torch.empty((N, m), dtype=torch.float16, device=X.device) for m in (Mq, Mk, Mv)]
    outs = list(out)
    if len(outs) != 3 or any(o.dtype != torch.float16 or not o.is_cuda or not o.is_contiguous()
                             or tuple(o.shape) != (N, m) for o, m in zip(outs, (Mq, Mk, Mv))):
        raise ValueError("out must be three contiguous CUDA fp16 tensors [N, Mq], [N, Mk], [N, Mv]")
    return outs


def gemm_qkv(w: PackedWeight, X, splits, bias=None, out=None, stream=None):
    """(Yq, Yk, Yv) token-major fp16 for a weight whose rows are three stacked
    projections of widths splits = (Mq, Mk, Mv), each row plus bias[m] (fp16
    [M] or None), via w4a16_gemm_qkv.  out: three contiguous CUDA fp16 tensors
    [N, Mq], [N, Mk], [N, Mv] to write, or None to allocate them."""
    N, K = X.shape
    outs = _qkv_outs(w, X, splits, bias, out)
    Mq, Mk, Mv = (int(v) for v in splits)
    _check(lib().w4a16_gemm_qkv(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(bias), Mq, Mk, Mv,
                                K, N, w.group, _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                _stream_ptr(stream)), "w4a16_gemm_qkv")
    return tuple(outs)


def add_rmsnorm_gemm_qkv(h, gamma, w: PackedWeight, splits, eps: float = 1e-6, d=None, r_out=None, bias=None,
                         out=None, flags: int = 0, stream=None):
    """gemm_qkv of the normalised residual stream in one launch, via
    w4a16_add_rmsnorm_gemm_qkv (N <= GEMV_MAX_TOKENS): X = add_rmsnorm(h, d)
    is formed inside the projection and never stored; r = h + d goes to r_out
    when given.  Returns (Yq, Yk, Yv)."""
    import torch

    N, K = h.shape
    outs = _qkv_outs(w, h, splits, bias, out)
    if gamma.dtype != torch.float16 or not gamma.is_cuda or not gamma.is_contiguous() or gamma.numel() != K:
        raise ValueError("gamma must be a contiguous CUDA fp16 tensor of K values")
    for name, t in (("d", d), ("r_out", r_out)):
        if t is not None and (t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous()
                              or tuple(t.shape) != (N, K)):
            raise ValueError(f"{name} must be a contiguous CUDA fp16 [N, K] tensor")
    Mq, Mk, Mv = (int(v) for v in splits)
    _check(lib().w4a16_add_rmsnorm_gemm_qkv(_ptr(h), _ptr(d), _ptr(gamma), float(eps), _ptr(r_out), _ptr(w.wq),
                                            _ptr(w.scales), _ptr(w.zeros), _ptr(bias), Mq, Mk, Mv, K, N, w.group,
                                            _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), int(flags),
                                            _stream_ptr(stream)), "w4a16_add_rmsnorm_gemm_qkv")
    return tuple(outs)


def gemm_ws(w: PackedWeight, X, Y=None, path: int = PATH_AUTO, workspace: Workspace | None = None,
            flags: int = 0, stream=None):
    """Y [N, M] fp16 = X [N, K] fp16 . dequant(W)^T via w4a16_gemm_ws, with a
    workspace (the caller's, or one kept per device and stream)."""
    import torch

    N, K = X.shape
    if K != w.K or X.dtype != torch.float16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA fp16 [N, K] tensor")
    if Y is None:
        Y = torch.empty((N, w.M), dtype=torch.float16, device=X.device)
    st = torch.cuda.current_stream(X.device) if stream is None else stream
    ws = workspace if workspace is not None else default_workspace(X.device, st)
    need = workspace_size(w.M, K, N, w.group) if path in (PATH_AUTO, PATH_GEMV_TC) else 0
    ws.ensure(need)
    _check(lib().w4a16_gemm_ws(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(Y), w.M, K, N,
                               w.group, path, _ptr(ws.buf), ws.nbytes, int(flags), _vp(st.cuda_stream)),
           "w4a16_gemm_ws")
    return Y


def gemm_qkv_ws(w: PackedWeight, X, splits, bias=None, out=None, workspace: Workspace | None = None,
                flags: int = 0, stream=None):
    """gemm_qkv through w4a16_gemm_qkv_ws (with a workspace)."""
    import torch

    N, K = X.shape
    outs = _qkv_outs(w, X, splits, bias, out)
    st = torch.cuda.current_stream(X.device) if stream is None else stream
    ws = workspace if workspace is not None else default_workspace(X.device, st)
    ws.ensure(workspace_size(w.M, K, N, w.group))
    Mq, Mk, Mv = (int(v) for v in splits)
    _check(lib().w4a16_gemm_qkv_ws(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(bias), Mq, Mk, Mv,
                                   K, N, w.group, _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), _ptr(ws.buf),
                                   ws.nbytes, int(flags), _vp(st.cuda_stream)), "w4a16_gemm_qkv_ws")
    return tuple(outs)


def gemm(w: PackedWeight, X, Y=None, stream=None):
    """Y [N, M] fp16 = X [N, K] fp16 . dequant(W)^T via w4a16_gemm."""
    import torch

    N, K = X.shape
    if K != w.K or X.dtype != torch.float16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA fp16 [N, K] tensor")
    if Y is None:
        Y = torch.empty((N, w.M), dtype=torch.float16, device=X.device)
    _check(lib().w4a16_gemm(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros), _ptr(X), _ptr(Y),
                            w.M, K, N, w.group, _stream_ptr(stream)), "w4a16_gemm")
    return Y


def dequant_debug(w: PackedWeight, W_out=None, stream=None):
    """fp16 W [M, K] from the packed buffers via w4a16_dequant_debug."""
    import torch

    if W_out is None:
        W_out = torch.empty((w.M, w.K), dtype=torch.float16, device=w.wq.device)
    _check(lib().w4a16_dequant_debug(_ptr(w.wq), _ptr(w.scales), _ptr(w.zeros),
                                     _ptr(W_out), w.M, w.K, w.group, _stream_ptr(stream)),
           "w4a16_dequant_debug")
    return W_out


def device_status(stream=None) -> int:
    """Synchronise and read/clear the device wait-timeout status."""
    st = _i(0)
    _check(lib().w4a16_device_status(_stream_ptr(stream), ctypes.byref(st)),
           "w4a16_device_status")
    return st.value


def selftest_wait_timeout(limit_cycles: int = 2_000_000, stream=None) -> None:
    """Launch the diagnostic kernel whose bounded wait must run out."""
    _check(lib().w4a16_selftest_wait_timeout(int(limit_cycles), _stream_ptr(stream)),
           "w4a16_selftest_wait_timeout")

"""Helpers shared by the GPU parity tests (no test functions here)."""
from __future__ import annotations

import numpy as np

# Tolerances of the parity bar: max |Y - Y_ref| <= 2e-3 * max |Y_ref| and
# ||Y - Y_ref||_2 / ||Y_ref||_2 <= 5e-4 over the compared elements, with Y_ref
# the fp64 oracle.  Budget: fp16 rounding of Y alone gives a relative L2 error
# near 2^-11 / sqrt(3) = 2.8e-4 and a max error <= 2^-11 * max |Y_ref|.
MAX_REL = 2e-3
L2_REL = 5e-4


def device_problem(p, device="cuda"):
    import torch

    q = torch.from_numpy(p.q).to(device)
    zeros = torch.from_numpy(p.zeros).to(device)
    scales = torch.from_numpy(p.scales.view(np.float16)).to(device)
    x = torch.from_numpy(p.x.view(np.float16)).to(device)
    return q, scales, zeros, x


def pack_problem(p, device="cuda"):
    from gemm_w4a16_b200 import w4a16

    q, scales, zeros, x = device_problem(p, device)
    w = w4a16.pack(q, scales, zeros)
    return w, x


def to_f64(y_fp16_tensor) -> np.ndarray:
    return y_fp16_tensor.float().cpu().numpy().astype(np.float64)


def errors(y: np.ndarray, ref: np.ndarray):
    d = y - ref
    max_ref = float(np.abs(ref).max())
    max_err = float(np.abs(d).max())
    l2 = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))
    return max_err, max_ref, l2


def assert_close(y: np.ndarray, ref: np.ndarray, what: str = ""):
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    max_err, max_ref, l2 = errors(y, ref)
    assert max_err <= MAX_REL * max_ref, f"{what}: max err {max_err:.3e} > {MAX_REL} * {max_ref:.3e}"
    assert l2 <= L2_REL, f"{what}: rel L2 {l2:.3e} > {L2_REL}"
    return max_err / max_ref, l2


def sample_rows(M: int, n: int = 96, seed: int = 0) -> np.ndarray:
    """Sampled output rows: both ends and lane-quarter edges, then from every
    128-row tile (every row block of the packed weight, so every tile a
    persistent CTA or a cluster takes) its first and last row and one random
    row inside it, plus n random rows."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 31, 32, 127, 128, M // 2, M - 129, M - 128, M - 2, M - 1]
    fixed = [r for r in fixed if 0 <= r < M]
    tiles = []
    for t0 in range(0, M, 128):
        t1 = min(M, t0 + 128)
        tiles += [t0, t1 - 1, int(rng.integers(t0, t1))]
    rnd = rng.choice(M, size=min(n, M), replace=False)
    return np.unique(np.concatenate([np.asarray(fixed + tiles, dtype=np.int64), rnd.astype(np.int64)]))

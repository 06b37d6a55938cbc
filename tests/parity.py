"""Comparison helpers for the GPU parity tests (test infrastructure; uses the oracle)."""
from __future__ import annotations

import numpy as np

from oracle import quant as Q

ROT_TOL = 1e-5     # rotated values: |y - y_ref| <= 1e-5 * max(|y_ref|, rms(row))
LIN_TOL = 1e-4     # linear output:  |C - C_ref| <= 1e-4 * max(|C_ref|, rms(row))
BOUNDARY = 1e-5    # decisions within 1e-5 of a rounding boundary are excluded (and counted)


def to_device(a32: np.ndarray, bf16: bool):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a32, dtype=np.float32))
    if bf16:
        t = t.to(torch.bfloat16)
    return t.cuda()


def padded_rows(a32: np.ndarray, bf16: bool = True):
    """Device rows whose leading dimension is rounded up to a multiple of 16 bytes."""
    import torch
    M, K = a32.shape
    per = 8 if bf16 else 4
    Kp = (K + per - 1) // per * per
    t = torch.zeros((M, Kp), dtype=torch.bfloat16 if bf16 else torch.float32, device="cuda")
    t[:, :K] = to_device(a32, bf16)
    return t[:, :K]


def assert_rotated_close(y_gpu: np.ndarray, y_ref: np.ndarray, tol: float = ROT_TOL):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    bound = tol * np.maximum(np.abs(y_ref), rms)
    err = np.abs(y_gpu - y_ref)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} rotated values outside {tol}: worst {np.max(err / np.maximum(bound, 1e-300)) * tol}"
    return float(np.max(err / np.maximum(np.abs(y_ref).max(axis=1, keepdims=True), 1e-300)))


def assert_codes_match(codes_gpu, scales_gpu, y_ref: np.ndarray, bits: int, G: int):
    """Codes and scales bit-exact except where the oracle's decision is within 1e-5 of a boundary.

    Returns the number of excluded code elements."""
    K = y_ref.shape[1]
    q_ref, s_ref = Q.quantize(y_ref, bits, G)
    cflag, gflag = Q.boundary_flags(y_ref, bits, G, BOUNDARY)
    q_gpu = Q.unpack(np.asarray(codes_gpu), bits, K)
    s_gpu = np.asarray(scales_gpu).view(np.uint16)
    s_bad = (s_gpu != s_ref.view(np.uint16)) & ~gflag
    assert not s_bad.any(), f"{s_bad.sum()} scales differ outside the boundary window"
    c_bad = (q_gpu != q_ref) & ~cflag
    assert not c_bad.any(), f"{c_bad.sum()} codes differ outside the boundary window (first at {np.argwhere(c_bad)[:3]})"
    return int(cflag.sum())


def assert_linear_close(C_gpu: np.ndarray, C_ref: np.ndarray, tol: float = LIN_TOL):
    C_gpu = np.asarray(C_gpu, dtype=np.float64)
    rms = np.sqrt(np.mean(C_ref ** 2, axis=1, keepdims=True))
    bound = tol * np.maximum(np.abs(C_ref), rms)
    bad = np.abs(C_gpu - C_ref) > bound
    assert not bad.any(), f"{bad.sum()} outputs outside {tol}"


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    g = np.random.default_rng(seed)
    rows = set([0, M - 1, M // 2])
    rows.update(g.choice(M, min(M, n), replace=False).tolist())
    return np.array(sorted(rows))

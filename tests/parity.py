"""Comparison helpers for the GPU parity tests (test infrastructure; uses the oracle).

Outputs of the library are written into poisoned, guarded buffers (``Guarded``): every
byte of the output starts as a value the kernel never produces, and a tail of guard bytes
follows it. After a call, ``check()`` asserts the guard is intact; the element-by-element
comparison then fails on any element the kernel did not write.

Every rounding-boundary exclusion that ``assert_codes_match`` makes is recorded in
``EXCLUSIONS`` and printed at the end of the pytest run (``conftest.py``).
"""
from __future__ import annotations

import os

import numpy as np

from oracle import quant as Q

ROT_TOL = 1e-5     # rotated values: |y - y_ref| <= 1e-5 * max(|y_ref|, rms(row))
LIN_TOL = 1e-4     # linear output:  |C - C_ref| <= 1e-4 * max(|C_ref|, rms(row))
BOUNDARY = 1e-5    # decisions within 1e-5 of a rounding boundary are excluded (and counted)

GUARD_BYTES = 512
GUARD_FILL = 0x5A
# poison values no kernel output can hold: int4 nibble 0x8 (-8) and int2 pair 0b10 (-2) are
# outside the symmetric levels, int8 0x80 (-128) too; all-ones bytes are a NaN in binary16, bf16 and fp32
POISON = {"codes4": 0x88, "codes2": 0xAA, "codes8": 0x80, "f16": 0xFF, "f32": 0xFF, "bf16": 0xFF, "i32": 0xAB}

# (test, what, excluded codes, excluded groups, total codes, total groups)
EXCLUSIONS: list[tuple] = []


class Guarded:
    """A device tensor of ``shape``/``dtype`` carved from a byte buffer whose output bytes are
    poisoned and whose tail holds ``GUARD_BYTES`` guard bytes."""

    def __init__(self, shape, dtype, poison: int):
        import torch
        self.shape = tuple(int(s) for s in shape)
        n = int(np.prod(self.shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.raw = torch.empty(n + GUARD_BYTES, dtype=torch.uint8, device="cuda")
        self.raw[:n].fill_(poison)
        self.raw[n:].fill_(GUARD_FILL)
        self.t = self.raw[:n].view(dtype).view(self.shape)

    def check(self):
        import torch
        torch.cuda.synchronize()
        tail = self.raw[self.nbytes:]
        bad = int((tail != GUARD_FILL).sum().item())
        assert bad == 0, f"{bad} guard bytes past the end of a {self.shape} output were overwritten"


def guarded_quant(lib, A, plan, bits: int, G: int):
    """rot_quant into poisoned, guarded codes and scales; returns host (codes, scales)."""
    import torch
    M, K = A.shape[0], plan.K
    c = Guarded((M, K * bits // 8), torch.uint8, POISON[f"codes{bits}"])
    s = Guarded((M, K // G), torch.float16, POISON["f16"])
    lib.rot_quant(A, plan, bits, G, codes=c.t, scales=s.t)
    c.check()
    s.check()
    return c.t, s.t


def guarded_apply(lib, A, plan, inverse: bool = False):
    """rot_apply into a NaN-poisoned, guarded fp32 output (rows padded to 16 bytes)."""
    import torch
    Kp = (plan.K + 3) // 4 * 4
    y = Guarded((A.shape[0], Kp), torch.float32, POISON["f32"])
    out = y.t[:, :plan.K]
    lib.rot_apply(A, plan, inverse=inverse, out=out)
    y.check()
    return out


def guarded_linear(lib, fn, Aq, As, Wq, Ws, G: int, dtype):
    """A W4A4 entry point (``fn`` = lib.w4a4_linear or a variant) into a NaN-poisoned,
    guarded output."""
    import torch
    C = Guarded((Aq.shape[0], Wq.shape[0]), dtype, POISON["f32" if dtype == torch.float32 else "bf16"])
    fn(Aq, As, Wq, Ws, G, out=C.t)
    C.check()
    return C.t


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
    assert np.isfinite(y_gpu).all(), "non-finite (unwritten or poisoned) rotated values"
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    bound = tol * np.maximum(np.abs(y_ref), rms)
    err = np.abs(y_gpu - y_ref)
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} rotated values outside {tol}: worst {np.max(err / np.maximum(bound, 1e-300)) * tol}"
    return float(np.max(err / np.maximum(np.abs(y_ref).max(axis=1, keepdims=True), 1e-300)))


def assert_codes_match(codes_gpu, scales_gpu, y_ref: np.ndarray, bits: int, G: int, what: str = ""):
    """Codes and scales bit-exact except where the oracle's decision is within 1e-5 of a boundary.

    The exclusions are recorded in ``EXCLUSIONS`` (printed at the end of the run).
    Returns the number of excluded code elements."""
    if hasattr(codes_gpu, "cpu"):
        codes_gpu = codes_gpu.cpu().numpy()
    if hasattr(scales_gpu, "cpu"):
        scales_gpu = scales_gpu.cpu().numpy()
    K = y_ref.shape[1]
    q_ref, s_ref = Q.quantize(y_ref, bits, G)
    cflag, gflag = Q.boundary_flags(y_ref, bits, G, BOUNDARY)
    q_gpu = Q.unpack(np.asarray(codes_gpu), bits, K)
    s_gpu = np.asarray(scales_gpu).view(np.uint16)
    s_bad = (s_gpu != s_ref.view(np.uint16)) & ~gflag
    assert not s_bad.any(), f"{s_bad.sum()} scales differ outside the boundary window"
    c_bad = (q_gpu != q_ref) & ~cflag
    assert not c_bad.any(), f"{c_bad.sum()} codes differ outside the boundary window (first at {np.argwhere(c_bad)[:3]})"
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    EXCLUSIONS.append((test, what or f"int{bits} G={G}", int(cflag.sum()), int(gflag.sum()), int(cflag.size),
                       int(gflag.size)))
    return int(cflag.sum())


def assert_linear_close(C_gpu: np.ndarray, C_ref: np.ndarray, tol: float = LIN_TOL):
    C_gpu = np.asarray(C_gpu, dtype=np.float64)
    assert np.isfinite(C_gpu).all(), "non-finite (unwritten or poisoned) outputs"
    rms = np.sqrt(np.mean(C_ref ** 2, axis=1, keepdims=True))
    bound = tol * np.maximum(np.abs(C_ref), rms)
    bad = np.abs(C_gpu - C_ref) > bound
    assert not bad.any(), f"{bad.sum()} outputs outside {tol}"


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    g = np.random.default_rng(seed)
    rows = set([0, M - 1, M // 2])
    rows.update(g.choice(M, min(M, n), replace=False).tolist())
    return np.array(sorted(rows))

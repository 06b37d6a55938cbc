"""W4A4 linear and the page-2 matmul quantisation-error metric, fp64 / int64.

Sources:
* Hadamard-Int4-Accuracy wiki, Hypothesis: W4A4 is a same-precision int4 MAC of
  4-bit activations and 4-bit weights; A.B = (A.Q).(Q.B) exactly, so the rotated
  operands are quantised instead.
* same page, Method: ``matmul_q_err(..., abits, bbits, rotate)`` measures the RMS
  error of the quantised product relative to the fp32 reference; the five printed
  rows are W8A8, W4A4 plain / + Hadamard, W4A8 (activations 8-bit, weights 4-bit)
  plain / + Hadamard.

Reading: "RMS rel" = ||C_q - C||_F / ||C||_F over all M x N outputs.
"""
from __future__ import annotations

import numpy as np

from . import quant as Q


def group_partials(qa: np.ndarray, qw: np.ndarray, G: int) -> np.ndarray:
    """P[m, n, g] = sum_{k in group g} qa[m, k] * qw[n, k], exact int64."""
    M, K = qa.shape
    N = qw.shape[0]
    a = qa.astype(np.int64).reshape(M, K // G, G)
    w = qw.astype(np.int64).reshape(N, K // G, G)
    return np.einsum("mgk,ngk->mng", a, w)


def w4a4_reference(qa: np.ndarray, sa16: np.ndarray, qw: np.ndarray, sw16: np.ndarray,
                   G: int) -> np.ndarray:
    """C[m, n] = sum_g float(sa[m,g]) * float(sw[n,g]) * P[m,n,g] in fp64."""
    P = group_partials(qa, qw, G).astype(np.float64)
    sa = sa16.astype(np.float64)
    sw = sw16.astype(np.float64)
    return np.einsum("mg,ng,mng->mn", sa, sw, P)


def w4a8_reference(qa8: np.ndarray, sa16: np.ndarray, qw: np.ndarray, sw16: np.ndarray, G: int) -> np.ndarray:
    """The W4A8 linear (int8 activation codes, int4 weight codes; the wiki's "W4A8 (act8/wt4)"
    row): the same definition, C[m, n] = sum_g float(sa[m,g]) * float(sw[n,g]) * P[m,n,g] with
    exact int64 group sums of the int8 x int4 products, in fp64."""
    return w4a4_reference(qa8, sa16, qw, sw16, G)


def two_sided_weights(B: np.ndarray, rot_in, rot_out) -> np.ndarray:
    """Offline weight preparation of a two-sided processor (HARP abstract: a two-sided orthogonal
    processor). With the input-side operator T (``rot_in``: rows x -> T x, size K) and the
    output-side operator U (``rot_out``: rows x -> U x, size N), B~ = T B U^T; returned as the rows
    of B~^T [N, K] (what is quantised): the rows of B (length N) go through U, then the columns
    of B U^T (length K) through T."""
    BU = rot_out(np.asarray(B, dtype=np.float64))        # rows of B -> U b: B U^T  [K, N]
    return rot_in(np.ascontiguousarray(BU.T))            # columns of B U^T -> T col: (T B U^T)^T


def unrotate_output(Ct: np.ndarray, rot_out_inv) -> np.ndarray:
    """Rows c~ = U c of the two-sided linear's output back to c = U^T c~ (``rot_out_inv``: rows
    x -> U^T x)."""
    return rot_out_inv(np.asarray(Ct, dtype=np.float64))


def _quant_dequant_rows(X: np.ndarray, bits: int, G: int) -> np.ndarray:
    q, s = Q.quantize(X, bits, G)
    return Q.dequantize(q, s, G).astype(np.float64)


def matmul_q_err(A: np.ndarray, B: np.ndarray, abits: int, bbits: int, rotate, G: int) -> float:
    """RMS relative error of the group-quantised product against A.B (fp64).

    ``rotate``: None/False for the plain product, else a callable applying the
    column operator T to rows (y = T a); A's rows become T a and B's columns T b.
    """
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    C = A @ B
    if rotate:
        Ar = rotate(A)
        Br = rotate(B.T)          # columns of B are rotated: (T B)^T = rows T b
    else:
        Ar, Br = A, B.T
    Aq = _quant_dequant_rows(Ar, abits, G)
    Bq = _quant_dequant_rows(Br, bbits, G)
    Cq = Aq @ Bq.T
    return float(np.linalg.norm(Cq - C) / np.linalg.norm(C))

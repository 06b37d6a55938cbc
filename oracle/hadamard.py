"""Sylvester Hadamard matrices and the randomized Hadamard transform (RHT), fp64.

Sources:
* Hadamard-Int4-Accuracy wiki (oRKLLM ork-driver, "Experiment -- Hadamard rotation
  for int4 (W4A4) accuracy"), Hypothesis: Q = H/sqrt(K) is orthonormal and
  symmetric, and A.B = (A.Q).(Q.B) exactly; Method: ``fwht_norm()`` is the fast
  Walsh-Hadamard transform followed by x 1/sqrt(K); Reproduce: plain FWHT needs a
  power-of-two K.
* HARP abstract (arXiv 2605.29843) and its gist.science summary, section 1
  (problem statement): the randomized Hadamard transform is O(d log d) and
  exactly orthogonal; "randomized" = random +-1 signs applied before the
  transform.

Convention (column operator): a row a of A is mapped to y = T a with
T = H_K D / sqrt(K), D = diag(signs). With signs all +1 this is the page-2 probe's
symmetric Q = H/sqrt(K).
"""
from __future__ import annotations

import numpy as np


def is_pow2(K: int) -> bool:
    return K >= 1 and (K & (K - 1)) == 0


def sylvester(K: int) -> np.ndarray:
    """Dense Sylvester Hadamard matrix, H[i, j] = (-1)^popcount(i & j), int8."""
    if not is_pow2(K):
        raise ValueError("Sylvester Hadamard matrices exist only for power-of-two K")
    i = np.arange(K, dtype=np.int64)
    return _sylvester_rows(i, K)


def _sylvester_rows(rows: np.ndarray, K: int) -> np.ndarray:
    """Rows ``rows`` of H_K, int8 in {+1,-1}."""
    j = np.arange(K, dtype=np.int64)
    x = rows[:, None] & j[None, :]
    # parity of popcount(x), bit by bit
    par = np.zeros_like(x)
    while np.any(x):
        par ^= x & 1
        x >>= 1
    return (1 - 2 * par).astype(np.int8)


def rht_matrix(K: int, signs: np.ndarray | None = None) -> np.ndarray:
    """Dense T = H_K D / sqrt(K) in fp64 (small K only)."""
    H = sylvester(K).astype(np.float64)
    d = np.ones(K) if signs is None else signs.astype(np.float64)
    return H * d[None, :] / np.sqrt(K)


def rht_apply(A: np.ndarray, signs: np.ndarray | None = None, *, inverse: bool = False,
              chunk: int = 512) -> np.ndarray:
    """y = T a for every row a of A (fp64), T = H_K D / sqrt(K).

    ``inverse`` applies T^T = D H_K / sqrt(K) instead. The dense product is done
    over chunks of output coordinates only to bound memory (H rows are generated
    on the fly from their closed form); no butterfly factorisation is used.
    """
    A = np.asarray(A, dtype=np.float64)
    M, K = A.shape
    d = np.ones(K) if signs is None else signs.astype(np.float64)
    out = np.empty((M, K), dtype=np.float64)
    inv_sqrt = 1.0 / np.sqrt(K)
    if not inverse:
        X = A * d[None, :]
        for i0 in range(0, K, chunk):
            rows = np.arange(i0, min(K, i0 + chunk), dtype=np.int64)
            Hc = _sylvester_rows(rows, K).astype(np.float64)
            out[:, i0:i0 + len(rows)] = (X @ Hc.T) * inv_sqrt
    else:
        for i0 in range(0, K, chunk):
            rows = np.arange(i0, min(K, i0 + chunk), dtype=np.int64)
            Hc = _sylvester_rows(rows, K).astype(np.float64)  # H symmetric
            out[:, i0:i0 + len(rows)] = (A @ Hc.T) * inv_sqrt
        out *= d[None, :]
    return out


def fwht_norm_loop(x: list[float]) -> list[float]:
    """Page-2 style in-place butterfly FWHT then x 1/sqrt(K), pure Python.

    For pins only (tiny K): each stage replaces (a, b) by (a + b, a - b) for the
    pairs at distance h = 1, 2, 4, ...; the result is scaled by 1/sqrt(K).
    """
    v = [float(t) for t in x]
    K = len(v)
    if not is_pow2(K):
        raise ValueError("plain FWHT needs a power-of-two length")
    h = 1
    while h < K:
        for start in range(0, K, 2 * h):
            for j in range(start, start + h):
                a, b = v[j], v[j + h]
                v[j], v[j + h] = a + b, a - b
        h *= 2
    s = 1.0 / K ** 0.5
    return [t * s for t in v]

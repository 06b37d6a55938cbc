"""HARP mixed-radix block-orthogonal processor, fp64, stage by stage.

Sources (HARP, arXiv 2605.29843):
* abstract: each rotation is a product of sparse butterfly-like block-orthogonal
  stages, non-power-of-two dimensions use mixed-radix schedules, and the
  processor initialises to the RHT up to a fixed permutation;
* gist.science summary, section 2.1 (core architecture): schedule
  b = (b_0..b_{m-1}) with prod b_t = d; stage t applies a block-diagonal
  orthogonal B_t to coordinate groups, separated by stride permutations;
  non-power-of-two radices use a deterministic orthogonal fallback (QR of a fixed
  Gaussian matrix); example 5120 = (8, 8, 8, 5, 2);
* section 2.2 (Hadamard preconditioning & initialisation):
  B_{t,c}(theta) = Q_{t,c}(theta) G_{b_t}; G is the normalised Sylvester-Hadamard
  matrix for powers of two, the QR fallback otherwise; Q is a Givens rotation for
  b_t = 2; at theta = 0, Q = I so B = G and HARP equals the RHT.

Readings where the pages leave a step open:
* digit addressing: coordinate i = sum_t d_t s_t with s_t = prod_{u<t} b_u
  (digit 0 least significant). Stage t mixes the b_t coordinates that differ only
  in digit t, base + r*s_t for r = 0..b_t-1, with block index
  c = low + high*s_t (low = digits below t, high = digits above t). With this
  "stride" convention the theta = 0 processor equals H_K D / sqrt(K) exactly, so
  the fixed permutation of the page is the identity.
* optional gather after stage t: x''[j] = x'[P_t[j]].
* Givens block: R(theta) = [[cos, -sin], [sin, cos]], B = R(theta) H_2 / sqrt(2).
* QR fallback: Q factor of a Gaussian b x b matrix with diag(R) > 0.
* base mixer used when a stage gives no parameters: H_b / sqrt(b) for a power of
  two b, the identity otherwise.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .hadamard import is_pow2, sylvester


def base_mixer(b: int) -> np.ndarray:
    if is_pow2(b):
        return sylvester(b).astype(np.float64) / np.sqrt(b)
    return np.eye(b)


def givens_blocks(theta: np.ndarray) -> np.ndarray:
    """B = R(theta) . H_2/sqrt(2) for each angle, shape [n, 2, 2]."""
    theta = np.asarray(theta, dtype=np.float64)
    c, s = np.cos(theta), np.sin(theta)
    R = np.empty(theta.shape + (2, 2))
    R[..., 0, 0], R[..., 0, 1] = c, -s
    R[..., 1, 0], R[..., 1, 1] = s, c
    return R @ base_mixer(2)


def qr_block(gauss: np.ndarray) -> np.ndarray:
    """Q of the QR factorisation of a square Gaussian matrix, diag(R) made positive."""
    Q, R = np.linalg.qr(np.asarray(gauss, dtype=np.float64))
    d = np.sign(np.diag(R))
    d[d == 0] = 1.0
    return Q * d[None, :]


def cayley(params: np.ndarray, b: int) -> np.ndarray:
    """Cayley map of a b x b skew-symmetric matrix S built from its b(b-1)/2 strictly upper
    entries (row-major order: S[i, j] = p_k for i < j, S[j, i] = -p_k):
    Q(S) = (I + S)^{-1} (I - S)  (= (I - S)(I + S)^{-1}; the two factors commute).

    Source: HARP gist.science summary, section 2.2: Q_{t,c}(theta) is a learnable orthogonal
    matrix, a Cayley map for b_t > 2, with Q(0) = I. Reading: the standard Cayley transform of a
    skew-symmetric matrix (orthogonal with determinant +1); the page does not fix the sign
    convention or the parameter order.
    """
    p = np.asarray(params, dtype=np.float64).reshape(-1)
    if p.size != b * (b - 1) // 2:
        raise ValueError("a b x b Cayley block takes b(b-1)/2 parameters")
    S = np.zeros((b, b))
    iu = np.triu_indices(b, 1)
    S[iu] = p
    S -= S.T
    eye = np.eye(b)
    return np.linalg.solve(eye + S, eye - S)


def cayley_blocks(params: np.ndarray, b: int, mixer: np.ndarray | None = None) -> np.ndarray:
    """B = Q(theta) G_b for each parameter row (HARP summary, section 2.2: B = Q(theta) G,
    G the base mixer: normalised Sylvester-Hadamard for powers of two, else the given fallback
    mixer, e.g. the QR of a fixed Gaussian). params: [n, b(b-1)/2] -> [n, b, b]."""
    G = base_mixer(b) if mixer is None else np.asarray(mixer, dtype=np.float64)
    P = np.asarray(params, dtype=np.float64).reshape(-1, b * (b - 1) // 2)
    return np.stack([cayley(p, b) @ G for p in P])


def quant_params_int8(theta: np.ndarray):
    """Store a stage's parameters in int8 (HARP gist.science summary, section 2.4: the
    parameters can be stored in int8 with minimal effect; section 4: 2.00 -> 2.05 bits per
    parameter). Reading: one symmetric absmax scale per stage, s = fp32(max|theta| / 127),
    codes q = clamp(round_half_away(theta / s), -127, 127); s = 0 gives q = 0.
    Returns (codes int8, scale float32)."""
    th = np.asarray(theta, dtype=np.float64)
    s = np.float32(np.max(np.abs(th)) / 127.0) if th.size else np.float32(0.0)
    if s == 0:
        return np.zeros(th.shape, dtype=np.int8), np.float32(0.0)
    v = th / np.float64(s)
    q = np.clip(np.sign(v) * np.floor(np.abs(v) + 0.5), -127, 127)
    return q.astype(np.int8), s


def dequant_params_int8(codes: np.ndarray, scale) -> np.ndarray:
    """theta = q * s in fp64 (s the stored fp32 scale)."""
    return np.asarray(codes, dtype=np.float64) * np.float64(np.float32(scale))


@dataclass
class HarpSpec:
    K: int
    radices: list[int]
    blocks: list[np.ndarray | None]          # per stage: None (base mixer) or [n, b, b], n in {1, K/b}
    perms: list[np.ndarray | None] = field(default_factory=list)
    signs: np.ndarray | None = None

    def __post_init__(self):
        if int(np.prod(self.radices)) != self.K:
            raise ValueError("product of radices must equal K")
        if not self.perms:
            self.perms = [None] * len(self.radices)


def spec_from_draws(draws, signs: np.ndarray | None, variant: str) -> HarpSpec:
    """Build a processor from the seeded draws of ``workloads.harp_draws``.

    variant:
      ``random``       Givens blocks from the angles, QR blocks from the Gaussians,
                       the drawn permutations between stages;
      ``init_identity`` theta = 0 (blocks = base mixers), identity for the
                       non-power-of-two radix, no permutations;
      ``init_qr``      theta = 0, QR-fallback block for the non-power-of-two
                       radix (page-4 reading of the initial state), no permutations.
    """
    radices = list(draws.radices)
    K = int(np.prod(radices))
    blocks: list[np.ndarray | None] = []
    for t, b in enumerate(radices):
        if variant == "random":
            if b == 2:
                blocks.append(givens_blocks(draws.angles[t]))
            else:
                blocks.append(np.stack([qr_block(gm) for gm in draws.gaussians[t]]))
        elif variant == "init_identity":
            blocks.append(None)
        elif variant == "init_qr":
            if b == 2 or is_pow2(b):
                blocks.append(None)
            else:
                blocks.append(qr_block(draws.gaussians[t][0])[None])
        else:
            raise ValueError(variant)
    perms = list(draws.perms) if variant == "random" else [None] * len(radices)
    return HarpSpec(K, radices, blocks, perms, signs)


def spec_from_q8(draws, signs: np.ndarray | None) -> HarpSpec:
    """A processor stored with int8 parameters (``workloads.harp_q8_draws``): per stage
    theta = code * scale (dequant_params_int8); Givens blocks for b = 2, Cayley blocks
    Q(theta) G_b for b > 2 with G_b the Sylvester-Hadamard mixer (powers of two) or the QR
    fallback of the drawn Gaussian; the drawn permutations between stages."""
    radices = list(draws.radices)
    K = int(np.prod(radices))
    blocks = []
    for t, b in enumerate(radices):
        th = dequant_params_int8(draws.codes[t], draws.scales[t])
        if b == 2:
            blocks.append(givens_blocks(th))
        else:
            mix = None if draws.mixer_gaussians[t] is None else qr_block(draws.mixer_gaussians[t])
            blocks.append(cayley_blocks(th, b, mix))
    return HarpSpec(K, radices, blocks, list(draws.perms), signs)


def _stage_blocks(spec: HarpSpec, t: int) -> np.ndarray:
    b = spec.radices[t]
    B = spec.blocks[t]
    return base_mixer(b)[None] if B is None else np.asarray(B, dtype=np.float64)


def stage_apply(X: np.ndarray, spec: HarpSpec, t: int, *, transpose: bool = False) -> np.ndarray:
    """Apply the block-diagonal stage S_t (or S_t^T) to every row of X (no permutation)."""
    M = X.shape[0]
    b = spec.radices[t]
    s_t = int(np.prod(spec.radices[:t])) if t else 1
    high = spec.K // (s_t * b)
    Xv = X.reshape(M, high, b, s_t)            # i = l + r*s_t + h*s_t*b
    B = _stage_blocks(spec, t)
    if transpose:
        B = np.swapaxes(B, -1, -2)
    if B.shape[0] == 1:
        Y = np.einsum("rs,mhsl->mhrl", B[0], Xv)
    else:
        Bc = B.reshape(high, s_t, b, b)          # block index c = l + h*s_t
        Y = np.einsum("hlrs,mhsl->mhrl", Bc, Xv)
    return Y.reshape(M, spec.K)


def harp_apply(A: np.ndarray, spec: HarpSpec, *, inverse: bool = False) -> np.ndarray:
    """y = T a for each row a, T = (P_{m-1} S_{m-1}) ... (P_0 S_0) D; ``inverse`` gives T^T a."""
    X = np.array(A, dtype=np.float64, copy=True)
    d = None if spec.signs is None else spec.signs.astype(np.float64)
    m = len(spec.radices)
    if not inverse:
        if d is not None:
            X *= d[None, :]
        for t in range(m):
            X = stage_apply(X, spec, t)
            if spec.perms[t] is not None:
                X = X[:, spec.perms[t]]
    else:
        for t in reversed(range(m)):
            P = spec.perms[t]
            if P is not None:
                Y = np.empty_like(X)
                Y[:, P] = X                    # inverse of the gather x''[j] = x'[P[j]]
                X = Y
            X = stage_apply(X, spec, t, transpose=True)
        if d is not None:
            X *= d[None, :]
    return X


def harp_dense(spec: HarpSpec) -> np.ndarray:
    """Dense K x K matrix T (small K only): column j is T e_j."""
    return harp_apply(np.eye(spec.K), spec).T


def stage_matrix_explicit(spec: HarpSpec, t: int) -> np.ndarray:
    """Explicit K x K matrix of S_t built coordinate by coordinate (pure loops, pins only)."""
    K, b = spec.K, spec.radices[t]
    s_t = int(np.prod(spec.radices[:t])) if t else 1
    B = _stage_blocks(spec, t)
    S = np.zeros((K, K))
    for base in range(K):
        digit = (base // s_t) % b
        if digit != 0:
            continue
        low = base % s_t
        high = base // (s_t * b)
        c = low + high * s_t
        Bc = B[0] if B.shape[0] == 1 else B[c]
        for r in range(b):
            for r2 in range(b):
                S[base + r * s_t, base + r2 * s_t] = Bc[r, r2]
    return S

"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a closed form, a
library routine, an independent construction, brute force on tiny inputs, or
numbers printed on the pages (``tests/golden/``).
"""
from fractions import Fraction
import os

import numpy as np
import pytest
import scipy.linalg

import workloads as W
from oracle import hadamard as Hd
from oracle import harp as Hp
from oracle import linear as L
from oracle import quant as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("K", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_sylvester_gram_is_K_identity(K):
    # H H^T = K I exactly in integers (Hadamard-Int4-Accuracy wiki, Hypothesis: Q = H/sqrt(K) orthonormal)
    H = Hd.sylvester(K).astype(np.int64)
    assert np.array_equal(H @ H.T, K * np.eye(K, dtype=np.int64))
    assert np.array_equal(H, H.T)  # symmetric


@pytest.mark.parametrize("K", [2, 8, 128, 2048])
def test_sylvester_matches_library_and_kronecker(K):
    H = Hd.sylvester(K)
    assert np.array_equal(H, scipy.linalg.hadamard(K))
    kr = np.array([[1]])
    while kr.shape[0] < K:
        kr = np.kron(np.array([[1, 1], [1, -1]]), kr)
    assert np.array_equal(H, kr)


def test_non_power_of_two_rejected():
    # "plain FWHT needs power-of-2 K" (Hadamard-Int4-Accuracy wiki, Reproduce)
    with pytest.raises(ValueError):
        Hd.sylvester(12)
    with pytest.raises(ValueError):
        Hd.fwht_norm_loop([1.0] * 6)


@pytest.mark.parametrize("K", [2, 4, 8, 16, 32, 64])
def test_fwht_loop_equals_dense(K):
    g = np.random.default_rng(K)
    X = g.standard_normal((5, K))
    dense = Hd.rht_apply(X)
    loop = np.array([Hd.fwht_norm_loop(list(r)) for r in X])
    assert np.max(np.abs(dense - loop)) < 1e-12


@pytest.mark.parametrize("K", [4, 64, 512, 2048])
def test_rht_orthonormal(K):
    Qm = Hd.rht_matrix(K)
    assert np.max(np.abs(Qm @ Qm.T - np.eye(K))) < 1e-12
    assert np.array_equal(Qm, Qm.T)
    s = W.signs(W.rng(K), K)
    T = Hd.rht_matrix(K, s)
    assert np.max(np.abs(T @ T.T - np.eye(K))) < 1e-12
    D = np.diag(s.astype(float))
    assert np.array_equal(D @ D, np.eye(K))


def test_rht_apply_matches_matrix_and_inverse():
    K = 256
    g = np.random.default_rng(1)
    s = W.signs(g, K)
    X = g.standard_normal((7, K))
    T = Hd.rht_matrix(K, s)
    Y = Hd.rht_apply(X, s, chunk=64)
    assert np.max(np.abs(Y - X @ T.T)) < 1e-12
    assert np.max(np.abs(Hd.rht_apply(Y, s, inverse=True) - X)) < 1e-12


def test_exact_equivalence_pr1():
    # A.B = (A.Q)(Q^T.B) exactly in full precision (wiki Hypothesis; HARP abstract)
    wl = W.make_workload("pr1")
    A, B = wl.A.astype(np.float64), wl.W.astype(np.float64)
    C = A @ B
    Ar = Hd.rht_apply(A, wl.signs)
    Br = Hd.rht_apply(B.T, wl.signs).T
    assert np.linalg.norm(C - Ar @ Br) / np.linalg.norm(C) < 1e-12


def test_rotation_scatters_outliers():
    # page-1 model card: rotation lowers the peak activation (context: "10x"); here only "much lower"
    wl = W.make_workload("pr1")
    Y = Hd.rht_apply(wl.A, wl.signs)
    assert np.abs(Y).max() < 0.5 * np.abs(wl.A).max()


# ----------------------------------------------------------------------------- HARP

def test_schedules_from_pages():
    with open(os.path.join(GOLDEN, "harp_schedules.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            d, *rad = [int(t) for t in line.split()]
            assert int(np.prod(rad)) == d
            Hp.HarpSpec(d, rad, [None] * len(rad))
    with pytest.raises(ValueError):
        Hp.HarpSpec(5120, [8, 8, 8, 5], [None] * 4)


def test_givens_blocks():
    th = np.random.default_rng(0).uniform(-np.pi, np.pi, 100)
    B = Hp.givens_blocks(th)
    I = np.einsum("nij,nkj->nik", B, B)
    assert np.max(np.abs(I - np.eye(2))) < 1e-12
    B0 = Hp.givens_blocks(np.zeros(1))[0]
    assert np.max(np.abs(B0 - np.array([[1, 1], [1, -1]]) / np.sqrt(2))) < 1e-15
    # theta rotates the Hadamard block: B(theta) = R(theta) B(0)
    t = 0.3
    R = np.array([[np.cos(t), -np.sin(t)], [np.sin(t), np.cos(t)]])
    assert np.max(np.abs(Hp.givens_blocks(np.array([t]))[0] - R @ B0)) < 1e-15


@pytest.mark.parametrize("b", [3, 5, 43])
def test_qr_block(b):
    G = np.random.default_rng(b).standard_normal((b, b))
    Qb = Hp.qr_block(G)
    assert np.max(np.abs(Qb @ Qb.T - np.eye(b))) < 1e-12
    R = Qb.T @ G
    assert np.max(np.abs(np.tril(R, -1))) < 1e-12      # upper triangular
    assert np.all(np.diag(R) > 0)                        # sign convention
    assert np.max(np.abs(Qb @ R - G)) < 1e-12


def _random_spec(radices, seed, per_block=True, perms=True, signs=True):
    K = int(np.prod(radices))
    g = np.random.default_rng(seed)
    blocks = []
    for b in radices:
        n = K // b if per_block else 1
        blocks.append(np.stack([Hp.qr_block(g.standard_normal((b, b))) for _ in range(n)]))
    P = [g.permutation(K) if (perms and t < len(radices) - 1) else None for t in range(len(radices))]
    s = (1 - 2 * g.integers(0, 2, K)).astype(np.int8) if signs else None
    return Hp.HarpSpec(K, list(radices), blocks, P, s)


@pytest.mark.parametrize("radices", [[2, 2, 3], [2, 3, 2, 2], [2, 43], [5, 3, 2], [3, 4]])
@pytest.mark.parametrize("per_block", [True, False])
def test_stage_apply_matches_explicit_loops(radices, per_block):
    spec = _random_spec(radices, 7, per_block=per_block)
    K = spec.K
    X = np.random.default_rng(3).standard_normal((4, K))
    for t in range(len(radices)):
        S = Hp.stage_matrix_explicit(spec, t)
        assert np.max(np.abs(Hp.stage_apply(X, spec, t) - X @ S.T)) < 1e-12
        assert np.max(np.abs(S @ S.T - np.eye(K))) < 1e-12
    # composite with signs and gathers, built from the explicit matrices
    T = np.diag(spec.signs.astype(float))
    for t in range(len(radices)):
        Pm = np.eye(K)[spec.perms[t]] if spec.perms[t] is not None else np.eye(K)
        T = Pm @ Hp.stage_matrix_explicit(spec, t) @ T
    assert np.max(np.abs(Hp.harp_dense(spec) - T)) < 1e-12
    assert np.max(np.abs(T @ T.T - np.eye(K))) < 1e-12
    Y = Hp.harp_apply(X, spec)
    assert np.max(np.abs(Hp.harp_apply(Y, spec, inverse=True) - X)) < 1e-12


@pytest.mark.parametrize("K", [2, 8, 64, 256, 2048])
def test_harp_init_equals_rht(K):
    # theta = 0 -> B = G (normalised Sylvester) -> HARP = RHT (gist.science summary, 2.2)
    n = int(np.log2(K))
    s = W.signs(W.rng(K + 1), K)
    spec = Hp.HarpSpec(K, [2] * n, [None] * n, signs=s)
    X = np.random.default_rng(0).standard_normal((3, K))
    assert np.max(np.abs(Hp.harp_apply(X, spec) - Hd.rht_apply(X, s))) < 1e-12
    # explicit Givens blocks at theta = 0 give the same processor
    spec2 = Hp.HarpSpec(K, [2] * n, [Hp.givens_blocks(np.zeros(K // 2))] * n, signs=s)
    assert np.max(np.abs(Hp.harp_apply(X, spec2) - Hd.rht_apply(X, s))) < 1e-12


def test_mixed_radix_init_5120_pattern():
    # 5120-style schedule scaled down: (8, 5, 2) with base mixers; identity radix-5 stage
    spec = Hp.HarpSpec(80, [8, 5, 2], [None] * 3)
    T = Hp.harp_dense(spec)
    assert np.max(np.abs(T @ T.T - np.eye(80))) < 1e-12
    # digits 0 (radix 8) and 2 (radix 2) form a 16-point Sylvester transform on {i: digit1 fixed}
    H8 = Hd.sylvester(8) / np.sqrt(8)
    H2 = Hd.sylvester(2) / np.sqrt(2)
    ref = np.kron(H2, np.kron(np.eye(5), H8))
    assert np.max(np.abs(T - ref)) < 1e-12


def test_harp11008_identity43_is_blockwise_rht():
    K = 11008
    s = W.signs(W.rng(5), K)
    spec = Hp.HarpSpec(K, [2] * 8 + [43], [None] * 9, signs=s)
    X = np.random.default_rng(2).standard_normal((3, K))
    Y = Hp.harp_apply(X, spec)
    for c in range(43):
        sl = slice(256 * c, 256 * (c + 1))
        ref = Hd.rht_apply(X[:, sl], s[sl])
        assert np.max(np.abs(Y[:, sl] - ref)) < 1e-12


def test_harp11008_random_orthonormal_sampled():
    d = W.harp_draws(2, [2] * 8 + [43])
    s = W.signs(W.rng(9), 11008)
    spec = Hp.spec_from_draws(d, s, "random")
    g = np.random.default_rng(4)
    idx = g.choice(11008, 64, replace=False)
    E = np.zeros((64, 11008))
    E[np.arange(64), idx] = 1.0
    Te = Hp.harp_apply(E, spec)          # rows T e_i
    assert np.max(np.abs(Te @ Te.T - np.eye(64))) < 1e-12
    x = g.standard_normal((2, 11008))
    assert np.allclose(np.linalg.norm(Hp.harp_apply(x, spec), axis=1), np.linalg.norm(x, axis=1),
                       rtol=1e-12, atol=0)


# ----------------------------------------------------------------------------- quantiser

def test_quantize_hand_cases():
    y = np.array([[7.0, 2.5, -2.5, 0.5, -0.5, 1.4999, 0.0, 3.5]])
    q, s = Q.quantize(y, 4, 8)
    assert s[0, 0] == np.float16(1.0)
    assert q.tolist() == [[7, 3, -3, 1, -1, 1, 0, 4]]
    # int2: levels -1..1, scale absmax/1
    q2, s2 = Q.quantize(np.array([[2.0, 1.0, -0.999, 0.5, -0.5, 0.49, 0, -2]]), 2, 8)
    assert s2[0, 0] == np.float16(2.0)
    assert q2.tolist() == [[1, 1, 0, 0, 0, 0, 0, -1]]   # v = 0.5 rounds away from zero


def test_quantize_zero_group_subnormal_scale_and_clamp():
    y = np.zeros((1, 16))
    y[0, 8:] = [6e-7, 3e-7, -1e-7, 0, 0, 0, 0, 0]
    q, s = Q.quantize(y, 4, 8)
    assert s[0, 0] == 0 and np.all(q[0, :8] == 0)            # all-zero group
    # 6e-7/7 rounds to the smallest binary16 subnormal 2^-24, so v = 6e-7 * 2^24 ~ 10 -> clamp to 7
    assert s[0, 1] == np.float16(2.0 ** -24)
    assert q[0, 8] == 7 and q[0, 9] == 5 and q[0, 10] == -2
    # a scale that underflows to zero gives zero codes
    qz, sz = Q.quantize(np.array([[1e-8, -1e-8, 0, 0]]), 4, 4)
    assert sz[0, 0] == 0 and np.all(qz == 0)
    # a scale that overflows binary16 gives zero codes (v = y / inf)
    qi, si = Q.quantize(np.array([[1e6, 3.0, -2.0, 0]]), 4, 4)
    assert np.isinf(si[0, 0]) and np.all(qi == 0)


def test_scale_fp16_rounding_ties_to_even():
    m = np.array([7 * (1 + 2.0 ** -11), 7 * (1 + 3 * 2.0 ** -11), 7.0 / 3, 7 * 65504.0, 7 * 65520.0],
                 dtype=np.float32)
    s = Q.scales_fp16(m, 4)
    assert s[0] == np.float16(1.0)
    assert s[1] == np.float16(1 + 2.0 ** -9)
    assert s[2].view(np.uint16) == 0x3555            # 1/3 in binary16
    assert s[3] == np.float16(65504.0)
    assert np.isinf(s[4])


def test_quantize_brute_force_exact_rationals():
    # independent scalar evaluation: absmax, fp16 scale, exact rational quotient, round half away
    g = np.random.default_rng(11)
    for bits, G in [(4, 8), (2, 4), (8, 16), (4, 32)]:
        y = g.standard_normal((6, 4 * G)) * np.exp(g.uniform(-3, 3, (6, 1)))
        y[:, 3] *= 20.0
        q, s = Q.quantize(y, bits, G)
        qm = 2 ** (bits - 1) - 1
        y32 = y.astype(np.float32)
        for m in range(y.shape[0]):
            for gi in range(y.shape[1] // G):
                grp = y32[m, gi * G:(gi + 1) * G]
                amax = max(abs(float(v)) for v in grp)
                sc = float(np.float16(np.float32(amax) / np.float32(qm)))
                assert sc == float(s[m, gi])
                for j, v in enumerate(grp):
                    if sc == 0:
                        ref = 0
                    else:
                        r = Fraction(float(v)) / Fraction(sc)
                        a = abs(r)
                        if abs(a - int(a) - Fraction(1, 2)) < Fraction(1, 10 ** 6):
                            continue  # fp32 division may round across an exact-rational tie
                        k = int(a + Fraction(1, 2))
                        ref = max(-qm, min(qm, k if r >= 0 else -k))
                    assert q[m, gi * G + j] == ref


def test_dequantize_error_bound():
    g = np.random.default_rng(12)
    y = g.standard_normal((8, 256))
    for bits in (2, 4, 8):
        q, s = Q.quantize(y, bits, 32)
        xh = Q.dequantize(q, s, 32)
        err = np.abs(xh - y.astype(np.float32)).reshape(8, 8, 32)
        bound = s.astype(np.float64)[..., None] * 0.5 * (1 + 1e-3)
        assert np.all(err <= bound + 1e-7 * np.abs(y).reshape(8, 8, 32))


def test_pack_layout_hand_cases():
    assert Q.pack(np.array([[1, -1]]), 4).tolist() == [[0xF1]]
    assert Q.pack(np.array([[7, -7]]), 4).tolist() == [[0x97]]
    assert Q.pack(np.array([[1, -1, 0, 1]]), 2).tolist() == [[0x4D]]
    assert Q.pack(np.array([[-1, 127, -127]]), 8).tolist() == [[0xFF, 0x7F, 0x81]]
    g = np.random.default_rng(5)
    for bits in (2, 4, 8):
        qm = 2 ** (bits - 1) - 1
        c = g.integers(-qm, qm + 1, (3, 64)).astype(np.int8)
        assert np.array_equal(Q.unpack(Q.pack(c, bits), bits, 64), c)


def test_boundary_flags_mark_ties():
    y = np.array([[7.0, 2.5, 2.5 + 1e-7, 2.3, -1.5, 0.1, 0.0, 3.0]])
    cf, gf = Q.boundary_flags(y, 4, 8)
    assert cf.tolist() == [[False, True, True, False, True, False, False, False]]
    assert not gf.any()
    # absmax/qmax at a binary16 midpoint flags the whole group
    y2 = np.array([[7 * (1 + 2.0 ** -11), 1.0, 0.2, 0.3]])
    cf2, gf2 = Q.boundary_flags(y2, 4, 4)
    assert gf2.all() and cf2.all()


# ----------------------------------------------------------------------------- W4A4 linear

def test_group_partials_brute_force():
    g = np.random.default_rng(3)
    M, N, K, G = 3, 5, 16, 8
    qa = g.integers(-7, 8, (M, K))
    qw = g.integers(-7, 8, (N, K))
    sa = g.uniform(0.01, 1, (M, K // G)).astype(np.float16)
    sw = g.uniform(0.01, 1, (N, K // G)).astype(np.float16)
    P = L.group_partials(qa, qw, G)
    C = L.w4a4_reference(qa, sa, qw, sw, G)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for gi in range(K // G):
                p = sum(int(qa[m, k]) * int(qw[n, k]) for k in range(gi * G, (gi + 1) * G))
                assert P[m, n, gi] == p
                tot += float(sa[m, gi]) * float(sw[n, gi]) * p
            assert abs(C[m, n] - tot) <= 1e-12 * max(1.0, abs(tot))
    # one group spanning K: C = sa sw (qa qw^T)
    C1 = L.w4a4_reference(qa, sa[:, :1], qw, sw[:, :1], K)
    ref = sa[:, :1].astype(float) * sw[:, :1].astype(float).T * (qa @ qw.T)
    assert np.max(np.abs(C1 - ref)) < 1e-12


def _page2_table():
    rows = {}
    with open(os.path.join(GOLDEN, "page2_synthetic_error_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, ab, bb, rot, g128, g32 = line.split()
            rows[name] = (int(ab), int(bb), int(rot), float(g128), float(g32))
    return rows


def test_page2_synthetic_error_table():
    """W4A4 RMS errors, plain vs Hadamard, on the page-2 synthetic setting.

    The page's RNG, B distribution and outlier fraction are not given, so values are
    pinned to a 20% band around the printed numbers, plus the page's three trend facts.
    """
    wl = W.make_workload("pr1")
    A, B = wl.A.astype(np.float64), wl.W.astype(np.float64)
    rot = lambda X: Hd.rht_apply(X, None)   # the page probe: plain Q = H/sqrt(K), no signs
    got = {}
    for name, (ab, bb, r, p128, p32) in _page2_table().items():
        for G, page in ((128, p128), (32, p32)):
            e = 100 * L.matmul_q_err(A, B, ab, bb, rot if r else None, G)
            got[(name, G)] = e
            assert abs(e - page) <= 0.2 * page, (name, G, e, page)
    for G in (128, 32):
        assert got[("W8A8_sanity", G)] < 3.0
        # Hadamard cuts W4A4 error substantially (page: 40-60% on the real weights)
        assert got[("W4A4_hadamard", G)] < 0.75 * got[("W4A4_plain", G)]
        # activations dominate: rotation barely changes W4A8
        assert abs(got[("W4A8_hadamard", G)] - got[("W4A8_plain", G)]) < 2.0
    assert got[("W4A4_plain", 32)] < got[("W4A4_plain", 128)]
    # with random signs (the RHT) the same holds
    e_sign = 100 * L.matmul_q_err(A, B, 4, 4, lambda X: Hd.rht_apply(X, wl.signs), 128)
    assert e_sign < 0.75 * got[("W4A4_plain", 128)]


def test_error_benefit_scales_with_outlier_severity():
    # page 2, fact 2: the benefit grows with outlier mass (x20 vs x4)
    g = W.rng(0)
    base = g.standard_normal((16, 2048)).astype(np.float32)
    ch = g.choice(2048, 21, replace=False)
    B = W.weights(1, 2048, 512, 0.02).astype(np.float64)
    rot = lambda X: Hd.rht_apply(X, None)
    gains = []
    for sc in (4.0, 20.0):
        A = base.copy()
        A[:, ch] *= sc
        plain = L.matmul_q_err(A, B, 4, 4, None, 128)
        had = L.matmul_q_err(A, B, 4, 4, rot, 128)
        gains.append(plain - had)
    assert gains[1] > gains[0] > 0


# ----------------------------------------------------------------------------- plain CPU baseline

@pytest.mark.parametrize("K,G,bits", [(2, 2, 4), (64, 16, 2), (256, 32, 4), (2048, 32, 4), (2048, 128, 4),
                                      (4096, 64, 2)])
def test_plain_cpu_baseline_matches_the_oracle(K, G, bits):
    """The scalar O(K log K) C baseline (fp32 butterflies) gives the oracle's codes and scales
    (fp64 dense RHT) everywhere outside the 1e-5 rounding-boundary windows, on heavy-tailed rows
    with outlier channels, with and without signs (the wiki's probe has none)."""
    from oracle import plain
    g = W.rng(K + G + bits)
    A = W.activations(g, 24, K, dist="student_t", t_scale=0.5, outlier_frac=0.01, outlier_scale=50.0, bf16=False)
    for s in (W.signs(g, K), None):
        codes, scales = plain.rht_quant(A, s, bits, G)
        y = Hd.rht_apply(A, s)
        q_ref, s_ref = Q.quantize(y, bits, G)
        cflag, gflag = Q.boundary_flags(y, bits, G)
        assert not ((scales.view(np.uint16) != s_ref.view(np.uint16)) & ~gflag).any()
        assert not ((Q.unpack(codes, bits, K) != q_ref) & ~cflag).any()


def test_plain_cpu_baseline_edge_cases():
    """Zero rows, scales in the binary16 subnormal range and past its largest finite value (inf
    scale, zero codes) take the same decisions as the oracle."""
    from oracle import plain
    K, G = 256, 32
    A = np.zeros((4, K), dtype=np.float32)
    A[1] = W.rng(2).standard_normal(K) * 1e-6
    A[2] = 3.0e5
    A[3, 5] = -4.0
    codes, scales = plain.rht_quant(A, None, 4, G)
    y = Hd.rht_apply(A, None)
    q_ref, s_ref = Q.quantize(y, 4, G)
    cflag, gflag = Q.boundary_flags(y, 4, G)
    assert np.array_equal(scales.view(np.uint16)[~gflag], s_ref.view(np.uint16)[~gflag])
    assert not ((Q.unpack(codes, 4, K) != q_ref) & ~cflag).any()
    # a constant row puts all its energy in coordinate 0 (no signs): group 0's scale overflows to inf
    assert np.isinf(scales[2, 0].astype(np.float32)) and (Q.unpack(codes, 4, K)[2] == 0).all()


# ----------------------------------------------------------------------------- Cayley blocks, int8 parameters

def test_cayley_b2_is_the_rotation_by_twice_the_arctangent():
    """Closed form: for S = [[0, t], [-t, 0]], (I + S)^{-1}(I - S) = [[1 - t^2, -2t], [2t, 1 - t^2]] / (1 + t^2),
    the rotation by 2 atan(t) (a textbook identity of the Cayley transform)."""
    for t in (0.0, 0.3, -1.7, 5.0):
        Q = Hp.cayley(np.array([t]), 2)
        phi = 2.0 * np.arctan(t)
        R = np.array([[np.cos(phi), -np.sin(phi)], [np.sin(phi), np.cos(phi)]])
        assert np.max(np.abs(Q - R)) < 1e-14


@pytest.mark.parametrize("b", [3, 5, 8, 43])
def test_cayley_orthogonal_det_one_and_inverse(b):
    g = W.rng(b)
    p = g.standard_normal(b * (b - 1) // 2) * 0.7
    Q = Hp.cayley(p, b)
    assert np.max(np.abs(Q @ Q.T - np.eye(b))) < 1e-12
    assert abs(np.linalg.det(Q) - 1.0) < 1e-10
    # the inverse map S = (I - Q)(I + Q)^{-1} gives back the skew-symmetric matrix
    S = (np.eye(b) - Q) @ np.linalg.inv(np.eye(b) + Q)
    iu = np.triu_indices(b, 1)
    assert np.max(np.abs(S + S.T)) < 1e-10 and np.max(np.abs(S[iu] - p)) < 1e-10
    assert np.array_equal(Hp.cayley(np.zeros_like(p), b), np.eye(b))   # Q(0) = I


def test_cayley_blocks_at_zero_are_the_base_mixer():
    """B(0) = G_b (summary 2.2): Sylvester-Hadamard for b = 8, the given fallback for b = 5."""
    assert np.max(np.abs(Hp.cayley_blocks(np.zeros((1, 28)), 8)[0] - Hd.sylvester(8) / np.sqrt(8))) < 1e-15
    G5 = Hp.qr_block(W.rng(1).standard_normal((5, 5)))
    assert np.array_equal(Hp.cayley_blocks(np.zeros((2, 10)), 5, G5)[1], G5)


def test_int8_parameter_storage():
    th = np.array([0.0, 1.0, -2.54, 2.54, 0.01, -1.27])
    q, s = Hp.quant_params_int8(th)
    assert s == np.float32(2.54 / 127)
    assert q.dtype == np.int8 and q[2] == -127 and q[3] == 127 and q[0] == 0
    back = Hp.dequant_params_int8(q, s)
    assert np.all(np.abs(back - th) <= float(s) / 2 + 1e-12)
    # a tie rounds away from zero: theta = 2.5 s exactly
    s0 = np.float32(0.5)
    q2, _ = Hp.quant_params_int8(np.array([63.5, 2.5 * float(s0), -1.25]))   # scale 0.5
    assert list(q2) == [127, 3, -3]
    z, sz = Hp.quant_params_int8(np.zeros(5))
    assert sz == 0 and not z.any()


# ----------------------------------------------------------------------------- two-sided processor

def test_two_sided_exact_equivalence():
    """(A T^T)(T B U^T) U = A B in fp64 to 1e-12, with T an RHT of size K and U a random HARP
    processor of size N (mixed radix with permutations), both applied through the oracle."""
    K, N = 256, 96
    g = W.rng(21)
    A = g.standard_normal((7, K))
    B = g.standard_normal((K, N))
    sT = W.signs(g, K)
    radU = [2, 3, 2, 2, 2, 2]
    spec = Hp.HarpSpec(N, radU, [np.stack([Hp.qr_block(g.standard_normal((b, b))) for _ in range(N // b)])
                                 for b in radU], [g.permutation(N).astype(np.int32), None, None, None, None, None],
                       (1 - 2 * g.integers(0, 2, N)).astype(np.int8))
    rot_in = lambda X: Hd.rht_apply(X, sT)
    rot_out = lambda X: Hp.harp_apply(X, spec)
    rot_out_inv = lambda X: Hp.harp_apply(X, spec, inverse=True)
    Bt = L.two_sided_weights(B, rot_in, rot_out)           # rows of (T B U^T)^T
    Ct = rot_in(A) @ Bt.T                                  # (A T^T)(T B U^T) = A B U^T
    C = L.unrotate_output(Ct, rot_out_inv)
    ref = A @ B
    assert np.linalg.norm(C - ref) / np.linalg.norm(ref) < 1e-12
    # each output row of the rotated product is U c (the output side is really rotated)
    assert np.linalg.norm(Ct - rot_out(ref)) / np.linalg.norm(ref) < 1e-12
    assert np.linalg.norm(Ct - ref) / np.linalg.norm(ref) > 0.1

"""GPU parity of the rotation and rotate+quantise kernels against the fp64 oracle."""
import numpy as np
import pytest

import workloads as W
from oracle import hadamard as Hd
from oracle import harp as Hp
from oracle import quant as Q
from parity import (assert_codes_match, assert_rotated_close, guarded_apply, guarded_quant, padded_rows,
                    sample_rows, to_device)

pytestmark = pytest.mark.gpu


def _acts(M, K, seed, bf16=True, scale=20.0):
    g = W.rng(seed)
    return W.activations(g, M, K, outlier_frac=0.01, outlier_scale=scale, bf16=bf16), W.signs(g, K)


# ----------------------------------------------------------------------------- RHT rotation

@pytest.mark.parametrize("K", [32, 64, 128, 256, 512, 1024, 2048, 4096, 8192])
@pytest.mark.parametrize("bf16", [True, False])
def test_rht_apply(lib, K, bf16):
    A, s = _acts(37, K, K, bf16)
    plan = lib.Plan.rht(K, s)
    assert plan.info()["chunk"] == K
    y = guarded_apply(lib, to_device(A, bf16), plan).cpu().numpy()
    assert_rotated_close(y, Hd.rht_apply(A, s))
    yi = guarded_apply(lib, to_device(A, bf16), plan, inverse=True).cpu().numpy()
    assert_rotated_close(yi, Hd.rht_apply(A, s, inverse=True))


@pytest.mark.parametrize("M", [1, 2, 3, 129])
def test_rht_apply_ragged_rows_and_stride(lib, M):
    import torch
    K = 2048
    A, s = _acts(M, K, 5)
    big = torch.zeros((M, K + 64), dtype=torch.bfloat16, device="cuda")
    big[:, :K] = to_device(A, True)
    plan = lib.Plan.rht(K, s)
    y = guarded_apply(lib, big[:, :K], plan).cpu().numpy()
    assert_rotated_close(y, Hd.rht_apply(A, s))


# ----------------------------------------------------------------------------- RHT quantise

@pytest.mark.parametrize("K,G,bits", [(32, 8, 4), (64, 16, 2), (128, 32, 4), (256, 128, 4), (256, 64, 2),
                                      (512, 256, 4), (1024, 32, 4), (2048, 32, 4), (2048, 128, 4),
                                      (2048, 2048, 4), (4096, 128, 4), (4096, 64, 2), (4096, 256, 4),
                                      (4096, 16, 2), (4096, 32, 4), (8192, 128, 4), (8192, 64, 2), (8192, 16, 2)])
def test_rht_quant(lib, K, G, bits):
    A, s = _acts(67, K, K + G + bits)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, True), plan, bits, G)
    y = Hd.rht_apply(A, s)
    assert_codes_match(codes, scales, y, bits, G)
    # exclusions stay rare: per-code windows well under 1e-3 of the codes, and scale windows
    # (binary16 midpoints are 2^-10 apart, the window 2e-5 wide) under 5% of the groups
    cflag, gflag = Q.boundary_flags(y, bits, G)
    assert (cflag & ~np.repeat(gflag, G, axis=1)).sum() < 1e-3 * A.size
    assert gflag.sum() <= max(6, 0.06 * gflag.size)


@pytest.mark.parametrize("G", [32, 128, 512])
@pytest.mark.parametrize("M", [1, 7, 600])
def test_rht_quant_k4096_strided_few_rows(lib, M, G):
    """K = 4096 bf16 int4 with few rows (one CTA per row) and past the few-row limit of 512 chunks
    (the one-warp-per-row kernel): rows with a pitch of K + 64 elements, every row against the oracle."""
    import torch
    K = 4096
    A, s = _acts(M, K, 11 * M + G)
    big = torch.zeros((M, K + 64), dtype=torch.bfloat16, device="cuda")
    big[:, :K] = to_device(A, True)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, big[:, :K], plan, 4, G)
    assert_codes_match(codes, scales, Hd.rht_apply(A, s), 4, G)


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 5, 2961])
def test_rht_quant_k2048_strided_ragged(lib, M, G):
    """K = 2048 bf16 int4 (the tensor-core first stage): rows with a pitch of K + 64 elements and
    row counts just past one round of the persistent slots; sampled rows against the oracle."""
    import torch
    K = 2048
    A, s = _acts(M, K, 7 * M + G)
    big = torch.zeros((M, K + 64), dtype=torch.bfloat16, device="cuda")
    big[:, :K] = to_device(A, True)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, big[:, :K], plan, 4, G)
    rows = sample_rows(M, 64)
    idx = rows.tolist()
    assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), Hd.rht_apply(A[rows], s), 4, G)


def test_rht_quant_fp32_input_and_page2_probe_without_signs(lib):
    wl = W.make_workload("pr1")
    for signs in (wl.signs, None):
        plan = lib.Plan.rht(2048, signs)
        for bits, G in wl.quant:
            codes, scales = guarded_quant(lib, to_device(wl.A, False), plan, bits, G)
            assert_codes_match(codes, scales, Hd.rht_apply(wl.A, signs), bits, G)


def test_quant_edge_cases(lib):
    import torch
    K, G = 256, 32
    s = W.signs(W.rng(1), K)
    A = np.zeros((6, K), dtype=np.float32)
    A[1] = 1e-30                      # tiny: scale underflows / subnormal
    A[2, :] = W.rng(2).standard_normal(K) * 1e-6   # subnormal binary16 scales
    A[3, :] = 3.0e5                   # scale above binary16 range -> inf, zero codes
    A[4, 7] = 5.0                     # one spike
    A[5] = W.rng(3).standard_normal(K)
    A = W.to_bf16_exact(A)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, True), plan, 4, G)
    assert_codes_match(codes, scales, Hd.rht_apply(A, s), 4, G)
    # empty input is a no-op
    e = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
    c0, s0 = lib.rot_quant(e, plan, 4, G)
    assert c0.shape == (0, K // 2)


def test_invalid_arguments(lib):
    import torch
    plan = lib.Plan.rht(256, None)
    A = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    for bits, G in [(3, 32), (4, 12), (4, 100), (2, 8)]:
        with pytest.raises(lib.RotError):
            lib.rot_quant(A, plan, bits, G)
    with pytest.raises(lib.RotError):
        lib.rot_quant(A[:, 1:], plan, 4, 32)   # misaligned base pointer


# ----------------------------------------------------------------------------- workloads at full size

@pytest.mark.parametrize("name", ["llama32_1b", "down_proj", "q_proj_prefill"])
def test_workload_full_size_sampled_rows(lib, name):
    wl = W.make_workload(name)
    plan = lib.Plan.rht(wl.K, wl.signs)
    dA = to_device(wl.A, True)
    rows = sample_rows(wl.M, 48)
    y_ref = Hd.rht_apply(wl.A[rows], wl.signs)
    y = guarded_apply(lib, dA, plan)[rows.tolist()].cpu().numpy()
    assert_rotated_close(y, y_ref)
    for bits, G in wl.quant:
        codes, scales = guarded_quant(lib, dA, plan, bits, G)
        idx = rows.tolist()
        assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), y_ref, bits, G)


# ----------------------------------------------------------------------------- dequantisation

@pytest.mark.parametrize("bits,G", [(4, 128), (2, 64), (4, 32)])
def test_dequant_roundtrip(lib, bits, G):
    K = 8192
    A, s = _acts(9, K, 77)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, True), plan, bits, G)
    c_np, s_np = codes.cpu().numpy(), scales.cpu().numpy()
    # rotated basis: exact q * s of the GPU's own codes
    xh = lib.rot_dequant(codes, scales, plan, bits, G).cpu().numpy()
    ref = Q.dequantize(Q.unpack(c_np, bits, K), s_np, G)
    assert np.array_equal(xh, ref)
    # original basis: T^T (q s)
    xo = lib.rot_dequant(codes, scales, plan, bits, G, inverse=True).cpu().numpy()
    assert_rotated_close(xo, Hd.rht_apply(ref.astype(np.float64), s, inverse=True))
    # round-trip error of the quantiser itself (oracle): reported, bounded
    y = Hd.rht_apply(A, s)
    rel = np.linalg.norm(ref - y) / np.linalg.norm(y)
    assert rel < (0.2 if bits == 4 else 0.8)


# ----------------------------------------------------------------------------- HARP

def _random_plan(lib, radices, seed, per_block=True, perms=True):
    K = int(np.prod(radices))
    g = np.random.default_rng(seed)
    blocks = []
    for b in radices:
        n = K // b if per_block else 1
        blocks.append(np.stack([Hp.qr_block(g.standard_normal((b, b))) for _ in range(n)]))
    P = [g.permutation(K).astype(np.int32) if (perms and t < len(radices) - 1) else None
         for t in range(len(radices))]
    s = (1 - 2 * g.integers(0, 2, K)).astype(np.int8)
    spec = Hp.HarpSpec(K, list(radices), [b.astype(np.float32).astype(np.float64) for b in blocks], P, s)
    plan = lib.Plan(K, radices, [b.astype(np.float32) for b in blocks], P, s)
    return spec, plan


@pytest.mark.parametrize("radices", [[2, 2, 3, 2], [2, 43], [3, 4, 2, 2], [5, 3, 2, 2], [2] * 6 + [43]])
@pytest.mark.parametrize("per_block", [True, False])
def test_harp_generic_apply_and_quant(lib, radices, per_block):
    spec, plan = _random_plan(lib, radices, 11, per_block)
    K = spec.K
    A, _ = _acts(21, K, 3)
    assert plan.info()["chunk"] == 0
    dA = padded_rows(A)            # leading dimension rounded up to 16 bytes
    y_ref = Hp.harp_apply(A, spec)
    y = guarded_apply(lib, dA, plan).cpu().numpy()
    assert_rotated_close(y, y_ref)
    yi = guarded_apply(lib, dA, plan, inverse=True).cpu().numpy()
    assert_rotated_close(yi, Hp.harp_apply(A, spec, inverse=True))
    if K % 8 == 0:
        codes, scales = guarded_quant(lib, dA, plan, 4, 8)
        assert_codes_match(codes, scales, y_ref, 4, 8)


@pytest.mark.parametrize("variant", ["init_identity", "init_qr", "random"])
def test_harp11008_full_size(lib, variant):
    wl = W.make_workload("harp11008")
    draws = W.harp_draws(2, wl.extra["radices"])
    plan = lib.harp_plan(draws, wl.signs, variant)
    spec = Hp.spec_from_draws(draws, wl.signs, variant)
    info = plan.info()
    assert info["chunk"] == (256 if variant == "init_identity" else 0)
    dA = to_device(wl.A, True)
    rows = sample_rows(wl.M, 24)
    y_ref = Hp.harp_apply(wl.A[rows], spec)
    y = guarded_apply(lib, dA, plan)[rows.tolist()].cpu().numpy()
    assert_rotated_close(y, y_ref)
    for bits, G in wl.quant:
        codes, scales = guarded_quant(lib, dA, plan, bits, G)
        idx = rows.tolist()
        assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), y_ref, bits, G)


# ----------------------------------------------------------------------------- fp32 input at large K

@pytest.mark.parametrize("K,G,bits", [(4096, 128, 4), (4096, 32, 4), (8192, 128, 4), (8192, 64, 2)])
def test_rht_quant_fp32_input_large_k(lib, K, G, bits):
    """fp32 activations (the weight-preparation input type) at K = 4096 / 8192, every element."""
    A, s = _acts(41, K, 3 * K + G + bits, bf16=False)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, False), plan, bits, G)
    assert_codes_match(codes, scales, Hd.rht_apply(A, s), bits, G)
    y = guarded_apply(lib, to_device(A, False), plan).cpu().numpy()
    assert_rotated_close(y, Hd.rht_apply(A, s))


# ----------------------------------------------------------------------------- offline weight preparation

@pytest.mark.parametrize("name", ["q_proj_prefill", "up_proj_prefill"])
def test_weight_prep_full_size(lib, name):
    """The offline step of the linear: the fp32 rows of W^T ([N, K] = [4096 or 11008, 4096]) through
    the same RHT plan as the activations and quantised to int4 G = 128, at full size; codes and
    scales of sampled rows bit-exact against the oracle's quantize(rht_apply(W^T)) outside the
    rounding-boundary windows [Hadamard-Int4-Accuracy wiki, Hypothesis: A.B = (A.Q)(Q.B), the
    weights take the rotation offline]."""
    wl = W.make_workload(name, M=16)
    bits, G = wl.quant[0]
    Wt = np.ascontiguousarray(wl.W.T)            # [N, K] fp32
    plan = lib.Plan.rht(wl.K, wl.signs)
    codes, scales = guarded_quant(lib, to_device(Wt, False), plan, bits, G)
    rows = sample_rows(Wt.shape[0], 64, seed=5)
    idx = rows.tolist()
    assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), Hd.rht_apply(Wt[rows], wl.signs),
                       bits, G, what=f"W^T {Wt.shape[0]}x{wl.K} int{bits} G={G}")

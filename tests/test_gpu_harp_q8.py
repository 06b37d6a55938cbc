"""GPU parity of HARP processors stored with int8 parameters (Givens blocks expanded on the device
at load, Cayley blocks for b > 2) and of the mixed-radix schedule 5120 = (8, 8, 8, 5, 2)
[HARP gist.science summary, 2.1 (schedules, 5120 example), 2.2 (B = Q(theta) G; Givens for b = 2,
Cayley for b > 2), 2.4 and 4 (int8 parameter storage)]."""
import numpy as np
import pytest

import workloads as W
from oracle import harp as Hp
from parity import (assert_codes_match, assert_rotated_close, guarded_apply, guarded_quant, padded_rows,
                    sample_rows, to_device)

pytestmark = pytest.mark.gpu


def test_harp11008_int8_params_per_block_cayley_full_size(lib):
    """K = 11008 = 2^8 * 43: eight Givens stages and 256 distinct Cayley blocks of radix 43 (times
    the QR fallback mixer), all from int8 codes, the drawn permutations; A[4096, 11008] bf16 at full
    size, sampled rows: rotated values, int4 G = 128 and int2 G = 64 codes against the oracle."""
    wl = W.make_workload("harp11008")
    draws = W.harp_q8_draws(4, wl.extra["radices"], per_block=True)
    plan = lib.harp_q8_plan(draws, wl.signs)
    spec = Hp.spec_from_q8(draws, wl.signs)
    assert plan.info()["chunk"] == 0
    dA = to_device(wl.A, True)
    rows = sample_rows(wl.M, 16)
    idx = rows.tolist()
    y_ref = Hp.harp_apply(wl.A[rows], spec)
    y = guarded_apply(lib, dA, plan)[idx].cpu().numpy()
    assert_rotated_close(y, y_ref)
    for bits, G in wl.quant:
        codes, scales = guarded_quant(lib, dA, plan, bits, G)
        assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), y_ref, bits, G)


@pytest.mark.parametrize("per_block", [True, False])
def test_harp5120_int8_params(lib, per_block):
    """5120 = (8, 8, 8, 5, 2): Cayley blocks for radix 8 (times H_8 / sqrt 8) and 5 (times the QR
    fallback), Givens for 2, int8 codes, permutations; every row and coordinate; the inverse too."""
    radices = [8, 8, 8, 5, 2]
    K = 5120
    draws = W.harp_q8_draws(9, radices, per_block=per_block)
    g = W.rng(10)
    A = W.activations(g, 96, K, outlier_frac=0.01, outlier_scale=20.0)
    s = W.signs(g, K)
    plan = lib.harp_q8_plan(draws, s)
    spec = Hp.spec_from_q8(draws, s)
    dA = to_device(A, True)
    y_ref = Hp.harp_apply(A, spec)
    assert_rotated_close(guarded_apply(lib, dA, plan).cpu().numpy(), y_ref)
    assert_rotated_close(guarded_apply(lib, dA, plan, inverse=True).cpu().numpy(), Hp.harp_apply(A, spec, inverse=True))
    for bits, G in ((4, 128), (8, 64), (2, 64)):
        codes, scales = guarded_quant(lib, dA, plan, bits, G)
        assert_codes_match(codes, scales, y_ref, bits, G)


def test_harp5120_initial_state_equals_base_mixers(lib):
    """theta = 0 (no codes): the 5120 processor is H_8 x H_8 x H_8 x I_5 x H_2 (normalised), the
    pages' initial state with the identity fallback; on the GPU through rot_plan_create_q8."""
    radices = [8, 8, 8, 5, 2]
    K = 5120
    g = W.rng(12)
    A = W.activations(g, 40, K, outlier_frac=0.01, outlier_scale=20.0)
    s = W.signs(g, K)
    plan = lib.Plan.q8(K, radices, [None] * 5, [0.0] * 5, signs=s)
    spec = Hp.HarpSpec(K, radices, [None] * 5, [None] * 5, s)
    y_ref = Hp.harp_apply(A, spec)
    assert_rotated_close(guarded_apply(lib, to_device(A, True), plan).cpu().numpy(), y_ref)
    codes, scales = guarded_quant(lib, to_device(A, True), plan, 4, 128)
    assert_codes_match(codes, scales, y_ref, 4, 128)


def test_harp11008_fp32_per_block_qr_full_size(lib):
    """The per-block stress variant of the fp32 processor: 256 distinct radix-43 QR blocks
    (1.9 MB) with the random Givens stages and permutations, at full size (sampled rows)."""
    wl = W.make_workload("harp11008")
    draws = W.harp_draws(2, wl.extra["radices"], per_block_gaussian=True)
    plan = lib.harp_plan(draws, wl.signs, "random")
    spec = Hp.spec_from_draws(draws, wl.signs, "random")
    dA = to_device(wl.A, True)
    rows = sample_rows(wl.M, 16)
    idx = rows.tolist()
    y_ref = Hp.harp_apply(wl.A[rows], spec)
    assert_rotated_close(guarded_apply(lib, dA, plan)[idx].cpu().numpy(), y_ref)
    codes, scales = guarded_quant(lib, dA, plan, 4, 128)
    assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), y_ref, 4, 128)

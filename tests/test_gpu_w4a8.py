"""GPU parity of the int8 quantiser and the W4A8 linear (int8 activations, int4 weights) against
the oracle [Hadamard-Int4-Accuracy wiki, Method: matmul_q_err(..., abits = 8, bbits = 4);
Results: the "W4A8 (act8/wt4)" rows; fact 3: int8 activations absorb the outliers]."""
import numpy as np
import pytest

import workloads as W
from oracle import hadamard as Hd
from oracle import harp as Hp
from oracle import linear as L
from oracle import quant as Q
from parity import (POISON, Guarded, assert_codes_match, assert_linear_close, guarded_quant, padded_rows,
                    sample_rows, to_device)

pytestmark = pytest.mark.gpu


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("K,G", [(256, 8), (1024, 32), (2048, 32), (2048, 128), (4096, 128), (8192, 128), (8192, 64)])
@pytest.mark.parametrize("bf16", [True, False])
def test_rht_quant_int8(lib, K, G, bf16):
    g = W.rng(K + G)
    A = W.activations(g, 45, K, outlier_frac=0.01, outlier_scale=20.0, bf16=bf16)
    s = W.signs(g, K)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, bf16), plan, 8, G)
    assert_codes_match(codes, scales, Hd.rht_apply(A, s), 8, G)


@pytest.mark.parametrize("radices,G", [([2, 2, 3, 2], 4), ([2] * 6 + [43], 64)])
def test_harp_quant_int8(lib, radices, G):
    K = int(np.prod(radices))
    g = np.random.default_rng(3)
    blocks = [np.stack([Hp.qr_block(g.standard_normal((b, b))) for _ in range(K // b)]) for b in radices]
    P = [g.permutation(K).astype(np.int32) if t < len(radices) - 1 else None for t in range(len(radices))]
    s = (1 - 2 * g.integers(0, 2, K)).astype(np.int8)
    spec = Hp.HarpSpec(K, list(radices), [b.astype(np.float32).astype(np.float64) for b in blocks], P, s)
    plan = lib.Plan(K, radices, [b.astype(np.float32) for b in blocks], P, s)
    A = W.activations(W.rng(7), 33, K, outlier_frac=0.01, outlier_scale=20.0)
    codes, scales = guarded_quant(lib, padded_rows(A), plan, 8, G)
    assert_codes_match(codes, scales, Hp.harp_apply(A, spec), 8, G)


def test_dequant_int8_roundtrip(lib):
    K, G = 4096, 128
    g = W.rng(2)
    A = W.activations(g, 9, K, outlier_frac=0.01, outlier_scale=20.0)
    s = W.signs(g, K)
    plan = lib.Plan.rht(K, s)
    codes, scales = guarded_quant(lib, to_device(A, True), plan, 8, G)
    xh = lib.rot_dequant(codes, scales, plan, 8, G).cpu().numpy()
    ref = Q.dequantize(Q.unpack(codes.cpu().numpy(), 8, K), scales.cpu().numpy(), G)
    assert np.array_equal(xh, ref)
    y = Hd.rht_apply(A, s)
    assert np.linalg.norm(ref - y) / np.linalg.norm(y) < 0.02


def _operands(seed, M, N, K, G):
    g = W.rng(seed)
    X = g.standard_normal((M, K)) * np.exp(g.uniform(-2, 2, (M, 1)))
    X[:, g.choice(K, max(1, K // 64), replace=False)] *= 20.0
    qa, sa = Q.quantize(X, 8, G)
    qw, sw = Q.quantize(g.standard_normal((N, K)) * 0.02, 4, G)
    return qa, sa, qw, sw


@pytest.mark.parametrize("M,N,K,G", [(1, 16, 128, 32), (3, 48, 256, 64), (129, 272, 384, 128), (64, 512, 4096, 128),
                                     (200, 176, 192, 32), (16, 256, 1024, 256), (300, 784, 640, 64),
                                     (5, 640, 1152, 96)])
def test_w4a8_group_partials_exact(lib, M, N, K, G):
    import torch
    qa, sa, qw, sw = _operands(M + N + K, M, N, K, G)
    out = Guarded((M, N, K // G), torch.int32, POISON["i32"])
    P = lib.w4a8_group_partials(_dev(qa), _dev(Q.pack(qw, 4)), G, out=out.t).cpu().numpy()
    out.check()
    assert np.array_equal(P, L.group_partials(qa, qw, G))


@pytest.mark.parametrize("M,N,K,G", [(1, 16, 128, 32), (3, 48, 256, 64), (129, 272, 384, 128), (64, 512, 4096, 128),
                                     (200, 176, 192, 32), (16, 256, 1024, 256), (300, 784, 640, 64),
                                     (5, 640, 1152, 96), (130, 208, 1344, 192), (1, 128, 1024, 128),
                                     (9, 176, 768, 256), (16, 48, 2560, 128)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_w4a8_linear_small(lib, M, N, K, G, out):
    import torch
    qa, sa, qw, sw = _operands(M * 7 + N + K, M, N, K, G)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    C = Guarded((M, N), dt, POISON["f32" if out == "f32" else "bf16"])
    lib.w4a8_linear(_dev(qa), _dev(sa), _dev(Q.pack(qw, 4)), _dev(sw), G, out=C.t)
    C.check()
    C_ref = L.w4a8_reference(qa, sa, qw, sw, G)
    assert_linear_close(C.t.float().cpu().numpy(), C_ref, tol=1e-4 if out == "f32" else 2 ** -8)


@pytest.mark.parametrize("name", ["q_proj_prefill", "up_proj_prefill", "q_proj_decode", "up_proj_decode"])
def test_w4a8_rotated_pipeline_full_size(lib, name):
    """The whole W4A8 path at the workload's full size: rotate + int8-quantise the bf16 activations,
    rotate + int4-quantise the rows of W^T (fp32), then the W4A8 linear. Sampled rows: activation
    codes and scales against the oracle (outside the rounding-boundary windows), and C against the
    oracle linear on the GPU's own codes at 1e-4."""
    import torch
    wl = W.make_workload(name)
    G = wl.quant[0][1]
    plan = lib.Plan.rht(wl.K, wl.signs)
    Aq, As = guarded_quant(lib, to_device(wl.A, True), plan, 8, G)
    Wt = np.ascontiguousarray(wl.W.T)
    Wq, Ws = guarded_quant(lib, to_device(Wt, False), plan, 4, G)
    C = Guarded((wl.M, Wt.shape[0]), torch.float32, POISON["f32"])
    lib.w4a8_linear(Aq.view(torch.int8), As, Wq, Ws, G, out=C.t)
    C.check()
    rows = sample_rows(wl.M, 16)
    idx = rows.tolist()
    assert_codes_match(Aq[idx].cpu().numpy(), As[idx].cpu().numpy(), Hd.rht_apply(wl.A[rows], wl.signs), 8, G,
                       what="A int8 G=128")
    qa = Q.unpack(Aq[idx].cpu().numpy(), 8, wl.K)
    qw = Q.unpack(Wq.cpu().numpy(), 4, wl.K)
    C_ref = L.w4a8_reference(qa, As[idx].cpu().numpy(), qw, Ws.cpu().numpy(), G)
    assert_linear_close(C.t[idx].cpu().numpy(), C_ref)


def test_w4a8_error_below_w4a4(lib):
    """Fact 3 of the wiki's Results: int8 activations absorb the outliers, so W4A8 (rotated) has a
    lower RMS relative error against the exact product than W4A4 (rotated), on the GPU path."""
    import torch
    wl = W.make_workload("q_proj_prefill", M=128)
    G = 128
    N = 512
    Wt = np.ascontiguousarray(wl.W.T[:N])
    plan = lib.Plan.rht(wl.K, wl.signs)
    dA = to_device(wl.A, True)
    Wq, Ws = lib.rot_quant(to_device(Wt, False), plan, 4, G)
    A8, S8 = lib.rot_quant(dA, plan, 8, G)
    A4, S4 = lib.rot_quant(dA, plan, 4, G)
    C8 = lib.w4a8_linear(A8.view(torch.int8), S8, Wq, Ws, G).cpu().numpy()
    C4 = lib.w4a4_linear(A4, S4, Wq, Ws, G).cpu().numpy()
    exact = wl.A.astype(np.float64) @ wl.W[:, :N].astype(np.float64)
    e8 = np.linalg.norm(C8 - exact) / np.linalg.norm(exact)
    e4 = np.linalg.norm(C4 - exact) / np.linalg.norm(exact)
    assert e8 < 0.8 * e4

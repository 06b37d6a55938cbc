"""GPU parity of the tcgen05 W4A4 linear against the oracle (exact int32 group sums,
fp32 output within 1e-4 relative), plus the end-to-end rotated pipeline."""
import numpy as np
import pytest

import workloads as W
from oracle import hadamard as Hd
from oracle import linear as L
from oracle import quant as Q
from parity import assert_codes_match, assert_linear_close, guarded_linear, guarded_quant, sample_rows, to_device

pytestmark = pytest.mark.gpu


def _codes(seed, rows, K, G):
    """Oracle-quantised rows of a heavy-tailed matrix: (codes int8, packed uint8, scales fp16)."""
    g = W.rng(seed)
    X = g.standard_normal((rows, K)) * np.exp(g.uniform(-2, 2, (rows, 1)))
    X[:, g.choice(K, max(1, K // 64), replace=False)] *= 20.0
    q, s = Q.quantize(X, 4, G)
    return q, Q.pack(q, 4), s


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,N,K,G", [(1, 16, 128, 32), (3, 48, 256, 64), (128, 256, 512, 128),
                                     (129, 272, 384, 128), (64, 512, 4096, 128), (200, 176, 192, 32),
                                     (16, 256, 1024, 256), (300, 784, 640, 64), (5, 640, 1152, 96),
                                     (33, 144, 640, 160), (5, 640, 192, 192)])
def test_group_partials_exact(lib, M, N, K, G):
    qa, pa, sa = _codes(M + K, M, K, G)
    qw, pw, sw = _codes(N + K + 1, N, K, G)
    import torch
    from parity import POISON, Guarded
    out = Guarded((M, N, K // G), torch.int32, POISON["i32"])
    P = lib.w4a4_group_partials(_dev(pa), _dev(pw), G, out=out.t).cpu().numpy()
    out.check()
    assert np.array_equal(P, L.group_partials(qa, qw, G))


@pytest.mark.parametrize("M,N,K,G", [(1, 16, 128, 32), (3, 48, 256, 64), (129, 272, 384, 128),
                                     (64, 512, 4096, 128), (200, 176, 192, 32), (16, 256, 1024, 256),
                                     (300, 784, 640, 64), (5, 640, 1152, 96), (130, 208, 1344, 192),
                                     (7, 96, 896, 224), (33, 144, 640, 160), (5, 640, 192, 192),
                                     (7, 96, 448, 224), (1, 128, 1024, 128), (9, 176, 768, 256),
                                     (16, 48, 2560, 128)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_w4a4_linear_small(lib, M, N, K, G, out):
    import torch
    qa, pa, sa = _codes(M + K + 7, M, K, G)
    qw, pw, sw = _codes(N + K + 9, N, K, G)
    C = guarded_linear(lib, lib.w4a4_linear, _dev(pa), _dev(sa), _dev(pw), _dev(sw), G,
                       torch.float32 if out == "f32" else torch.bfloat16)
    C_ref = L.w4a4_reference(qa, sa, qw, sw, G)
    if out == "f32":
        assert_linear_close(C.cpu().numpy(), C_ref)
    else:
        # bf16 output: the fp32 result rounded once (8-bit mantissa)
        assert_linear_close(C.float().cpu().numpy(), C_ref, tol=2 ** -8)


def test_w4a4_empty_M(lib):
    import torch
    _, pw, sw = _codes(1, 32, 256, 128)
    Aq = torch.empty((0, 128), dtype=torch.uint8, device="cuda")
    As = torch.empty((0, 2), dtype=torch.float16, device="cuda")
    C = lib.w4a4_linear(Aq, As, _dev(pw), _dev(sw), 128)
    assert C.shape == (0, 32)


@pytest.mark.parametrize("name", ["q_proj_prefill", "up_proj_prefill", "q_proj_decode", "up_proj_decode"])
def test_w4a4_workload_oracle_codes(lib, name):
    """Full-size linear on oracle-quantised codes (parity isolates the GEMM; the codes of the
    workload's activation and weight shapes are quantised without rotation to keep the oracle fast)."""
    import torch
    wl = W.make_workload(name)
    bits, G = wl.quant[0]
    rows = sample_rows(wl.M, 24)
    qa, sa = Q.quantize(wl.A, bits, G)
    qw, sw = Q.quantize(np.ascontiguousarray(wl.W.T), bits, G)
    C = guarded_linear(lib, lib.w4a4_linear, _dev(Q.pack(qa, 4)), _dev(sa), _dev(Q.pack(qw, 4)), _dev(sw), G,
                       torch.float32).cpu().numpy()
    C_ref = L.w4a4_reference(qa[rows], sa[rows], qw, sw, G)
    assert_linear_close(C[rows], C_ref)


@pytest.mark.parametrize("M", [16, 256])
def test_w4a4_end_to_end_rotated_pipeline(lib, M):
    """The whole path on the GPU: rotate + quantise the activations (bf16) and the rows of W^T
    (fp32, the offline step) with one RHT plan, then the linear. Checked element by element:
    the GPU codes and scales of both operands equal the oracle's outside the rounding-boundary
    windows, and the GPU linear on the GPU codes is within 1e-4 of the oracle linear on those
    same codes. The page-2 accuracy trend (rotation lowers the W4A4 error against the exact
    product) holds as well [Hadamard-Int4-Accuracy wiki, Hypothesis and Results]."""
    import torch
    wl = W.make_workload("q_proj_prefill", M=M)
    bits, G = wl.quant[0]
    N = 512                                           # the first 512 output columns of q_proj
    Wt = np.ascontiguousarray(wl.W.T[:N])             # [N, K]
    plan = lib.Plan.rht(wl.K, wl.signs)
    Aq, As = guarded_quant(lib, to_device(wl.A, True), plan, bits, G)
    Wq, Ws = guarded_quant(lib, to_device(Wt, False), plan, bits, G)
    assert_codes_match(Aq, As, Hd.rht_apply(wl.A, wl.signs), bits, G, what="A int4 G=128")
    assert_codes_match(Wq, Ws, Hd.rht_apply(Wt, wl.signs), bits, G, what="W^T int4 G=128")
    C = guarded_linear(lib, lib.w4a4_linear, Aq, As, Wq, Ws, G, torch.float32).cpu().numpy()
    qa, sa = Q.unpack(Aq.cpu().numpy(), 4, wl.K), As.cpu().numpy()
    qw, sw = Q.unpack(Wq.cpu().numpy(), 4, wl.K), Ws.cpu().numpy()
    assert_linear_close(C, L.w4a4_reference(qa, sa, qw, sw, G))
    exact = wl.A.astype(np.float64) @ wl.W[:, :N].astype(np.float64)
    err_rot = np.linalg.norm(C - exact) / np.linalg.norm(exact)
    qa0, sa0 = Q.quantize(wl.A, bits, G)
    qw0, sw0 = Q.quantize(Wt, bits, G)
    err_plain = np.linalg.norm(L.w4a4_reference(qa0, sa0, qw0, sw0, G) - exact) / np.linalg.norm(exact)
    assert err_rot < 0.8 * err_plain


@pytest.mark.parametrize("name", ["q_proj_prefill", "q_proj_decode", "up_proj_prefill"])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_w4a4_linear_act_full_size(lib, name, out):
    """The one-call online path (rotate + quantise the bf16 activations into a workspace, then the
    linear, launched as a programmatic dependent): the workspace codes and scales against the
    oracle on sampled rows, and C against the oracle linear on those codes."""
    import torch
    from parity import POISON, Guarded
    wl = W.make_workload(name)
    bits, G = wl.quant[0]
    plan = lib.Plan.rht(wl.K, wl.signs)
    Wq, Ws = guarded_quant(lib, to_device(np.ascontiguousarray(wl.W.T), False), plan, bits, G)
    N = Wq.shape[0]
    nbytes = lib.w4a4_linear_act_workspace(wl.M, wl.K, G)
    ws = Guarded((nbytes,), torch.uint8, POISON["codes4"])
    dt = torch.float32 if out == "f32" else torch.bfloat16
    C = Guarded((wl.M, N), dt, POISON["f32" if out == "f32" else "bf16"])
    lib.w4a4_linear_act(to_device(wl.A, True), plan, Wq, Ws, G, out=C.t, workspace=ws.t)
    C.check()
    ws.check()
    lib.check_device()
    cbytes = -(-wl.M * wl.K // 2 // 16) * 16
    codes = ws.t[:wl.M * wl.K // 2].view(wl.M, wl.K // 2)
    scales = ws.t[cbytes:cbytes + wl.M * (wl.K // G) * 2].view(torch.float16).view(wl.M, wl.K // G)
    rows = sample_rows(wl.M, 16)
    idx = rows.tolist()
    assert_codes_match(codes[idx].cpu().numpy(), scales[idx].cpu().numpy(), Hd.rht_apply(wl.A[rows], wl.signs),
                       bits, G, what="w4a4_linear_act workspace")
    qa, sa = Q.unpack(codes[idx].cpu().numpy(), 4, wl.K), scales[idx].cpu().numpy()
    C_ref = L.w4a4_reference(qa, sa, Q.unpack(Wq.cpu().numpy(), 4, wl.K), Ws.cpu().numpy(), G)
    assert_linear_close(C.t[idx].float().cpu().numpy(), C_ref, tol=1e-4 if out == "f32" else 2 ** -8)

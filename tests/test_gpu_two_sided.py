"""GPU parity of the two-sided processor [HARP abstract: a learnable structured two-sided
orthogonal processor; HARP gist.science summary, sections 1 and 3]: weights prepared on the GPU
as B~ = T B U^T (rows of B through the output-side plan U with rot_apply, then the columns through
the input-side RHT T with rot_quant), the linear, and the output rows returned to c = U^T c~ by
w4a4_linear_rot. Checked against the oracle on the GPU's own codes (1e-4), the weight codes
against the oracle's preparation, and the product against the exact A B."""
import numpy as np
import pytest

import workloads as W
from oracle import hadamard as Hd
from oracle import harp as Hp
from oracle import linear as L
from oracle import quant as Q
from parity import POISON, Guarded, assert_codes_match, assert_linear_close, guarded_quant, sample_rows, to_device

pytestmark = pytest.mark.gpu


def _out_side(lib, name, N):
    """Output-side plan U and the oracle's row operators x -> U x, x -> U^T x."""
    if name == "rht":
        sU = W.signs(W.rng(77), N)
        return lib.Plan.rht(N, sU), (lambda X: Hd.rht_apply(X, sU)), (lambda X: Hd.rht_apply(X, sU, inverse=True))
    draws = W.harp_draws(5, [2] * 8 + [43])
    sU = W.signs(W.rng(78), N)
    spec = Hp.spec_from_draws(draws, sU, "random")
    return (lib.harp_plan(draws, sU, "random"), (lambda X: Hp.harp_apply(X, spec)),
            (lambda X: Hp.harp_apply(X, spec, inverse=True)))


@pytest.mark.parametrize("wname,uname,M", [("q_proj_prefill", "rht", 16), ("q_proj_prefill", "rht", 256),
                                           ("up_proj_prefill", "harp", 64), ("up_proj_prefill", "harp", 200)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_two_sided_linear(lib, wname, uname, M, out):
    import torch
    wl = W.make_workload(wname, M=M)
    bits, G = wl.quant[0]
    N = wl.W.shape[1]
    T = lib.Plan.rht(wl.K, wl.signs)
    U, rot_out, rot_out_inv = _out_side(lib, uname, N)
    # offline: B~^T = (T (B U^T))^T on the GPU
    BU = lib.rot_apply(to_device(wl.W, False), U)                  # rows of B through U: [K, N]
    Bt = BU.t().contiguous()                                       # columns of B U^T as rows: [N, K]
    Wq, Ws = guarded_quant(lib, Bt, T, bits, G)
    Aq, As = guarded_quant(lib, to_device(wl.A, True), T, bits, G)
    dt = torch.float32 if out == "f32" else torch.bfloat16
    C = Guarded((M, N), dt, POISON["f32" if out == "f32" else "bf16"])
    lib.w4a4_linear_rot(Aq, As, Wq, Ws, G, U, out=C.t)
    C.check()
    lib.check_device()
    C = C.t.float().cpu().numpy()
    # weight preparation against the oracle on sampled output columns n: T (B U^T)[:, n]
    ns = sample_rows(N, 12, seed=3)
    u_rows = rot_out_inv(np.eye(N)[ns])                            # U^T e_n = row n of U
    y_w = Hd.rht_apply((wl.W.astype(np.float64) @ u_rows.T).T, wl.signs)
    assert_codes_match(Wq[ns.tolist()].cpu().numpy(), Ws[ns.tolist()].cpu().numpy(), y_w, bits, G,
                       what=f"two-sided W~^T rows ({uname} U)")
    # the linear + output-side rotation against the oracle on the GPU's own codes
    rows = sample_rows(M, 24)
    qa, sa = Q.unpack(Aq.cpu().numpy(), 4, wl.K)[rows], As.cpu().numpy()[rows]
    qw, sw = Q.unpack(Wq.cpu().numpy(), 4, wl.K), Ws.cpu().numpy()
    C_ref = L.unrotate_output(L.w4a4_reference(qa, sa, qw, sw, G), rot_out_inv)
    assert_linear_close(C[rows], C_ref, tol=1e-4 if out == "f32" else 2 ** -8)
    # the two-sided product stays close to the exact one (W4A4 quantisation error only)
    exact = wl.A[rows].astype(np.float64) @ wl.W.astype(np.float64)
    assert np.linalg.norm(C[rows] - exact) / np.linalg.norm(exact) < 0.25

"""The bounded-wait failure path of the kernels, exercised without faulting the GPU.

Every device-side wait of the fused rotation kernels and of the W4A4 tile kernel gives up
after a bound of wall time, records ROT_ETIMEOUT and returns. Through the library's testing
hook (rot_test_inject) the next launch skips issuing copies, so no copy or MMA is in flight
and the waits on them run out; the bound is shortened to 20 ms for the test. Each test then
checks that rot_check_device reports ROT_ETIMEOUT once, that the record is cleared, and that
the next ordinary call on the same context matches the oracle.
"""
import numpy as np
import pytest

import workloads as W
from oracle import hadamard as Hd
from oracle import linear as L
from oracle import quant as Q
from parity import assert_codes_match, assert_linear_close, guarded_linear, guarded_quant, to_device

pytestmark = pytest.mark.gpu

WAIT_NS = 20_000_000


@pytest.mark.parametrize("K,G", [(2048, 32), (8192, 128)])
def test_rotation_staging_wait_gives_up_then_recovers(lib, K, G):
    g = W.rng(K + 1)
    A = W.activations(g, 300, K, outlier_frac=0.01, outlier_scale=20.0)
    s = W.signs(g, K)
    plan = lib.Plan.rht(K, s)
    dA = to_device(A, True)
    lib.check_device()                       # nothing recorded before
    lib.test_inject(lib.ROT_TEST_ROTATION_COPY, WAIT_NS)
    try:
        lib.rot_quant(dA, plan, 4, G)
        with pytest.raises(lib.RotError) as e:
            lib.check_device()
        assert e.value.status == lib.ROT_ETIMEOUT
    finally:
        lib.test_inject(lib.ROT_TEST_NONE, 0)
    lib.check_device()                       # the record was cleared by the first check
    codes, scales = guarded_quant(lib, dA, plan, 4, G)
    assert_codes_match(codes, scales, Hd.rht_apply(A, s), 4, G)
    lib.check_device()


def test_w4a4_pipeline_waits_give_up_then_recover(lib):
    import torch
    M, N, K, G = 256, 384, 1024, 128          # the tcgen05 tile kernel (M > 64)
    g = W.rng(5)
    qa, sa = Q.quantize(g.standard_normal((M, K)), 4, G)
    qw, sw = Q.quantize(g.standard_normal((N, K)) * 0.02, 4, G)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Aq, As, Wq, Ws = dev(Q.pack(qa, 4)), dev(sa), dev(Q.pack(qw, 4)), dev(sw)
    lib.check_device()
    lib.test_inject(lib.ROT_TEST_W4A4_LOADS, WAIT_NS)
    try:
        lib.w4a4_linear(Aq, As, Wq, Ws, G)
        with pytest.raises(lib.RotError) as e:
            lib.check_device()
        assert e.value.status == lib.ROT_ETIMEOUT
    finally:
        lib.test_inject(lib.ROT_TEST_NONE, 0)
    lib.check_device()
    C = guarded_linear(lib, lib.w4a4_linear, Aq, As, Wq, Ws, G, torch.float32)
    assert_linear_close(C.cpu().numpy(), L.w4a4_reference(qa, sa, qw, sw, G))
    lib.check_device()


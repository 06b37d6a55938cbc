"""w4a4_linear_noalloc through the C ABI: the split-K path with bf16 output accumulates in
the library's static device buffer instead of a stream-ordered temporary. Two consecutive
calls of each entry point on the same operands agree with each other (the split-K sum
order may differ: fp32 rounding only) and with the oracle."""
import numpy as np
import pytest

import workloads as W
from oracle import linear as L
from oracle import quant as Q
from parity import assert_linear_close

pytestmark = pytest.mark.gpu


def _operands(seed, M, N, K, G):
    g = W.rng(seed)
    X = g.standard_normal((M, K)) * np.exp(g.uniform(-1, 1, (M, 1)))
    Wt = g.standard_normal((N, K)) * 0.02
    qa, sa = Q.quantize(X, 4, G)
    qw, sw = Q.quantize(Wt, 4, G)
    return qa, sa, qw, sw


@pytest.mark.parametrize("M,N,K,G", [(16, 4096, 4096, 128), (16, 1024, 2048, 256), (5, 640, 1024, 64)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_noalloc_matches_allocating_entry(lib, M, N, K, G, out):
    import torch
    qa, sa, qw, sw = _operands(M + N + K, M, N, K, G)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Aq, As, Wq, Ws = dev(Q.pack(qa, 4)), dev(sa), dev(Q.pack(qw, 4)), dev(sw)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    runs = []
    for _ in range(2):
        runs.append(lib.w4a4_linear(Aq, As, Wq, Ws, G, out_dtype=dt).float().cpu().numpy())
        runs.append(lib.w4a4_linear_noalloc(Aq, As, Wq, Ws, G, out_dtype=dt).float().cpu().numpy())
    lib.check_device()   # raises if a device-side wait gave up
    ref = runs[0]
    # bf16: two fp32 sums that differ in the last bits may round one bf16 ulp apart (<= 2^-7)
    tol = 2 ** -7 if out == "bf16" else 1e-6
    for r in runs[1:]:
        scale = np.maximum(np.abs(ref), np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True)))
        assert np.all(np.abs(r - ref) <= tol * scale + 1e-30)
    C_ref = L.w4a4_reference(qa, sa, qw, sw, G)
    assert_linear_close(runs[1], C_ref, tol=2 ** -8 if out == "bf16" else 1e-4)


def test_noalloc_rejects_shapes_beyond_its_buffer(lib):
    """M * N above the static buffer on the split path (bf16 output): ROT_EINVAL before any launch.
    72 output tiles of 128 x 128 leave more than half of the 148 SMs idle, so K is split."""
    import torch
    M, N, K, G = 256, 4608, 256, 128
    Aq = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    As = torch.zeros((M, K // G), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    Ws = torch.zeros((N, K // G), dtype=torch.float16, device="cuda")
    with pytest.raises(lib.RotError) as e:
        lib.w4a4_linear_noalloc(Aq, As, Wq, Ws, G, out_dtype=torch.bfloat16)
    assert e.value.status == lib.ROT_EINVAL
    # the allocating entry point takes the same shape
    C = lib.w4a4_linear(Aq, As, Wq, Ws, G, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.count_nonzero(C).item() == 0

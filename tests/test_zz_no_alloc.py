"""w4a4_linear_noalloc through the C ABI.

This entry point is for callers that cannot allocate device memory while they run the
linear: a serving runtime that reserves all device memory up front and hands out fixed
buffers, or code running while the stream is captured into a CUDA graph, where a
stream-ordered allocation would become part of the graph. Its only difference from
w4a4_linear is where the split-K fp32 partial sums of a bf16 output go: a static buffer of
the library instead of a stream-ordered temporary.

Checked here: two consecutive calls of each entry point on the same operands agree with
each other (the split-K summation order may differ: fp32 rounding only) and with the oracle;
the calls leave the device's stream-ordered memory pool untouched (its high-water mark stays
at zero, and the same check does see the allocating entry point's temporary); shapes beyond
the static buffer are refused before any launch. This file is collected last.
"""
import ctypes as C

import numpy as np
import pytest

import workloads as W
from oracle import linear as L
from oracle import quant as Q
from parity import assert_linear_close

pytestmark = pytest.mark.gpu

_USED_MEM_HIGH = 8   # cudaMemPoolAttrUsedMemHigh


def _operands(seed, M, N, K, G):
    g = W.rng(seed)
    X = g.standard_normal((M, K)) * np.exp(g.uniform(-1, 1, (M, 1)))
    Wt = g.standard_normal((N, K)) * 0.02
    qa, sa = Q.quantize(X, 4, G)
    qw, sw = Q.quantize(Wt, 4, G)
    return qa, sa, qw, sw


def _dev_operands(qa, sa, qw, sw):
    import torch
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return dev(Q.pack(qa, 4)), dev(sa), dev(Q.pack(qw, 4)), dev(sw)


@pytest.mark.parametrize("M,N,K,G", [(128, 1024, 4096, 128), (96, 2048, 2048, 256), (5, 640, 1024, 64),
                                     (16, 4096, 4096, 128)])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_noalloc_matches_allocating_entry(lib, M, N, K, G, out):
    import torch
    if M > 64 or G % 128:
        # these shapes take the tile kernel's split-K path, where the bf16 output needs the buffer
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert lib.w4a4_tile_plan(M, N, K, G, sms)["splits"] > 1
    qa, sa, qw, sw = _operands(M + N + K, M, N, K, G)
    Aq, As, Wq, Ws = _dev_operands(qa, sa, qw, sw)
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
    assert_linear_close(runs[3], C_ref, tol=2 ** -8 if out == "bf16" else 1e-4)


def _cudart():
    # the runtime the library itself resolved (same soname), so it sees the same device pools
    return C.CDLL("libcudart.so.12")


def _pool_used_high(rt, dev: int) -> int:
    pool = C.c_void_p()
    assert rt.cudaDeviceGetDefaultMemPool(C.byref(pool), C.c_int(dev)) == 0
    v = C.c_uint64(0)
    assert rt.cudaMemPoolGetAttribute(pool, C.c_int(_USED_MEM_HIGH), C.byref(v)) == 0
    return int(v.value)


def _pool_reset_high(rt, dev: int):
    pool = C.c_void_p()
    assert rt.cudaDeviceGetDefaultMemPool(C.byref(pool), C.c_int(dev)) == 0
    zero = C.c_uint64(0)
    assert rt.cudaMemPoolSetAttribute(pool, C.c_int(_USED_MEM_HIGH), C.byref(zero)) == 0


def test_noalloc_leaves_the_memory_pool_untouched(lib):
    """The bf16 split-K path, where w4a4_linear takes a stream-ordered temporary from the
    device's default memory pool: w4a4_linear_noalloc leaves the pool's high-water mark at zero
    over two calls; the allocating entry point then raises it (so the check can see one)."""
    import torch
    if torch.cuda.get_allocator_backend() != "native":
        pytest.skip("torch itself allocates from the stream-ordered pool under this configuration")
    M, N, K, G = 128, 1024, 4096, 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert lib.w4a4_tile_plan(M, N, K, G, sms)["splits"] > 1
    qa, sa, qw, sw = _operands(11, M, N, K, G)
    Aq, As, Wq, Ws = _dev_operands(qa, sa, qw, sw)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dev = torch.cuda.current_device()
    rt = _cudart()
    torch.cuda.synchronize()
    _pool_reset_high(rt, dev)
    for _ in range(2):
        lib.w4a4_linear_noalloc(Aq, As, Wq, Ws, G, out=out)
    torch.cuda.synchronize()
    assert _pool_used_high(rt, dev) == 0
    C_na = out.float().cpu().numpy()
    lib.w4a4_linear(Aq, As, Wq, Ws, G, out=out)
    torch.cuda.synchronize()
    assert _pool_used_high(rt, dev) >= M * N * 4
    C_ref = L.w4a4_reference(qa, sa, qw, sw, G)
    assert_linear_close(C_na, C_ref, tol=2 ** -8)
    assert_linear_close(out.float().cpu().numpy(), C_ref, tol=2 ** -8)


def test_noalloc_rejects_shapes_beyond_its_buffer(lib):
    """M * N above the static buffer on the split path (bf16 output): ROT_EINVAL before any launch."""
    import torch
    M, N, K, G = 256, 4608, 256, 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tp = lib.w4a4_tile_plan(M, N, K, G, sms)
    assert tp["splits"] > 1, "the shape must take the split-K path on this device"
    assert M * N > (1 << 20)
    Aq = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    As = torch.zeros((M, K // G), dtype=torch.float16, device="cuda")
    Wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    Ws = torch.zeros((N, K // G), dtype=torch.float16, device="cuda")
    with pytest.raises(lib.RotError) as e:
        lib.w4a4_linear_noalloc(Aq, As, Wq, Ws, G, out_dtype=torch.bfloat16)
    assert e.value.status == lib.ROT_EINVAL
    # the allocating entry point takes the same shape
    C_ = lib.w4a4_linear(Aq, As, Wq, Ws, G, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.count_nonzero(C_).item() == 0

"""CPU checks of the C-ABI library: it loads, exports every declared entry point, its host
helpers match the oracle, and argument errors are reported before any device work."""
import os
import re

import numpy as np
import pytest

import workloads as W
from oracle import harp as Hp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rot_b200.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:rot_status|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("rot_plan_create", "rot_plan_destroy", "rot_quant", "rot_dequant", "rot_apply", "w4a4_linear"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib._lib, name), name
    assert "sm_100a" in lib.version()


def test_givens_blocks_match_oracle(lib):
    th = W.rng(3).uniform(-np.pi, np.pi, 1000)
    got = lib.harp_givens_blocks(th).astype(np.float64)
    ref = Hp.givens_blocks(th)
    assert np.max(np.abs(got - ref)) < 1e-6


@pytest.mark.parametrize("b", [3, 5, 43])
def test_qr_block_matches_oracle(lib, b):
    g = W.rng(b).standard_normal((b, b))
    got = lib.harp_qr_block(g).astype(np.float64)
    ref = Hp.qr_block(g)
    assert np.max(np.abs(got - ref)) < 1e-5
    assert np.max(np.abs(got @ got.T - np.eye(b))) < 1e-5


def test_null_plan_is_rejected_without_a_device(lib):
    import ctypes as C
    st = lib._lib.rot_quant(C.c_void_p(0), lib.ROT_BF16, 1, 16, C.c_void_p(0), 4, 16, C.c_void_p(0),
                            C.c_void_p(0), C.c_void_p(0))
    assert st == lib.ROT_EINVAL
    assert "plan" in lib.last_error()
    st = lib._lib.rot_apply(C.c_void_p(0), lib.ROT_BF16, 1, 16, C.c_void_p(0), 0, C.c_void_p(0), 16, C.c_void_p(0))
    assert st == lib.ROT_EINVAL


def test_bad_w4a4_shapes_rejected_without_a_device(lib):
    import ctypes as C
    buf = (C.c_uint8 * 64)()
    p = C.cast(buf, C.c_void_p)
    # G not a multiple of 32
    st = lib._lib.w4a4_linear(p, p, p, p, 1, 16, 128, 48, p, lib.ROT_F32, C.c_void_p(0))
    assert st == lib.ROT_EINVAL
    # N not a multiple of 16
    st = lib._lib.w4a4_linear(p, p, p, p, 1, 24, 128, 32, p, lib.ROT_F32, C.c_void_p(0))
    assert st == lib.ROT_EINVAL


def test_plan_create_rejects_bad_schedules(lib):
    import ctypes as C
    h = C.c_void_p()
    rad = (C.c_int * 2)(2, 3)
    st = lib._lib.rot_plan_create(C.byref(h), 8, 2, rad, None, None, None, None)
    assert st == lib.ROT_EINVAL and "product" in lib.last_error()
    rad1 = (C.c_int * 1)(1)
    st = lib._lib.rot_plan_create(C.byref(h), 1, 1, rad1, None, None, None, None)
    assert st == lib.ROT_EINVAL
    s = (C.c_int8 * 2)(1, 0)
    rad2 = (C.c_int * 1)(2)
    st = lib._lib.rot_plan_create(C.byref(h), 2, 1, rad2, None, None, None, s)
    assert st == lib.ROT_EINVAL and "signs" in lib.last_error()


def _w4a4_plan_cases():
    cases = []
    for M in (1, 65, 129, 2048, 5000):
        for N in (16, 272, 4096, 11008):
            for G in (32, 64, 96, 128, 160, 192, 224, 256):
                for K in (192, 448, 1344, 4096, 11008):
                    if K % G == 0 and K % 64 == 0:
                        cases.append((M, N, K, G))
    return cases


def test_w4a4_tile_plan_invariants(lib):
    """Host planner of the tcgen05 W4A4 kernel: every K split starts and ends on a K-block and a
    group boundary, none is empty, the splits cover K, and K is split only when the output tiles
    leave more than half of the SMs idle."""
    from math import gcd
    cases = _w4a4_plan_cases()
    assert len(cases) > 100
    for sms in (1, 20, 148):
        for M, N, K, G in cases:
            pl = lib.w4a4_tile_plan(M, N, K, G, sms)
            unit = (G * 128 // gcd(G, 128)) // 128
            nkb = -(-K // 128)
            tiles = -(-M // 128) * -(-N // 128)
            assert (pl["tiles_m"], pl["tiles_n"]) == (-(-M // 128), -(-N // 128))
            kb = pl["kb_per_split"]
            assert kb >= 1 and kb % unit == 0, (M, N, K, G, sms, pl)
            assert pl["splits"] == -(-nkb // kb)
            assert (pl["splits"] - 1) * kb < nkb                       # no empty split
            assert all((s * kb * 128) % G == 0 for s in range(pl["splits"]))
            assert pl["units"] == tiles * pl["splits"]
            assert pl["grid"] == min(pl["units"], sms)
            if 2 * tiles > sms:
                assert pl["splits"] == 1
            if pl["splits"] > 1:
                assert pl["splits"] * tiles <= max(sms, tiles)


def test_w4a4_tile_plan_k_below_one_lcm_range(lib):
    """K smaller than lcm(G, 128): one split of one whole lcm range (a floor division here once
    gave zero K-blocks per split)."""
    for M, N, K, G in ((5, 640, 192, 192), (7, 96, 448, 224), (3, 48, 192, 96)):
        pl = lib.w4a4_tile_plan(M, N, K, G, 148)
        assert pl["splits"] == 1 and pl["kb_per_split"] >= -(-K // 128)


def test_w4a4_tile_plan_partials_never_split(lib):
    pl = lib.w4a4_tile_plan(16, 256, 4096, 128, 148, partials=True)
    assert pl["splits"] == 1 and pl["units"] == 2


def test_w4a4_tile_plan_rejects_bad_shapes(lib):
    for args in ((0, 256, 4096, 128, 148), (16, 256, 4096, 96, 148), (16, 256, 4096, 512, 148),
                 (16, 250, 4096, 128, 148), (16, 256, 4096, 128, 0), (16, 256, 4000, 32, 148)):
        with pytest.raises(lib.RotError) as e:
            lib.w4a4_tile_plan(*args)
        assert e.value.status == lib.ROT_EINVAL


def test_binding_rejects_host_tensors_before_any_kernel(lib):
    """A host tensor's address must never reach a kernel: the binding refuses it (ROT_EINVAL)
    before calling the library, with no device needed."""
    import types
    import torch
    fake_plan = types.SimpleNamespace(K=256, handle=None)
    A = torch.zeros((4, 256), dtype=torch.bfloat16)
    for call in (lambda: lib.rot_quant(A, fake_plan, 4, 32),
                 lambda: lib.rot_apply(A, fake_plan),
                 lambda: lib.rot_dequant(torch.zeros((4, 128), dtype=torch.uint8),
                                         torch.zeros((4, 8), dtype=torch.float16), fake_plan, 4, 32),
                 lambda: lib.w4a4_linear(torch.zeros((4, 64), dtype=torch.uint8), torch.zeros((4, 1), dtype=torch.float16),
                                         torch.zeros((16, 64), dtype=torch.uint8), torch.zeros((16, 1), dtype=torch.float16),
                                         128),
                 lambda: lib.w4a4_group_partials(torch.zeros((4, 64), dtype=torch.uint8),
                                                 torch.zeros((16, 64), dtype=torch.uint8), 128),
                 lambda: lib.rot_quant(np.zeros((4, 256), dtype=np.float32), fake_plan, 4, 32)):
        with pytest.raises(lib.RotError) as e:
            call()
        assert e.value.status == lib.ROT_EINVAL
        assert "CUDA" in str(e.value) or "torch tensor" in str(e.value)


def test_binding_rejects_operands_on_another_device(lib):
    """Operands must live on the current device (the library launches there): the binding's
    device check raises ROT_EINVAL for any other index, before an address reaches a kernel."""
    lib._check_device(0, 0, "A")
    lib._check_device(3, 3, "A")
    for idx, cur in ((1, 0), (0, 2), (None, 0)):
        with pytest.raises(lib.RotError) as e:
            lib._check_device(idx, cur, "Wq")
        assert e.value.status == lib.ROT_EINVAL and "Wq" in str(e.value)


def test_test_inject_rejects_unknown_faults(lib):
    """The testing hook refuses unknown faults and negative bounds (host only, no device)."""
    with pytest.raises(lib.RotError) as e:
        lib.test_inject(7, 0)
    assert e.value.status == lib.ROT_EINVAL
    with pytest.raises(lib.RotError):
        lib.test_inject(0, -1)
    lib.test_inject(lib.ROT_TEST_NONE, 0)


@pytest.mark.parametrize("b", [2, 3, 5, 8, 43])
def test_cayley_block_matches_oracle(lib, b):
    g = W.rng(b + 100)
    p = g.standard_normal(b * (b - 1) // 2) * 0.4
    mix = None if b in (2, 8) else Hp.qr_block(g.standard_normal((b, b))).astype(np.float32)
    got = lib.harp_cayley_block(p, b, mix).astype(np.float64)
    ref = Hp.cayley_blocks(p[None], b, None if mix is None else mix.astype(np.float64))[0]
    assert np.max(np.abs(got - ref)) < 2e-6
    assert np.max(np.abs(got @ got.T - np.eye(b))) < 2e-6


def test_plan_q8_rejects_bad_arguments_without_a_device(lib):
    import ctypes as C
    h = C.c_void_p()
    rad = (C.c_int * 2)(2, 3)
    codes = (C.c_int8 * 3)(1, 2, 3)
    cp = (C.POINTER(C.c_int8) * 2)(C.cast(codes, C.POINTER(C.c_int8)), C.POINTER(C.c_int8)())
    # a stage with codes but no scales / n_blocks
    st = lib._lib.rot_plan_create_q8(C.byref(h), 6, 2, rad, cp, None, None, None, None, None)
    assert st == lib.ROT_EINVAL
    # a radix-2 stage given a mixer
    mix = (C.c_float * 4)(1, 0, 0, 1)
    mp = (C.POINTER(C.c_float) * 2)(C.cast(mix, C.POINTER(C.c_float)), C.POINTER(C.c_float)())
    st = lib._lib.rot_plan_create_q8(C.byref(h), 6, 2, rad, None, None, None, mp, None, None)
    assert st == lib.ROT_EINVAL and "mixer" in lib.last_error()

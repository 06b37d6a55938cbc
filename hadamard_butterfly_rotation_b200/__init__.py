"""Python binding of the B200 rotation / group-quantisation / W4A4 library (``include/rot_b200.h``).

Argument marshalling only: every step runs in the CUDA library ``_lib/librot_b200.so``
(build it with ``python hadamard_butterfly_rotation_b200/build.py``). PyTorch supplies
device memory and the current CUDA stream. Importing this package without the built
library raises ImportError; there is no CPU fallback.

Names follow the C ABI: ``Plan`` (rot_plan_create / rot_plan_destroy), ``rot_apply``,
``rot_quant``, ``rot_dequant``, ``w4a4_linear``, ``w4a4_group_partials``, ``w4a8_linear``,
``w4a8_group_partials``,
``harp_givens_blocks``, ``harp_qr_block``, ``check_device``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("ROT_B200_LIB") or os.path.join(_HERE, "_lib", "librot_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python hadamard_butterfly_rotation_b200/build.py)")

_lib = C.CDLL(LIB_PATH)

ROT_OK, ROT_EINVAL, ROT_EUNSUPPORTED, ROT_ECUDA, ROT_ETIMEOUT, ROT_ENOMEM = range(6)
ROT_F32, ROT_BF16 = 0, 1
_STATUS = {0: "ROT_OK", 1: "ROT_EINVAL", 2: "ROT_EUNSUPPORTED", 3: "ROT_ECUDA", 4: "ROT_ETIMEOUT", 5: "ROT_ENOMEM"}

_vp, _i64, _i32, _int = C.c_void_p, C.c_int64, C.c_int32, C.c_int
_lib.rot_plan_create.argtypes = [C.POINTER(_vp), _int, _int, C.POINTER(_int), C.POINTER(C.POINTER(C.c_float)),
                                 C.POINTER(_i64), C.POINTER(C.POINTER(_i32)), C.POINTER(C.c_int8)]
_lib.rot_plan_destroy.argtypes = [_vp]
_lib.rot_plan_info.argtypes = [_vp, C.POINTER(_int), C.POINTER(_int)]
_lib.rot_apply.argtypes = [_vp, _int, _i64, _i64, _vp, _int, _vp, _i64, _vp]
_lib.rot_quant.argtypes = [_vp, _int, _i64, _i64, _vp, _int, _int, _vp, _vp, _vp]
_lib.rot_dequant.argtypes = [_vp, _vp, _i64, _vp, _int, _int, _int, _vp, _vp]
_lib.w4a4_linear.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _int, _vp]
_lib.w4a4_linear_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _int, _vp]
_lib.w4a4_group_partials.argtypes = [_vp, _vp, _i64, _i64, _i64, _int, _vp, _vp]
_lib.w4a8_linear.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _int, _vp]
_lib.w4a4_linear_rot.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _vp, _vp, _int, _vp]
_lib.w4a4_linear_act_workspace.argtypes = [_i64, _i64, _int, C.POINTER(C.c_size_t)]
_lib.w4a4_linear_act.argtypes = [_vp, _int, _i64, _i64, _vp, _vp, _vp, _i64, _int, _vp, _int, _vp, C.c_size_t, _vp]
_lib.w4a8_group_partials.argtypes = [_vp, _vp, _i64, _i64, _i64, _int, _vp, _vp]
_lib.w4a4_tile_plan.argtypes = [_i64, _i64, _i64, _int, _int, _int, C.POINTER(_i64)]
_lib.rot_harp_givens_blocks.argtypes = [C.POINTER(C.c_double), _i64, C.POINTER(C.c_float)]
_lib.rot_harp_qr_block.argtypes = [C.POINTER(C.c_double), _int, C.POINTER(C.c_float)]
_lib.rot_harp_cayley_block.argtypes = [C.POINTER(C.c_double), _int, C.POINTER(C.c_float), C.POINTER(C.c_float)]
_lib.rot_plan_create_q8.argtypes = [C.POINTER(_vp), _int, _int, C.POINTER(_int), C.POINTER(C.POINTER(C.c_int8)),
                                    C.POINTER(C.c_float), C.POINTER(_i64), C.POINTER(C.POINTER(C.c_float)),
                                    C.POINTER(C.POINTER(_i32)), C.POINTER(C.c_int8)]
_lib.rot_check_device.argtypes = []
_lib.rot_test_inject.argtypes = [_int, _i64]
_lib.rot_last_error.restype = C.c_char_p
_lib.rot_version.restype = C.c_char_p
for _f in ("rot_plan_create", "rot_plan_destroy", "rot_plan_info", "rot_apply", "rot_quant", "rot_dequant",
           "w4a4_linear", "w4a4_linear_noalloc", "w4a4_group_partials", "w4a8_linear", "w4a8_group_partials",
           "w4a4_linear_rot", "w4a4_linear_act_workspace", "w4a4_linear_act",
           "w4a4_tile_plan", "rot_harp_givens_blocks",
           "rot_harp_qr_block", "rot_check_device", "rot_test_inject", "rot_harp_cayley_block", "rot_plan_create_q8"):
    getattr(_lib, _f).restype = _int


class RotError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def _check(st: int):
    if st != ROT_OK:
        raise RotError(st, _lib.rot_last_error().decode())


def version() -> str:
    return _lib.rot_version().decode()


def last_error() -> str:
    return _lib.rot_last_error().decode()


def _stream(stream):
    import torch
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return ROT_BF16
    if t.dtype == torch.float32:
        return ROT_F32
    raise TypeError(f"activations must be bf16 or fp32, got {t.dtype}")


def _ptr(t) -> C.c_void_p:
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _check_device(index, current: int, name: str):
    """The library launches on the current CUDA device: an operand on another device would be
    read and written from the wrong GPU. ROT_EINVAL unless ``index`` is the current device."""
    if index is None or int(index) != int(current):
        raise RotError(ROT_EINVAL, f"{name} is on cuda:{index}, but the current device is cuda:{current} "
                                   "(call under torch.cuda.device(...) of the operands' device)")


def _arg(t, name: str, *, dtype=None, shape=None, strided_rows: bool = False):
    """Check a tensor argument before its address reaches a kernel: on the current CUDA device
    (a host address, or another GPU's memory, would be dereferenced by the wrong device), of the
    expected dtype and shape, and laid out as the C ABI reads it (dense rows; with strided_rows,
    unit stride along a row only)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise RotError(ROT_EINVAL, f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise RotError(ROT_EINVAL, f"{name} must be on a CUDA device, not {t.device}")
    _check_device(t.device.index, torch.cuda.current_device(), name)
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise RotError(ROT_EINVAL, f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise RotError(ROT_EINVAL, f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.numel() > 0:
        if strided_rows:
            if t.dim() != 2 or t.stride(1) != 1:
                raise RotError(ROT_EINVAL, f"{name} must be 2-D with unit stride along its rows")
        elif not t.is_contiguous():
            raise RotError(ROT_EINVAL, f"{name} must be contiguous")
    return C.c_void_p(t.data_ptr())


class Plan:
    """A rotation plan T = (P_{m-1} S_{m-1}) ... (P_0 S_0) D on the current CUDA device.

    radices: schedule (prod == K); stage_params[t]: None (base mixer) or float32 array of
    shape [n_blocks, b, b] (n_blocks 1 or K/b); perms[t]: None or int32 permutation
    applied after stage t as a gather; signs: None or int8 +-1 of length K.
    """

    def __init__(self, K: int, radices, stage_params=None, perms=None, signs=None):
        import torch  # noqa: F401  (ensures the CUDA runtime is initialised by torch)
        m = len(radices)
        self.K = int(K)
        self.radices = [int(b) for b in radices]
        rad = (_int * m)(*self.radices)
        keep = []
        sp = None
        nb = None
        if stage_params is not None and any(p is not None for p in stage_params):
            sp = (C.POINTER(C.c_float) * m)()
            nb = (_i64 * m)()
            for t, prm in enumerate(stage_params):
                if prm is None:
                    sp[t] = C.POINTER(C.c_float)()
                    nb[t] = 0
                else:
                    a = np.ascontiguousarray(prm, dtype=np.float32)
                    b = self.radices[t]
                    if a.size % (b * b):
                        raise ValueError("stage params must hold whole b x b blocks")
                    keep.append(a)
                    sp[t] = a.ctypes.data_as(C.POINTER(C.c_float))
                    nb[t] = a.size // (b * b)
        pp = None
        if perms is not None and any(p is not None for p in perms):
            pp = (C.POINTER(_i32) * m)()
            for t, P in enumerate(perms):
                if P is None:
                    pp[t] = C.POINTER(_i32)()
                else:
                    a = np.ascontiguousarray(P, dtype=np.int32)
                    keep.append(a)
                    pp[t] = a.ctypes.data_as(C.POINTER(_i32))
        sg = None
        if signs is not None:
            s = np.ascontiguousarray(signs, dtype=np.int8)
            keep.append(s)
            sg = s.ctypes.data_as(C.POINTER(C.c_int8))
        h = _vp()
        _check(_lib.rot_plan_create(C.byref(h), self.K, m, rad, sp, nb, pp, sg))
        self._h = h

    @classmethod
    def q8(cls, K: int, radices, codes, scales, mixers=None, perms=None, signs=None) -> "Plan":
        """Plan from int8-stored HARP parameters (rot_plan_create_q8): codes[t] None or int8
        ([n_blocks] for radix 2, [n_blocks, b(b-1)/2] otherwise), scales[t] fp32 (theta =
        code * scale), mixers[t] None or a b x b fp32 base mixer, perms / signs as for Plan."""
        import torch  # noqa: F401
        m = len(radices)
        radices = [int(b) for b in radices]
        keep = []
        cp = (C.POINTER(C.c_int8) * m)()
        nb = (_i64 * m)()
        for t, q in enumerate(codes):
            if q is None:
                cp[t] = C.POINTER(C.c_int8)()
            else:
                a = np.ascontiguousarray(q, dtype=np.int8)
                keep.append(a)
                cp[t] = a.ctypes.data_as(C.POINTER(C.c_int8))
                nb[t] = a.shape[0]
        sc = (C.c_float * m)(*[float(x) for x in scales])
        mp = None
        if mixers is not None and any(x is not None for x in mixers):
            mp = (C.POINTER(C.c_float) * m)()
            for t, g in enumerate(mixers):
                if g is None:
                    mp[t] = C.POINTER(C.c_float)()
                else:
                    a = np.ascontiguousarray(g, dtype=np.float32)
                    keep.append(a)
                    mp[t] = a.ctypes.data_as(C.POINTER(C.c_float))
        pp = None
        if perms is not None and any(p is not None for p in perms):
            pp = (C.POINTER(_i32) * m)()
            for t, P in enumerate(perms):
                if P is None:
                    pp[t] = C.POINTER(_i32)()
                else:
                    a = np.ascontiguousarray(P, dtype=np.int32)
                    keep.append(a)
                    pp[t] = a.ctypes.data_as(C.POINTER(_i32))
        sg = None
        if signs is not None:
            sgn = np.ascontiguousarray(signs, dtype=np.int8)
            keep.append(sgn)
            sg = sgn.ctypes.data_as(C.POINTER(C.c_int8))
        h = _vp()
        _check(_lib.rot_plan_create_q8(C.byref(h), int(K), m, (_int * m)(*radices), cp, sc, nb, mp, pp, sg))
        self = cls.__new__(cls)
        self.K = int(K)
        self.radices = radices
        self._h = h
        return self

    @classmethod
    def rht(cls, K: int, signs=None) -> "Plan":
        """Randomized Hadamard transform of size K (power of two): radix-2 base mixers."""
        n = int(K).bit_length() - 1
        if (1 << n) != K:
            raise ValueError("the randomized Hadamard transform needs a power-of-two K")
        return cls(K, [2] * n, signs=signs)

    @property
    def handle(self):
        return self._h

    def info(self):
        k, ch = _int(), _int()
        _check(_lib.rot_plan_info(self._h, C.byref(k), C.byref(ch)))
        return {"K": k.value, "chunk": ch.value}

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _lib.rot_plan_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rot_apply(A, plan: Plan, *, inverse: bool = False, out=None, stream=None):
    """y = T a (or T^T a) for every row of A (cuda bf16/fp32 [M, >=K]); fp32 [M, K] out."""
    import torch
    pa = _arg(A, "A", dtype=(torch.bfloat16, torch.float32), strided_rows=True)
    M = A.shape[0]
    if out is None:
        Kp = (plan.K + 3) // 4 * 4   # 16-byte aligned rows
        out = torch.empty((M, Kp), dtype=torch.float32, device=A.device)[:, :plan.K]
    po = _arg(out, "out", dtype=torch.float32, strided_rows=True)
    _check(_lib.rot_apply(pa, _dtype_code(A), M, A.stride(0), plan.handle, int(inverse), po, out.stride(0),
                          _stream(stream)))
    return out


def rot_quant(A, plan: Plan, bits: int, G: int, *, codes=None, scales=None, stream=None):
    """Fused rotate + group quantise + pack (bits 2, 4 or 8). Returns (codes uint8 [M, K*bits/8],
    scales fp16 [M, K/G]); int8 codes can be viewed as torch.int8 for w4a8_linear."""
    import torch
    pa = _arg(A, "A", dtype=(torch.bfloat16, torch.float32), strided_rows=True)
    M = A.shape[0]
    K = plan.K
    if codes is None:
        codes = torch.empty((M, K * bits // 8), dtype=torch.uint8, device=A.device)
    if scales is None:
        scales = torch.empty((M, K // G), dtype=torch.float16, device=A.device)
    pc = _arg(codes, "codes", dtype=torch.uint8, shape=(M, K * bits // 8))
    ps = _arg(scales, "scales", dtype=torch.float16, shape=(M, K // G) if G > 0 else None)
    _check(_lib.rot_quant(pa, _dtype_code(A), M, A.stride(0), plan.handle, bits, G, pc, ps, _stream(stream)))
    return codes, scales


def rot_dequant(codes, scales, plan: Plan, bits: int, G: int, *, inverse: bool = False, out=None, stream=None):
    """x_hat = q * s (rotated basis) or T^T (q * s) (original basis); fp32 [M, K]."""
    import torch
    pc = _arg(codes, "codes", dtype=torch.uint8)
    M = codes.shape[0]
    ps = _arg(scales, "scales", dtype=torch.float16)
    if out is None:
        out = torch.empty((M, plan.K), dtype=torch.float32, device=codes.device)
    po = _arg(out, "out", dtype=torch.float32, shape=(M, plan.K))
    _check(_lib.rot_dequant(pc, ps, M, plan.handle, bits, G, int(inverse), po, _stream(stream)))
    return out


def _w4a4_args(Aq, As, Wq, Ws, G: int):
    """Shapes (M, N, K) and checked addresses of the W4A4 operands (As / Ws may be None)."""
    import torch
    pw = _arg(Wq, "Wq", dtype=torch.uint8)
    if Wq.dim() != 2:
        raise RotError(ROT_EINVAL, "Wq must be 2-D [N, K/2]")
    N, K = Wq.shape[0], Wq.shape[1] * 2
    if G <= 0 or K % G != 0:
        raise RotError(ROT_EINVAL, f"G = {G} must divide K = {K}")
    pa = _arg(Aq, "Aq", dtype=torch.uint8)
    if Aq.dim() != 2 or Aq.shape[1] * 2 != K:
        raise RotError(ROT_EINVAL, f"Aq must be [M, {K // 2}] like Wq")
    M = Aq.shape[0]
    ps_a = _arg(As, "As", dtype=torch.float16, shape=(M, K // G)) if As is not None else C.c_void_p(0)
    ps_w = _arg(Ws, "Ws", dtype=torch.float16, shape=(N, K // G)) if Ws is not None else C.c_void_p(0)
    return M, N, K, (pa, ps_a, pw, ps_w)


def w4a4_linear(Aq, As, Wq, Ws, G: int, *, out_dtype=None, out=None, stream=None):
    """C = sum_g sA sW (qA qW^T)_g for int4 codes Aq [M, K/2], Wq [N, K/2]; fp32 or bf16 [M, N]."""
    import torch
    M, N, K, ptrs = _w4a4_args(Aq, As, Wq, Ws, G)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=Wq.device)
    po = _arg(out, "out", dtype=(torch.float32, torch.bfloat16), shape=(M, N))
    cd = ROT_BF16 if out.dtype == torch.bfloat16 else ROT_F32
    _check(_lib.w4a4_linear(*ptrs, M, N, K, G, po, cd, _stream(stream)))
    return out


def w4a4_linear_rot(Aq, As, Wq, Ws, G: int, out_plan: Plan, *, out_dtype=None, out=None, stream=None):
    """Two-sided processor: the linear on weights prepared as B~ = T B U^T, then every output row
    returned to c = U^T c~ with the output-side plan U (size N)."""
    import torch
    M, N, K, ptrs = _w4a4_args(Aq, As, Wq, Ws, G)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=Wq.device)
    po = _arg(out, "out", dtype=(torch.float32, torch.bfloat16), shape=(M, N))
    cd = ROT_BF16 if out.dtype == torch.bfloat16 else ROT_F32
    _check(_lib.w4a4_linear_rot(*ptrs, M, N, K, G, out_plan.handle, po, cd, _stream(stream)))
    return out


def w4a4_linear_act_workspace(M: int, K: int, G: int) -> int:
    n = C.c_size_t()
    _check(_lib.w4a4_linear_act_workspace(M, K, G, C.byref(n)))
    return int(n.value)


def w4a4_linear_act(A, plan: Plan, Wq, Ws, G: int, *, out_dtype=None, out=None, workspace=None, stream=None):
    """rot_quant of the activations A (bf16/fp32 [M, >=K]) into a workspace, then the linear.
    Returns C; the workspace (uint8, allocated here if not given) holds the codes and scales."""
    import torch
    pa = _arg(A, "A", dtype=(torch.bfloat16, torch.float32), strided_rows=True)
    pw = _arg(Wq, "Wq", dtype=torch.uint8)
    M, K, N = A.shape[0], plan.K, Wq.shape[0]
    if Wq.dim() != 2 or Wq.shape[1] * 2 != K:
        raise RotError(ROT_EINVAL, f"Wq must be [N, {K // 2}]")
    ps_w = _arg(Ws, "Ws", dtype=torch.float16, shape=(N, K // G) if G > 0 and K % G == 0 else None)
    nbytes = w4a4_linear_act_workspace(M, K, G)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=A.device)
    pws = _arg(workspace, "workspace", dtype=torch.uint8)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=A.device)
    po = _arg(out, "out", dtype=(torch.float32, torch.bfloat16), shape=(M, N))
    cd = ROT_BF16 if out.dtype == torch.bfloat16 else ROT_F32
    _check(_lib.w4a4_linear_act(pa, _dtype_code(A), M, A.stride(0), plan.handle, pw, ps_w, N, G, po, cd, pws,
                                workspace.numel(), _stream(stream)))
    return out


def w4a4_linear_noalloc(Aq, As, Wq, Ws, G: int, *, out_dtype=None, out=None, stream=None):
    """w4a4_linear that never allocates device memory (static split-K buffer; see the header)."""
    import torch
    M, N, K, ptrs = _w4a4_args(Aq, As, Wq, Ws, G)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=Wq.device)
    po = _arg(out, "out", dtype=(torch.float32, torch.bfloat16), shape=(M, N))
    cd = ROT_BF16 if out.dtype == torch.bfloat16 else ROT_F32
    _check(_lib.w4a4_linear_noalloc(*ptrs, M, N, K, G, po, cd, _stream(stream)))
    return out


def w4a4_group_partials(Aq, Wq, G: int, *, out=None, stream=None):
    """Exact int32 group sums P[m, n, g] of the W4A4 contraction."""
    import torch
    M, N, K, ptrs = _w4a4_args(Aq, None, Wq, None, G)
    if out is None:
        out = torch.empty((M, N, K // G), dtype=torch.int32, device=Wq.device)
    po = _arg(out, "out", dtype=torch.int32, shape=(M, N, K // G))
    _check(_lib.w4a4_group_partials(ptrs[0], ptrs[2], M, N, K, G, po, _stream(stream)))
    return out


def _w4a8_args(Aq, As, Wq, Ws, G: int):
    """Shapes (M, N, K) and checked addresses of the W4A8 operands (int8 Aq [M, K]; As / Ws may be None)."""
    import torch
    pw = _arg(Wq, "Wq", dtype=torch.uint8)
    if Wq.dim() != 2:
        raise RotError(ROT_EINVAL, "Wq must be 2-D [N, K/2]")
    N, K = Wq.shape[0], Wq.shape[1] * 2
    if G <= 0 or K % G != 0:
        raise RotError(ROT_EINVAL, f"G = {G} must divide K = {K}")
    pa = _arg(Aq, "Aq", dtype=(torch.int8, torch.uint8))
    if Aq.dim() != 2 or Aq.shape[1] != K:
        raise RotError(ROT_EINVAL, f"Aq must be int8 [M, {K}]")
    M = Aq.shape[0]
    ps_a = _arg(As, "As", dtype=torch.float16, shape=(M, K // G)) if As is not None else C.c_void_p(0)
    ps_w = _arg(Ws, "Ws", dtype=torch.float16, shape=(N, K // G)) if Ws is not None else C.c_void_p(0)
    return M, N, K, (pa, ps_a, pw, ps_w)


def w4a8_linear(Aq, As, Wq, Ws, G: int, *, out_dtype=None, out=None, stream=None):
    """C = sum_g sA sW (qA qW^T)_g for int8 codes Aq [M, K] (rot_quant bits=8) and int4 Wq [N, K/2]."""
    import torch
    M, N, K, ptrs = _w4a8_args(Aq, As, Wq, Ws, G)
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype or torch.float32, device=Wq.device)
    po = _arg(out, "out", dtype=(torch.float32, torch.bfloat16), shape=(M, N))
    cd = ROT_BF16 if out.dtype == torch.bfloat16 else ROT_F32
    _check(_lib.w4a8_linear(*ptrs, M, N, K, G, po, cd, _stream(stream)))
    return out


def w4a8_group_partials(Aq, Wq, G: int, *, out=None, stream=None):
    """Exact int32 group sums P[m, n, g] of the W4A8 contraction."""
    import torch
    M, N, K, ptrs = _w4a8_args(Aq, None, Wq, None, G)
    if out is None:
        out = torch.empty((M, N, K // G), dtype=torch.int32, device=Wq.device)
    po = _arg(out, "out", dtype=torch.int32, shape=(M, N, K // G))
    _check(_lib.w4a8_group_partials(ptrs[0], ptrs[2], M, N, K, G, po, _stream(stream)))
    return out


def w4a4_tile_plan(M: int, N: int, K: int, G: int, sms: int, partials: bool = False) -> dict:
    """Host: the tile kernel's work list for a shape (see ``include/rot_b200.h``)."""
    out = (_i64 * 6)()
    _check(_lib.w4a4_tile_plan(M, N, K, G, sms, int(partials), out))
    keys = ("tiles_m", "tiles_n", "splits", "kb_per_split", "units", "grid")
    return {k: int(v) for k, v in zip(keys, out)}


def harp_givens_blocks(theta) -> np.ndarray:
    """Host: R(theta) H_2 / sqrt(2) blocks, float32 [n, 2, 2]."""
    th = np.ascontiguousarray(theta, dtype=np.float64)
    out = np.empty((th.size, 2, 2), dtype=np.float32)
    _check(_lib.rot_harp_givens_blocks(th.ctypes.data_as(C.POINTER(C.c_double)), th.size,
                                       out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def harp_qr_block(g) -> np.ndarray:
    """Host: Q factor (diag(R) > 0) of a square matrix, float32 [b, b]."""
    a = np.ascontiguousarray(g, dtype=np.float64)
    b = a.shape[0]
    out = np.empty((b, b), dtype=np.float32)
    _check(_lib.rot_harp_qr_block(a.ctypes.data_as(C.POINTER(C.c_double)), b,
                                  out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def harp_cayley_block(params, b: int, mixer=None) -> np.ndarray:
    """Host: B = Q(theta) G (Cayley map of the b(b-1)/2 parameters times the mixer), float32 [b, b]."""
    p = np.ascontiguousarray(params, dtype=np.float64)
    out = np.empty((b, b), dtype=np.float32)
    mx = None
    if mixer is not None:
        mx = np.ascontiguousarray(mixer, dtype=np.float32)
    _check(_lib.rot_harp_cayley_block(p.ctypes.data_as(C.POINTER(C.c_double)), int(b),
                                      mx.ctypes.data_as(C.POINTER(C.c_float)) if mx is not None else None,
                                      out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def harp_q8_plan(draws, signs) -> Plan:
    """Plan of an int8-stored HARP processor (``workloads.harp_q8_draws``): the fallback mixers of
    non-power-of-two radices are the library's QR of the drawn Gaussians."""
    mixers = [None if gm is None else harp_qr_block(gm) for gm in draws.mixer_gaussians]
    K = int(np.prod(draws.radices))
    return Plan.q8(K, draws.radices, draws.codes, draws.scales, mixers, draws.perms, signs)


def harp_plan(draws, signs, variant: str) -> Plan:
    """Plan for a HARP processor built from seeded draws (``workloads.harp_draws``).

    variant: ``random`` (Givens blocks per block from the angles, QR blocks from the
    Gaussians, the drawn permutations), ``init_identity`` (theta = 0, identity for
    non-power-of-two radices, no permutations) or ``init_qr`` (theta = 0, QR fallback
    mixer for non-power-of-two radices).
    """
    radices = list(draws.radices)
    K = int(np.prod(radices))
    params = []
    for t, b in enumerate(radices):
        if variant == "random":
            if b == 2:
                params.append(harp_givens_blocks(draws.angles[t]))
            else:
                params.append(np.stack([harp_qr_block(gm) for gm in draws.gaussians[t]]))
        elif variant == "init_identity":
            params.append(None)
        elif variant == "init_qr":
            params.append(None if (b & (b - 1)) == 0 else harp_qr_block(draws.gaussians[t][0])[None])
        else:
            raise ValueError(variant)
    perms = list(draws.perms) if variant == "random" else None
    return Plan(K, radices, params, perms, signs)


def check_device():
    """Synchronise and raise if a bounded device wait gave up since the last check."""
    _check(_lib.rot_check_device())


ROT_TEST_NONE, ROT_TEST_ROTATION_COPY, ROT_TEST_W4A4_LOADS = 0, 1, 2


def test_inject(fault: int, wait_ns: int = 0):
    """Testing hook (rot_test_inject): make the next launch of one kernel family skip its copies
    so that its bounded waits run out, and/or set the wait bound (0 = defaults)."""
    _check(_lib.rot_test_inject(int(fault), int(wait_ns)))

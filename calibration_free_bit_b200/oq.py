"""Thin ctypes binding over liboq.so (C ABI in include/oq.h).

Argument marshalling only: every step of the path runs in liboq's sm_100a kernels.  PyTorch
supplies device memory and the stream.  If liboq.so is missing this module raises at import
of the library (there is no CPU fallback): build it with ``python -m
calibration_free_bit_b200.build`` or ``__graft_entry__.build()``.

Names follow the C ABI: oq_build_rpbh, oq_lloyd_max, oq_quantize_weight, oq_quantize_act,
oq_linear (plus oq_check and the introspection calls used by the tests).
"""
from __future__ import annotations

import ctypes as C
import os
import re
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liboq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "oq.h")

OQ_OK, OQ_EINVAL, OQ_EUNSUPPORTED, OQ_ECUDA, OQ_EDEVICE, OQ_ENOMEM = 0, -1, -2, -3, -4, -5
OQ_F32, OQ_BF16 = 0, 1

_lib = None


class OQError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"liboq error {code}: {msg}")
        self.code = code


def lib():
    """Load liboq.so once and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise OQError(OQ_EUNSUPPORTED, f"{LIB_PATH} is missing: the CUDA extension has not been "
                      "built (run `python -m calibration_free_bit_b200.build`)")
    L = C.CDLL(LIB_PATH)
    vp, i32, u64 = C.c_void_p, C.c_int, C.c_uint64
    L.oq_build_rpbh.argtypes = [i32, i32, u64, C.POINTER(vp)]
    L.oq_build_block_rht.argtypes = [i32, i32, u64, C.POINTER(vp)]
    L.oq_rpbh_tables.argtypes = [vp, vp, vp]
    L.oq_lloyd_max.argtypes = [i32, i32, C.POINTER(vp)]
    L.oq_lloyd_max_marginal.argtypes = [i32, i32, i32, C.POINTER(vp)]
    L.oq_codebook_values.argtypes = [vp, vp, vp]
    L.oq_codebook_grid.argtypes = [vp, C.POINTER(i32), C.POINTER(C.c_double), vp]
    L.oq_quantize_weight.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.oq_quantize_act.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.oq_quantize_act_gelu.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.oq_linear.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp]
    L.oq_quantized_linear.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, vp, i32, vp,
                                      i32, vp]
    L.oq_linear_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, vp, i32, vp]
    L.oq_check.argtypes = [vp]
    L.oq_free_rpbh.argtypes = [vp]
    L.oq_free_rpbh.restype = None
    L.oq_free_codebook.argtypes = [vp]
    L.oq_free_codebook.restype = None
    L.oq_debug_arm_wait_timeout.argtypes = [i32, C.c_longlong]
    L.oq_timing_enable.argtypes = [i32]
    L.oq_timing_collect.argtypes = [vp, i32, C.POINTER(i32)]
    L.oq_last_error.restype = C.c_char_p
    L.oq_version.restype = C.c_char_p
    for name in ("oq_build_rpbh", "oq_build_block_rht", "oq_rpbh_tables", "oq_lloyd_max", "oq_lloyd_max_marginal",
                 "oq_codebook_values",
                 "oq_codebook_grid", "oq_quantize_weight", "oq_quantize_act",
                 "oq_quantize_act_gelu", "oq_linear", "oq_quantized_linear",
                 "oq_linear_noalloc", "oq_check", "oq_timing_enable", "oq_timing_collect",
                 "oq_debug_arm_wait_timeout"):
        getattr(L, name).restype = i32
    _lib = L
    return L


def header_functions() -> list[str]:
    """Names of the functions include/oq.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(oq_[a-z0-9_]+)\s*\(", text)))


def _check(rc: int):
    if rc != OQ_OK:
        raise OQError(rc, lib().oq_last_error().decode())


def _stream(stream) -> Optional[int]:
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return OQ_F32
    if t.dtype == torch.bfloat16:
        return OQ_BF16
    raise OQError(OQ_EINVAL, f"unsupported dtype {t.dtype} (fp32 or bf16)")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise OQError(OQ_EINVAL, "tensors must be contiguous")
    return t.data_ptr()


class RPBH:
    """Handle of an RPBH rotation (oq_build_rpbh), or of its Block-RHT ablation without the
    leading permutation (oq_build_block_rht, permute=False)."""

    def __init__(self, d: int, h: int, seed: int = 0, permute: bool = True):
        self._h = C.c_void_p()
        build = lib().oq_build_rpbh if permute else lib().oq_build_block_rht
        _check(build(d, h, seed, C.byref(self._h)))
        self.d, self.h, self.seed, self.permute = d, h, seed, permute

    @property
    def handle(self):
        return self._h

    def tables(self):
        perm = np.empty(self.d, dtype=np.int32)
        sign = np.empty(self.d, dtype=np.int8)
        _check(lib().oq_rpbh_tables(self._h, perm.ctypes.data, sign.ctypes.data))
        return perm, sign

    def __del__(self):
        if getattr(self, "_h", None) and self._h.value and _lib is not None:
            _lib.oq_free_rpbh(self._h)
            self._h = C.c_void_p()


MARGINALS = {"gauss": 0, "exact": 1}      # OQ_MARGINAL_GAUSSIAN, OQ_MARGINAL_EXACT


class Codebook:
    """Handle of a Lloyd-Max codebook (oq_lloyd_max_marginal): for N(0, 1/d) ("gauss") or for
    the exact coordinate marginal f_d ("exact")."""

    def __init__(self, d: int, bits: int, marginal: str = "gauss"):
        self._h = C.c_void_p()
        _check(lib().oq_lloyd_max_marginal(d, bits, MARGINALS[marginal], C.byref(self._h)))
        self.d, self.bits, self.marginal = d, bits, marginal

    @property
    def handle(self):
        return self._h

    def values(self):
        L = 1 << self.bits
        c = np.empty(L, dtype=np.float64)
        t = np.empty(L - 1, dtype=np.float64)
        _check(lib().oq_codebook_values(self._h, c.ctypes.data, t.ctypes.data))
        return c, t

    def grid(self):
        G = C.c_int(0)
        delta = C.c_double(0)
        _check(lib().oq_codebook_grid(self._h, C.byref(G), C.byref(delta), None))
        table = np.empty(G.value + 1, dtype=np.uint32)
        _check(lib().oq_codebook_grid(self._h, C.byref(G), C.byref(delta), table.ctypes.data))
        return G.value, delta.value, table

    def __del__(self):
        if getattr(self, "_h", None) and self._h.value and _lib is not None:
            _lib.oq_free_codebook(self._h)
            self._h = C.c_void_p()


def oq_build_rpbh(d: int, h: int, seed: int = 0) -> RPBH:
    return RPBH(d, h, seed)


def oq_build_block_rht(d: int, h: int, seed: int = 0) -> RPBH:
    return RPBH(d, h, seed, permute=False)


def oq_lloyd_max(d: int, bits: int, marginal: str = "gauss") -> Codebook:
    return Codebook(d, bits, marginal)


def _rows_out(x: torch.Tensor, bits: int, codes, norms):
    rows, d = x.shape
    if codes is None:
        codes = torch.empty((rows, d * bits // 8), dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty(rows, dtype=torch.float32, device=x.device)
    return codes, norms


def oq_quantize_weight(r: RPBH, cw: Codebook, W: torch.Tensor, W_codes=None, row_norms=None,
                       stream=None):
    """Offline weight step: returns (W_codes uint8 [out, d*bw/8], row_norms fp32 [out])."""
    W_codes, row_norms = _rows_out(W, cw.bits, W_codes, row_norms)
    _check(lib().oq_quantize_weight(r.handle, cw.handle, _ptr(W), _dtype_code(W), W.shape[0],
                                    W.shape[1], _ptr(W_codes), _ptr(row_norms), _stream(stream)))
    return W_codes, row_norms


def oq_quantize_act(r: RPBH, ca: Codebook, x: torch.Tensor, x_codes=None, s=None, stream=None,
                    gelu: bool = False):
    """Online activation step: returns (x_codes uint8 [T, d*ba/8], s fp32 [T]); with
    gelu=True the codes and norms are those of GELU(x) (oq_quantize_act_gelu, bf16 x)."""
    x_codes, s = _rows_out(x, ca.bits, x_codes, s)
    fn = lib().oq_quantize_act_gelu if gelu else lib().oq_quantize_act
    _check(fn(r.handle, ca.handle, _ptr(x), _dtype_code(x), x.shape[0], x.shape[1],
              _ptr(x_codes), _ptr(s), _stream(stream)))
    return x_codes, s


def _out(y, T, N, out_dtype, device):
    if y is None:
        return torch.empty((T, N), dtype=out_dtype, device=device)
    if y.dtype not in (torch.float32, torch.bfloat16) or tuple(y.shape) != (T, N):
        raise ValueError(f"y must be fp32 or bf16 of shape {(T, N)}")
    return y


def oq_linear(ca: Codebook, cw: Codebook, x_codes: torch.Tensor, s: torch.Tensor,
              W_codes: torch.Tensor, row_norms: torch.Tensor, y=None, stream=None,
              out_dtype=torch.float32):
    """Codebook linear layer: y [T, out] = s_t rn_o sum_k ca[xc] cw[wc], fp32 or bf16 (the
    dtype of y when given, else out_dtype)."""
    T, N, d = x_codes.shape[0], W_codes.shape[0], ca.d
    y = _out(y, T, N, out_dtype, x_codes.device)
    _check(lib().oq_linear(ca.handle, cw.handle, _ptr(x_codes), _ptr(s), _ptr(W_codes),
                           _ptr(row_norms), T, d, N, _ptr(y), _dtype_code(y), _stream(stream)))
    return y


OQ_FORWARD_GELU = 1


def oq_quantized_linear(r: RPBH, ca: Codebook, cw: Codebook, x: torch.Tensor,
                        W_codes: torch.Tensor, row_norms: torch.Tensor, y=None, s=None,
                        stream=None, out_dtype=torch.float32, gelu: bool = False):
    """The online path in one call: y = oq_linear(oq_quantize_act(x)) without x_codes in
    memory (with gelu=True: of GELU(x)).  Returns y; the norms go to s when given."""
    T, d, N = x.shape[0], x.shape[1], W_codes.shape[0]
    y = _out(y, T, N, out_dtype, x.device)
    _check(lib().oq_quantized_linear(r.handle, ca.handle, cw.handle, _ptr(x), _dtype_code(x),
                                     _ptr(W_codes), _ptr(row_norms), T, d, N, _ptr(y),
                                     _dtype_code(y), _ptr(s), OQ_FORWARD_GELU if gelu else 0,
                                     _stream(stream)))
    return y


def oq_linear_noalloc(ca: Codebook, cw: Codebook, x_codes: torch.Tensor, s: torch.Tensor,
                      W_codes: torch.Tensor, row_norms: torch.Tensor, y: torch.Tensor,
                      stream=None):
    """oq_linear with the library's fixed workspace: the caller passes y; nothing is
    allocated on the device (see include/oq.h for the size limit and sharing rules)."""
    T, N, d = x_codes.shape[0], W_codes.shape[0], ca.d
    y = _out(y, T, N, None, x_codes.device)
    _check(lib().oq_linear_noalloc(ca.handle, cw.handle, _ptr(x_codes), _ptr(s), _ptr(W_codes),
                                   _ptr(row_norms), T, d, N, _ptr(y), _dtype_code(y),
                                   _stream(stream)))
    return y


def oq_check(stream=None):
    _check(lib().oq_check(_stream(stream)))


KERNEL_NAMES = {1: "quantize", 2: "decode", 3: "gemm", 4: "fused", 5: "aux"}
OQ_KERNEL_QUANTIZE, OQ_KERNEL_DECODE, OQ_KERNEL_GEMM, OQ_KERNEL_FUSED = 1, 2, 3, 4
OQ_KERNEL_AUX = 5


def oq_debug_arm_wait_timeout(kernel: int, limit_cycles: int):
    """Arm the one-shot test of the bounded waits for this thread's next launch of `kernel`
    (OQ_KERNEL_QUANTIZE or OQ_KERNEL_GEMM; 0 disarms); see include/oq.h."""
    _check(lib().oq_debug_arm_wait_timeout(kernel, limit_cycles))


class _TimingRecord(C.Structure):
    _fields_ = [("kernel", C.c_int), ("ms", C.c_float)]


def oq_timing_enable(on: bool = True):
    """Bracket every kernel this thread launches through liboq with CUDA events."""
    _check(lib().oq_timing_enable(1 if on else 0))


def oq_timing_collect(capacity: int = 1 << 20):
    """Wait for the pending timing events; returns [(kernel name, ms), ...] in launch order."""
    buf = (_TimingRecord * capacity)()
    n = C.c_int(0)
    _check(lib().oq_timing_collect(buf, capacity, C.byref(n)))
    return [(KERNEL_NAMES.get(buf[i].kernel, str(buf[i].kernel)), buf[i].ms)
            for i in range(n.value)]


def version() -> str:
    return lib().oq_version().decode()

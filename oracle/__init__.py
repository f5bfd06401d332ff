"""fp64 CPU oracle of the routed sparse-MoE block (ctypes front end).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  It
shares no code with the CUDA library (``routed_expert_ffn_06_b200``); the only
thing both sides take from a common place is the seeded input generator
``routed_expert_ffn_06_b200.synth``, which holds none of the block's
arithmetic.  The arithmetic itself is in ``oracle.c`` (plain C, fp64).

Parity pins for each function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

PRENORM = 1
RESIDUAL = 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (-O2, OpenMP, IEEE math)."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC),
                                             os.path.getmtime(os.path.join(HERE, "oracle.h")))):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
                           "-o", tmp, SRC, "-lm"])
    os.replace(tmp, LIB)
    return LIB


class _Layer(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("E", ctypes.c_int32), ("F", ctypes.c_int32),
                ("Fs", ctypes.c_int32), ("k", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("Wr", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("expert_slot", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("shared_codes", ctypes.c_void_p),
                ("shared_scales", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_double
        L.orc_half_to_double.restype = dbl
        L.orc_half_to_double.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_double.restype = dbl
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_double_to_bf16.argtypes = [dbl]
        L.orc_codes_bytes.restype = ctypes.c_int64
        L.orc_codes_bytes.argtypes = [i32, i32, i32]
        L.orc_read_code.restype = i32
        L.orc_read_code.argtypes = [vp, i32, i32, i32, i32, i32]
        L.orc_dequant.restype = dbl
        L.orc_dequant.argtypes = [vp, vp, i32, i32, i32, i32, i32]
        L.orc_dequant_matrix.argtypes = [vp, vp, i32, i32, i32, vp]
        L.orc_router_logits.argtypes = [vp, vp, i32, vp]
        L.orc_select_topk_f32.argtypes = [vp, i32, i32, i32, vp]
        L.orc_select_topk_f64.argtypes = [vp, i32, i32, i32, vp]
        L.orc_renorm_weights.argtypes = [vp, vp, i32, i32, i32, vp]
        L.orc_bucket.argtypes = [vp, i32, i32, i32, vp, vp, vp]
        L.orc_silu.restype = dbl
        L.orc_silu.argtypes = [dbl]
        L.orc_expert_ffn.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        L.orc_rmsnorm_bf16.argtypes = [vp, i32, i32, dbl, vp]
        L.orc_block_forward.restype = ctypes.c_int
        L.orc_block_forward.argtypes = [vp, vp, i32, vp, i32, vp, i32, vp, vp, vp, vp]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_set_num_threads.argtypes = [i32]
    return _lib


# ------------------------------------------------------------------ helpers
def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _np(t, dtype=None):
    """torch tensor / numpy array -> contiguous numpy array on the host."""
    if t is None:
        return None
    if hasattr(t, "detach"):
        import torch
        t = t.detach().cpu()
        if t.dtype in (torch.bfloat16, torch.float16):
            t = t.view(torch.int16)
        t = t.contiguous().numpy()
    a = np.ascontiguousarray(t)
    if dtype is not None:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return a


def half_to_double(h: int) -> float:
    return lib().orc_half_to_double(int(h) & 0xFFFF)


def bf16_to_double(b: int) -> float:
    return lib().orc_bf16_to_double(int(b) & 0xFFFF)


def double_to_bf16(v: float) -> int:
    return lib().orc_double_to_bf16(float(v))


def silu(z: float) -> float:
    return lib().orc_silu(float(z))


def codes_bytes(R: int, K: int, bits: int) -> int:
    return lib().orc_codes_bytes(R, K, bits)


def read_code(codes, R, K, bits, row, col) -> int:
    c = _np(codes, np.uint8)
    return lib().orc_read_code(_p(c), R, K, bits, row, col)


def dequant_matrix(codes, scales, R: int, K: int, bits: int) -> np.ndarray:
    c = _np(codes, np.uint8)
    s = _np(scales, np.uint16)
    W = np.empty((R, K), dtype=np.float64)
    lib().orc_dequant_matrix(_p(c), _p(s), R, K, bits, _p(W))
    return W


def select_topk_f32(logits, k: int) -> np.ndarray:
    L = _np(logits, np.float32)
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int32)
    lib().orc_select_topk_f32(_p(L), T, E, k, _p(ids))
    return ids


def select_topk_f64(logits, k: int) -> np.ndarray:
    L = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = L.shape
    ids = np.empty((T, k), dtype=np.int32)
    lib().orc_select_topk_f64(_p(L), T, E, k, _p(ids))
    return ids


def renorm_weights(logits, ids) -> np.ndarray:
    L = np.ascontiguousarray(logits, dtype=np.float64)
    I = np.ascontiguousarray(ids, dtype=np.int32)
    T, E = L.shape
    k = I.shape[1]
    w = np.empty((T, k), dtype=np.float64)
    lib().orc_renorm_weights(_p(L), _p(I), T, E, k, _p(w))
    return w


def bucket(ids, E: int):
    I = np.ascontiguousarray(_np(ids), dtype=np.int32)
    T, k = I.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    entries = np.empty(T * k, dtype=np.int32)
    lib().orc_bucket(_p(I), T, k, E, _p(counts), _p(offsets), _p(entries))
    return counts, offsets, entries


def expert_ffn(codes, scales, d: int, F: int, bits: int, x) -> np.ndarray:
    c = _np(codes, np.uint8)
    s = _np(scales, np.uint16)
    xv = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty(d, dtype=np.float64)
    lib().orc_expert_ffn(_p(c), _p(s), d, F, bits, _p(xv), _p(y))
    return y


def rmsnorm_bf16(x_bf16_bits, eps: float = 1e-6) -> np.ndarray:
    x = np.ascontiguousarray(_np(x_bf16_bits), dtype=np.uint16)
    T, d = x.shape
    out = np.empty_like(x)
    lib().orc_rmsnorm_bf16(_p(x), T, d, eps, _p(out))
    return out


class OracleLayer:
    """Host copies of one layer's tensors, laid out as the oracle reads them."""

    def __init__(self, layer, bias_override=None):
        sh = layer.shape
        self.shape = sh
        self.Wr = _np(layer.router_w, np.float32)
        b = bias_override if bias_override is not None else layer.router_bias
        self.bias = None if b is None else _np(b, np.float32)
        self.slot = np.ascontiguousarray(_np(layer.expert_slot), dtype=np.int32)
        self.codes = _np(layer.codes, np.uint8)
        self.scales = _np(layer.scales, np.uint16)
        self.shared_codes = _np(layer.shared_codes, np.uint8)
        self.shared_scales = _np(layer.shared_scales, np.uint16)
        self._s = _Layer(sh.d, sh.E, sh.F, sh.Fs, sh.k, sh.bits, _p(self.Wr).value,
                         None if self.bias is None else _p(self.bias).value,
                         _p(self.slot).value, _p(self.codes).value, _p(self.scales).value,
                         None if self.shared_codes is None else _p(self.shared_codes).value,
                         None if self.shared_scales is None else _p(self.shared_scales).value)

    def router_logits(self, x) -> np.ndarray:
        xv = np.ascontiguousarray(x, dtype=np.float64)
        T = xv.shape[0]
        out = np.empty((T, self.shape.E), dtype=np.float64)
        lib().orc_router_logits(ctypes.byref(self._s), _p(xv), T, _p(out))
        return out

    def block_forward(self, x_bf16, rows=None, sel_logits=None, flags: int = 0):
        """Returns dict(y [n,d] f64, logits [n,E] f64, ids [n,k], w [n,k])."""
        x = np.ascontiguousarray(_np(x_bf16), dtype=np.uint16)
        T, d = x.shape
        rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
        n = T if rws is None else len(rws)
        sl = None if sel_logits is None else np.ascontiguousarray(_np(sel_logits),
                                                                   dtype=np.float32)
        y = np.empty((n, d), dtype=np.float64)
        lg = np.empty((n, self.shape.E), dtype=np.float64)
        ids = np.empty((n, self.shape.k), dtype=np.int32)
        w = np.empty((n, self.shape.k), dtype=np.float64)
        rc = lib().orc_block_forward(ctypes.byref(self._s), _p(x), T, _p(rws), n, _p(sl), flags,
                                     _p(y), _p(lg), _p(ids), _p(w))
        if rc:
            raise RuntimeError(f"oracle block_forward failed ({rc})")
        return dict(y=y, logits=lg, ids=ids, w=w)


def set_num_threads(n: int) -> None:
    lib().orc_set_num_threads(int(n))


def num_threads() -> int:
    return lib().orc_num_threads()

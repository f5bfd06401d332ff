"""ctypes binding of the C ABI in ``include/moe.h``.

Argument marshalling only: every step of the block runs in the CUDA kernels
of ``libmoe.so``.  There is no fallback path; if the library is missing or no
sm_100 GPU is current, the calls raise.

Functions keep the C names (``moe_route_topk``, ``moe_expert_ffn_decode``,
``moe_expert_ffn_prefill``, ``moe_block_forward``, ...).  Tensors are torch
tensors on the current CUDA device; the stream is torch's current stream unless
one is passed.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
          3: "MOE_ERR_WORKSPACE_TOO_SMALL", 4: "MOE_ERR_MISALIGNED", 5: "MOE_ERR_CUDA",
          6: "MOE_ERR_DEVICE_CHECK", 7: "MOE_ERR_TIMEOUT", 8: "MOE_ERR_NO_DEVICE"}

F_PRENORM = 1
F_RESIDUAL = 2
F_DETERMINISTIC = 4
F_DEBUG = 8

# moe_workspace_set_debug_withhold sites
WITHHOLD_PREFILL_ARRIVE = 1

EXPORTS = ["moe_workspace_bytes", "moe_workspace_init", "moe_workspace_error",
           "moe_workspace_set_wait_limit", "moe_workspace_set_debug_withhold", "moe_router_split",
           "moe_route_topk",
           "moe_expert_ffn_decode", "moe_expert_ffn_prefill", "moe_block_forward",
           "moe_block_forward_noalloc", "moe_adapt_workspace_bytes", "moe_adapt_layout",
           "moe_status_string", "moe_build_info", "moe_pack_host"]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class moe_layer(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("ffn", ctypes.c_int32), ("top_k", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("group", ctypes.c_int32), ("shared_ffn", ctypes.c_int32),
                ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("expert_slot", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("shared_codes", ctypes.c_void_p),
                ("shared_scales", ctypes.c_void_p), ("router_pref", ctypes.c_void_p),
                ("route_counts", ctypes.c_void_p), ("l2_next", ctypes.c_void_p),
                ("router_w_split", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with "
                           "`python -m routed_expert_ffn_06_b200.build` (needs nvcc)")
    L = ctypes.CDLL(path)
    vp, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    st = ctypes.c_int
    P = ctypes.POINTER(moe_layer)
    L.moe_workspace_bytes.restype = sz
    L.moe_workspace_bytes.argtypes = [P, i32]
    L.moe_workspace_init.restype = st
    L.moe_workspace_init.argtypes = [vp, sz, vp]
    L.moe_workspace_error.restype = st
    L.moe_workspace_error.argtypes = [vp, sz, ctypes.POINTER(u32), vp]
    L.moe_router_split.restype = st
    L.moe_router_split.argtypes = [P, vp, vp]
    L.moe_workspace_set_wait_limit.restype = st
    L.moe_workspace_set_wait_limit.argtypes = [vp, sz, u32, vp]
    L.moe_workspace_set_debug_withhold.restype = st
    L.moe_workspace_set_debug_withhold.argtypes = [vp, sz, u32, vp]
    L.moe_route_topk.restype = st
    L.moe_route_topk.argtypes = [P, vp, i32, u32, vp, vp, vp, vp, sz, vp]
    L.moe_expert_ffn_decode.restype = st
    L.moe_expert_ffn_decode.argtypes = [P, vp, i32, vp, vp, vp, u32, vp, sz, vp]
    L.moe_expert_ffn_prefill.restype = st
    L.moe_expert_ffn_prefill.argtypes = [P, vp, i32, vp, vp, vp, vp, vp, u32, vp, sz, vp]
    L.moe_block_forward.restype = st
    L.moe_block_forward.argtypes = [P, vp, i32, vp, u32, vp, sz, vp]
    L.moe_block_forward_noalloc.restype = st
    L.moe_block_forward_noalloc.argtypes = [P, vp, i32, vp, u32, vp]
    L.moe_adapt_workspace_bytes.restype = sz
    L.moe_adapt_workspace_bytes.argtypes = [P, i32]
    L.moe_adapt_layout.restype = st
    L.moe_adapt_layout.argtypes = [P, ctypes.c_float, i32, vp, vp, sz, vp]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [st]
    L.moe_build_info.restype = ctypes.c_char_p
    L.moe_build_info.argtypes = []
    L.moe_pack_host.restype = st
    L.moe_pack_host.argtypes = [vp, i32, i32, i32, vp, vp]
    _lib = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def make_layer_struct(layer, router_pref=None, route_counts=None) -> moe_layer:
    """moe_layer for a ``synth.Layer`` whose tensors live on the GPU;
    router_pref: optional fp32 [E] selection bonus; route_counts: optional fp32
    [E] routing counters (both on the same device)."""
    sh = layer.shape
    return moe_layer(sh.d, sh.E, sh.F, sh.k, sh.bits, 32, sh.Fs, _ptr(layer.router_w),
                     _ptr(layer.router_bias), _ptr(layer.expert_slot), _ptr(layer.codes),
                     _ptr(layer.scales), _ptr(layer.shared_codes), _ptr(layer.shared_scales),
                     _ptr(router_pref), _ptr(route_counts))


def moe_router_split(layer: moe_layer, stream=None) -> torch.Tensor:
    """The layer's router weights split into bf16 hi and lo parts ([2][E][d],
    bf16 bits as int16) on the current device; set it as
    layer.router_w_split (keep the tensor alive while the struct is used)."""
    out = torch.empty(2, layer.n_experts, layer.d_model, dtype=torch.int16, device="cuda")
    _check(load().moe_router_split(ctypes.byref(layer), _ptr(out), _stream(stream)),
           "moe_router_split")
    return out


def link_l2_next(structs, cyclic: bool = True) -> None:
    """Name, in each moe_layer of a sequence, the one run after it (the last
    names the first when cyclic), so that each decode step prefetches the next
    layer's router and shared expert into L2.  The structs must outlive the
    calls (and any graph captured from them)."""
    n = len(structs)
    for i, L in enumerate(structs):
        j = i + 1
        if j == n:
            if not cyclic:
                L.l2_next = None
                continue
            j = 0
        L.l2_next = ctypes.addressof(structs[j])


def moe_workspace_bytes(layer: moe_layer, max_tokens: int) -> int:
    return load().moe_workspace_bytes(ctypes.byref(layer), int(max_tokens))


def moe_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(load().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def moe_workspace_error(ws: torch.Tensor, stream=None):
    code = ctypes.c_uint32(0)
    st = load().moe_workspace_error(_ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(code),
                                    _stream(stream))
    return st, code.value


def moe_workspace_set_wait_limit(ws: torch.Tensor, limit_us: int, stream=None) -> None:
    _check(load().moe_workspace_set_wait_limit(_ptr(ws), ws.numel() * ws.element_size(),
                                               int(limit_us), _stream(stream)),
           "moe_workspace_set_wait_limit")


def moe_workspace_set_debug_withhold(ws: torch.Tensor, site: int, stream=None) -> None:
    _check(load().moe_workspace_set_debug_withhold(_ptr(ws), ws.numel() * ws.element_size(),
                                                   int(site), _stream(stream)),
           "moe_workspace_set_debug_withhold")


def alloc_workspace(layer: moe_layer, max_tokens: int, device=None) -> torch.Tensor:
    n = moe_workspace_bytes(layer, max_tokens)
    if n == 0:
        raise MoEError(1, "moe_workspace_bytes")
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    moe_workspace_init(ws)
    return ws


def moe_route_topk(layer: moe_layer, x, T: int, flags: int, logits, ids, w, ws, stream=None):
    _check(load().moe_route_topk(ctypes.byref(layer), _ptr(x), int(T), int(flags), _ptr(logits),
                                 _ptr(ids), _ptr(w), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_route_topk")


def moe_expert_ffn_decode(layer: moe_layer, x, T: int, ids, w, y, flags: int, ws, stream=None):
    _check(load().moe_expert_ffn_decode(ctypes.byref(layer), _ptr(x), int(T), _ptr(ids), _ptr(w),
                                        _ptr(y), int(flags), _ptr(ws), ws.numel(),
                                        _stream(stream)),
           "moe_expert_ffn_decode")


def moe_expert_ffn_prefill(layer: moe_layer, x, T: int, ids, w, y, offsets, entries, flags: int,
                           ws, stream=None):
    _check(load().moe_expert_ffn_prefill(ctypes.byref(layer), _ptr(x), int(T), _ptr(ids), _ptr(w),
                                         _ptr(y), _ptr(offsets), _ptr(entries), int(flags),
                                         _ptr(ws), ws.numel(), _stream(stream)),
           "moe_expert_ffn_prefill")


def moe_block_forward(layer: moe_layer, x, T: int, y, flags: int, ws, stream=None):
    _check(load().moe_block_forward(ctypes.byref(layer), _ptr(x), int(T), _ptr(y), int(flags),
                                    _ptr(ws), ws.numel(), _stream(stream)),
           "moe_block_forward")


def moe_block_forward_noalloc(layer: moe_layer, x, T: int, y, flags: int, stream=None):
    """Decode-window block forward on the library's static device scratch."""
    _check(load().moe_block_forward_noalloc(ctypes.byref(layer), _ptr(x), int(T), _ptr(y),
                                            int(flags), _stream(stream)),
           "moe_block_forward_noalloc")


def moe_adapt_workspace_bytes(layer: moe_layer, max_swaps: int) -> int:
    return load().moe_adapt_workspace_bytes(ctypes.byref(layer), int(max_swaps))


def moe_adapt_layout(layer: moe_layer, decay: float, max_swaps: int, swaps_done, ws, stream=None):
    """Re-order the layer's slots by its routing counters (include/moe.h)."""
    _check(load().moe_adapt_layout(ctypes.byref(layer), float(decay), int(max_swaps),
                                   _ptr(swaps_done), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)),
           "moe_adapt_layout")


def moe_pack_host(w, bits: int):
    """Quantise and pack one host fp32 matrix [rows, cols] (include/moe_pack.h).
    Returns (codes uint8 [rows/16, cols/32*16*(8|12)], scales int16 holding
    fp16 bits [rows/16, cols/32*16]), host tensors."""
    import torch
    if w.device.type != "cpu" or w.dtype != torch.float32 or w.dim() != 2:
        raise ValueError("moe_pack_host takes a 2-D host float32 tensor")
    w = w.contiguous()
    rows, cols = w.shape
    gb = 8 if bits == 2 else 12
    codes = torch.empty(max(rows // 16, 1), max(cols // 32, 1) * 16 * gb, dtype=torch.uint8)
    scales = torch.empty(max(rows // 16, 1), max(cols // 32, 1) * 16, dtype=torch.int16)
    _check(load().moe_pack_host(w.data_ptr(), int(rows), int(cols), int(bits), codes.data_ptr(),
                                scales.data_ptr()), "moe_pack_host")
    return codes, scales


def moe_status_string(status: int) -> str:
    return load().moe_status_string(int(status)).decode()


def moe_build_info() -> str:
    return load().moe_build_info().decode()

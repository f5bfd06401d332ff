"""Helpers shared by the GPU parity tests."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from routed_expert_ffn_06_b200 import moe, synth

# Tolerances of the block output against the fp64 oracle.
MAX_REL = 2e-2   # per token: max_i |y - ŷ| / max_i |ŷ|, worst token
RMS_REL = 3e-3   # ||y - ŷ||_2 / ||ŷ||_2 over the whole output


def errors(y_gpu, y_ref):
    """(max rel, rms rel) of a device output against the oracle's fp64."""
    y = y_gpu.float().cpu().double().numpy() if torch.is_tensor(y_gpu) else np.asarray(y_gpu)
    r = np.asarray(y_ref, dtype=np.float64)
    diff = y - r
    per_tok = np.abs(diff).max(axis=1) / np.maximum(np.abs(r).max(axis=1), 1e-30)
    rms = np.linalg.norm(diff) / max(np.linalg.norm(r), 1e-30)
    return float(per_tok.max()), float(rms)


def assert_close(y_gpu, y_ref, max_rel=MAX_REL, rms_rel=RMS_REL):
    mr, rr = errors(y_gpu, y_ref)
    assert mr <= max_rel and rr <= rms_rel, f"max rel {mr:.3e} (<= {max_rel}), rms rel {rr:.3e} (<= {rms_rel})"
    return mr, rr


def logit_bound(layer, x_in: np.ndarray) -> np.ndarray:
    """1e-4 * (sum_i |x_i Wr_ei| + |b_e|): the fp32 logit tolerance."""
    Wr = np.abs(layer.router_w.double().cpu().numpy())
    b = 0.0 if layer.router_bias is None else np.abs(layer.router_bias.double().cpu().numpy())
    return 1e-4 * (np.abs(x_in) @ Wr.T + b)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().view(torch.int16).numpy().view(np.uint16)


class GpuBlock:
    """One layer on the GPU plus its workspace, driven through the C ABI."""

    def __init__(self, layer, max_tokens: int):
        self.layer = layer
        self.L = moe.make_layer_struct(layer)
        self.ws = moe.alloc_workspace(self.L, max_tokens)
        self.sh = layer.shape

    def route(self, x, flags=0):
        T = x.shape[0]
        logits = torch.empty(T, self.sh.E, dtype=torch.float32, device="cuda")
        ids = torch.empty(T, self.sh.k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, self.sh.k, dtype=torch.float32, device="cuda")
        moe.moe_route_topk(self.L, x, T, flags, logits, ids, w, self.ws)
        return logits, ids, w

    def decode(self, x, ids, w, flags=0):
        y = torch.empty_like(x)
        moe.moe_expert_ffn_decode(self.L, x, x.shape[0], ids, w, y, flags, self.ws)
        return y

    def prefill(self, x, ids, w, flags=0, want_buckets=False):
        T = x.shape[0]
        y = torch.empty_like(x)
        off = ent = None
        if want_buckets:
            off = torch.empty(self.sh.E + 1, dtype=torch.int32, device="cuda")
            ent = torch.empty(T * self.sh.k, dtype=torch.int32, device="cuda")
        moe.moe_expert_ffn_prefill(self.L, x, T, ids, w, y, off, ent, flags, self.ws)
        return (y, off, ent) if want_buckets else y

    def block(self, x, flags=0):
        y = torch.empty_like(x)
        moe.moe_block_forward(self.L, x, x.shape[0], y, flags, self.ws)
        return y

    def error_word(self):
        return moe.moe_workspace_error(self.ws)


def router_oracle(layer):
    """The oracle for one layer's router only: host copies of the router
    tensors (its router reads no expert bytes, so those stay where they are)."""
    z8 = torch.zeros(16, dtype=torch.uint8)
    z16 = torch.zeros(16, dtype=torch.float16)
    lite = synth.Layer(layer.shape, layer.router_w.cpu(), None if layer.router_bias is None
                       else layer.router_bias.cpu(), layer.expert_slot.cpu(), z8, z16, None, None)
    return oracle.OracleLayer(lite)


def routing_check(layer, x, logits, ids, w, flags=0):
    """Routing of every token of one layer against the oracle: selection on
    the device's fp32 logits, logits within the fp32 bound of the oracle's
    fp64 router, weights as in oracle_check."""
    lg = logits.cpu().numpy()
    ids_g = ids.cpu().numpy()
    assert np.array_equal(oracle.select_topk_f32(lg, layer.shape.k), ids_g), "routing differs"
    if flags & moe.F_PRENORM:
        xin = oracle.rmsnorm_bf16(bf16_bits(x))
        xin = torch.from_numpy(xin.view(np.int16)).view(torch.bfloat16).double().numpy()
    else:
        xin = x.cpu().double().numpy()
    lg64 = router_oracle(layer).router_logits(xin)
    assert np.all(np.abs(lg - lg64) <= logit_bound(layer, xin)), "router logits outside the fp32 bound"
    wg = w.cpu().double().numpy()
    sel = np.take_along_axis(lg.astype(np.float64), ids_g.astype(np.int64), axis=1)
    own = np.exp(sel - sel.max(1, keepdims=True))
    own /= own.sum(1, keepdims=True)
    assert np.allclose(wg, own, rtol=1e-5, atol=1e-6), "weights differ from the softmax of the logits"
    ref = oracle.renorm_weights(lg64, ids_g)
    dl = np.take_along_axis(np.abs(lg.astype(np.float64) - lg64), ids_g.astype(np.int64),
                            axis=1).max(1, keepdims=True)
    assert np.all(np.abs(wg - ref) <= ref * (np.expm1(2 * dl) + 1e-5) + 1e-6), \
        "routing weights outside the logit-error bound"


def oracle_check(layer, x, logits, ids, w, y, flags=0, rows=None, oflags=None):
    """Compare one GPU block result with the oracle (selection on the GPU's
    fp32 logits).  Returns (max rel, rms rel)."""
    OL = oracle.OracleLayer(layer.to("cpu") if layer.codes.is_cuda else layer)
    of = 0
    if flags & moe.F_PRENORM:
        of |= oracle.PRENORM
    if flags & moe.F_RESIDUAL:
        of |= oracle.RESIDUAL
    lg = logits.cpu().numpy()
    r = OL.block_forward(bf16_bits(x), rows=rows, sel_logits=lg, flags=of)
    rr = np.arange(x.shape[0]) if rows is None else np.asarray(rows)
    ids_g = ids.cpu().numpy()[rr]
    assert np.array_equal(ids_g, r["ids"]), "routing differs from the oracle's selection"
    # logits within the fp32 bound of the oracle's fp64 logits
    if flags & moe.F_PRENORM:
        xin = oracle.rmsnorm_bf16(bf16_bits(x)[rr])
        xin = torch.from_numpy(xin.view(np.int16)).view(torch.bfloat16).double().numpy()
    else:
        xin = x.cpu().double().numpy()[rr]
    bound = logit_bound(layer, xin)
    assert np.all(np.abs(lg[rr] - r["logits"]) <= bound), "router logits outside the fp32 bound"
    # The weights are the softmax of the selected logits, which the device
    # knows to fp32 accuracy only: (a) against the softmax, in fp64, of the
    # device's own selected logits (the weight arithmetic alone), tightly; (b)
    # against the oracle's weights within the propagated logit error,
    # |dw_j| <= w_j * expm1(2 max_i |dl_i|) over the selected i.
    wg = w.cpu().double().numpy()[rr]
    sel = np.take_along_axis(lg[rr].astype(np.float64), ids_g.astype(np.int64), axis=1)
    own = np.exp(sel - sel.max(1, keepdims=True))
    own /= own.sum(1, keepdims=True)
    assert np.allclose(wg, own, rtol=1e-5, atol=1e-6), "weights differ from the softmax of the logits"
    dl = np.take_along_axis(np.abs(lg[rr].astype(np.float64) - r["logits"]),
                            ids_g.astype(np.int64), axis=1).max(1, keepdims=True)
    assert np.all(np.abs(wg - r["w"]) <= r["w"] * (np.expm1(2 * dl) + 1e-5) + 1e-6), \
        "routing weights outside the logit-error bound"
    assert np.allclose(wg.sum(1), 1.0, atol=1e-6)
    yg = y.float().cpu().double().numpy()[rr]
    return assert_close(yg, r["y"])

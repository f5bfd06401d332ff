"""Stacked layers (the 48-layer decode stack and the prefill + decode mix),
teacher-forced per layer: each layer's GPU output is compared with the oracle
run on that layer's GPU input and the GPU's fp32 logits, through
moe_block_forward with pre-norm and residual.  The mix also re-ranks the
experts (router bias permuted) between passes, as its drifting workload does."""
import numpy as np
import pytest
import torch

import oracle

from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock, oracle_check, routing_check

pytestmark = pytest.mark.gpu

FLAGS = moe.F_PRENORM | moe.F_RESIDUAL


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run_layers(layers, x, rows=None):
    """x through the layers; every layer checked against the oracle."""
    T = x.shape[0]
    for layer in layers:
        gb = GpuBlock(layer, T)
        logits, ids, w = gb.route(x, FLAGS)
        y = gb.block(x, FLAGS)
        torch.cuda.synchronize()
        oracle_check(layer, x, logits, ids, w, y, flags=FLAGS, rows=rows)
        assert gb.error_word() == (0, 0)
        x = y
    return x


@pytest.mark.parametrize("T", [1, 4])
def test_decode_stack_teacher_forced(T):
    wl = synth.WORKLOADS["decode_stack"]
    layers = [synth.make_layer(wl["shape"], seed=0, layer=l, device="cuda", bias=wl["bias"],
                               slot=wl["slot"]) for l in range(3)]
    x = synth.make_tokens(T, wl["shape"].d, seed=11 + T, device="cuda")
    y = _run_layers(layers, x)
    assert torch.isfinite(y.float()).all()


def test_mix_prefill_then_decode_with_drift():
    """A prefill chunk through three 3-bit layers, then a decode window, then
    the expert ranking drifts (bias permuted) and the window runs again."""
    wl = synth.WORKLOADS["mix"]
    sh = wl["shape"]
    layers = [synth.make_layer(sh, seed=0, layer=l, device="cuda", bias=wl["bias"],
                               slot=wl["slot"]) for l in range(3)]
    chunk = synth.make_tokens(512, sh.d, seed=1, device="cuda")
    rows = np.unique(np.random.default_rng(2).choice(512, 40, replace=False))
    _run_layers(layers, chunk, rows=rows)
    win = synth.make_tokens(4, sh.d, seed=3, device="cuda")
    _run_layers(layers, win)
    for layer in layers:
        layer.router_bias.copy_(synth.permute_profile(layer, seed=0, epoch=1))
    _run_layers(layers, win)


def test_decode_stack_all_48_layers():
    """The whole 48-layer 3-bit decode stack, one 4-token step through
    moe_block_forward with pre-norm and residual, teacher-forced.  At every
    layer the routing of every token is checked against the oracle (selection
    on the device's fp32 logits, logits within the fp32 bound of the oracle's
    fp64 router, weights); at the first, a middle and the last layer the
    outputs too.  Layers are generated one at a time, so the stack's 34 GB never
    sit on the device together."""
    wl = synth.WORKLOADS["decode_stack"]
    sh = wl["shape"]
    T = 4
    x = synth.make_tokens(T, sh.d, seed=77, device="cuda")
    for l in range(48):
        layer = synth.make_layer(sh, seed=0, layer=l, device="cuda", bias=wl["bias"],
                                 slot=wl["slot"])
        gb = GpuBlock(layer, T)
        logits, ids, w = gb.route(x, FLAGS)
        y = gb.block(x, FLAGS)
        torch.cuda.synchronize()
        if l in (0, 24, 47):
            oracle_check(layer, x, logits, ids, w, y, flags=FLAGS)
        else:
            routing_check(layer, x, logits, ids, w, flags=FLAGS)
        assert gb.error_word() == (0, 0)
        assert torch.isfinite(y.float()).all()
        x = y
        del layer, gb


def test_mix_prefill_chunk_all_48_layers():
    """One full 8192-token chunk of the mix through all 48 3-bit layers with
    pre-norm and residual, teacher-forced.  At every layer the selection of
    every token equals the oracle's on the device's fp32 logits; at the first,
    a middle and the last layer a seeded sample of 24 tokens is checked in full
    (logits, weights, outputs) against the oracle."""
    wl = synth.WORKLOADS["mix"]
    sh = wl["shape"]
    T = wl["chunk"]
    x = synth.make_tokens(T, sh.d, seed=5, device="cuda")
    rows = np.unique(np.random.default_rng(5).choice(T, 24, replace=False))
    for l in range(48):
        layer = synth.make_layer(sh, seed=0, layer=l, device="cuda", bias=wl["bias"],
                                 slot=wl["slot"])
        gb = GpuBlock(layer, T)
        logits, ids, w = gb.route(x, FLAGS)
        y = gb.block(x, FLAGS)
        torch.cuda.synchronize()
        if l in (0, 24, 47):
            oracle_check(layer, x, logits, ids, w, y, flags=FLAGS, rows=rows)
        else:
            assert np.array_equal(oracle.select_topk_f32(logits.cpu().numpy(), sh.k),
                                  ids.cpu().numpy()), f"routing differs at layer {l}"
        assert gb.error_word() == (0, 0)
        x = y
        del layer, gb

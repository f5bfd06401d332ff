"""Stacked layers (the 48-layer decode stack and the prefill + decode mix),
teacher-forced per layer: each layer's GPU output is compared with the oracle
run on that layer's GPU input and the GPU's fp32 logits, through
moe_block_forward with pre-norm and residual.  The mix also re-ranks the
experts (router bias permuted) between passes, as its drifting workload does."""
import numpy as np
import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock, oracle_check

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

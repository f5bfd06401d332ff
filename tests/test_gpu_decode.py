"""GPU parity of the router and the decode / verify-window step against the
fp64 oracle, through the C ABI.  Routing must match bit for bit given the
device's fp32 logits; outputs within max rel 2e-2 / RMS rel 3e-3."""
import numpy as np
import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock, assert_close, errors, oracle_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _layer(shape, **kw):
    kw.setdefault("bias", "normal")
    return synth.make_layer(shape, device="cuda", **kw)


# -------------------------------------------------------------- tiny config
def test_tiny_config_block():
    """d=64, 16 experts (ffn 32) + shared (ffn 32), top-2, 4 tokens, 2-bit, seed 0."""
    wl = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(4, 64, seed=0, device="cuda")
    gb = GpuBlock(layer, 8)
    logits, ids, w = gb.route(x)
    y = gb.decode(x, ids, w)
    oracle_check(layer, x, logits, ids, w, y)
    y2 = gb.block(x)
    assert torch.equal(y, y2)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("T", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("E,k,Fs", [(16, 2, 32), (37, 5, 0), (64, 16, 64), (8, 8, 32), (12, 1, 32)])
def test_small_shapes(bits, T, E, k, Fs):
    sh = synth.MoEShape(d=96, E=E, F=64, Fs=Fs, k=k, bits=bits)
    layer = _layer(sh, seed=T * 7 + E, bias_std=1.0)
    x = synth.make_tokens(T, 96, seed=T, device="cuda")
    gb = GpuBlock(layer, 8)
    logits, ids, w = gb.route(x)
    y = gb.decode(x, ids, w)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("flags", [moe.F_PRENORM, moe.F_RESIDUAL, moe.F_PRENORM | moe.F_RESIDUAL])
def test_flags_small(flags):
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=64, k=4, bits=3)
    layer = _layer(sh, seed=3)
    x = (synth.make_tokens(4, 128, seed=9, device="cuda").float() * 3.0).to(torch.bfloat16)
    gb = GpuBlock(layer, 8)
    logits, ids, w = gb.route(x, flags)
    y = gb.decode(x, ids, w, flags)
    oracle_check(layer, x, logits, ids, w, y, flags=flags)


def test_zero_tokens_is_a_noop():
    sh = synth.MoEShape(d=64, E=16, F=32, Fs=32, k=2, bits=2)
    gb = GpuBlock(_layer(sh), 4)
    x = torch.ones(1, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.full((1, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_block_forward(gb.L, x, 0, y, 0, gb.ws)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_zero_input_gives_zero():
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=64, k=4, bits=2)
    gb = GpuBlock(_layer(sh), 4)
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    assert torch.count_nonzero(gb.block(x)) == 0


def test_out_of_range_ids_are_flagged_not_read():
    sh = synth.MoEShape(d=64, E=16, F=32, Fs=32, k=2, bits=2)
    layer = _layer(sh)
    gb = GpuBlock(layer, 4)
    x = synth.make_tokens(2, 64, device="cuda")
    ids = torch.tensor([[3, 99], [-1, 5]], dtype=torch.int32, device="cuda")
    w = torch.full((2, 2), 0.5, dtype=torch.float32, device="cuda")
    gb.decode(x, ids, w)
    st, code = gb.error_word()
    assert st == 6 and code & 2
    assert gb.error_word() == (0, 0)      # the read clears it


# --------------------------------------------------------------- full size
@pytest.fixture(scope="module")
def decode_layer():
    wl = synth.WORKLOADS["decode"]
    return synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"], slot=wl["slot"])


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_decode_full_size(decode_layer, T):
    """d=2048, 512 experts ffn 512 + shared, top-10, 2-bit, Zipf(1.1) popularity."""
    gb = GpuBlock(decode_layer, 8)
    x = synth.make_tokens(T, 2048, seed=100 + T, device="cuda")
    logits, ids, w = gb.route(x)
    y = gb.decode(x, ids, w)
    mr, rr = oracle_check(decode_layer, x, logits, ids, w, y)
    print(f"T={T}: max rel {mr:.2e} rms rel {rr:.2e}")
    assert gb.error_word() == (0, 0)


def test_decode_window_invariance(decode_layer):
    """A verify window gives each token what it gets alone: same routing,
    outputs equal within tolerance."""
    gb = GpuBlock(decode_layer, 8)
    x = synth.make_tokens(4, 2048, seed=55, device="cuda")
    _, ids4, w4 = gb.route(x)
    y4 = gb.decode(x, ids4, w4)
    for t in range(4):
        _, ids1, w1 = gb.route(x[t:t + 1])
        y1 = gb.decode(x[t:t + 1].clone(), ids1, w1)
        assert torch.equal(ids1[0], ids4[t])
        assert_close(y4[t:t + 1].float().cpu().double().numpy(), y1.float().cpu().double().numpy(),
                     max_rel=1e-2, rms_rel=3e-3)


def test_decode_slot_layout_invariance():
    """The same experts packed into other slots: bit-identical output."""
    sh = synth.MoEShape(d=512, E=64, F=128, Fs=128, k=6, bits=3)
    a = synth.make_layer(sh, seed=4, device="cuda", bias="normal", slot="identity")
    b = synth.make_layer(sh, seed=4, device="cuda", bias="normal", slot="random")
    assert not torch.equal(a.expert_slot, b.expert_slot)
    x = synth.make_tokens(4, 512, seed=8, device="cuda")
    ya = GpuBlock(a, 4).block(x)
    yb = GpuBlock(b, 4).block(x)
    assert torch.equal(ya, yb)


def test_decode_3bit_stack_layer_prenorm_residual():
    """One layer of the 48-layer 3-bit stack, with pre-norm and residual."""
    wl = synth.WORKLOADS["decode_stack"]
    layer = synth.make_layer(wl["shape"], seed=0, layer=7, device="cuda", bias=wl["bias"],
                             slot=wl["slot"])
    gb = GpuBlock(layer, 4)
    x = (synth.make_tokens(4, 2048, seed=7, device="cuda").float() * 20).to(torch.bfloat16)
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    logits, ids, w = gb.route(x, flags)
    y = gb.decode(x, ids, w, flags)
    oracle_check(layer, x, logits, ids, w, y, flags=flags)


@pytest.mark.parametrize("T", [4, 8])
def test_decode_wide_model(T):
    """d = 4096 (the largest supported model width), 4- and 8-token windows,
    3-bit: routing and outputs match the oracle."""
    sh = synth.MoEShape(d=4096, E=32, F=64, Fs=64, k=4, bits=3)
    layer = synth.make_layer(sh, seed=12, device="cuda", bias="normal")
    x = synth.make_tokens(T, sh.d, seed=T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y = gb.decode(x, ids, w)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T,F", [(1, 1920), (8, 640)])
def test_decode_widest_experts_it_takes(T, F):
    """The widest experts (routed and shared) the decode kernels take for a 1-
    and an 8-token window, with the largest top-k (16): routing and outputs
    match the oracle."""
    sh = synth.MoEShape(d=256, E=20, F=F, Fs=F, k=16, bits=2)
    layer = synth.make_layer(sh, seed=15, device="cuda", bias="normal")
    x = synth.make_tokens(T, sh.d, seed=16 + T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y = gb.decode(x, ids, w)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T", [1, 8])
def test_wide_experts_take_the_prefill_step(T):
    """Experts too wide for the decode kernels' stages (ffn 4096): the decode
    call rejects the shape before enqueuing anything, and the block forward
    runs the prefill step instead, matching the oracle."""
    sh = synth.MoEShape(d=256, E=20, F=4096, Fs=4096, k=16, bits=2)
    layer = synth.make_layer(sh, seed=15, device="cuda", bias="normal")
    x = synth.make_tokens(T, sh.d, seed=16 + T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    with pytest.raises(moe.MoEError) as err:
        gb.decode(x, ids, w)
    assert err.value.status == 2          # MOE_ERR_UNSUPPORTED_SHAPE
    y = gb.block(x)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T", [5, 8])
def test_block_forward_uses_decode_up_to_eight_tokens(T):
    """moe_block_forward on a 5- and an 8-token window (decode path): routing
    and outputs match the oracle, and equal the expert step called directly."""
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=6, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(T, 2048, seed=30 + T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y = gb.block(x)
    yd = gb.decode(x, ids, w)
    torch.cuda.synchronize()
    assert torch.equal(y, yd)
    oracle_check(layer, x, logits, ids, w, y)


@pytest.mark.parametrize("T", [9, 16, 33, 64])
def test_block_forward_middle_windows(T):
    """Windows wider than the decode kernels: 9..32 tokens run as consecutive
    decode windows of up to 8 tokens (the measured crossover), wider ones on
    the prefill step.  Routing and outputs match the oracle; up to 32 tokens
    the output equals the explicit 8-token decode calls byte for byte."""
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=8, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(T, 2048, seed=60 + T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y = gb.block(x)
    torch.cuda.synchronize()
    oracle_check(layer, x, logits, ids, w, y)
    if T <= 32:
        parts = []
        for t0 in range(0, T, 8):
            xs = x[t0:t0 + 8].clone()
            _, i8, w8 = gb.route(xs)
            parts.append(gb.decode(xs, i8, w8))
        torch.cuda.synchronize()
        assert torch.equal(y, torch.cat(parts))
    assert gb.error_word() == (0, 0)


def test_l2_prefetch_of_the_next_layer_changes_no_result():
    """Naming the next layer (its router and shared expert prefetched into L2
    by this layer's expert step) is a hint: outputs equal, byte for byte, the
    same chain without it, for decode windows and sub-windows."""
    wl = synth.WORKLOADS["decode_stack"]
    layers = [synth.make_layer(wl["shape"], seed=0, layer=l, device="cuda", bias=wl["bias"],
                               slot=wl["slot"]) for l in range(3)]
    plain = [moe.make_layer_struct(l) for l in layers]
    linked = [moe.make_layer_struct(l) for l in layers]
    moe.link_l2_next(linked)
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    for T in (1, 4, 12):
        x = synth.make_tokens(T, 2048, seed=70 + T, device="cuda")
        outs = []
        for structs in (plain, linked):
            ws = moe.alloc_workspace(structs[0], T)
            h = x
            for L in structs:
                y = torch.empty_like(h)
                moe.moe_block_forward(L, h, T, y, flags, ws)
                h = y
            torch.cuda.synchronize()
            assert moe.moe_workspace_error(ws) == (0, 0)
            outs.append(h)
        assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("T", [12, 32])
def test_block_forward_middle_windows_prenorm_residual(T):
    """The middle windows with pre-norm and residual (the stack's flags) on
    the 3-bit layer: byte-equal to explicit decode calls on the 8-token pieces,
    and within tolerance of the oracle."""
    wl = synth.WORKLOADS["decode_stack"]
    layer = synth.make_layer(wl["shape"], seed=0, layer=3, device="cuda", bias=wl["bias"],
                             slot=wl["slot"])
    x = (synth.make_tokens(T, 2048, seed=90 + T, device="cuda").float() * 3).to(torch.bfloat16)
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    gb = GpuBlock(layer, T)
    y = gb.block(x, flags)
    parts, routed = [], []
    for t0 in range(0, T, 8):   # the router of each 8-token piece, as the block runs it
        xs = x[t0:t0 + 8].clone()
        r = gb.route(xs, flags)
        routed.append(r)
        parts.append(gb.decode(xs, r[1], r[2], flags))
    torch.cuda.synchronize()
    assert torch.equal(y, torch.cat(parts))
    logits, ids, w = (torch.cat([r[i] for r in routed]) for i in range(3))
    oracle_check(layer, x, logits, ids, w, y, flags=flags)
    assert gb.error_word() == (0, 0)

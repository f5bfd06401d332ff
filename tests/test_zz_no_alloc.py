"""moe_block_forward_noalloc: the decode-window block forward on the library's
static device scratch, for callers that cannot allocate device memory (a host
with no device allocator, a step loop that must not call cudaMalloc because it
synchronises the device).  Called through the C ABI, it must give exactly the
bytes of the workspace entry point (moe_block_forward: same kernels, same
inputs), on calls in a row and on calls queued back to back on one stream with
no host synchronisation between them, and reject what its 2 MiB scratch cannot
hold before enqueuing anything.

This file sorts last so that a run stopping at its first failure has already
run every other test."""
import ctypes

import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _reference(L, x, T, flags):
    """moe_block_forward on a workspace of its own."""
    ws = moe.alloc_workspace(L, T)
    y = torch.empty_like(x)
    moe.moe_block_forward(L, x, T, y, flags, ws)
    return y


def _two_calls_match(layer, T, seed, flags=0):
    L = moe.make_layer_struct(layer)
    x = synth.make_tokens(T, layer.shape.d, seed=seed, device="cuda")
    if flags & moe.F_PRENORM:
        x = (x.float() * 3).to(torch.bfloat16)
    y_ref = _reference(L, x, T, flags)
    for _ in range(2):
        y = torch.full_like(x, float("nan"))
        moe.moe_block_forward_noalloc(L, x, T, y, flags)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), "no-alloc output differs from the workspace entry point"


@pytest.mark.parametrize("T", [1, 2, 3, 4])
def test_noalloc_matches_workspace_path_full_size(T):
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=3, device="cuda", bias=wl["bias"], slot=wl["slot"])
    _two_calls_match(layer, T, seed=40 + T)


def test_noalloc_matches_workspace_path_3bit_prenorm_residual():
    wl = synth.WORKLOADS["decode_stack"]
    layer = synth.make_layer(wl["shape"], seed=0, layer=5, device="cuda", bias=wl["bias"],
                             slot=wl["slot"])
    _two_calls_match(layer, 4, seed=7, flags=moe.F_PRENORM | moe.F_RESIDUAL)


def test_noalloc_tiny_config():
    wl = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"], slot=wl["slot"])
    _two_calls_match(layer, 4, seed=0)


def test_noalloc_back_to_back_on_one_stream():
    """Three calls with different inputs and separate outputs queued on one
    stream with one synchronisation at the end: each must equal the workspace
    entry point run on its own."""
    wl = synth.WORKLOADS["decode"]
    layers = [synth.make_layer(wl["shape"], seed=20 + i, device="cuda", bias=wl["bias"],
                               slot=wl["slot"]) for i in range(2)]
    Ls = [moe.make_layer_struct(l) for l in layers]
    cases = [(0, 4, 100), (1, 1, 101), (0, 3, 102)]
    xs = [synth.make_tokens(T, wl["shape"].d, seed=s, device="cuda") for _, T, s in cases]
    refs = [_reference(Ls[li], x, T, 0) for (li, T, _), x in zip(cases, xs)]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    ys = [torch.full_like(x, float("nan")) for x in xs]
    with torch.cuda.stream(stream):
        for (li, T, _), x, y in zip(cases, xs, ys):
            moe.moe_block_forward_noalloc(Ls[li], x, T, y, 0, stream)
    stream.synchronize()
    for y, r in zip(ys, refs):
        assert torch.equal(y, r), "queued no-alloc call differs from the workspace entry point"


def _status(L, x, T, y):
    lib = moe.load()
    return lib.moe_block_forward_noalloc(ctypes.byref(L), moe._ptr(x), T, moe._ptr(y), 0, None)


def test_noalloc_rejects_long_windows_and_large_shapes():
    wl = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"], slot=wl["slot"])
    L = moe.make_layer_struct(layer)
    x = synth.make_tokens(8, 64, seed=1, device="cuda")
    y = torch.empty_like(x)
    assert _status(L, x, 5, y) == 2            # MOE_ERR_UNSUPPORTED_SHAPE: T > 4
    # a layer whose decode workspace exceeds 2 MiB (d 4096, 1024 experts, ffn 4096,
    # top-16, 3-bit): rejected by size before any weight is read
    big = moe.moe_layer(4096, 1024, 4096, 16, 3, 32, 4096, 4096, 4096, 4096, 4096, 4096, 4096, 4096)
    assert moe.moe_workspace_bytes(big, 4) > (2 << 20)
    xb = torch.zeros(4, 4096, dtype=torch.bfloat16, device="cuda")
    yb = torch.empty_like(xb)
    assert _status(big, xb, 4, yb) == 3        # MOE_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()

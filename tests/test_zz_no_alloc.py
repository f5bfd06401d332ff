"""moe_block_forward_noalloc: the decode-window block forward on the library's
static device scratch, through the C ABI.  It must agree with the workspace
entry point (moe_block_forward) on two calls in a row, and reject what its
2 MiB scratch cannot hold before enqueuing anything."""
import ctypes

import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth
from _util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _two_calls_match(layer, T, seed, flags=0):
    L = moe.make_layer_struct(layer)
    ws = moe.alloc_workspace(L, T)
    x = synth.make_tokens(T, layer.shape.d, seed=seed, device="cuda")
    if flags & moe.F_PRENORM:
        x = (x.float() * 3).to(torch.bfloat16)
    y_ref = torch.empty_like(x)
    moe.moe_block_forward(L, x, T, y_ref, flags, ws)
    for _ in range(2):
        y = torch.full_like(x, float("nan"))
        moe.moe_block_forward_noalloc(L, x, T, y, flags)
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all()
        assert_close(y.float().cpu().double().numpy(), y_ref.float().cpu().double().numpy())


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

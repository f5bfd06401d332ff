"""The bounded-wait error path, exercised without a fault.

Every pipeline wait in the kernels gives up after a limit, records
MOE_ERR_TIMEOUT in the workspace's error word and stops issuing work; the
thread block then waits for the copies and MMAs it already issued before it
ends.  The test switch moe_workspace_set_debug_withhold(site 1) makes one
producer warp of the prefill gate/up GEMM skip one plain mbarrier arrive (the
first k-step's stage, thread block 0) in calls that pass MOE_F_DEBUG, so the
MMA issuer's wait on that stage runs out.  With a host-set limit of a few
milliseconds the call must end within a fraction of the default one-second
limit, report the timeout, and leave the workspace and the GPU usable: the
next call equals a reference call on a workspace of its own, byte for byte,
and leaves the error word clear."""
import time

import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock

pytestmark = pytest.mark.gpu

LIMIT_US = 5000
T = 64          # above the decode sub-windows: the prefill expert step runs


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _setup(workload, seed):
    wl = synth.WORKLOADS[workload]
    layer = synth.make_layer(wl["shape"], seed=seed, device="cuda", bias=wl["bias"],
                             slot=wl["slot"])
    x = synth.make_tokens(T, wl["shape"].d, seed=seed + 1, device="cuda")
    ref = GpuBlock(layer, T)
    y_ref = ref.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert ref.error_word() == (0, 0)
    return layer, x, y_ref


@pytest.mark.parametrize("workload", ["decode", "decode_stack"])   # 2-bit and 3-bit GEMMs
def test_withheld_arrive_times_out_and_the_next_call_is_clean(workload):
    layer, x, y_ref = _setup(workload, seed=11)
    gb = GpuBlock(layer, T)
    gb.block(x, moe.F_DEBUG)                      # warm: modules loaded, workspace used once
    torch.cuda.synchronize()
    assert gb.error_word() == (0, 0)

    moe.moe_workspace_set_wait_limit(gb.ws, LIMIT_US)
    moe.moe_workspace_set_debug_withhold(gb.ws, moe.WITHHOLD_PREFILL_ARRIVE)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gb.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    status, code = gb.error_word()
    assert status == 7 and code & 1, (status, code)          # MOE_ERR_TIMEOUT, kErrTimeout
    assert LIMIT_US * 1e-6 <= elapsed < 0.5, elapsed          # the host-set limit, not 1 s

    # the GPU and the workspace stay usable: switch off, default limit
    moe.moe_workspace_set_debug_withhold(gb.ws, 0)
    moe.moe_workspace_set_wait_limit(gb.ws, 0)
    y = gb.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert gb.error_word() == (0, 0)


def test_switch_needs_the_debug_flag():
    """Without MOE_F_DEBUG the switch is ignored: a correct call, no error."""
    layer, x, _ = _setup("decode", seed=21)
    ref = GpuBlock(layer, T)
    y_ref = ref.block(x)
    gb = GpuBlock(layer, T)
    moe.moe_workspace_set_wait_limit(gb.ws, LIMIT_US)
    moe.moe_workspace_set_debug_withhold(gb.ws, moe.WITHHOLD_PREFILL_ARRIVE)
    y = gb.block(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("n", [4, 16, T, 1024])
def test_short_limit_alone_changes_nothing(n):
    """A 50 ms limit on calls that do not withhold anything: every path
    (decode, decode sub-windows, prefill) gives the reference bytes and no
    error."""
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=31, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(n, wl["shape"].d, seed=32, device="cuda")
    y_ref = GpuBlock(layer, n).block(x, moe.F_DEBUG)
    gb = GpuBlock(layer, n)
    moe.moe_workspace_set_wait_limit(gb.ws, 50_000)
    y = gb.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert gb.error_word() == (0, 0)


def test_workspace_init_restores_the_defaults():
    """moe_workspace_init zeroes the control block: limit back to the default,
    switch off."""
    layer, x, y_ref = _setup("decode", seed=41)
    gb = GpuBlock(layer, T)
    moe.moe_workspace_set_wait_limit(gb.ws, LIMIT_US)
    moe.moe_workspace_set_debug_withhold(gb.ws, moe.WITHHOLD_PREFILL_ARRIVE)
    moe.moe_workspace_init(gb.ws)
    y = gb.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert gb.error_word() == (0, 0)

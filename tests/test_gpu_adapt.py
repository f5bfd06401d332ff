"""Adaptive frequency-ordered slot layout (moe_adapt_layout) and the routing
counters behind it, through the C ABI.

The pages' expert cache follows the session's routing with decayed counters
and swaps hot experts in, a bounded number per round ("Strata: Run a 125B
Model on a 12 GB GPU with MoE Expert Hot Cache", section "How It Works";
"Strata illustrated", section on the expert cache).  Here the slot order plays
the cache's part.  Checked: the counters equal the router's picks exactly;
the new slot table, the swap count and the decayed counts equal a host
restatement of the rule; every expert's packed bytes arrive intact in its new
slot; block outputs are bit-identical before and after; a slot table that is
not a permutation moves nothing and is reported."""
import numpy as np
import pytest
import torch

from routed_expert_ffn_06_b200 import build, moe, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _plan(counts, slot, max_swaps):
    """Host restatement: rank by count (descending, ties to the lower expert
    index), then swap the expert of rank r into slot r while under budget."""
    E = len(counts)
    order = sorted(range(E), key=lambda e: (-float(counts[e]), e))
    slot = list(slot)
    at = [0] * E
    for e, s in enumerate(slot):
        at[s] = e
    nsw = 0
    for r in range(E):
        if nsw >= max_swaps:
            break
        e = order[r]
        s = slot[e]
        if s == r:
            continue
        other = at[r]
        slot[e], at[r] = r, e
        slot[other], at[s] = s, other
        nsw += 1
    return np.array(slot, dtype=np.int32), nsw


def _adapt(L, decay, max_swaps):
    ws = torch.zeros(moe.moe_adapt_workspace_bytes(L, max_swaps) + 256, dtype=torch.uint8,
                     device="cuda")
    ws = ws[(-ws.data_ptr()) % 256:]
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_adapt_layout(L, decay, max_swaps, done, ws)
    torch.cuda.synchronize()
    return int(done.item()), ws


def test_counters_count_every_pick():
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=41, device="cuda", bias=wl["bias"], slot=wl["slot"])
    sh = layer.shape
    counts = torch.zeros(sh.E, dtype=torch.float32, device="cuda")
    L = moe.make_layer_struct(layer, route_counts=counts)
    ws = moe.alloc_workspace(L, 64)
    expect = np.zeros(sh.E, np.int64)
    for T, seed in [(1, 1), (4, 2), (8, 3), (64, 4)]:
        x = synth.make_tokens(T, sh.d, seed=seed, device="cuda")
        ids = torch.empty(T, sh.k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, sh.k, dtype=torch.float32, device="cuda")
        moe.moe_route_topk(L, x, T, 0, None, ids, w, ws)
        torch.cuda.synchronize()
        expect += np.bincount(ids.cpu().numpy().ravel(), minlength=sh.E)
        y = torch.empty_like(x)
        moe.moe_block_forward(L, x, T, y, 0, ws)   # the same routing, counted again
        torch.cuda.synchronize()
        expect += np.bincount(ids.cpu().numpy().ravel(), minlength=sh.E)
    assert np.array_equal(counts.cpu().numpy().astype(np.int64), expect)


@pytest.mark.parametrize("max_swaps", [0, 5, 96, 1000])
def test_adapt_layout_moves_hot_experts_and_keeps_outputs(max_swaps):
    sh = synth.MoEShape(d=256, E=64, F=64, Fs=64, k=6, bits=3)
    layer = synth.make_layer(sh, seed=42, device="cuda", bias="normal", slot="random")
    g = torch.Generator().manual_seed(9)
    counts = torch.randint(0, 6, (sh.E,), generator=g).float().cuda()   # many equal counts
    L = moe.make_layer_struct(layer, route_counts=counts)
    x = synth.make_tokens(5, sh.d, seed=43, device="cuda")
    bws = moe.alloc_workspace(L, 8)
    y0 = torch.empty_like(x)
    moe.moe_block_forward(L, x, 5, y0, moe.F_DETERMINISTIC, bws)
    torch.cuda.synchronize()
    old_slot = layer.expert_slot.cpu().numpy().copy()
    old_codes = layer.codes.cpu().numpy().copy()
    old_scales = layer.scales.cpu().numpy().copy()
    c0 = counts.cpu().numpy().copy()
    want_slot, want_n = _plan(c0, old_slot, max_swaps)
    done, _ = _adapt(L, 0.5, max_swaps)
    assert done == want_n
    new_slot = layer.expert_slot.cpu().numpy()
    assert np.array_equal(new_slot, want_slot)
    assert np.array_equal(counts.cpu().numpy(), c0 * np.float32(0.5))
    codes, scales = layer.codes.cpu().numpy(), layer.scales.cpu().numpy()
    for e in range(sh.E):
        assert np.array_equal(codes[new_slot[e]], old_codes[old_slot[e]])
        assert np.array_equal(scales[new_slot[e]], old_scales[old_slot[e]])
    y1 = torch.empty_like(x)
    # the routing counters change the layer struct's view nothing: same routing
    moe.moe_block_forward(L, x, 5, y1, moe.F_DETERMINISTIC, bws)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    # the hottest experts now hold the lowest slots (as far as the budget allowed)
    if max_swaps >= sh.E:
        order = sorted(range(sh.E), key=lambda e: (-float(c0[e]), e))
        assert [int(new_slot[e]) for e in order] == list(range(sh.E))


def test_adapt_layout_rejects_a_table_that_is_not_a_permutation():
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=0, k=4, bits=2)
    layer = synth.make_layer(sh, seed=44, device="cuda", bias="normal", slot="identity")
    counts = torch.arange(sh.E, dtype=torch.float32, device="cuda")
    layer.expert_slot[3] = layer.expert_slot[4]     # a duplicate
    L = moe.make_layer_struct(layer, route_counts=counts)
    before = layer.codes.clone()
    done, ws = _adapt(L, 0.5, 8)
    assert done == 0
    assert torch.equal(layer.codes, before)
    st, code = moe.moe_workspace_error(ws)
    assert code & 2

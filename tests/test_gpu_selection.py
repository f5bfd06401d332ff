"""Device-side selection rules on exactly tied and non-finite fp32 logits.

The router keeps the top_k of 512 expert scores per token ("Strata open-source
runtime: a 12GB card runs the 125B Qwen3 model", section "the model itself");
equal fp32 logits go to the lower expert index and NaN ranks below every
number.  Random logits almost never tie, so these tests build ties on purpose:
duplicated router rows (identical dot products, bit for bit) and a zero router
whose logits are exactly the bias.  Both router paths are covered: the decode
window (T <= 8) and the long-batch tensor-core router with its top-k kernel.
Selection must equal the oracle's selection on the device's own fp32 logits,
id for id; the weights are the softmax of the selected logits."""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock, assert_close, bf16_bits, oracle_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


SHAPE = synth.MoEShape(d=256, E=64, F=64, Fs=64, k=10, bits=2)
FULL = synth.WORKLOADS["decode"]["shape"]


def _check_selection(logits, ids, w, k):
    lg = logits.cpu().numpy()
    ref = oracle.select_topk_f32(lg, k)
    got = ids.cpu().numpy()
    assert np.array_equal(got, ref), f"selection differs from the oracle:\n{got}\nvs\n{ref}"
    sel = np.take_along_axis(lg.astype(np.float64), got.astype(np.int64), axis=1)
    if np.isfinite(sel).all():
        own = np.exp(sel - sel.max(1, keepdims=True))
        own /= own.sum(1, keepdims=True)
        assert np.allclose(w.cpu().double().numpy(), own, rtol=1e-5, atol=1e-6)


def _count_ties(logits, ids, k):
    """(ties inside the selection, ties across the k / k+1 boundary) over all tokens."""
    lg = logits.cpu().numpy()
    inside = boundary = 0
    for t in range(lg.shape[0]):
        sel = lg[t, ids[t].cpu().numpy()]
        inside += len(sel) - len(np.unique(sel))
        rest = np.delete(lg[t], ids[t].cpu().numpy())
        boundary += int(np.any(rest == sel[-1]))
    return inside, boundary


def _duplicate_rows(layer, group):
    """Router rows and bias copied within groups of `group` consecutive experts."""
    E = layer.shape.E
    src = (torch.arange(E, device=layer.router_w.device) // group) * group
    layer.router_w.copy_(layer.router_w[src].clone())
    if layer.router_bias is not None:
        layer.router_bias.copy_(layer.router_bias[src].clone())
    return layer


@pytest.mark.parametrize("T", [1, 4, 8, 9, 64])
@pytest.mark.parametrize("shape", [SHAPE, FULL], ids=["small", "full"])
def test_ties_from_duplicated_router_rows(T, shape):
    """Groups of 4 identical router rows (and biases): every logit is shared by
    four experts, so both the selected set and the boundary carry ties."""
    layer = _duplicate_rows(synth.make_layer(shape, seed=11, device="cuda", bias="normal",
                                             bias_std=0.3), 4)
    x = synth.make_tokens(T, shape.d, seed=12, device="cuda")
    gb = GpuBlock(layer, max(T, 8))
    logits, ids, w = gb.route(x)
    torch.cuda.synchronize()
    inside, boundary = _count_ties(logits, ids, shape.k)
    assert inside > 0 and boundary > 0, "the test input produced no ties"
    _check_selection(logits, ids, w, shape.k)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T", [2, 8, 16])
def test_ties_from_zero_router_and_tied_bias(T):
    """A zero router makes every logit exactly its bias; the bias takes a few
    distinct values, so ties fill the selection and cross the boundary."""
    layer = synth.make_layer(SHAPE, seed=13, device="cuda", bias="normal")
    layer.router_w.zero_()
    g = torch.Generator().manual_seed(5)
    vals = torch.tensor([0.75, 0.5, 0.5, -0.25, 1.0, 0.0])
    layer.router_bias.copy_(vals[torch.randint(0, len(vals), (SHAPE.E,), generator=g)].cuda())
    x = synth.make_tokens(T, SHAPE.d, seed=14, device="cuda")
    gb = GpuBlock(layer, max(T, 8))
    logits, ids, w = gb.route(x)
    torch.cuda.synchronize()
    assert torch.equal(logits, layer.router_bias.expand(T, -1)), "zero router: logits != bias"
    inside, boundary = _count_ties(logits, ids, SHAPE.k)
    assert inside > 0 and boundary > 0
    _check_selection(logits, ids, w, SHAPE.k)
    # every token has the same logits, hence the same (lowest-index) selection
    assert (ids == ids[0:1]).all()


@pytest.mark.parametrize("T", [3, 8, 40])
def test_nan_logits_rank_last_and_flag(T):
    """NaN in the bias makes those experts' logits NaN for every token: they are
    never selected while k finite logits remain, and MOE_F_DEBUG reports the
    non-finite value through the error word (bit 4)."""
    layer = synth.make_layer(SHAPE, seed=15, device="cuda", bias="normal", bias_std=2.0)
    nan_ids = [0, 3, 17, 40, 63]
    layer.router_bias[nan_ids] = float("nan")
    # make the NaN experts the ones the bias alone would otherwise pick first
    layer.router_w[nan_ids] *= 10.0
    x = synth.make_tokens(T, SHAPE.d, seed=16, device="cuda")
    gb = GpuBlock(layer, max(T, 8))
    logits, ids, w = gb.route(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert torch.isnan(logits[:, nan_ids]).all()
    assert not np.isin(ids.cpu().numpy(), nan_ids).any(), "a NaN logit was selected"
    _check_selection(logits, ids, w, SHAPE.k)
    st, code = gb.error_word()
    assert code & 4, f"non-finite logit not flagged (error word {code:#x})"
    # the whole block with those logits: finite output, the oracle's result
    y = gb.block(x, moe.F_DEBUG)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    lg2, ids2, _ = gb.route(x)
    torch.cuda.synchronize()
    OL = oracle.OracleLayer(layer.to("cpu"))
    r = OL.block_forward(bf16_bits(x), sel_logits=lg2.cpu().numpy())
    assert np.array_equal(ids2.cpu().numpy(), r["ids"])
    assert_close(y, r["y"])
    gb.error_word()


def test_fewer_finite_logits_than_k_selects_nan_by_lowest_index():
    """With only 3 finite logits and k = 10 the rest of the selection is NaN
    experts in ascending index order (NaN below every number, ties to the
    lower index)."""
    layer = synth.make_layer(SHAPE, seed=17, device="cuda", bias="normal")
    finite = [5, 30, 50]
    mask = torch.ones(SHAPE.E, dtype=torch.bool)
    mask[finite] = False
    layer.router_bias[mask.cuda()] = float("nan")
    for T in (2, 12):
        x = synth.make_tokens(T, SHAPE.d, seed=18, device="cuda")
        gb = GpuBlock(layer, max(T, 8))
        logits, ids, _ = gb.route(x)
        torch.cuda.synchronize()
        got = ids.cpu().numpy()
        assert np.array_equal(got, oracle.select_topk_f32(logits.cpu().numpy(), SHAPE.k))
        assert (np.sort(got[:, :3], axis=1) == np.array(finite)).all()
        nan_part = [e for e in range(SHAPE.E) if e not in finite][:7]
        assert (got[:, 3:] == np.array(nan_part)).all()


@pytest.mark.parametrize("T", [1, 4, 8, 40])
def test_selection_bonus_prefers_the_given_experts(T):
    """router_pref (the pages' "router prefers experts already on the card"):
    selection ranks logit + bonus in fp32 with the usual tie and NaN rules, the
    weights are the softmax of the unbiased logits.  Decode-window router (T <=
    8) and long-batch router (T = 40); the block output matches the oracle
    selecting on the same shifted logits."""
    wl = synth.WORKLOADS["decode"]
    sh = wl["shape"]
    layer = synth.make_layer(sh, seed=31, device="cuda", bias=wl["bias"], slot=wl["slot"])
    g = torch.Generator().manual_seed(7)
    preferred = torch.randperm(sh.E, generator=g)[:96]
    pref = torch.zeros(sh.E, dtype=torch.float32)
    pref[preferred] = 0.5
    pref = pref.cuda()
    L = moe.make_layer_struct(layer, pref)
    ws = moe.alloc_workspace(L, max(T, 8))
    x = synth.make_tokens(T, sh.d, seed=32, device="cuda")
    logits = torch.empty(T, sh.E, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, sh.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, sh.k, dtype=torch.float32, device="cuda")
    moe.moe_route_topk(L, x, T, 0, logits, ids, w, ws)
    y = torch.empty_like(x)
    moe.moe_block_forward(L, x, T, y, 0, ws)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    shifted = (lg + pref.cpu().numpy()).astype(np.float32)
    got = ids.cpu().numpy()
    assert np.array_equal(got, oracle.select_topk_f32(shifted, sh.k))
    assert not np.array_equal(got, oracle.select_topk_f32(lg, sh.k)), "the bonus changed nothing"
    sel = np.take_along_axis(lg.astype(np.float64), got.astype(np.int64), axis=1)
    own = np.exp(sel - sel.max(1, keepdims=True))
    assert np.allclose(w.cpu().double().numpy(), own / own.sum(1, keepdims=True), rtol=1e-5, atol=1e-6)
    r = oracle.OracleLayer(layer.to("cpu")).block_forward(bf16_bits(x), sel_logits=shifted)
    assert np.array_equal(got, r["ids"])
    assert_close(y, r["y"])


@pytest.mark.parametrize("T", [1, 4, 16])
def test_faster_mode_top_k_minus_one_full_size(T):
    """The pages' "Faster" speed mode (5 of 6 experts, release 0.2.5) read as
    top-(k-1): the decode layer run with top_k = 9 instead of 10 matches the
    oracle on the decode and prefill paths."""
    wl = synth.WORKLOADS["decode"]
    sh = synth.MoEShape(bits=2, d=2048, E=512, F=512, Fs=512, k=9)
    layer = synth.make_layer(sh, seed=33, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(T, sh.d, seed=34, device="cuda")
    gb = GpuBlock(layer, max(T, 8))
    logits, ids, w = gb.route(x)
    y = gb.block(x)
    torch.cuda.synchronize()
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)

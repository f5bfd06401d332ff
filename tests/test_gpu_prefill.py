"""GPU parity of the prefill step (bucketing + tcgen05 grouped GEMMs) against
the fp64 oracle, through the C ABI.  Bucketing is compared bit for bit; outputs
within max rel 2e-2 / RMS rel 3e-3 (sampled rows at full size)."""
import numpy as np
import pytest
import torch

import oracle
from routed_expert_ffn_06_b200 import build, moe, synth
from _util import GpuBlock, assert_close, logit_bound, oracle_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _check_buckets(ids, off, ent, E):
    counts, offsets, entries = oracle.bucket(ids.cpu().numpy(), E)
    assert np.array_equal(off.cpu().numpy(), offsets), "bucket offsets differ"
    assert np.array_equal(ent.cpu().numpy(), entries), "bucket entries differ"


@pytest.mark.parametrize("T", [5, 16, 33, 100, 300])
def test_tiny_config_prefill(T):
    wl = synth.WORKLOADS["tiny"]
    layer = synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"], slot=wl["slot"])
    x = synth.make_tokens(T, 64, seed=T, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y, off, ent = gb.prefill(x, ids, w, want_buckets=True)
    _check_buckets(ids, off, ent, 16)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("shape", [dict(d=128, E=32, F=64, Fs=64, k=4),
                                   dict(d=256, E=64, F=128, Fs=0, k=6),
                                   dict(d=192, E=40, F=96, Fs=160, k=3),
                                   dict(d=160, E=24, F=64, Fs=32, k=2),
                                   dict(d=128, E=16, F=64, Fs=0, k=1),
                                   dict(d=96, E=6, F=64, Fs=32, k=6)])
def test_prefill_small_shapes(bits, shape):
    sh = synth.MoEShape(bits=bits, **shape)
    layer = synth.make_layer(sh, seed=11, device="cuda", bias="normal", bias_std=1.0)
    T = 700
    x = synth.make_tokens(T, sh.d, seed=3, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y, off, ent = gb.prefill(x, ids, w, want_buckets=True)
    _check_buckets(ids, off, ent, sh.E)
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("flags", [moe.F_PRENORM | moe.F_RESIDUAL, moe.F_RESIDUAL])
def test_prefill_flags(flags):
    sh = synth.MoEShape(d=256, E=32, F=128, Fs=128, k=4, bits=3)
    layer = synth.make_layer(sh, seed=5, device="cuda", bias="normal")
    x = (synth.make_tokens(160, 256, seed=4, device="cuda").float() * 5).to(torch.bfloat16)
    gb = GpuBlock(layer, 160)
    logits, ids, w = gb.route(x, flags)
    y = gb.prefill(x, ids, w, flags)
    oracle_check(layer, x, logits, ids, w, y, flags=flags)


def test_prefill_matches_decode_on_a_window():
    """The same 4 tokens through both expert paths agree."""
    wl = synth.WORKLOADS["decode"]
    layer = synth.make_layer(wl["shape"], seed=2, device="cuda", bias=wl["bias"], slot=wl["slot"])
    gb = GpuBlock(layer, 8)
    x = synth.make_tokens(4, 2048, seed=21, device="cuda")
    logits, ids, w = gb.route(x)
    yd = gb.decode(x, ids, w)
    yp = gb.prefill(x, ids, w)
    assert_close(yp.float().cpu().double().numpy(), yd.float().cpu().double().numpy(),
                 max_rel=1e-2, rms_rel=3e-3)


def test_prefill_full_size_chunk():
    """8192 tokens, d=2048, 512 experts ffn 512 + shared, top-10, 2-bit,
    router bias ~ N(0, 0.5): all routing exact, buckets exact, outputs on a
    seeded sample of 96 rows against the oracle."""
    wl = synth.WORKLOADS["prefill"]
    layer = synth.make_layer(wl["shape"], seed=0, device="cuda", bias=wl["bias"],
                             bias_std=wl["bias_std"], slot=wl["slot"])
    T = wl["T"]
    x = synth.make_tokens(T, 2048, seed=0, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y, off, ent = gb.prefill(x, ids, w, want_buckets=True)
    torch.cuda.synchronize()
    # routing on every token: oracle selection on the device's fp32 logits
    assert np.array_equal(oracle.select_topk_f32(logits.cpu().numpy(), 10), ids.cpu().numpy())
    _check_buckets(ids, off, ent, 512)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, T - 1], rng.choice(T, 93, replace=False)]))
    mr, rr = oracle_check(layer, x, logits, ids, w, y, rows=rows)
    print(f"prefill 8192: max rel {mr:.2e} rms rel {rr:.2e}")
    counts = np.diff(off.cpu().numpy())
    print("experts hit", int((counts > 0).sum()), "median", int(np.median(counts)),
          "max", int(counts.max()))
    assert gb.error_word() == (0, 0)


def test_prefill_out_of_range_ids_are_flagged_not_read():
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=64, k=4, bits=2)
    layer = synth.make_layer(sh, seed=1, device="cuda", bias="normal")
    T = 40
    x = synth.make_tokens(T, 128, seed=2, device="cuda")
    gb = GpuBlock(layer, T)
    _, ids, w = gb.route(x)
    bad = ids.clone()
    bad[3, 1] = 99
    bad[17, 0] = -5
    y = gb.prefill(x, bad, w)
    torch.cuda.synchronize()
    st, code = gb.error_word()
    assert st == 6 and code & 2
    assert torch.isfinite(y.float()).all()
    # tokens untouched by the bad entries match the clean run
    y_ok = gb.prefill(x, ids, w)
    keep = [t for t in range(T) if t not in (3, 17)]
    assert torch.equal(y[keep], y_ok[keep])


@pytest.mark.parametrize("bits", [2, 3])
def test_prefill_deterministic_mode(bits):
    """MOE_F_DETERMINISTIC: the fixed-order combine matches the oracle, repeats
    bit for bit, and agrees with the reducing combine within rounding."""
    sh = synth.MoEShape(d=256, E=48, F=128, Fs=96, k=6, bits=bits)
    layer = synth.make_layer(sh, seed=9, device="cuda", bias="normal", bias_std=1.0)
    T = 900
    x = synth.make_tokens(T, sh.d, seed=5, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    f = moe.F_DETERMINISTIC | moe.F_RESIDUAL
    y1 = gb.prefill(x, ids, w, f)
    y2 = gb.prefill(x, ids, w, f)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    oracle_check(layer, x, logits, ids, w, y1, flags=moe.F_RESIDUAL)
    y3 = gb.prefill(x, ids, w, moe.F_RESIDUAL)
    assert_close(y3.float().cpu().double().numpy(), y1.float().cpu().double().numpy(),
                 max_rel=1e-2, rms_rel=1e-3)
    assert gb.error_word() == (0, 0)


def test_prefill_deterministic_slot_layout_invariance():
    """The same experts packed into other slots: bit-identical deterministic
    prefill output."""
    sh = synth.MoEShape(d=256, E=64, F=128, Fs=128, k=6, bits=3)
    a = synth.make_layer(sh, seed=4, device="cuda", bias="normal", slot="identity")
    b = synth.make_layer(sh, seed=4, device="cuda", bias="normal", slot="random")
    assert not torch.equal(a.expert_slot, b.expert_slot)
    T = 500
    x = synth.make_tokens(T, 256, seed=8, device="cuda")
    ga, gb = GpuBlock(a, T), GpuBlock(b, T)
    _, ids, w = ga.route(x)
    ya = ga.prefill(x, ids, w, moe.F_DETERMINISTIC)
    yb = gb.prefill(x, ids, w, moe.F_DETERMINISTIC)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)


def test_prefill_full_size_deterministic_matches_sampled_oracle():
    """8192-token chunk with the fixed-order combine: sampled rows against the
    oracle and bitwise repeatability."""
    wl = synth.WORKLOADS["prefill"]
    layer = synth.make_layer(wl["shape"], seed=1, device="cuda", bias=wl["bias"],
                             bias_std=wl["bias_std"], slot=wl["slot"])
    T = wl["T"]
    x = synth.make_tokens(T, 2048, seed=1, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y1 = gb.prefill(x, ids, w, moe.F_DETERMINISTIC)
    y2 = gb.prefill(x, ids, w, moe.F_DETERMINISTIC)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rows = np.random.default_rng(1).choice(T, 48, replace=False)
    oracle_check(layer, x, logits, ids, w, y1, rows=rows)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T,d,E", [(9, 64, 16), (300, 96, 40), (1000, 2048, 512)])
def test_router_large_T_tensor_core(T, d, E):
    """Routing of a long batch (tensor-core logits, split bf16 router weights):
    logits within the fp32 bound of the oracle's fp64 logits, selection equal
    to the oracle's on the device logits, weights summing to one."""
    sh = synth.MoEShape(d=d, E=E, F=64, Fs=0, k=min(10, E // 2), bits=2)
    layer = synth.make_layer(sh, seed=T, device="cuda", bias="normal")
    x = synth.make_tokens(T, d, seed=T + 1, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    torch.cuda.synchronize()
    lg = logits.cpu().numpy()
    OL = oracle.OracleLayer(layer.to("cpu"))
    xv = x.cpu().double().numpy()
    ref = OL.router_logits(xv)
    bound = logit_bound(layer, xv)
    assert np.all(np.abs(lg - ref) <= bound), float(np.max(np.abs(lg - ref) / bound))
    assert np.array_equal(oracle.select_topk_f32(lg, sh.k), ids.cpu().numpy())
    assert np.allclose(w.sum(1).cpu().numpy(), 1.0, atol=1e-5)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("T,d,E", [(9, 64, 16), (300, 96, 40), (1000, 2048, 512)])
def test_router_presplit_weights_give_the_same_routing(T, d, E):
    """Router weights split once by moe_router_split and handed over as
    router_w_split: the same logits, ids and weights, bit for bit, as the
    split the router makes in the workspace on every call; and the split
    itself is hi = bf16(Wr), lo = bf16(Wr - hi) (torch's round to nearest
    even)."""
    sh = synth.MoEShape(d=d, E=E, F=64, Fs=0, k=min(10, E // 2), bits=2)
    layer = synth.make_layer(sh, seed=T + 7, device="cuda", bias="normal")
    x = synth.make_tokens(T, d, seed=T + 8, device="cuda")
    gb = GpuBlock(layer, T)
    ref = gb.route(x)
    split = moe.moe_router_split(gb.L)
    gb.L.router_w_split = split.data_ptr()
    got = gb.route(x)
    torch.cuda.synchronize()
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
    wr = layer.router_w.float()
    hi = wr.to(torch.bfloat16)
    lo = (wr - hi.float()).to(torch.bfloat16)
    assert torch.equal(split[0], hi.view(torch.int16))
    assert torch.equal(split[1], lo.view(torch.int16))
    assert gb.error_word() == (0, 0)


def test_prefill_hot_experts_split_into_many_chunks():
    """Every token routes to the same k experts (router bias far above the
    token logits), so k buckets hold all T tokens, several 128-token chunks
    each, and every other routed bucket is empty."""
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=64, k=4, bits=3)
    layer = synth.make_layer(sh, seed=7, device="cuda", bias="normal")
    hot = [3, 11, 20, 31]
    b = torch.zeros(sh.E, dtype=torch.float32)
    b[hot] = torch.tensor([12.0, 11.5, 11.0, 10.5])
    layer.router_bias.copy_(b.to("cuda"))
    T = 600
    x = synth.make_tokens(T, sh.d, seed=8, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    assert sorted(ids.unique().tolist()) == hot
    y, off, ent = gb.prefill(x, ids, w, want_buckets=True)
    _check_buckets(ids, off, ent, sh.E)
    counts = np.diff(off.cpu().numpy())[:sh.E]
    assert counts[hot].tolist() == [T] * 4 and int(counts.sum()) == 4 * T
    oracle_check(layer, x, logits, ids, w, y)
    assert gb.error_word() == (0, 0)


def test_prefill_zero_tokens_is_a_noop():
    sh = synth.MoEShape(d=128, E=32, F=64, Fs=64, k=4, bits=2)
    layer = synth.make_layer(sh, seed=1, device="cuda", bias="normal")
    gb = GpuBlock(layer, 16)
    x = torch.ones(1, 128, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    w = torch.zeros(1, 4, dtype=torch.float32, device="cuda")
    y = torch.full((1, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn_prefill(gb.L, x, 0, ids, w, y, None, None, 0, gb.ws)
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)
    assert gb.error_word() == (0, 0)


@pytest.mark.parametrize("d,F,T,n_rows", [(4096, 1024, 40, 8), (256, 4096, 300, 20)])
def test_prefill_widest_shapes(d, F, T, n_rows):
    """The largest supported model width (4096) or expert width (4096) with
    the largest top-k (16), 3-bit: buckets exact, and routing and outputs
    against the oracle on the first and last token and a seeded sample."""
    sh = synth.MoEShape(d=d, E=20, F=F, Fs=F, k=16, bits=3)
    layer = synth.make_layer(sh, seed=13, device="cuda", bias="normal")
    x = synth.make_tokens(T, d, seed=14, device="cuda")
    gb = GpuBlock(layer, T)
    logits, ids, w = gb.route(x)
    y, off, ent = gb.prefill(x, ids, w, want_buckets=True)
    _check_buckets(ids, off, ent, sh.E)
    rng = np.random.default_rng(T)
    rows = np.unique(np.concatenate([[0, T - 1], rng.choice(T, n_rows - 2, replace=False)]))
    oracle_check(layer, x, logits, ids, w, y, rows=rows)
    assert gb.error_word() == (0, 0)

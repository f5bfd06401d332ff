"""Pins of the fp64 oracle to things other than itself.

Each test checks one oracle function against a closed form, an invariant, a
library routine on a special case, brute force, hand-packed bytes, or a figure
printed on the pages.  A plausible slip in the oracle (dropped term, wrong
sign, transposed operand, wrong bit position, wrong tie-break) fails at least
one of them.  No GPU is needed.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from routed_expert_ffn_06_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- formats
def test_half_to_double_exhaustive():
    """Every fp16 bit pattern against numpy's binary16 conversion."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_bf16_to_double_exhaustive():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in range(65536)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_double_to_bf16_matches_library_on_float32_values():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormals
                        (rng.standard_normal(2000) * 1e38).astype(np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.double_to_bf16(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_double_to_bf16_ties_to_even():
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80       # tie -> even (1.0)
    assert oracle.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82   # tie -> even (1 + 2^-6)
    assert oracle.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81  # above tie
    assert oracle.double_to_bf16(-(1.0 + 2.0 ** -8)) == 0xBF80
    assert oracle.double_to_bf16((2 - 2.0 ** -8) * 2.0 ** 127) == 0x7F80  # overflow tie -> inf
    assert oracle.double_to_bf16((2 - 2.0 ** -7) * 2.0 ** 127) == 0x7F7F  # largest finite


# ------------------------------------------------------- packed-layout reader
def _parse_values(spec: str):
    out = []
    for part in spec.split(";"):
        part = part.strip()
        if " x" in part:
            vals, rep = part.rsplit(" x", 1)
            out += [float(v) for v in vals.split(",")] * int(rep)
        else:
            out += [float(v) for v in part.split(",")]
    return out


def _golden_groups():
    rows = []
    with open(os.path.join(GOLDEN, "dequant_groups.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, bits, hexb, scale, vals = [p.strip() for p in line.split("|")]
            rows.append((name, int(bits), bytes.fromhex(hexb), int(scale, 16),
                         _parse_values(vals)))
    return rows


@pytest.mark.parametrize("case", _golden_groups(), ids=lambda c: c[0])
@pytest.mark.parametrize("row", [0, 5, 15])
def test_dequant_hand_packed_group(case, row):
    """One hand-packed group placed at tile row `row` of a 16 x 32 matrix; the
    other rows hold a different pattern so a wrong row offset shows."""
    name, bits, gbytes, scale, expect = case
    gb = synth.group_bytes(bits)
    assert len(gbytes) == gb and len(expect) == 32
    codes = bytearray(16 * gb)
    for r in range(16):  # filler rows: every code 1 (2-bit word 0x55.., 3-bit hi plane 0)
        codes[r * 8:(r + 1) * 8] = b"\x55" * 8
    codes[row * 8:(row + 1) * 8] = gbytes[:8]
    if bits == 3:
        codes[128 + row * 4:128 + (row + 1) * 4] = gbytes[8:]
    scales = np.full(16, 0x3C00, dtype=np.uint16)
    scales[row] = scale
    W = oracle.dequant_matrix(np.frombuffer(bytes(codes), dtype=np.uint8), scales, 16, 32, bits)
    assert np.array_equal(W[row], np.array(expect))
    other = [r for r in range(16) if r != row]
    assert np.all(W[other] == 1.0 * (1 - (1 << (bits - 1))))


@pytest.mark.parametrize("bits", [2, 3])
def test_reader_inverts_independent_packer(bits):
    """Random codes and scales laid out by the packer in the synth module
    (an independent implementation of the layout, written with tensor
    reshapes) read back exactly, over several tiles and groups."""
    g = torch.Generator().manual_seed(7 + bits)
    R, K = 48, 96
    q = torch.randint(0, 1 << bits, (1, R, K // 32, 32), generator=g, dtype=torch.uint8)
    s = (torch.randn(1, R, K // 32, generator=g) * 0.1).to(torch.float16)
    codes, scales = synth.pack_codes(q, s, bits)
    W = oracle.dequant_matrix(codes[0], scales[0], R, K, bits)
    qn = q.reshape(R, K).numpy().astype(np.int64)
    sn = s[0].float().numpy().astype(np.float64).repeat(32, axis=1)
    assert np.array_equal(W, sn * (qn - (1 << (bits - 1))))
    for row, col in [(0, 0), (17, 45), (47, 95), (31, 64)]:
        assert oracle.read_code(codes[0], R, K, bits, row, col) == qn[row, col]


@pytest.mark.parametrize("bits", [2, 3])
def test_pack_of_dequant_round_trips_bytes(bits):
    """pack(dequant(block)) == block for representable blocks (every group
    holds a code 0, so its largest-magnitude value fixes the scale)."""
    g = torch.Generator().manual_seed(11 + bits)
    R, K = 32, 64
    q = torch.randint(0, 1 << bits, (1, R, K // 32, 32), generator=g, dtype=torch.uint8)
    q[..., 5] = 0
    s = (torch.rand(1, R, K // 32, generator=g) * 0.2 + 0.01).to(torch.float16)
    codes, scales = synth.pack_codes(q, s, bits)
    W = oracle.dequant_matrix(codes[0], scales[0], R, K, bits)
    c2, s2 = synth.pack_matrices(torch.from_numpy(W).unsqueeze(0), bits)
    assert torch.equal(c2, codes) and torch.equal(s2.view(torch.int16), scales.view(torch.int16))


# ------------------------------------------------------------------- router
def _tiny_layer(**kw):
    sh = kw.pop("shape", synth.MoEShape(d=64, E=16, F=32, Fs=32, k=2, bits=2))
    return synth.make_layer(sh, seed=kw.pop("seed", 0), **kw)


def test_router_one_hot_and_zero_inputs():
    L = _tiny_layer(bias="normal", bias_std=0.5)
    OL = oracle.OracleLayer(L)
    Wr = L.router_w.double().numpy()
    b = L.router_bias.double().numpy()
    x = np.zeros((3, 64))
    x[0, 5] = 1.0
    x[1, 63] = -2.0
    lg = OL.router_logits(x)
    assert np.array_equal(lg[0], Wr[:, 5] + b)
    assert np.array_equal(lg[1], -2.0 * Wr[:, 63] + b)
    assert np.array_equal(lg[2], b)


# ---------------------------------------------------------------- selection
def test_topk_matches_library_sort():
    rng = np.random.default_rng(3)
    L = rng.standard_normal((64, 512)).astype(np.float32)
    ids = oracle.select_topk_f32(L, 10)
    for t in range(64):
        order = sorted(range(512), key=lambda e: (-float(L[t, e]), e))
        assert list(ids[t]) == order[:10]


def test_topk_ties_lower_index_and_nan_last():
    L = np.array([[1.0, 3.0, 3.0, 2.0, 3.0, -1.0],
                  [np.nan, 0.0, np.nan, -np.inf, 0.0, -0.0],
                  [np.nan, np.nan, np.nan, np.nan, np.nan, np.nan]], dtype=np.float32)
    ids = oracle.select_topk_f32(L, 4)
    assert list(ids[0]) == [1, 2, 4, 3]
    assert list(ids[1]) == [1, 4, 5, 3]        # -0.0 == 0.0: index order; -inf before NaN
    assert list(ids[2]) == [0, 1, 2, 3]


def test_topk_permutation_equivariance():
    rng = np.random.default_rng(4)
    L = rng.standard_normal((8, 512)).astype(np.float32)
    perm = rng.permutation(512)
    ids = oracle.select_topk_f32(L, 10)
    ids_p = oracle.select_topk_f32(L[:, perm], 10)   # expert perm[e'] is now called e'
    assert np.array_equal(perm[ids_p], ids)


def test_renorm_weights_closed_forms():
    w = oracle.renorm_weights(np.array([[0.0, math.log(3.0), -50.0]]), np.array([[1, 0]]))
    assert np.allclose(w, [[0.75, 0.25]], rtol=0, atol=1e-15)
    w = oracle.renorm_weights(np.array([[2.0, 2.0, 2.0, 2.0]]), np.array([[3, 1, 0, 2]]))
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)
    rng = np.random.default_rng(5)
    L = rng.standard_normal((16, 512)) * 3
    ids = oracle.select_topk_f64(L, 10)
    w = oracle.renorm_weights(L, ids)
    assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)           # descending logits -> descending weights
    ref = scipy.special.softmax(np.take_along_axis(L, ids, 1), axis=1)
    assert np.allclose(w, ref, rtol=1e-13, atol=0)


def test_renorm_with_all_experts_is_full_softmax():
    rng = np.random.default_rng(6)
    L = rng.standard_normal((4, 16)) * 2
    ids = oracle.select_topk_f64(L, 16)
    w = oracle.renorm_weights(L, ids)
    full = scipy.special.softmax(L, axis=1)
    assert np.allclose(w, np.take_along_axis(full, ids, 1), rtol=1e-13, atol=0)


# ---------------------------------------------------------------- bucketing
def test_bucket_hand_example():
    ids = np.array([[2, 0], [0, 1], [2, 1]], dtype=np.int32)   # T=3, k=2, E=4
    counts, offsets, entries = oracle.bucket(ids, 4)
    assert list(counts) == [2, 2, 2, 0]
    assert list(offsets) == [0, 2, 4, 6, 6]
    # expert 0: (t0,j1)=1, (t1,j0)=2; expert 1: (t1,j1)=3, (t2,j1)=5; expert 2: (t0,j0)=0, (t2,j0)=4
    assert list(entries) == [1, 2, 3, 5, 0, 4]


def test_bucket_invariants_random():
    rng = np.random.default_rng(8)
    T, k, E = 300, 10, 64
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, entries = oracle.bucket(ids, E)
    assert counts.sum() == T * k and offsets[-1] == T * k
    assert sorted(entries.tolist()) == list(range(T * k))          # each (t, j) exactly once
    for e in range(E):
        seg = entries[offsets[e]:offsets[e + 1]]
        assert np.all(ids.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg // k) > 0)                        # tokens strictly ascending
    assert np.array_equal(counts, np.bincount(ids.reshape(-1), minlength=E))


# --------------------------------------------------------------------- FFN
SILU_1 = 0.7310585786300049      # 1 / (1 + e^-1), textbook value
SILU_M1 = -0.2689414213699951    # -1 / (1 + e)


def _hand_expert(d, F, bits, entries):
    """Pack an expert whose codes are all 2^(b-1) (weight 0) except the listed
    (matrix, row, col, code, scale) entries; every scale is `scale` there, 1.0
    elsewhere."""
    off = 1 << (bits - 1)
    shapes = [(F, d), (F, d), (d, F)]
    cs, ss = [], []
    for mi, (R, K) in enumerate(shapes):
        q = torch.full((1, R, K // 32, 32), off, dtype=torch.uint8)
        s = torch.ones(1, R, K // 32, dtype=torch.float16)
        for (m, r, c, code, scale) in entries:
            if m == mi:
                q[0, r, c // 32, c % 32] = code
                s[0, r, c // 32] = scale
        c_, s_ = synth.pack_codes(q, s, bits)
        cs.append(c_[0])
        ss.append(s_[0])
    return torch.cat(cs), torch.cat(ss)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("sign", [1, -1])
def test_expert_ffn_one_hot_closed_form(bits, sign):
    d, F = 64, 32
    off = 1 << (bits - 1)
    f0, i0, i1 = 7, 41, 18
    # Wg[f0,i0] = 0.5, Wu[f0,i0] = 0.25, Wd[i1,f0] = 2.0
    codes, scales = _hand_expert(d, F, bits, [(0, f0, i0, off + 1, 0.5), (1, f0, i0, off + 1, 0.25),
                                              (2, i1, f0, off + 1, 2.0)])
    x = np.zeros(d)
    x[i0] = 2.0 * sign                    # g = +-1, u = +-0.5
    y = oracle.expert_ffn(codes, scales, d, F, bits, x)
    expect = np.zeros(d)
    expect[i1] = 2.0 * (SILU_1 if sign > 0 else SILU_M1) * 0.5 * sign
    assert np.allclose(y, expect, rtol=1e-15, atol=0)


def test_silu_values():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - SILU_1) < 1e-16
    assert abs(oracle.silu(-1.0) - SILU_M1) < 1e-16
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12


# -------------------------------------------------------------------- block
def _x(T, d, seed=0):
    return synth.make_tokens(T, d, seed=seed)


def test_block_zero_input_gives_zero():
    L = _tiny_layer()
    r = oracle.OracleLayer(L).block_forward(torch.zeros(4, 64, dtype=torch.bfloat16))
    assert np.all(r["y"] == 0.0)
    assert np.all(r["ids"] == [0, 1])          # all logits 0: lowest indices
    assert np.allclose(r["w"], 0.5)


def _zero_down(L):
    """Repack every routed expert with Wd = 0 (codes 2^(b-1))."""
    sh = L.shape
    off = 1 << (sh.bits - 1)
    q = torch.full((1, sh.d, sh.F // 32, 32), off, dtype=torch.uint8)
    c, s = synth.pack_codes(q, torch.ones(1, sh.d, sh.F // 32, dtype=torch.float16), sh.bits)
    nd = oracle.codes_bytes(sh.d, sh.F, sh.bits)
    L.codes[:, -nd:] = c[0]
    L.scales[:, -(sh.d * sh.F // 32):] = s[0]
    return L


def test_block_routed_zero_gives_shared_only():
    L = _zero_down(_tiny_layer())
    x = _x(4, 64)
    OL = oracle.OracleLayer(L)
    r = OL.block_forward(x)
    xd = x.double().numpy()
    for t in range(4):
        s = oracle.expert_ffn(L.shared_codes, L.shared_scales, 64, 32, 2, xd[t])
        assert np.array_equal(r["y"][t], s)


def _brute_force(L, x, sel_logits=None):
    """Dense evaluation of every expert, then a combine with weights that are
    zero off the selected set (selection by a library sort)."""
    sh = L.shape
    OL = oracle.OracleLayer(L)
    xd = x.double().numpy()
    lg = OL.router_logits(xd)
    slot = L.expert_slot.numpy()
    cb, ns = sh.codes_bytes, sh.n_scales
    ys = []
    for t in range(x.shape[0]):
        Y = np.stack([oracle.expert_ffn(L.codes[slot[e]], L.scales[slot[e]], sh.d, sh.F, sh.bits,
                                        xd[t]) for e in range(sh.E)])
        sl = (lg[t].astype(np.float32) if sel_logits is None else sel_logits[t])
        order = np.lexsort((np.arange(sh.E), -sl.astype(np.float64)))[:sh.k]
        wfull = np.zeros(sh.E)
        wfull[order] = scipy.special.softmax(lg[t][order])
        y = wfull @ Y
        if sh.Fs:
            y = y + oracle.expert_ffn(L.shared_codes, L.shared_scales, sh.d, sh.Fs, sh.bits, xd[t])
        ys.append(y)
    return np.stack(ys)


@pytest.mark.parametrize("bits", [2, 3])
def test_block_equals_brute_force_enumeration(bits):
    sh = synth.MoEShape(d=64, E=16, F=32, Fs=32, k=2, bits=bits)
    L = synth.make_layer(sh, seed=0, bias="normal", bias_std=0.5)
    x = _x(4, 64)
    r = oracle.OracleLayer(L).block_forward(x)
    assert np.allclose(r["y"], _brute_force(L, x), rtol=1e-12, atol=1e-15)


def test_block_all_experts_selected_is_dense_softmax_mixture():
    sh = synth.MoEShape(d=64, E=16, F=32, Fs=0, k=16, bits=2)
    L = synth.make_layer(sh, seed=2, bias="normal")
    x = _x(3, 64, seed=2)
    r = oracle.OracleLayer(L).block_forward(x)
    OL = oracle.OracleLayer(L)
    xd = x.double().numpy()
    p = scipy.special.softmax(OL.router_logits(xd), axis=1)
    slot = L.expert_slot.numpy()
    for t in range(3):
        Y = np.stack([oracle.expert_ffn(L.codes[slot[e]], L.scales[slot[e]], 64, 32, 2, xd[t])
                      for e in range(16)])
        assert np.allclose(r["y"][t], p[t] @ Y, rtol=1e-12, atol=1e-15)


def test_block_identical_experts_is_routing_independent():
    """Every routed expert the same: y = S(x) + E(x) whatever is selected,
    because the selected weights sum to 1."""
    L = _tiny_layer(bias="normal", bias_std=3.0)
    L.codes[:] = L.codes[0]
    L.scales[:] = L.scales[0]
    x = _x(4, 64, seed=5)
    r = oracle.OracleLayer(L).block_forward(x)
    xd = x.double().numpy()
    for t in range(4):
        e = oracle.expert_ffn(L.codes[0], L.scales[0], 64, 32, 2, xd[t])
        s = oracle.expert_ffn(L.shared_codes, L.shared_scales, 64, 32, 2, xd[t])
        assert np.allclose(r["y"][t], s + e, rtol=1e-13, atol=1e-15)


def test_block_zero_weight_expert_contributes_nothing():
    """Forcing a selected expert's output to zero (its Wd = 0) removes exactly
    its weighted term."""
    L = _tiny_layer(bias="normal")
    x = _x(4, 64, seed=9)
    OL = oracle.OracleLayer(L)
    r = OL.block_forward(x)
    e0 = int(r["ids"][0, 0])
    L2 = _tiny_layer(bias="normal")
    slot = int(L2.expert_slot[e0])
    sh = L2.shape
    off = 1 << (sh.bits - 1)
    nd = oracle.codes_bytes(sh.d, sh.F, sh.bits)
    q = torch.full((1, sh.d, sh.F // 32, 32), off, dtype=torch.uint8)
    c, s = synth.pack_codes(q, torch.ones(1, sh.d, sh.F // 32, dtype=torch.float16), sh.bits)
    L2.codes[slot, -nd:] = c[0]
    r2 = oracle.OracleLayer(L2).block_forward(x)
    ye = oracle.expert_ffn(L.codes[slot], L.scales[slot], 64, 32, 2, x.double().numpy()[0])
    assert np.allclose(r["y"][0] - r2["y"][0], r["w"][0, 0] * ye, rtol=1e-12, atol=1e-15)


def test_block_slot_layout_invariance():
    """Packing the same experts into other slots changes nothing."""
    a = _tiny_layer(slot="identity")
    b = _tiny_layer(slot="random")
    assert not torch.equal(a.expert_slot, b.expert_slot)
    x = _x(4, 64, seed=3)
    ya = oracle.OracleLayer(a).block_forward(x)["y"]
    yb = oracle.OracleLayer(b).block_forward(x)["y"]
    assert np.array_equal(ya, yb)


def test_block_selects_on_given_fp32_logits():
    """In parity mode the selection follows the supplied fp32 logits."""
    L = _tiny_layer()
    x = _x(4, 64, seed=4)
    forced = np.zeros((4, 16), dtype=np.float32)
    forced[:, 3] = 1.0
    forced[:, 9] = 1.0          # tie 3 vs 9 -> 3 first
    r = oracle.OracleLayer(L).block_forward(x, sel_logits=forced)
    assert np.all(r["ids"] == [3, 9])
    assert np.allclose(r["y"], _brute_force(L, x, sel_logits=forced), rtol=1e-12, atol=1e-15)


def test_prenorm_and_residual():
    L = _tiny_layer(bias="normal")
    OL = oracle.OracleLayer(L)
    c = torch.full((2, 64), 3.0).to(torch.bfloat16)       # constant rows: RMSNorm -> 1
    ones = torch.ones(2, 64, dtype=torch.bfloat16)
    y_pn = OL.block_forward(c, flags=oracle.PRENORM)["y"]
    y_1 = OL.block_forward(ones)["y"]
    assert np.array_equal(y_pn, y_1)
    xn = oracle.rmsnorm_bf16(c.view(torch.int16).numpy().view(np.uint16))
    assert np.all(xn == 0x3F80)
    x = _x(3, 64, seed=6)
    y0 = OL.block_forward(x)["y"]
    y1 = OL.block_forward(x, flags=oracle.RESIDUAL)["y"]
    assert np.allclose(y1 - y0, x.double().numpy(), rtol=0, atol=1e-12)


def test_rmsnorm_against_library():
    x = _x(5, 256, seed=10)
    xn = oracle.rmsnorm_bf16(x.view(torch.int16).numpy().view(np.uint16))
    ref = torch.nn.functional.rms_norm(x.double(), (256,), eps=1e-6)
    got = torch.from_numpy(xn.view(np.int16)).view(torch.bfloat16).double()
    # same value up to the final bf16 rounding (one bf16 ulp)
    assert torch.all((got - ref).abs() <= ref.abs() * 2.0 ** -8 + 1e-30)


# ------------------------------------------------------------- page figures
def _figures():
    out = {}
    with open(os.path.join(GOLDEN, "pages_figures.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, val, _src = [p.strip() for p in line.split("|")]
                out[name] = float(val)
    return out


def test_expert_byte_counts_match_pages():
    fig = _figures()
    assert fig["experts_per_layer"] * fig["layers"] == fig["experts_total"]
    d, F = 2048, 512
    per3 = oracle.codes_bytes(F, d, 3) * 2 + oracle.codes_bytes(d, F, 3) + 3 * F * d // 32 * 2
    per2 = oracle.codes_bytes(F, d, 2) * 2 + oracle.codes_bytes(d, F, 2) + 3 * F * d // 32 * 2
    assert per3 == 1376256 and per2 == 983040
    assert per3 == synth.codes_bytes_per_expert(d, F, 3) + synth.scales_per_expert(d, F) * 2
    # 48 layers x top-10 experts at the 3-bit layout: within 0.5% of the
    # CPU pool's 663.6 MB per token
    per_token = fig["layers"] * fig["routed_per_token"] * per3
    assert abs(per_token / fig["cpu_pool_bytes_per_token"] - 1) < 0.005
    # all experts of the model at ~2.0 bits/weight is about the "Q2_0 ~34 GB" figure
    q2 = fig["experts_total"] * per2
    assert abs(q2 / fig["q2_0_expert_bytes_total"] - 1) < 0.35


def test_selection_bonus_reading_against_brute_force():
    """Resident-preferring routing is read as top-k of (logit + bonus) in fp32,
    weights from the logits alone.  With a bonus far above the logit spread on
    a preferred set S (|S| >= k), the selection must be the top-k of S by
    logit (ties to the lower index), and the renormalised weights the softmax
    of those logits: checked against a brute-force sort on random rows."""
    rng = np.random.default_rng(5)
    E, k = 64, 10
    for trial in range(20):
        L = rng.standard_normal((3, E)).astype(np.float32)
        S = np.sort(rng.choice(E, size=rng.integers(k, 30), replace=False))
        bonus = np.zeros(E, np.float32)
        bonus[S] = 1000.0
        ids = oracle.select_topk_f32((L + bonus).astype(np.float32), k)
        for t in range(3):
            order = sorted(S, key=lambda e: (-float(L[t, e]), e))[:k]
            assert list(ids[t]) == order
        w = oracle.renorm_weights(L.astype(np.float64), ids)
        sel = np.take_along_axis(L.astype(np.float64), ids.astype(np.int64), axis=1)
        ref = np.exp(sel - sel.max(1, keepdims=True))
        assert np.allclose(w, ref / ref.sum(1, keepdims=True), rtol=1e-12)

"""Seeded synthetic inputs for the routed sparse-MoE block.

This module is the one place both sides of the parity check take their inputs
from: the CUDA path (through :mod:`routed_expert_ffn_06_b200.moe`) and the fp64
oracle under ``oracle/``.  It holds none of the block's arithmetic (no router,
no selection, no dequantisation, no FFN).  It only draws random tensors and
writes expert weights in the packed low-bit layout, the way an offline
quantiser would hand them to the engine.

Packed layout (the format every reader of ``codes``/``scales`` follows)
-----------------------------------------------------------------------
One expert is three matrices, each stored as ``R x K`` with ``K`` the
contracted dimension:  ``Wg`` (F x d), ``Wu`` (F x d), ``Wd`` (d x F), in that
order.  Each row is split into groups of 32 consecutive ``K`` elements; a group
holds 32 unsigned codes ``q`` of ``b`` bits and one fp16 scale ``s``; the
weight it encodes is ``s * (q - 2**(b-1))``.

* Rows are taken in tiles of 16.  Inside a tile the group words are ordered
  group-major: word ``(c, r)`` (group ``c``, row ``r`` of the tile) sits at
  ``(c*16 + r) * 8`` bytes from the tile start.
* 2-bit: one 8-byte little-endian word per group.  Code ``j`` (column
  ``32c + j``) is written as ``j = 8m + 2t + h`` (m in 0..3, t in 0..3, h in
  0..1) and occupies bits ``32h + 8t + 2m`` .. ``+1``.
* 3-bit: the low two bits of every code form the 8-byte word above; the high
  bit of code ``j`` sits at bit ``16h + 4t + m`` of a 4-byte word.  A tile
  stores all its 8-byte words first (``nG*16*8`` bytes) and then all its
  4-byte words, ordered the same way (``(c*16 + r) * 4``).
* Scales: fp16, one per (row, group), tile-interleaved the same way: the
  scale of group ``c`` of tile row ``r`` is element ``c*16 + r`` of the tile's
  ``16*nG`` scales.
* An expert's bytes are ``Wg`` tiles, then ``Wu`` tiles, then ``Wd`` tiles;
  its scales follow the same order.  Expert ``e`` lives in slot
  ``expert_slot[e]``: ``codes[slot]`` / ``scales[slot]``.

Quantiser (test-data preparation only): per group, ``m`` is the signed element
of largest magnitude, ``s = fp16(m / -2**(b-1))`` and
``q = clamp(round_half_even(w / s) + 2**(b-1), 0, 2**b - 1)``; an all-zero
group gets ``s = 0`` and ``q = 2**(b-1)``.  The GPU and the oracle consume the
same bytes, so the quantiser's own rounding never enters a parity check.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass, field

import torch

GROUP = 32
TILE_ROWS = 16


def group_bytes(bits: int) -> int:
    """Packed bytes of one group of 32 codes (scale not included)."""
    if bits == 2:
        return 8
    if bits == 3:
        return 12
    raise ValueError(f"bits must be 2 or 3, got {bits}")


def codes_bytes_per_expert(d: int, F: int, bits: int) -> int:
    return 3 * F * d // GROUP * group_bytes(bits)


def scales_per_expert(d: int, F: int) -> int:
    return 3 * F * d // GROUP


# --------------------------------------------------------------------------
# seeds
# --------------------------------------------------------------------------
def _splitmix64(z: int) -> int:
    z = (z + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    return z ^ (z >> 31)


def derive_seed(*parts) -> int:
    """Stable 63-bit seed from (master seed, tags...): SplitMix64 chained over
    the parts (strings hashed with BLAKE2b so the result does not depend on
    Python's per-process string hashing)."""
    h = 0x243F6A8885A308D3
    for p in parts:
        if isinstance(p, str):
            v = int.from_bytes(hashlib.blake2b(p.encode(), digest_size=8).digest(), "little")
        else:
            v = int(p) & 0xFFFFFFFFFFFFFFFF
        h = _splitmix64(h ^ v)
    return h & 0x7FFFFFFFFFFFFFFF


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(*parts))
    return g


# --------------------------------------------------------------------------
# packer
# --------------------------------------------------------------------------
def quantize_groups(W: torch.Tensor, bits: int):
    """Group-of-32 symmetric quantiser.  W: [..., R, K] float.  Returns
    (q uint8 [..., R, K/32, 32], s fp16 [..., R, K/32])."""
    off = 1 << (bits - 1)
    qmax = (1 << bits) - 1
    *lead, R, K = W.shape
    if K % GROUP:
        raise ValueError("K must be a multiple of 32")
    Wg = W.reshape(*lead, R, K // GROUP, GROUP).float()
    idx = Wg.abs().argmax(dim=-1, keepdim=True)
    m = torch.gather(Wg, -1, idx)
    s16 = (m / float(-off)).to(torch.float16)
    s = s16.float()
    zero = s == 0
    q = torch.round(Wg / torch.where(zero, torch.ones_like(s), s)) + off
    q = q.clamp(0, qmax)
    q = torch.where(zero.expand_as(q), torch.full_like(q, off), q).to(torch.uint8)
    return q, s16.squeeze(-1)


def pack_codes(q: torch.Tensor, s16: torch.Tensor, bits: int):
    """Lay quantised groups out in the packed format.

    q: uint8 [B, R, nG, 32] codes, s16: fp16 [B, R, nG].  Returns
    (codes uint8 [B, R*nG*group_bytes], scales fp16 [B, R*nG])."""
    B, R, nG, G = q.shape
    assert G == GROUP
    if R % TILE_ROWS:
        raise ValueError("row count must be a multiple of 16")
    dev = q.device
    qi = q.to(torch.int32)
    # code j = 8m + 2t + h  ->  view [.., m, t, h]
    lo = (qi & 3).reshape(B, R, nG, 4, 4, 2)
    sh = torch.tensor([0, 2, 4, 6], device=dev, dtype=torch.int32).view(4, 1, 1)
    byte_th = (lo << sh).sum(dim=3)                       # [B,R,nG,t,h]
    low = byte_th.permute(0, 1, 2, 4, 3).reshape(B, R, nG, 8)   # byte = 4h + t
    tiles = R // TILE_ROWS
    low = low.reshape(B, tiles, TILE_ROWS, nG, 8).permute(0, 1, 3, 2, 4)
    low = low.reshape(B, tiles, nG * TILE_ROWS * 8)
    if bits == 2:
        tile_bytes = low
    elif bits == 3:
        hb = ((qi >> 2) & 1).reshape(B, R, nG, 4, 2, 2, 2)   # [m, t_hi, t_lo, h]
        m_idx = torch.arange(4, device=dev, dtype=torch.int32).view(4, 1, 1, 1)
        tlo = torch.arange(2, device=dev, dtype=torch.int32).view(1, 1, 2, 1)
        byte = (hb << (4 * tlo + m_idx)).sum(dim=(3, 5))  # [B,R,nG,t_hi,h]
        hi = byte.permute(0, 1, 2, 4, 3).reshape(B, R, nG, 4)   # byte = 2h + t_hi
        hi = hi.reshape(B, tiles, TILE_ROWS, nG, 4).permute(0, 1, 3, 2, 4)
        hi = hi.reshape(B, tiles, nG * TILE_ROWS * 4)
        tile_bytes = torch.cat([low, hi], dim=-1)
    else:
        raise ValueError("bits must be 2 or 3")
    codes = tile_bytes.reshape(B, -1).to(torch.uint8)
    scales = s16.reshape(B, tiles, TILE_ROWS, nG).permute(0, 1, 3, 2).reshape(B, -1)
    return codes.contiguous(), scales.contiguous()


def pack_matrices(W: torch.Tensor, bits: int):
    """Quantise and pack a batch of matrices W [B, R, K]."""
    q, s16 = quantize_groups(W, bits)
    return pack_codes(q, s16, bits)


# --------------------------------------------------------------------------
# layers and tokens
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class MoEShape:
    d: int
    E: int
    F: int
    Fs: int
    k: int
    bits: int

    @property
    def codes_bytes(self) -> int:
        return codes_bytes_per_expert(self.d, self.F, self.bits)

    @property
    def n_scales(self) -> int:
        return scales_per_expert(self.d, self.F)

    @property
    def shared_codes_bytes(self) -> int:
        return codes_bytes_per_expert(self.d, self.Fs, self.bits) if self.Fs else 0

    @property
    def shared_n_scales(self) -> int:
        return scales_per_expert(self.d, self.Fs) if self.Fs else 0


@dataclass
class Layer:
    """One routed-MoE layer's tensors (all on one device)."""
    shape: MoEShape
    router_w: torch.Tensor          # fp32 [E, d]
    router_bias: torch.Tensor | None  # fp32 [E]
    expert_slot: torch.Tensor       # int32 [E]
    codes: torch.Tensor             # uint8 [E, codes_bytes]  (indexed by slot)
    scales: torch.Tensor            # fp16  [E, n_scales]     (indexed by slot)
    shared_codes: torch.Tensor | None
    shared_scales: torch.Tensor | None
    rank: torch.Tensor | None = None  # int64 [E] popularity rank (1 = hottest)
    meta: dict = field(default_factory=dict)

    def to(self, device) -> "Layer":
        mv = lambda t: None if t is None else t.to(device)
        return Layer(self.shape, mv(self.router_w), mv(self.router_bias), mv(self.expert_slot),
                     mv(self.codes), mv(self.scales), mv(self.shared_codes), mv(self.shared_scales),
                     mv(self.rank), dict(self.meta))


def zipf_profile(E: int, s: float, c: float, gen: torch.Generator):
    """Popularity ranks and router bias for Zipf(s) expert popularity.

    rank[e] is a seeded permutation of 1..E; bias[e] = c * ln p_rank[e] with
    p_r = r**-s / sum_r' r'**-s."""
    perm = torch.randperm(E, generator=gen)
    rank = perm.to(torch.int64) + 1
    r = torch.arange(1, E + 1, dtype=torch.float64)
    logZ = math.log(float((r ** -s).sum()))
    bias = c * (-s * torch.log(rank.to(torch.float64)) - logZ)
    return rank, bias.to(torch.float32)


def make_expert_weights(shape: MoEShape, F: int, seed: int, tag, layer: int, e: int, device,
                        weight_std: float):
    """Float weights of one expert: (Wg [F,d], Wu [F,d], Wd [d,F]) ~ N(0, std)."""
    g = _gen(device, seed, tag, "expert", layer, e)
    d = shape.d
    Wg = torch.randn(F, d, generator=g, device=device) * weight_std
    Wu = torch.randn(F, d, generator=g, device=device) * weight_std
    Wd = torch.randn(d, F, generator=g, device=device) * weight_std
    return Wg, Wu, Wd


def _pack_experts(shape, F, seed, tag, layer, ids, device, weight_std, bits):
    Ws = [make_expert_weights(shape, F, seed, tag, layer, e, device, weight_std) for e in ids]
    parts_c, parts_s = [], []
    for mi in range(3):
        c, s = pack_matrices(torch.stack([w[mi] for w in Ws]), bits)
        parts_c.append(c)
        parts_s.append(s)
    return torch.cat(parts_c, dim=1), torch.cat(parts_s, dim=1)


def make_layer(shape: MoEShape, seed: int = 0, layer: int = 0, device="cpu", *, tag: str = "moe",
               weight_std: float = 0.05, router_std: float = 0.02, bias: str = "none",
               bias_std: float = 0.5, zipf_s: float = 1.1, zipf_c: float = 0.46,
               slot: str = "random", chunk: int = 64) -> Layer:
    """Generate one layer.

    bias: "none" | "zipf" (popularity ~ Zipf(zipf_s) through c*ln p_rank) |
          "normal" (N(0, bias_std)).
    slot: "identity" | "random" (seeded permutation) | "profile" (slots in
          descending popularity: slot = rank - 1; needs bias="zipf")."""
    device = torch.device(device)
    d, E = shape.d, shape.E
    g = _gen(device, seed, tag, "router", layer)
    router_w = (torch.randn(E, d, generator=g, device=device) * router_std).float()
    gc = _gen("cpu", seed, tag, "profile", layer)
    rank = None
    if bias == "none":
        router_bias = None
    elif bias == "zipf":
        rank, b = zipf_profile(E, zipf_s, zipf_c, gc)
        router_bias = b.to(device)
    elif bias == "normal":
        router_bias = (torch.randn(E, generator=gc) * bias_std).float().to(device)
    else:
        raise ValueError(bias)
    gs = _gen("cpu", seed, tag, "slots", layer)
    if slot == "identity":
        expert_slot = torch.arange(E, dtype=torch.int32)
    elif slot == "random":
        expert_slot = torch.randperm(E, generator=gs).to(torch.int32)
    elif slot == "profile":
        if rank is None:
            raise ValueError("slot='profile' needs a popularity profile (bias='zipf')")
        expert_slot = (rank - 1).to(torch.int32)
    else:
        raise ValueError(slot)
    expert_slot = expert_slot.to(device)

    codes = torch.empty(E, shape.codes_bytes, dtype=torch.uint8, device=device)
    scales = torch.empty(E, shape.n_scales, dtype=torch.float16, device=device)
    slots_cpu = expert_slot.cpu()
    for e0 in range(0, E, chunk):
        ids = list(range(e0, min(E, e0 + chunk)))
        c, s = _pack_experts(shape, shape.F, seed, tag, layer, ids, device, weight_std, shape.bits)
        dst = slots_cpu[e0:e0 + len(ids)].to(device=device, dtype=torch.int64)
        codes.index_copy_(0, dst, c)
        scales.index_copy_(0, dst, s)
    shared_codes = shared_scales = None
    if shape.Fs:
        c, s = _pack_experts(shape, shape.Fs, seed, tag + "/shared", layer, [0], device,
                             weight_std, shape.bits)
        shared_codes, shared_scales = c[0].contiguous(), s[0].contiguous()
    return Layer(shape, router_w.contiguous(), router_bias, expert_slot.contiguous(), codes,
                 scales, shared_codes, shared_scales, rank,
                 dict(seed=seed, layer=layer, tag=tag, bias=bias, slot=slot))


def make_tokens(T: int, d: int, seed: int = 0, step: int = 0, device="cpu", *, tag: str = "moe",
                std: float = 1.0) -> torch.Tensor:
    """Activations x ~ N(0, std) rounded to bf16, [T, d]."""
    g = _gen(device, seed, tag, "tokens", step)
    return (torch.randn(T, d, generator=g, device=device) * std).to(torch.bfloat16)


def permute_profile(layer: Layer, seed: int, epoch: int) -> torch.Tensor:
    """Routing drift: the Zipf bias re-assigned by a fresh seeded permutation
    of the experts (the packed slot layout is left as it was)."""
    if layer.router_bias is None:
        raise ValueError("layer has no bias to permute")
    g = _gen("cpu", seed, layer.meta.get("tag", "moe"), "drift", layer.meta.get("layer", 0), epoch)
    perm = torch.randperm(layer.shape.E, generator=g).to(layer.router_bias.device)
    return layer.router_bias[perm].contiguous()


# --------------------------------------------------------------------------
# named workloads (sizes and distributions of the five configurations)
# --------------------------------------------------------------------------
FULL = dict(d=2048, E=512, F=512, Fs=512, k=10)

WORKLOADS = {
    # 1 layer, d=64, 16 experts (ffn 32) + shared (ffn 32), top-2, 4 tokens, 2-bit, seed 0
    "tiny": dict(shape=MoEShape(d=64, E=16, F=32, Fs=32, k=2, bits=2), T=4, bias="none",
                 slot="random"),
    # 1 layer, full size, 2-bit, Zipf(1.1) popularity, frequency-ordered slots, T = 1..4
    "decode": dict(shape=MoEShape(bits=2, **FULL), T=(1, 2, 3, 4), bias="zipf", slot="profile"),
    # 48 layers, 3-bit, Zipf profile, frequency-ordered slots, 4 tokens/step, 256 steps
    "decode_stack": dict(shape=MoEShape(bits=3, **FULL), T=4, layers=48, steps=256, bias="zipf",
                         slot="profile"),
    # 1 layer, 8192 tokens, 2-bit, bias ~ N(0, 0.5)
    "prefill": dict(shape=MoEShape(bits=2, **FULL), T=8192, bias="normal", bias_std=0.5,
                    slot="random"),
    # 48 layers, 3-bit: 4 x 8192-token chunks then 512 decode steps of 4 tokens, ranking drift/64
    "mix": dict(shape=MoEShape(bits=3, **FULL), T=4, layers=48, chunk=8192, chunks=4,
                decode_steps=512, drift_every=64, bias="zipf", slot="profile"),
}

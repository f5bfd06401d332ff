"""moe_pack_host, the host-side quantiser and packer of include/moe_pack.h, on
the CPU: bytes identical to the seeded input generator's packer, codes read
back by the oracle's own reader, the quantiser's tie, rounding and zero-group
rules on hand-made groups, and argument validation."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from routed_expert_ffn_06_b200 import build, moe, synth


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load()


def _dequant(W, bits):
    codes, scales = moe.moe_pack_host(W, bits)
    R, K = W.shape
    return oracle.dequant_matrix(codes.numpy().reshape(-1), scales.numpy().view(np.uint16).reshape(-1),
                                 R, K, bits), codes, scales


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("R,K", [(16, 32), (48, 96), (128, 2048)])
def test_bytes_match_the_generator_packer(bits, R, K):
    g = torch.Generator().manual_seed(R * 7 + K + bits)
    W = torch.randn(R, K, generator=g) * 0.05
    W[3, :32] = 0.0                                  # an all-zero group
    codes, scales = moe.moe_pack_host(W, bits)
    c_ref, s_ref = synth.pack_matrices(W.unsqueeze(0), bits)
    assert torch.equal(codes.reshape(-1), c_ref.reshape(-1))
    assert torch.equal(scales.reshape(-1), s_ref.reshape(-1).view(torch.int16))


@pytest.mark.parametrize("bits", [2, 3])
def test_oracle_reads_values_within_one_step(bits):
    """Every read-back value is s * (q - 2^(b-1)) with |w - w'| <= |s| (at most
    half a step, plus half a step where the top code is clamped)."""
    g = torch.Generator().manual_seed(bits)
    W = torch.randn(32, 256, generator=g)
    deq, _, scales = _dequant(W, bits)
    s = np.abs(scales.numpy().view(np.float16).astype(np.float64))   # tile-interleaved
    s = s.reshape(2, 8, 16).transpose(0, 2, 1).reshape(32, 8)         # -> [row][group]
    step = np.repeat(s, 32, axis=1)
    assert np.all(np.abs(W.double().numpy() - deq) <= step * (1 + 1e-12))
    q, s16 = synth.quantize_groups(W, bits)
    off = 1 << (bits - 1)
    ref = s16.double().unsqueeze(-1) * (q.double() - off)
    assert np.array_equal(deq, ref.reshape(32, 256).numpy())


def test_hand_groups_2bit():
    """Largest magnitude first on ties, round half to even, clamp at the top
    code, and the zero group."""
    W = torch.zeros(16, 96)
    # group 0 of row 0: m = -1 -> s = 0.5; 0.25/0.5 = 0.5 -> 0; 0.75/0.5 = 1.5 -> 2
    # -> code 4, clamped to 3; -0.25/0.5 = -0.5 -> 0
    W[0, :4] = torch.tensor([-1.0, 0.25, 0.75, -0.25])
    # group 1 of row 0: +0.7 and -0.7 tie; the first (+0.7) sets s = fp16(-0.35)
    W[0, 32 + 5] = 0.7
    W[0, 32 + 9] = -0.7
    # group 2 of row 0 stays all zero
    deq, _, scales = _dequant(W, 2)
    assert deq[0, :5].tolist() == [-1.0, 0.0, 0.5, 0.0, 0.0]
    s = float(torch.tensor(-0.35).to(torch.float16))
    assert deq[0, 32 + 5] == s * (0 - 2) and deq[0, 32 + 9] == s * (3 - 2)
    assert np.all(deq[0, 64:] == 0.0) and np.all(deq[1:] == 0.0)
    sc = scales.numpy().view(np.uint16)[0]          # tile 0: element c*16 + r
    # the zero group's scale is fp16(+0 / -2) = -0 (bits 0x8000)
    assert sc[0] == 0x3800 and sc[16] == np.float16(s).view(np.uint16) and sc[32] == 0x8000


def test_hand_group_3bit_codes():
    """3-bit: m = 4 -> s = -1; codes are w/s + 4, read back bit by bit."""
    W = torch.zeros(16, 32)
    W[0] = torch.tensor([4.0, 3, 2, 1, 0, -1, -2, -3] * 4)
    deq, codes, _ = _dequant(W, 3)
    assert deq[0].tolist() == W[0].tolist()
    c = codes.numpy().reshape(-1)
    got = [oracle.read_code(c, 16, 32, 3, 0, j) for j in range(32)]
    assert got == [0, 1, 2, 3, 4, 5, 6, 7] * 4


def test_argument_validation():
    lib = moe.load()
    w = np.zeros((16, 32), dtype=np.float32)
    c = np.zeros(16 * 12, dtype=np.uint8)
    s = np.zeros(16, dtype=np.uint16)
    P = lambda a: a.ctypes.data
    assert lib.moe_pack_host(P(w), 16, 32, 2, P(c), P(s)) == 0
    assert lib.moe_pack_host(None, 16, 32, 2, P(c), P(s)) == 1
    assert lib.moe_pack_host(P(w), 16, 32, 2, None, P(s)) == 1
    assert lib.moe_pack_host(P(w), 8, 32, 2, P(c), P(s)) == 2
    assert lib.moe_pack_host(P(w), 16, 48, 2, P(c), P(s)) == 2
    assert lib.moe_pack_host(P(w), 16, 32, 4, P(c), P(s)) == 2
    assert lib.moe_pack_host(P(w), 0, 32, 2, P(c), P(s)) == 2

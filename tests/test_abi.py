"""The C ABI library: it loads, exports every entry point the headers in
include/ declare, and its host-side validation answers before touching a GPU."""
import ctypes
import os
import re

import pytest

from routed_expert_ffn_06_b200 import build, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load()


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for h in sorted(os.listdir(inc)):
        if h.endswith(".h"):
            src = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, h)).read(), flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["moe_route_topk", "moe_expert_ffn_decode", "moe_expert_ffn_prefill",
              "moe_block_forward", "moe_workspace_bytes"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(_declared()) <= set(moe.EXPORTS) | set(_declared())


def _layer(**kw):
    base = dict(d_model=64, n_experts=16, ffn=32, top_k=2, bits=2, group=32, shared_ffn=32)
    base.update(kw)
    L = moe.moe_layer(**base)
    fake = 0x7F0000000000  # 256-aligned fake device addresses: never dereferenced on the host
    L.router_w = fake
    L.expert_slot = fake + 0x1000
    L.codes = fake + 0x2000
    L.scales = fake + 0x100000
    L.shared_codes = fake + 0x200000
    L.shared_scales = fake + 0x300000
    return L


def test_workspace_bytes(lib):
    L = _layer()
    n1 = moe.moe_workspace_bytes(L, 1)
    n4 = moe.moe_workspace_bytes(L, 4)
    n8k = moe.moe_workspace_bytes(L, 8192)
    assert 0 < n1 <= n4 < n8k
    assert n8k % 256 == 0
    assert moe.moe_workspace_bytes(_layer(bits=4), 4) == 0
    assert moe.moe_workspace_bytes(_layer(d_model=48), 4) == 0


@pytest.mark.parametrize("bad,status", [
    (dict(bits=4), 2), (dict(group=64), 2), (dict(d_model=48), 2), (dict(ffn=40), 2),
    (dict(top_k=17), 2), (dict(top_k=0), 2), (dict(n_experts=1), 2), (dict(n_experts=2048), 2),
    (dict(shared_ffn=-32), 2), (dict(d_model=8192), 2),
])
def test_shape_validation(lib, bad, status):
    L = _layer(**bad)
    rc = lib.moe_block_forward(ctypes.byref(L), 0x7F0000400000, 4, 0x7F0000500000, 0,
                               0x7F0000600000, 1 << 30, None)
    assert rc == status


def test_pointer_and_size_validation(lib):
    L = _layer()
    ws, x, y = 0x7F0000600000, 0x7F0000400000, 0x7F0000500000
    P = ctypes.byref
    assert lib.moe_block_forward(P(L), None, 4, y, 0, ws, 1 << 30, None) == 1
    assert lib.moe_block_forward(P(L), x, -1, y, 0, ws, 1 << 30, None) == 1
    assert lib.moe_block_forward(P(L), x + 2, 4, y, 0, ws, 1 << 30, None) == 4     # misaligned x
    assert lib.moe_block_forward(P(L), x, 4, y, 0, ws + 16, 1 << 30, None) == 4    # ws not 256-aligned
    assert lib.moe_block_forward(P(L), x, 4, y, 0, ws, 64, None) == 3              # too small
    assert lib.moe_expert_ffn_decode(P(L), x, 9, x, x, y, 0, ws, 1 << 30, None) == 2  # T > 8
    assert lib.moe_expert_ffn_decode(P(L), x, 4, x, x, x, 0, ws, 1 << 30, None) == 1  # y aliases x
    assert lib.moe_route_topk(P(L), x, 4, 1 << 7, None, x, x, ws, 1 << 30, None) == 1  # bad flag
    L2 = _layer()
    L2.codes = 0x7F0000002008
    assert lib.moe_block_forward(P(L2), x, 4, y, 0, ws, 1 << 30, None) == 4
    L3 = _layer()
    L3.shared_codes = None
    assert lib.moe_block_forward(P(L3), x, 4, y, 0, ws, 1 << 30, None) == 1
    assert lib.moe_block_forward(None, x, 4, y, 0, ws, 1 << 30, None) == 1


def test_no_gpu_reports_no_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = _layer()
    rc = lib.moe_block_forward(ctypes.byref(L), 0x7F0000400000, 4, 0x7F0000500000, 0,
                               0x7F0000600000, 1 << 30, None)
    assert rc == 8


def test_status_strings(lib):
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(3)
    assert "sm_100a" in moe.moe_build_info()


def test_decode_rejects_experts_too_wide_for_its_stages(lib):
    """The decode step checks that its shared-memory stages hold the layer
    before anything else touches the device: ffn 4096 at d 256 is a valid layer
    that only the prefill step takes (MOE_ERR_UNSUPPORTED_SHAPE, not a launch
    failure), while ffn 512 passes the shape checks and stops at the missing
    device."""
    x, y, ids, w, ws = 0x7F0000400000, 0x7F0000500000, 0x7F0000700000, 0x7F0000800000, 0x7F0000600000
    wide = _layer(d_model=256, n_experts=20, ffn=4096, shared_ffn=4096, top_k=16)
    assert lib.moe_expert_ffn_decode(ctypes.byref(wide), x, 1, ids, w, y, 0, ws, 1 << 30, None) == 2
    ok = _layer(d_model=256, n_experts=20, ffn=512, shared_ffn=512, top_k=16)
    assert lib.moe_expert_ffn_decode(ctypes.byref(ok), x, 8, ids, w, y, 0, ws, 1 << 30, None) == 8


def test_block_forward_takes_prefill_for_experts_too_wide_for_decode(lib):
    """Path choice on the host, seen through the workspace it demands: a
    4-token window of a layer within the decode kernels' width runs the decode
    path, which needs only a leading part of the workspace (so one byte short
    of the full size passes and the call stops at the missing device); with
    ffn 4096 the same window takes the prefill path, which needs it all."""
    x, y = 0x7F0000400000, 0x7F0000500000
    for ffn, want in [(512, 8), (4096, 3)]:
        L = _layer(d_model=256, n_experts=20, ffn=ffn, shared_ffn=ffn, top_k=16)
        full = lib.moe_workspace_bytes(ctypes.byref(L), 4)
        assert full > 0
        rc = lib.moe_block_forward(ctypes.byref(L), x, 4, y, 0, 0x7F0000600000, full - 1, None)
        assert rc == want, (ffn, rc)


def test_block_forward_middle_windows_need_only_the_decode_workspace(lib):
    """Windows of 9..32 tokens run as consecutive decode windows, which need
    only the decode part of the workspace (one byte short of the full size
    passes and stops at the missing device); 33 tokens take the prefill step
    and need it all."""
    x, y = 0x7F0000400000, 0x7F0000500000
    L = _layer(d_model=256, n_experts=20, ffn=512, shared_ffn=512, top_k=16)
    for T, want in [(9, 8), (16, 8), (32, 8), (33, 3)]:
        full = lib.moe_workspace_bytes(ctypes.byref(L), T)
        rc = lib.moe_block_forward(ctypes.byref(L), x, T, y, 0, 0x7F0000600000, full - 1, None)
        assert rc == want, (T, rc)


def test_wait_limit_and_withhold_switch_validation(lib):
    """The control-block setters check their arguments on the host; valid
    calls stop at the missing device."""
    ws = 0x7F0000600000
    set_limit, set_site = lib.moe_workspace_set_wait_limit, lib.moe_workspace_set_debug_withhold
    assert set_limit(None, 1 << 20, 1000, None) == 1
    assert set_limit(ws, 64, 1000, None) == 1                  # smaller than the control block
    assert set_limit(ws + 16, 1 << 20, 1000, None) == 4        # not 256-aligned
    assert set_limit(ws, 1 << 20, 60_000_001, None) == 1       # above 60 s
    assert set_limit(ws, 1 << 20, 999, None) == 1              # below the 1 ms floor
    assert set_site(ws, 1 << 20, 2, None) == 1                 # no such site
    assert set_site(None, 1 << 20, 1, None) == 1
    assert set_site(ws + 16, 1 << 20, 1, None) == 4
    import torch
    if not torch.cuda.is_available():
        assert set_limit(ws, 1 << 20, 60_000_000, None) == 8
        assert set_limit(ws, 1 << 20, 0, None) == 8
        assert set_site(ws, 1 << 20, moe.WITHHOLD_PREFILL_ARRIVE, None) == 8


def test_l2_next_layer_is_validated(lib):
    """A next layer named for the L2 prefetch must pass the layer checks
    (MOE_ERR_INVALID_ARG otherwise); a valid one lets the call reach the
    missing device."""
    x, y, ws = 0x7F0000400000, 0x7F0000500000, 0x7F0000600000
    L = _layer()
    bad = _layer(bits=4)
    L.l2_next = ctypes.addressof(bad)
    assert lib.moe_block_forward(ctypes.byref(L), x, 4, y, 0, ws, 1 << 30, None) == 1
    good = _layer(n_experts=32)
    L.l2_next = ctypes.addressof(good)
    import torch
    if not torch.cuda.is_available():
        assert lib.moe_block_forward(ctypes.byref(L), x, 4, y, 0, ws, 1 << 30, None) == 8
    structs = [_layer() for _ in range(3)]
    moe.link_l2_next(structs)
    assert [s.l2_next for s in structs] == [ctypes.addressof(structs[1]),
                                            ctypes.addressof(structs[2]),
                                            ctypes.addressof(structs[0])]


def test_router_split_validation(lib):
    """moe_router_split checks the layer and its output pointer on the host;
    a misaligned pre-split router in the layer is rejected by every call."""
    L = _layer()
    out = 0x7F0000900000
    assert lib.moe_router_split(ctypes.byref(L), None, None) == 1
    assert lib.moe_router_split(ctypes.byref(L), out + 2, None) == 4
    assert lib.moe_router_split(ctypes.byref(_layer(bits=4)), out, None) == 2
    import torch
    if not torch.cuda.is_available():
        assert lib.moe_router_split(ctypes.byref(L), out, None) == 8
    L.router_w_split = out + 8
    x, y, ws = 0x7F0000400000, 0x7F0000500000, 0x7F0000600000
    assert lib.moe_block_forward(ctypes.byref(L), x, 64, y, 0, ws, 1 << 30, None) == 4


def test_middle_windows_of_a_wide_layer_take_the_prefill_step(lib):
    """Windows of 9..32 tokens use the decode kernels only for layers within
    their width: with ffn 4096 at d 256 a 16-token window takes the prefill
    step and needs the whole workspace (one byte short is too small)."""
    x, y = 0x7F0000400000, 0x7F0000500000
    L = _layer(d_model=256, n_experts=20, ffn=4096, shared_ffn=4096, top_k=16)
    full = lib.moe_workspace_bytes(ctypes.byref(L), 16)
    assert lib.moe_block_forward(ctypes.byref(L), x, 16, y, 0, 0x7F0000600000, full - 1, None) == 3


def test_header_compiles_as_c99_and_ctypes_mirrors_moe_layer(tmp_path):
    """include/moe.h is a C header: it compiles as strict C99, and the ctypes
    mirror of moe_layer in the binding has the C struct's size and field
    offsets (measured by a program compiled against the header)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    fields = [f for f, _ in moe.moe_layer._fields_]
    src = ["#include <stddef.h>", "#include <stdint.h>", "#include <stdio.h>", '#include "moe.h"',
           "int main(void) {", '  printf("%zu\\n", sizeof(moe_layer));']
    src += [f'  printf("%zu\\n", offsetof(moe_layer, {f}));' for f in fields]
    src += ["  return 0;", "}"]
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    out = [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True,
                                          text=True).stdout.split()]
    assert out[0] == ctypes.sizeof(moe.moe_layer)
    assert out[1:] == [getattr(moe.moe_layer, f).offset for f in fields]

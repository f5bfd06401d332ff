"""The layer-split pipeline's GPU step on one rank: three 3-bit layers of the
decode stack driven by LayerSplitPipeline with cuda_layer_step give exactly
the bytes of the same block forwards called in sequence.  (Several GPUs are
not available to this suite; the hand-off between ranks is covered on host
ranks in test_pipeline.py.)"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

from routed_expert_ffn_06_b200 import build, moe, synth
from routed_expert_ffn_06_b200.pipeline import LayerSplitPipeline, cuda_layer_step

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_pipeline_equals_the_block_chain():
    build.build()
    moe.load()
    wl = synth.WORKLOADS["decode_stack"]
    layers = [synth.make_layer(wl["shape"], seed=0, layer=l, device="cuda", bias=wl["bias"],
                               slot=wl["slot"]) for l in range(3)]
    structs = [moe.make_layer_struct(l) for l in layers]
    ws = moe.alloc_workspace(structs[0], 8)
    flags = moe.F_PRENORM | moe.F_RESIDUAL
    xs = [synth.make_tokens(T, 2048, seed=9, step=T, device="cuda") for T in (4, 1, 8)]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        pipe = LayerSplitPipeline(3, cuda_layer_step(structs, ws, flags))
        out = pipe.run(xs, [x.shape for x in xs], device="cuda")
        torch.cuda.synchronize()
        for x, y in zip(xs, out):
            ref = x
            for L in structs:
                nxt = torch.empty_like(ref)
                moe.moe_block_forward(L, ref, ref.shape[0], nxt, flags, ws)
                ref = nxt
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
    finally:
        dist.destroy_process_group()

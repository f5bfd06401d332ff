"""The layer-split pipeline across ranks (routed_expert_ffn_06_b200/pipeline.py)
on two and three host ranks (gloo).  Each rank owns a contiguous block of four
tiny routed-MoE layers; the per-layer step is the fp64 oracle with pre-norm and
residual, its output rounded to bf16 as the GPU stack carries it.  The last
rank's outputs must equal the same layers applied in sequence in one process,
byte for byte, for micro-batches of different window sizes."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

N_LAYERS = 4
WINDOWS = (4, 1, 3, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_step():
    import oracle
    from routed_expert_ffn_06_b200 import synth
    sh = synth.WORKLOADS["tiny"]["shape"]
    layers = [oracle.OracleLayer(synth.make_layer(sh, seed=0, layer=l, bias="normal"))
              for l in range(N_LAYERS)]

    def step(l, x):
        bits = x.contiguous().view(torch.int16).numpy().view(np.uint16)
        y = layers[l].block_forward(bits, flags=oracle.PRENORM | oracle.RESIDUAL)["y"]
        return torch.from_numpy(y).to(torch.bfloat16)
    return step, sh


def _inputs(sh):
    from routed_expert_ffn_06_b200 import synth
    return [(synth.make_tokens(T, sh.d, seed=5, step=i).float() * 2).to(torch.bfloat16)
            for i, T in enumerate(WINDOWS)]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from routed_expert_ffn_06_b200.pipeline import LayerSplitPipeline
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    step, sh = _oracle_step()
    xs = _inputs(sh)
    pipe = LayerSplitPipeline(N_LAYERS, step)
    out = pipe.run(xs if rank == 0 else None, [x.shape for x in xs], device="cpu")
    if rank == world - 1:
        ref = []
        for x in xs:
            for l in range(N_LAYERS):
                x = step(l, x)
            ref.append(x)
        q.put((rank, list(pipe.layers), all(torch.equal(a, b) for a, b in zip(out, ref)),
               len(out)))
    else:
        q.put((rank, list(pipe.layers), out is None, 0))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_layer_split_pipeline_equals_the_sequential_stack(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    owned = [l for _, layers, _, _ in out for l in layers]
    assert owned == list(range(N_LAYERS))          # every layer once, in order
    for rank, _, ok, n in out:
        assert ok, f"rank {rank}"
    assert out[-1][3] == len(WINDOWS)


def test_layer_range_partitions_contiguously():
    from routed_expert_ffn_06_b200.pipeline import layer_range
    for n in (1, 4, 7, 48):
        for w in (1, 2, 3, 8):
            blocks = [list(layer_range(n, r, w)) for r in range(w)]
            assert sum(blocks, []) == list(range(n))
            sizes = [len(b) for b in blocks]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        layer_range(4, 2, 2)

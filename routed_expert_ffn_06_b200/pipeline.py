"""Layer-split pipeline across GPUs: each rank owns a contiguous block of the
stack's layers and hands the activations of every micro-batch (a verify window
or a prefill chunk) to the next rank.

The pages split a model across two cards the same way: every card keeps the
experts of its own layers and the prompt flows from card to card, which reads
long prompts 18-20% faster ("Why Strata is fast on low-VRAM GPUs", section
"two cards in relay"; "Strata illustrated", further reading on the multi-GPU
pipeline).  Here the hand-off is a point-to-point send of the micro-batch's
activations, T x d bf16 (16 KiB for a 4-token window of d = 2048), through
torch.distributed: NCCL over NVLink between GPUs, gloo on the host.  No
collective and no multicast is involved.

The schedule is the plain one for a chain: rank r receives micro-batch m from
rank r - 1 (rank 0 takes it from the caller), runs its layers on it, and
sends it on without waiting for the send to complete, so rank r works on
micro-batch m + 1 while rank r + 1 works on m.  The last rank returns the
outputs.  The per-layer step is a callable, so the same schedule drives the
CUDA block forward (``cuda_layer_step``) and, in the host tests, the oracle.

Every rank takes the same steps in the same order: one receive (ranks > 0) and
one send (ranks < world - 1) per micro-batch.
"""
from __future__ import annotations

from typing import Callable, List, Sequence

import torch
import torch.distributed as dist


def layer_range(n_layers: int, rank: int, world: int) -> range:
    """The layers rank `rank` owns: a contiguous block, the first
    n_layers % world ranks one layer longer."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    base, extra = divmod(n_layers, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


class LayerSplitPipeline:
    """One rank's part of a layer-split pipeline.

    step(l, x) runs layer l on activations x (a [T, d] bf16 tensor on this
    rank's device) and returns the new activations.  group: the process group
    (default: the world)."""

    def __init__(self, n_layers: int, step: Callable[[int, torch.Tensor], torch.Tensor],
                 group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.layers = layer_range(n_layers, self.rank, self.world)
        self.step = step

    def _peer(self, r: int) -> int:
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def run(self, micro_batches: Sequence[torch.Tensor] | None, shapes: Sequence[torch.Size],
            device, dtype=torch.bfloat16) -> List[torch.Tensor] | None:
        """Push the micro-batches through the pipeline.  Rank 0 passes them
        (the others pass None); every rank passes their shapes.  The last rank
        returns the outputs, the others None."""
        first, last = self.rank == 0, self.rank == self.world - 1
        if first and (micro_batches is None or len(micro_batches) != len(shapes)):
            raise ValueError("rank 0 supplies one tensor per shape")
        outputs, pending = [], []
        for m, shape in enumerate(shapes):
            if first:
                x = micro_batches[m].to(device)
            else:
                x = torch.empty(shape, dtype=dtype, device=device)
                dist.recv(x, src=self._peer(self.rank - 1), group=self.group)
            for l in self.layers:
                x = self.step(l, x)
            if last:
                outputs.append(x)
            else:
                pending.append(dist.isend(x.contiguous(), dst=self._peer(self.rank + 1),
                                          group=self.group))
        for req in pending:
            req.wait()
        return outputs if last else None


def cuda_layer_step(layer_structs, ws, flags: int, stream=None):
    """A pipeline step on this rank's GPU: the block forward of layer l (the
    structs are indexed by global layer number; only this rank's are used)."""
    from routed_expert_ffn_06_b200 import moe

    def step(l: int, x: torch.Tensor) -> torch.Tensor:
        y = torch.empty_like(x)
        moe.moe_block_forward(layer_structs[l], x, x.shape[0], y, flags, ws, stream)
        return y
    return step

"""Data-parallel plumbing of the adapter-only backward.

The layer shards by tokens with replicated weights, so the forward has no
exchange. The backward has one: every rank's adapter gradients dA, dB are
summed over the ranks before the optimizer step. Only the adapters train and
only they carry optimizer state (Principle 3 of "Reversible Sparse MoE Single
Node"), so this is the only data that crosses GPUs.

FlatGrads keeps the six gradient tensors of one layer as views of a single
fp32 buffer, so the exchange is one all-reduce per layer rather than six.
allreduce_adapter_grads sums it with torch.distributed: NCCL between GPUs,
gloo on CPU. With async_op=True it returns the work handle, so the sum of one
layer can overlap the backward of the next.
"""
from __future__ import annotations

import ctypes

from . import Grads


class FlatGrads:
    """dA[p] [E][r][in_p] and dB[p] [E][out_p][r] (p = gate, up, down; the storage
    layouts of lora_a / lora_b) as views of one zeroed fp32 buffer, with the
    tqp_adapter_grads struct pointing at them. r is a multiple of 8, so every
    view starts on a 32-byte boundary."""

    def __init__(self, E: int, d: int, f: int, r: int, device="cuda"):
        import torch
        dims = [(f, d), (f, d), (d, f)]                     # (out, in) per projection
        shapes = [(E, r, inn) for (_, inn) in dims] + [(E, out, r) for (out, _) in dims]
        counts = [a * b * c for (a, b, c) in shapes]
        self.flat = torch.zeros(sum(counts), dtype=torch.float32, device=device)
        views, off = [], 0
        for shape, n in zip(shapes, counts):
            views.append(self.flat[off:off + n].view(shape))
            off += n
        self.dA, self.dB = views[:3], views[3:]
        self.struct = Grads()
        for p in range(3):
            self.struct.dA[p] = self.dA[p].data_ptr() if r > 0 else None
            self.struct.dB[p] = self.dB[p].data_ptr() if r > 0 else None

    def ref(self):
        return ctypes.byref(self.struct)

    def zero_(self) -> None:
        self.flat.zero_()


def allreduce_adapter_grads(grads, group=None, async_op: bool = False):
    """Sum a layer's adapter gradients over the ranks of `group`, in place.

    grads: a FlatGrads or a flat fp32 tensor. Returns the work handle when
    async_op is set (wait on it before reading the gradients), else None. With
    no process group, one rank, or no adapters (rank 0), nothing is exchanged.
    """
    import torch.distributed as dist
    t = grads.flat if isinstance(grads, FlatGrads) else grads
    if t.numel() == 0 or not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return None
    work = dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
    return work if async_op else None


def adapter_dp_step(local_backward, grads, optimizer=None, group=None):
    """One data-parallel training step of a layer's adapters.

    local_backward(grads) fills `grads` with the gradients of this rank's token
    shard (overwriting them); the buffer is then summed over the ranks with one
    all-reduce, so every rank holds the gradient of the union of the shards
    (each expert's adapter gradient is a sum over the rows routed to it, so the
    shards' sums add up to the full batch's); finally optimizer.step(grads)
    runs the same update on every rank, which keeps the replicas identical.
    Every rank must call this with the same layer in the same order.
    """
    local_backward(grads)
    allreduce_adapter_grads(grads, group)
    if optimizer is not None:
        optimizer.step(grads)
    return grads


def layer_dp_step(layer, x_shard, dy_shard, dx_shard, grads, optimizer=None, group=None, ws=None, status=None,
                  stream=None):
    """adapter_dp_step with the library's layer backward as the local step:
    tqp_moe_layer_bwd on this rank's tokens (x_shard bf16, dy_shard fp32)."""
    from . import tqp_moe_layer_bwd

    def local(g):
        tqp_moe_layer_bwd(x_shard, dy_shard, layer, dx_shard, g, ws=ws, status=status, stream=stream)

    return adapter_dp_step(local, grads, optimizer, group)

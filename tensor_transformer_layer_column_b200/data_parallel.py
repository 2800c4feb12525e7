"""Data-parallel replicas: the parameter-gradient all-reduce, overlapped with the backward.

"3D decomposition in practice" and "What actually limits throughput in
production" (blog): beside tensor parallelism inside a node, whole replicas
of the model train on different batches, and their parameter gradients are
all-reduced once per step; that reduction is off the critical path, running
while the rest of the backward pass computes.

The layer's backward finishes its parameter gradients in three groups, in
this order (tp_layer_bwd_notify records one event per group; the
one-shard-per-GPU driver calls back at the same points):
  "mlp"   w1, b1, w2, b2, ln2_g, ln2_b   (the MLP backward and LN2's run first)
  "attn"  wqkv, bqkv, wout
  "ln1"   ln1_g, ln1_b, bout             (LN1's backward, last, also sums bout)
``GradBuckets`` lays each group's gradients out in one flat buffer, so one
collective reduces a group; ``GradientAllReduce`` issues that collective on
a side stream that first waits on the group's event, so the MLP gradients
cross the network while the attention backward computes.

The reduction is a SUM over the replicas (with a loss averaged over the
global batch, the upstream gradient already carries the 1/replicas factor
and the sum is the gradient of that loss), or an average when asked (the
collective's own AVG on NCCL; on backends without it, a sum then a scale).
torch.distributed does the communication (NCCL over NVLink / NVSwitch on
GPUs, gloo on CPU); nothing of the layer's arithmetic happens here.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

# Gradient groups of the pre-LN layer, in the order the backward completes them.
LAYER_GROUPS = {
    "mlp": ("w1", "b1", "w2", "b2", "ln2_g", "ln2_b"),
    "attn": ("wqkv", "bqkv", "wout"),
    "ln1": ("ln1_g", "ln1_b", "bout"),
}
ALIGN = 128    # elements between views: every gradient starts 256-byte aligned


class GradBuckets:
    """Flat per-group gradient buffers and the per-parameter views into them."""

    def __init__(self, shapes: Dict[str, Sequence[int]], groups: Dict[str, Sequence[str]],
                 dtype=torch.bfloat16, device="cuda"):
        self.groups = {g: tuple(n for n in names if n in shapes) for g, names in groups.items()}
        self.flat: Dict[str, torch.Tensor] = {}
        self.views: Dict[str, torch.Tensor] = {}
        for g, names in self.groups.items():
            offs, total = [], 0
            for n in names:
                offs.append(total)
                numel = 1
                for s in shapes[n]:
                    numel *= int(s)
                total += (numel + ALIGN - 1) // ALIGN * ALIGN
            buf = torch.zeros(max(total, 1), dtype=dtype, device=device)
            self.flat[g] = buf
            for n, o in zip(names, offs):
                numel = 1
                for s in shapes[n]:
                    numel *= int(s)
                self.views[n] = buf[o:o + numel].view(*shapes[n])

    def grads(self) -> Dict[str, torch.Tensor]:
        return dict(self.views)


class GradientAllReduce:
    """All-reduce of GradBuckets groups over the data-parallel process group,
    each issued as soon as its group is ready, on a side stream on GPUs."""

    def __init__(self, buckets: GradBuckets, group=None, average: bool = False):
        import torch.distributed as dist
        self.dist = dist
        self.buckets = buckets
        self.group = group
        self.average = average
        self.world = dist.get_world_size(group)
        self.backend = dist.get_backend(group)
        self.cuda = next(iter(buckets.flat.values())).is_cuda
        self.side = torch.cuda.Stream() if self.cuda else None
        self._events: Dict[str, torch.cuda.Event] = {}
        self._works: List = []
        self.order: List[str] = []

    def events(self) -> Dict[str, "torch.cuda.Event"]:
        """One CUDA event per group, materialised so that its handle can be
        given to tp_layer_bwd_notify."""
        if not self._events:
            for g in self.buckets.groups:
                e = torch.cuda.Event()
                e.record()          # creates the underlying cudaEvent_t
                self._events[g] = e
            torch.cuda.current_stream().synchronize()
        return self._events

    def _op(self):
        if self.average and self.backend == "nccl":
            return self.dist.ReduceOp.AVG
        return self.dist.ReduceOp.SUM

    def launch(self, group_name: str, event: Optional["torch.cuda.Event"] = None):
        """Start the all-reduce of one group.  On a GPU it waits, on the side
        stream, for `event` (recorded after the group's producing kernels), or
        for everything enqueued so far on the current stream."""
        buf = self.buckets.flat[group_name]
        self.order.append(group_name)
        if not self.cuda:
            self._works.append(self.dist.all_reduce(buf, op=self._op(), group=self.group,
                                                    async_op=True))
            return
        if event is None:
            event = torch.cuda.Event()
            event.record()
        self.side.wait_event(event)
        with torch.cuda.stream(self.side):
            self._works.append(self.dist.all_reduce(buf, op=self._op(), group=self.group,
                                                    async_op=True))

    def mark(self, group_name: str):
        """Callback form for drivers that call back when a group is ready
        (tensor_parallel.layer_backward's on_grads_ready)."""
        self.launch(group_name)

    def finish(self):
        """Make the current stream (or the host, on CPU) wait for every launched
        reduction, then scale by 1/replicas when averaging without AVG."""
        for w in self._works:
            w.wait()
        if self.cuda:
            torch.cuda.current_stream().wait_stream(self.side)
        self._works.clear()
        if self.average and self._op() == self.dist.ReduceOp.SUM and self.world > 1:
            for buf in self.buckets.flat.values():
                buf.mul_(1.0 / self.world)


def sharded_layer_buckets(layer, device="cuda"):
    """GradBuckets for a ShardedLayer (pre-LN) and the gradient dict its
    backward takes, whose tensors are views into the buckets: the library
    writes each gradient straight into its group's flat buffer.  The layer's
    gradient names are "d" + the parameter name (dw1, dbqkv, dln1_g, ...)."""
    meta = layer.alloc_grads(meta=True)
    shapes = {k[1:]: tuple(v.shape) for k, v in meta.items()}
    buckets = GradBuckets(shapes, LAYER_GROUPS, device=device)
    return buckets, {k: buckets.views[k[1:]] for k in meta}

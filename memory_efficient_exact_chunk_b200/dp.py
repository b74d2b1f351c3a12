"""Data-parallel replicas of the streamed stack backward with one fp32 gradient reduce-scatter
per step (skill page, Architecture Overview and Practical Guidance, Distributed Training: a
ZeRO-2 compatible variant whose ranks communicate for the optimizer step only, never for the
gradients of single chunks).  Each rank keeps 1/N of the summed gradient, as ZeRO-2 partitions
it.

Each rank runs the whole streamed backward on its own sequences; the chunk loop is unchanged
and no chunk-level data crosses ranks.  The fp32 gradients accumulate into buckets: one flat
buffer per unit whose gradient becomes final at one point of the backward (the LM head with the
final-norm gain right after the LM-head pass, each layer after its streamed backward, the
embedding at the end).  As soon as a bucket is final its reduce-scatter is queued on the
process group.  With NCCL the collective runs on the group's own stream, ordered after the
work already queued on the caller's stream, so the exchange of layer l overlaps the backward of
layer l-1.  After `GradReducer.wait()` every rank holds, for each bucket, the sum over ranks of
its own contiguous 1/N slice of the flat buffer.

Layout: tensors of a bucket are packed in order, each starting on a 64-element (256-byte)
boundary (the library wants 16-byte aligned gradient pointers); the bucket is padded to a
multiple of 64 * world elements so that every rank's shard starts 256-byte aligned.  This
module only arranges buffers and orders collectives; every gradient is computed by libsbp.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

from . import sbp

ALIGN = 64          # elements (fp32): 256 bytes


def _round_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def _numel(shape) -> int:
    n = 1
    for s in shape:
        n *= int(s)
    return n


def stack_buckets(layers: List[dict], lm_shape, final_shape, embed_shape) -> List[Tuple[str, list]]:
    """Bucket plan of the stack, in the order the backward finalises them:
    [("head", [("lm_head", shape), ("final_g", shape)]), ("layer{L-1}", [...]), ...,
     ("layer0", [...]), ("embed", [("embed", shape)])]."""
    plan = [("head", [("lm_head", tuple(lm_shape)), ("final_g", tuple(final_shape))])]
    for li in range(len(layers) - 1, -1, -1):
        W = layers[li]
        plan.append((f"layer{li}", [(n, tuple(W[n].shape)) for n in sbp.WEIGHT_FIELDS
                                    if W.get(n) is not None]))
    plan.append(("embed", [("embed", tuple(embed_shape))]))
    return plan


class ShardedGrads:
    """Flat fp32 gradient buckets, the per-tensor views the library accumulates into, and this
    rank's reduced shard of each bucket."""

    def __init__(self, plan: Sequence[Tuple[str, list]], world: int, rank: int, device):
        import torch
        if world < 1 or not 0 <= rank < world:
            raise ValueError(f"bad rank {rank} of world {world}")
        self.world, self.rank = world, rank
        self.order = [name for name, _ in plan]
        self.flat: Dict[str, object] = {}
        self.out: Dict[str, object] = {}
        self.views: Dict[str, Dict[str, object]] = {}
        self.offsets: Dict[str, Dict[str, int]] = {}
        for name, tensors in plan:
            off = 0
            offs = {}
            for tname, shape in tensors:
                offs[tname] = off
                off = _round_up(off + _numel(shape), ALIGN)
            total = _round_up(max(off, 1), ALIGN * world)
            flat = torch.zeros(total, dtype=torch.float32, device=device)
            self.flat[name] = flat
            self.offsets[name] = offs
            self.views[name] = {t: flat[offs[t]:offs[t] + _numel(s)].view(s) for t, s in tensors}
            self.out[name] = torch.zeros(total // world, dtype=torch.float32, device=device)

    def shard_range(self, bucket: str) -> Tuple[int, int]:
        """[lo, hi) element range of the bucket's flat buffer that this rank owns."""
        n = self.flat[bucket].numel() // self.world
        return self.rank * n, (self.rank + 1) * n

    def zero_(self):
        for t in self.flat.values():
            t.zero_()

    def stack_grads(self, n_layers: int) -> dict:
        """The gradient dict in the layout the stack functions take (views of the buckets)."""
        g = {"lm_head": self.views["head"]["lm_head"], "final_g": self.views["head"]["final_g"],
             "embed": self.views["embed"]["embed"], "layers": []}
        for li in range(n_layers):
            v = self.views[f"layer{li}"]
            g["layers"].append({n: v.get(n) for n in sbp.WEIGHT_FIELDS})
        return g


class GradReducer:
    """Queues one reduce-scatter (sum) per bucket as the backward finalises it.  Every rank must
    call `ready` for the same buckets in the same order, then `wait`."""

    def __init__(self, grads: ShardedGrads, group=None):
        self.g = grads
        self.group = group
        self.works = []
        self.issued: List[str] = []

    def ready(self, bucket: str):
        import torch.distributed as dist
        if bucket in self.issued:
            raise RuntimeError(f"bucket {bucket} reduced twice in one step")
        expected = self.g.order[len(self.issued)]
        if bucket != expected:
            raise RuntimeError(f"bucket {bucket} out of order (expected {expected})")
        self.issued.append(bucket)
        if self.g.world == 1 and self.group is None and not dist.is_initialized():
            self.g.out[bucket].copy_(self.g.flat[bucket])      # a single replica, no group
            return
        self.works.append(dist.reduce_scatter_tensor(self.g.out[bucket], self.g.flat[bucket],
                                                     op=dist.ReduceOp.SUM, group=self.group,
                                                     async_op=True))

    def wait(self):
        """Orders the caller's stream after every queued collective and resets for the next
        step.  All buckets must have been reduced."""
        if len(self.issued) != len(self.g.order):
            missing = [b for b in self.g.order if b not in self.issued]
            raise RuntimeError(f"step ended with buckets not reduced: {missing}")
        for w in self.works:
            w.wait()
        self.works.clear()
        self.issued.clear()


def dp_stack_step(cfg: sbp.LayerCfg, embed, layers: List[dict], final_g, lm_w, ids, targets,
                  loss_weights, grads: ShardedGrads, reducer: GradReducer, ws=None):
    """One data-parallel step on this rank's sequences: forward (layer-input checkpoints),
    streamed backward with the bucket reduce-scatters queued as each bucket is final, wait.
    Runs on torch's current stream (the collectives are ordered after it).  The loss weights
    carry the global normaliser (sum over all ranks' loss tokens), so the reduced gradient is
    that of the global loss.  Returns this rank's loss (device [1])."""
    from . import stack
    ws = ws or stack.Workspaces(embed.device)
    grads.zero_()
    xs, hf, rstd = stack.stack_forward(cfg, embed, layers, final_g, ids, ws)
    res = stack.stack_backward_from(cfg, layers, final_g, lm_w, ids, targets, loss_weights, xs,
                                    hf, rstd, ws, grads=grads.stack_grads(len(layers)),
                                    on_final=reducer.ready)
    reducer.wait()
    return res.loss

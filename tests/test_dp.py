"""The data-parallel gradient path (memory_efficient_exact_chunk_b200/dp.py) on CPU: bucket
layout and alignment, the reduce-scatter protocol with world size 2 on the gloo backend (each
rank ends with the sum over ranks of its own shard of every bucket), and the ordering checks.
The GPU test runs one data-parallel step of a small stack through libsbp on a one-rank NCCL
group and compares the reduced gradients with the fp64 oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from memory_efficient_exact_chunk_b200 import dp


def _plan():
    layers = [{"wq": torch.empty(8, 6), "wk": torch.empty(4, 6), "wv": torch.empty(4, 6),
               "bq": None, "bk": None, "bv": None, "wo": torch.empty(6, 8),
               "ln1_g": torch.empty(6), "ln2_g": torch.empty(6), "w_gate": torch.empty(10, 6),
               "w_up": torch.empty(10, 6), "w_down": torch.empty(6, 10)} for _ in range(2)]
    return dp.stack_buckets(layers, (17, 6), (6,), (17, 6))


def _fill(g, rank):
    """Gives every gradient view values that depend on the rank, as the backward would."""
    gen = torch.Generator().manual_seed(1000 + rank)
    for name in g.order:
        for t in g.views[name].values():
            t.copy_(torch.randn(t.shape, generator=gen))


def test_bucket_layout():
    plan = _plan()
    assert [b for b, _ in plan] == ["head", "layer1", "layer0", "embed"]
    for world in (1, 2, 3, 8):
        for rank in range(world):
            g = dp.ShardedGrads(plan, world, rank, "cpu")
            for name, tensors in plan:
                flat = g.flat[name]
                assert flat.numel() % (dp.ALIGN * world) == 0
                lo, hi = g.shard_range(name)
                assert (hi - lo) * world == flat.numel() and lo % dp.ALIGN == 0
                assert g.out[name].numel() == hi - lo
                end = 0
                for tname, shape in tensors:
                    off = g.offsets[name][tname]
                    assert off % dp.ALIGN == 0 and off >= end
                    v = g.views[name][tname]
                    assert tuple(v.shape) == shape
                    assert v.data_ptr() == flat.data_ptr() + 4 * off     # a view, not a copy
                    end = off + v.numel()
                assert end <= flat.numel()
    g = dp.ShardedGrads(plan, 2, 0, "cpu")
    sg = g.stack_grads(2)
    assert sg["layers"][0]["bq"] is None and sg["layers"][1]["wq"].shape == (8, 6)
    sg["lm_head"].fill_(3.0)
    assert float(g.flat["head"][:17 * 6].sum()) == 3.0 * 17 * 6
    with pytest.raises(ValueError):
        dp.ShardedGrads(plan, 2, 2, "cpu")


def test_reducer_order_checks_single_replica():
    g = dp.ShardedGrads(_plan(), 1, 0, "cpu")
    r = dp.GradReducer(g)
    _fill(g, 0)
    with pytest.raises(RuntimeError):
        r.ready("layer1")                      # "head" comes first
    r.ready("head")
    with pytest.raises(RuntimeError):
        r.ready("head")                        # twice in one step
    with pytest.raises(RuntimeError):
        r.wait()                               # buckets left
    for b in ("layer1", "layer0", "embed"):
        r.ready(b)
    r.wait()
    for b in g.order:
        assert torch.equal(g.out[b], g.flat[b])
    r.ready("head")                            # the next step starts over


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = _plan()
        g = dp.ShardedGrads(plan, world, rank, "cpu")
        r = dp.GradReducer(g)
        for step in range(2):                  # buffers and reducer are reused across steps
            g.zero_()
            _fill(g, rank + 10 * step)
            for b in g.order:
                r.ready(b)
            r.wait()
            # expected: the sum over ranks of this rank's shard, rebuilt from the seeds
            others = [dp.ShardedGrads(plan, world, q, "cpu") for q in range(world)]
            for q, o in enumerate(others):
                _fill(o, q + 10 * step)
            for b in g.order:
                lo, hi = g.shard_range(b)
                want = sum(o.flat[b][lo:hi] for o in others)
                err = float((g.out[b] - want).abs().max())
                out[(rank, step, b)] = err
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_scatter_gloo_world2():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(out)
    assert len(res) == 2 * 2 * 4
    assert max(res.values()) <= 1e-6, res


@pytest.mark.gpu
def test_dp_stack_step_one_rank_nccl():
    """One data-parallel step of a 2-layer fp32 stack (GQA, shifted targets, 3 sequences)
    through libsbp with the reduce-scatters on a one-rank NCCL group: the reduced shard is the
    whole gradient, checked against the fp64 oracle within 1e-5."""
    from oracle import sbp_oracle as O
    from memory_efficient_exact_chunk_b200 import sbp, synth
    from tests.helpers import f64, oracle_cfg, rel_fro, to_dev
    from tests.test_gpu_stack import NAMES, make_stack
    L = synth.LayerShape(64, 4, 2, 16, 96, 1e-6, 10000.0)
    B, T, V, D = 3, 96, 300, 4
    layers, E, fg, lm, ids, y, w = make_stack(11, L, 2, V, B, T, "f32", "shifted_tail",
                                              from_frac=0.25)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"))
    try:
        Ld = [{n: (to_dev(W[n], "f32") if W.get(n) is not None else None) for n in NAMES}
              for W in layers]
        cfg = sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn,
                            L.rms_eps, L.rope_theta, sbp.SBP_F32, D)
        plan = dp.stack_buckets(Ld, lm.shape, fg.shape, E.shape)
        g = dp.ShardedGrads(plan, 1, 0, "cuda")
        r = dp.GradReducer(g, group=dist.group.WORLD)
        i32 = lambda a: torch.from_numpy(a.reshape(-1).astype(np.int32)).cuda()
        for _ in range(2):                     # the second step reuses buffers and reducer
            loss = dp.dp_stack_step(cfg, to_dev(E, "f32"), Ld, to_dev(fg, "f32"),
                                    to_dev(lm, "f32"), i32(ids), i32(y),
                                    torch.from_numpy(w.reshape(-1)).cuda(), g, r)
        torch.cuda.synchronize()
        out = {b: g.out[b].cpu().numpy().astype(np.float64) for b in g.order}
    finally:
        dist.destroy_process_group()
    l0, g0 = O.stack_forward_backward(oracle_cfg(O, L), f64(E),
                                      [{n: f64(W.get(n)) for n in NAMES} for W in layers],
                                      f64(fg), f64(lm), ids, y, f64(w))
    assert abs(float(loss.item()) - l0) <= 1e-5 * abs(l0)

    def part(bucket, name, shape):
        o = g.offsets[bucket][name]
        return out[bucket][o:o + int(np.prod(shape))].reshape(shape)

    errs = {"lm_head": rel_fro(part("head", "lm_head", lm.shape), g0["lm_head"]),
            "final_g": rel_fro(part("head", "final_g", fg.shape), g0["final_g"]),
            "embed": rel_fro(part("embed", "embed", E.shape), g0["embed"])}
    for li in range(2):
        for n in g.offsets[f"layer{li}"]:
            errs[f"L{li}.{n}"] = rel_fro(part(f"layer{li}", n, layers[li][n].shape),
                                         g0["layers"][li][n])
    bad = {k: v for k, v in errs.items() if not v <= 1e-5}
    assert not bad, errs

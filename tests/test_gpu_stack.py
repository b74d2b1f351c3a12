"""GPU parity of a whole stack (embedding, layers, final norm, LM-head CE) composed from the C
ABI, against the fp64 oracle.  The tiny fp32 model runs at its full size (T = 256, D = 4)."""
import numpy as np
import pytest

from oracle import sbp_oracle as O
from memory_efficient_exact_chunk_b200 import synth
from tests.helpers import f64, oracle_cfg, rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu
NAMES = ("ln1_g", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "ln2_g", "w_gate", "w_up", "w_down")


def make_stack(seed, L, n_layers, V, B, T, dtype, loss_kind, **lkw):
    rng = np.random.default_rng(seed)
    bf = dtype == "bf16"
    layers = [synth.layer_weights(rng, L, bf) for _ in range(n_layers)]
    E = synth.normal(rng, (V, L.d_model), 0.02, bf)
    fg = np.ones(L.d_model, np.float32)
    lm = synth.normal(rng, (V, L.d_model), 0.02, bf)
    ids = synth.token_ids(rng, B, T, V)
    if loss_kind == "sft_all":
        y = synth.token_ids(rng, B, T, V)
    else:
        y = synth.shifted_targets(ids)
    w = synth.loss_weights(loss_kind, B, T, **lkw)
    return layers, E, fg, lm, ids, y, w


def run_gpu(L, layers, E, fg, lm, ids, y, w, D, dtype):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, stack
    B, T = ids.shape
    code = sbp.SBP_BF16 if dtype == "bf16" else sbp.SBP_F32
    cfg = sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn, L.rms_eps,
                        L.rope_theta, code, D)
    Ld = [{n: (to_dev(W[n], dtype) if W.get(n) is not None else None) for n in NAMES}
          for W in layers]
    r = stack.stack_backward(cfg, to_dev(E, dtype), Ld, to_dev(fg, dtype), to_dev(lm, dtype),
                             torch.from_numpy(ids.reshape(-1).astype(np.int32)).cuda(),
                             torch.from_numpy(y.reshape(-1).astype(np.int32)).cuda(),
                             torch.from_numpy(w.reshape(-1)).cuda())
    torch.cuda.synchronize()
    g = r.grads
    return (to_np(r.loss)[0], to_np(g["lm_head"]), to_np(g["final_g"]), to_np(g["embed"]),
            [{n: to_np(v) for n, v in lg.items() if v is not None} for lg in g["layers"]])


def _bf16_store(a):
    """The bf16 model keeps its layer-input checkpoints and the final-norm output in bf16."""
    return synth.bf16_round(np.asarray(a, np.float32)).astype(np.float64)


def check(L, stack_in, D, dtype, tol, store=True):
    """Every gradient against the oracle in the plain per-tensor relative Frobenius error.
    ``store``: on the bf16 path, give the oracle the bf16 rounding of the tensors the stack
    keeps between its passes (layer-input checkpoints, final-norm output); False runs the
    oracle on its own fp64 values throughout.  The bf16 key-bias gradients are held to the
    looser plain bound of test_gpu_layer (a sum with heavy cancellation) and, in addition, to
    ``tol`` against the sum of their absolute summands."""
    from tests.test_gpu_layer import BK_BF16_PLAIN
    layers, E, fg, lm, ids, y, w = stack_in
    loss, dlm, dfg, dE, dls = run_gpu(L, layers, E, fg, lm, ids, y, w, D, dtype)
    scales = []
    l0, g0 = O.stack_forward_backward(oracle_cfg(O, L), f64(E),
                                      [{n: f64(W.get(n)) for n in NAMES} for W in layers],
                                      f64(fg), f64(lm), ids, y, f64(w),
                                      store=_bf16_store if (dtype == "bf16" and store) else None,
                                      sum_scales=scales)
    assert abs(loss - l0) <= tol * abs(l0)
    errs = {"lm_head": rel_fro(dlm, g0["lm_head"]), "final_g": rel_fro(dfg, g0["final_g"]),
            "embed": rel_fro(dE, g0["embed"])}
    limits = {}
    summand = {}
    for i, lg in enumerate(dls):
        for n, v in lg.items():
            errs[f"L{i}.{n}"] = rel_fro(v, g0["layers"][i][n])
            if n == "bk" and dtype == "bf16":
                limits[f"L{i}.{n}"] = BK_BF16_PLAIN
                summand[f"L{i}.{n}"] = float(np.linalg.norm(f64(v) - g0["layers"][i][n]) /
                                             np.linalg.norm(scales[i][n]))
    print("stack errors:", {k: float(f"{v:.3g}") for k, v in errs.items()},
          "bk vs summands:", {k: float(f"{v:.3g}") for k, v in summand.items()})
    bad = {k: v for k, v in errs.items() if not v <= limits.get(k, tol)}
    bad.update({f"{k}/summands": v for k, v in summand.items() if not v <= tol})
    assert not bad, bad


def test_tiny_fp32_stack_full_size():
    """The tiny fp32 decoder (T 256, d 64, 4 heads of 16, MLP 172, vocab 512, mean CE over all
    tokens) at D = 4: every gradient within 1e-5 of the oracle."""
    wl = synth.WORKLOADS["tiny_stack_f32"]
    s = make_stack(0, wl.layer, 1, wl.vocab, 1, wl.seq_len, "f32", "sft_all")
    check(wl.layer, s, wl.num_chunks, "f32", 1e-5)


@pytest.mark.parametrize("store", [True, False])
def test_bf16_gqa_stack_shifted_targets(store):
    L = synth.LayerShape(128, 4, 2, 32, 192, 1e-5, 500000.0)
    s = make_stack(1, L, 2, 700, 1, 256, "bf16", "shifted_tail", from_frac=0.25)
    check(L, s, 4, "bf16", 1e-2, store=store)


@pytest.mark.parametrize("store", [True, False])
def test_bf16_grpo_batched_stack(store):
    L = synth.LayerShape(128, 4, 1, 32, 160, 1e-6, 1e6, qkv_bias=True)
    rng = np.random.default_rng(9)
    B, T, V = 3, 128, 600
    layers, E, fg, lm, ids, y, _ = make_stack(2, L, 2, V, B, T, "bf16", "shifted_tail",
                                              from_frac=0.25)
    w = synth.loss_weights("grpo", B, T, prompt_len=32, advantages=rng.standard_normal(B))
    check(L, (layers, E, fg, lm, ids, y, w), 4, "bf16", 1e-2, store=store)

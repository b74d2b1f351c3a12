"""GPU parity of the DPO objective (include/sbp_dpo.h) against the fp64 oracle: the streamed
LM-head forward (per-token CE), the DPO loss and per-token weights, and a whole DPO step of a
small stack.  Tolerances: 1e-5 (fp32 path), 1e-2 per tensor (bf16 inputs); D = 1 vs D > 1
within 1e-5."""
import numpy as np
import pytest

from oracle import sbp_oracle as O
from memory_efficient_exact_chunk_b200 import synth
from tests.helpers import f64, oracle_cfg, rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu
NAMES = ("ln1_g", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "ln2_g", "w_gate", "w_up", "w_down")


@pytest.mark.parametrize("dtype,N,d,V,D", [("f32", 600, 64, 1000, 3), ("bf16", 600, 128, 1500, 3),
                                           ("bf16", 1000, 256, 4100, 1)])
def test_lmhead_forward_token_ce(dtype, N, d, V, D):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    h, W, y, w = synth.lmhead_inputs(30 + N, N, d, V, bf16=(dtype == "bf16"), from_frac=0.2)
    hd, Wd = to_dev(h, dtype), to_dev(W, dtype)
    yd, wd = torch.from_numpy(y).cuda(), torch.from_numpy(w).cuda()
    ce = torch.full((N,), float("nan"), device="cuda")
    loss = torch.zeros(1, device="cuda")
    ws = sbp.lmhead_ce_forward(hd, Wd, yd, wd, D, ce, loss_out=loss)
    sbp.device_status(ws)
    ce0 = O.lmhead_token_ce(f64(h), f64(W), y, w)
    got = to_np(ce)
    assert np.all(got[w == 0] == 0)
    tol = 1e-5 if dtype == "f32" else 1e-4
    assert rel_fro(got, ce0) <= tol
    assert abs(to_np(loss)[0] - np.sum(f64(w) * ce0)) <= tol * abs(np.sum(f64(w) * ce0))


@pytest.mark.parametrize("P,T", [(1, 7), (3, 300), (5, 1025)])
def test_dpo_token_weights(P, T):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    rng = np.random.default_rng(P * 1000 + T)
    ce = np.abs(rng.standard_normal(2 * P * T)).astype(np.float32) * 3.0
    m = (rng.random(2 * P * T) > 0.25).astype(np.float32)
    ref = (-(m * ce).reshape(2 * P, T).sum(1) + rng.standard_normal(2 * P) * 4).astype(np.float32)
    beta = 0.2
    loss = torch.zeros(1, device="cuda")
    w = torch.full((2 * P * T,), float("nan"), device="cuda")
    lp = torch.zeros(2 * P, device="cuda")
    sbp.dpo_token_weights(P, T, torch.from_numpy(ce).cuda(), torch.from_numpy(m).cuda(),
                          torch.from_numpy(ref).cuda(), beta, loss, w, seq_logp=lp)
    torch.cuda.synchronize()
    l0, w0, lp0 = O.dpo_objective(f64(ce), f64(m), f64(ref), beta, P, T)
    # fp32 arithmetic: a sequence log-probability (a sum of up to T terms) carries an absolute
    # error up to ~4 eps32 sum|m ce|, and Delta (a difference of such sums with the fp32 ref)
    # twice that; loss and weights move by beta |dDelta| at most (d loss / d Delta and
    # d log coef / d Delta are bounded by beta)
    d_delta = 2 * 4 * 2.0 ** -23 * float(np.max(np.abs(m * ce).reshape(2 * P, T).sum(1)))
    assert abs(to_np(loss)[0] - l0) <= max(1e-6 * abs(l0), beta * d_delta)
    assert rel_fro(to_np(lp), lp0) <= 1e-6
    assert rel_fro(to_np(w), w0) <= max(1e-5, beta * d_delta)
    assert np.all(to_np(w)[m == 0] == 0)


def _dpo_inputs(seed, L, V, P, T, bf):
    rng = np.random.default_rng(seed)
    layers = [synth.layer_weights(rng, L, bf)]
    E = synth.normal(rng, (V, L.d_model), 0.02 if bf else 0.5, bf)
    fg = np.ones(L.d_model, np.float32)
    lm = synth.normal(rng, (V, L.d_model), 0.02 if bf else 0.5, bf)
    ids = synth.token_ids(rng, 2 * P, T, V)
    y = synth.shifted_targets(ids)
    m = np.zeros((2 * P, T), np.float32)
    m[:, T // 4:T - 1] = 1.0                         # response predictions after a prompt
    # reference log-probabilities near the policy's own, so that beta Delta is O(1)
    cfg = oracle_cfg(O, L)
    x = f64(E)[ids]
    for W in layers:
        x = O.decoder_layer_forward(cfg, {n: f64(W.get(n)) for n in NAMES}, x)
    hf, _ = O.rmsnorm_forward(x, f64(fg), cfg.rms_eps)
    ce = O.lmhead_token_ce(hf.reshape(2 * P * T, -1), f64(lm), y.reshape(-1), m.reshape(-1))
    logp = -(m * ce.reshape(2 * P, T)).sum(1)
    ref = (logp + rng.standard_normal(2 * P) * 2.0).astype(np.float32)
    return layers, E, fg, lm, ids, y, m, ref


def _gpu_dpo(L, inp, D, dtype, beta):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, stack
    layers, E, fg, lm, ids, y, m, ref = inp
    B, T = ids.shape
    code = sbp.SBP_BF16 if dtype == "bf16" else sbp.SBP_F32
    cfg = sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn, L.rms_eps,
                        L.rope_theta, code, D)
    Ld = [{n: (to_dev(W[n], dtype) if W.get(n) is not None else None) for n in NAMES}
          for W in layers]
    ws = stack.Workspaces(torch.device("cuda"))
    r = stack.stack_dpo_step(cfg, to_dev(E, dtype), Ld, to_dev(fg, dtype), to_dev(lm, dtype),
                             torch.from_numpy(ids.reshape(-1).astype(np.int32)).cuda(),
                             torch.from_numpy(y.reshape(-1).astype(np.int32)).cuda(),
                             torch.from_numpy(m.reshape(-1)).cuda(), torch.from_numpy(ref).cuda(),
                             beta, ws)
    torch.cuda.synchronize()
    g = r.grads
    out = {"lm_head": to_np(g["lm_head"]), "final_g": to_np(g["final_g"]),
           "embed": to_np(g["embed"])}
    for n, v in g["layers"][0].items():
        if v is not None:
            out[f"L0.{n}"] = to_np(v)
    return to_np(r.loss)[0], out


def _bf16_store(a):
    """The bf16 model keeps its layer-input checkpoints and the final-norm output in bf16."""
    return synth.bf16_round(np.asarray(a, np.float32)).astype(np.float64)


def _oracle_dpo(L, inp, beta, bf16, store=True):
    layers, E, fg, lm, ids, y, m, ref = inp
    loss, g, _ = O.stack_dpo(oracle_cfg(O, L), f64(E),
                             [{n: f64(W.get(n)) for n in NAMES} for W in layers], f64(fg),
                             f64(lm), ids, y, f64(m), f64(ref), beta,
                             store=_bf16_store if (bf16 and store) else None)
    out = {"lm_head": g["lm_head"], "final_g": g["final_g"], "embed": g["embed"]}
    for n, v in g["layers"][0].items():
        out[f"L0.{n}"] = v
    return loss, out


@pytest.mark.parametrize("dtype,L,P,T,D,tol,store", [
    ("f32", synth.LayerShape(64, 4, 4, 16, 172, 1e-6, 10000.0), 1, 128, 4, 1e-5, False),
    ("bf16", synth.LayerShape(128, 4, 2, 32, 192, 1e-5, 500000.0), 2, 256, 4, 1e-2, True),
    ("bf16", synth.LayerShape(128, 4, 2, 32, 192, 1e-5, 500000.0), 2, 256, 4, 1e-2, False),
])
def test_stack_dpo_step_matches_oracle(dtype, L, P, T, D, tol, store):
    """store=False: the oracle keeps every tensor in fp64 (no bf16 rounding of the stored
    checkpoints), so the whole bf16 error is measured."""
    inp = _dpo_inputs(7, L, 600, P, T, dtype == "bf16")
    beta = 0.5
    loss, g = _gpu_dpo(L, inp, D, dtype, beta)
    l0, g0 = _oracle_dpo(L, inp, beta, dtype == "bf16", store)
    assert abs(loss - l0) <= tol * abs(l0), (loss, l0)
    errs = {k: rel_fro(v, g0[k]) for k, v in g.items()}
    print("dpo errors:", {k: float(f"{v:.3g}") for k, v in errs.items()})
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, errs


def test_stack_dpo_chunk_invariance():
    L = synth.LayerShape(128, 4, 2, 32, 192, 1e-5, 500000.0)
    inp = _dpo_inputs(8, L, 600, 2, 512, True)
    l1, g1 = _gpu_dpo(L, inp, 1, "bf16", 0.3)
    for D in (2, 4):
        lD, gD = _gpu_dpo(L, inp, D, "bf16", 0.3)
        assert abs(lD - l1) <= 1e-6 * abs(l1)
        for k in g1:
            assert rel_fro(gD[k], g1[k]) <= 1e-5, (D, k, rel_fro(gD[k], g1[k]))

"""Pins for the fp64 oracle: each check ties the oracle to something other than itself
(finite differences, closed forms, special cases that reduce to a library routine, exact
invariants the StreamBP pages state).  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import sbp_oracle as O
from memory_efficient_exact_chunk_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def tiny_cfg(H=4, Hkv=2, hd=4, d=16, f=24, eps=1e-6, theta=10000.0):
    return O.LayerConfig(d, H, Hkv, hd, f, eps, theta)


def tiny_weights(cfg, seed=0, bias=True, std=0.3):
    rng = np.random.default_rng(seed)
    d, dq, dkv, f = cfg.d_model, cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.ffn
    W = {
        "ln1_g": 1.0 + 0.2 * rng.standard_normal(d),
        "wq": std * rng.standard_normal((dq, d)),
        "wk": std * rng.standard_normal((dkv, d)),
        "wv": std * rng.standard_normal((dkv, d)),
        "wo": std * rng.standard_normal((d, dq)),
        "ln2_g": 1.0 + 0.2 * rng.standard_normal(d),
        "w_gate": std * rng.standard_normal((f, d)),
        "w_up": std * rng.standard_normal((f, d)),
        "w_down": std * rng.standard_normal((d, f)),
        "bq": std * rng.standard_normal(dq) if bias else None,
        "bk": std * rng.standard_normal(dkv) if bias else None,
        "bv": std * rng.standard_normal(dkv) if bias else None,
    }
    return W


# ------------------------------------------------------------------------------------------
# chunk bounds: golden values worked from the rule on the skill page (Implementation).
# ------------------------------------------------------------------------------------------
def test_chunk_bounds_golden():
    with open(os.path.join(HERE, "golden", "chunk_bounds.txt")) as fh:
        rows = [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]
    assert rows
    for r in rows:
        T, D = int(r[0]), int(r[1])
        want = [tuple(int(v) for v in s.split(":")) for s in r[2:]]
        assert O.chunk_bounds(T, D) == want


def test_chunk_bounds_cover_and_reject():
    for T in range(1, 40):
        for D in range(1, T + 1):
            b = O.chunk_bounds(T, D)
            assert b[0][0] == 0 and b[-1][1] == T
            assert all(b[i][1] == b[i + 1][0] for i in range(D - 1))
    with pytest.raises(ValueError):
        O.chunk_bounds(4, 5)
    with pytest.raises(ValueError):
        O.chunk_bounds(4, 0)


# ------------------------------------------------------------------------------------------
# Token-wise pieces
# ------------------------------------------------------------------------------------------
def test_rmsnorm_matches_library_and_unit_rms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7, 33))
    g = 1 + 0.1 * rng.standard_normal(33)
    y, r = O.rmsnorm_forward(x, g, 1e-5)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (33,), torch.from_numpy(g), eps=1e-5)
    assert np.allclose(y, ref.numpy(), rtol=1e-13, atol=1e-13)
    y1, _ = O.rmsnorm_forward(x, np.ones(33), 0.0)
    assert np.allclose(np.sqrt(np.mean(y1 ** 2, axis=-1)), 1.0, rtol=1e-13)


def test_rope_closed_form_hd2():
    # hd = 2: inv_freq = 1, the pair (x0, x1) is a plane rotation by the position.
    x = np.array([[[0.3, -1.7]]] * 4)                   # [T=4, heads=1, 2]
    cos, sin = O.rope_tables(np.arange(4), 2, 10000.0)
    y = O.rope_forward(x, cos, sin)
    for t in range(4):
        c, s = math.cos(t), math.sin(t)
        assert np.allclose(y[t, 0], [c * 0.3 + s * 1.7, s * 0.3 - c * 1.7], atol=1e-15)


def test_rope_orthogonal_relative_and_frequencies():
    rng = np.random.default_rng(2)
    hd = 8
    x = rng.standard_normal((6, 3, hd))
    cos, sin = O.rope_tables(np.arange(6), hd, 500000.0)
    y = O.rope_forward(x, cos, sin)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    assert np.allclose(O.rope_backward(y, cos, sin), x, atol=1e-13)      # inverse = transpose
    assert np.allclose(y[0], x[0], atol=0)                                # position 0
    # q_m . k_n depends only on m - n
    q = rng.standard_normal(hd)
    k = rng.standard_normal(hd)
    cs, sn = O.rope_tables(np.arange(12), hd, 500000.0)
    rq = O.rope_forward(np.tile(q, (12, 1, 1)), cs, sn)[:, 0]
    rk = O.rope_forward(np.tile(k, (12, 1, 1)), cs, sn)[:, 0]
    assert abs(rq[5] @ rk[2] - rq[9] @ rk[6]) < 1e-12
    # the rotation angle of pair j at position 1 is theta^(-2j/hd) (rotate-half pairing j, j+hd/2)
    e = np.zeros((2, 1, hd))
    e[:, 0, 1] = 1.0
    r = O.rope_forward(e, *O.rope_tables(np.arange(2), hd, 500000.0))
    ang = 500000.0 ** (-2.0 * 1 / hd)
    assert np.isclose(r[1, 0, 1], math.cos(ang)) and np.isclose(r[1, 0, 1 + hd // 2], math.sin(ang))


def test_silu_and_swiglu_library():
    x = np.linspace(-8, 8, 101)
    assert np.allclose(O.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(), rtol=1e-14)
    assert O.silu(np.array(0.0)) == 0.0


# ------------------------------------------------------------------------------------------
# Attention forward: library cross-check and special cases
# ------------------------------------------------------------------------------------------
def test_attention_matches_library_sdpa_gqa():
    rng = np.random.default_rng(3)
    T, H, Hkv, hd = 9, 6, 2, 5
    q = rng.standard_normal((T, H, hd))
    k = rng.standard_normal((T, Hkv, hd))
    v = rng.standard_normal((T, Hkv, hd))
    out, _ = O.attention_forward(q, k, v)
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                           enable_gqa=True)
    assert np.allclose(out, ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_attention_prefix_rows_match_full():
    rng = np.random.default_rng(4)
    T, H, Hkv, hd = 10, 4, 1, 3
    q = rng.standard_normal((T, H, hd))
    k = rng.standard_normal((T, Hkv, hd))
    v = rng.standard_normal((T, Hkv, hd))
    full, _ = O.attention_forward(q, k, v)
    part, _ = O.attention_forward(q[6:9], k[:9], v[:9], q_start=6)
    assert np.allclose(part, full[6:9], rtol=1e-13, atol=1e-14)


def test_attention_special_cases():
    rng = np.random.default_rng(5)
    # one token: the softmax has one key, the output is v of the head's KV head
    q = rng.standard_normal((1, 4, 3))
    k = rng.standard_normal((1, 2, 3))
    v = rng.standard_normal((1, 2, 3))
    out, _ = O.attention_forward(q, k, v)
    assert np.allclose(out[0], np.repeat(v[0], 2, axis=0), atol=1e-15)
    # equal keys: uniform weights over the causal prefix -> running mean of v
    T = 7
    q = rng.standard_normal((T, 2, 3))
    k = np.tile(rng.standard_normal((1, 1, 3)), (T, 1, 1))
    v = rng.standard_normal((T, 1, 3))
    out, _ = O.attention_forward(q, k, v)
    want = np.cumsum(v[:, 0], axis=0) / np.arange(1, T + 1)[:, None]
    assert np.allclose(out[:, 0], want, atol=1e-13) and np.allclose(out[:, 1], want, atol=1e-13)


def test_attention_logsumexp_closed_forms():
    """lse of a causal score row, pinned by closed forms: one key gives the score itself
    (q.k / sqrt(hd): catches the scale); keys equal per KV head give score + log(t + 1) (the
    causal count of keys seen by query t, offset by q_start: catches the mask) with head h
    reading KV head h // (H / Hkv) (catches the GQA mapping)."""
    rng = np.random.default_rng(11)
    hd = 8
    q = rng.standard_normal((1, 2, hd))
    k = rng.standard_normal((1, 1, hd))
    lse = O.attention_logsumexp(q, k)
    assert np.allclose(lse[0], [q[0, 0] @ k[0, 0] / math.sqrt(hd), q[0, 1] @ k[0, 0] / math.sqrt(hd)],
                       rtol=1e-14, atol=1e-15)
    T, H, Hkv, q0 = 6, 4, 2, 3
    kv = rng.standard_normal((Hkv, hd))
    k = np.tile(kv[None], (q0 + T, 1, 1))
    q = rng.standard_normal((T, H, hd))
    lse = O.attention_logsumexp(q, k, q_start=q0)
    for t in range(T):
        for h in range(H):
            want = q[t, h] @ kv[h // (H // Hkv)] / math.sqrt(hd) + math.log(q0 + t + 1)
            assert abs(lse[t, h] - want) <= 1e-12 * max(1.0, abs(want)), (t, h)


# ------------------------------------------------------------------------------------------
# Layer: residual structure, finite differences, causality, chunk invariance
# ------------------------------------------------------------------------------------------
def test_layer_identity_when_output_projections_zero():
    cfg = tiny_cfg()
    W = tiny_weights(cfg)
    W["wo"] = np.zeros_like(W["wo"])
    W["w_down"] = np.zeros_like(W["w_down"])
    x = np.random.default_rng(6).standard_normal((2, 8, cfg.d_model))
    assert np.array_equal(O.decoder_layer_forward(cfg, W, x), x)


def _fd_check(fun, arr, idxs, analytic, h=1e-6, rtol=1e-6, atol=1e-9):
    for idx in idxs:
        old = arr[idx]
        arr[idx] = old + h
        fp = fun()
        arr[idx] = old - h
        fm = fun()
        arr[idx] = old
        num = (fp - fm) / (2 * h)
        assert abs(num - analytic[idx]) <= atol + rtol * abs(num), (idx, num, analytic[idx])


@pytest.mark.parametrize("bias", [True, False])
def test_layer_backward_finite_differences(bias):
    cfg = tiny_cfg()
    W = tiny_weights(cfg, seed=7, bias=bias)
    rng = np.random.default_rng(8)
    B, T = 2, 8
    x = rng.standard_normal((B, T, cfg.d_model))
    dy = rng.standard_normal((B, T, cfg.d_model))

    def loss():
        return float(np.sum(O.decoder_layer_forward(cfg, W, x) * dy))

    dx, g = O.decoder_layer_backward(cfg, W, x, dy)
    pick = lambda shape, n: [tuple(int(rng.integers(0, s)) for s in shape) for _ in range(n)]
    _fd_check(loss, x, pick(x.shape, 12), dx)
    for name in O.WEIGHT_NAMES:
        if W[name] is None:
            continue
        _fd_check(loss, W[name], pick(W[name].shape, 5), g[name])


def test_layer_causality_exact_zero():
    """Gradient of a chunk's output w.r.t. later tokens is exactly 0 (causal masking; skill
    page, Architecture Overview)."""
    cfg = tiny_cfg()
    W = tiny_weights(cfg, seed=9)
    rng = np.random.default_rng(10)
    x = rng.standard_normal((1, 12, cfg.d_model))
    for (s, e) in O.chunk_bounds(12, 3):
        dy = np.zeros_like(x)
        dy[0, s:e] = rng.standard_normal((e - s, cfg.d_model))
        dx, _ = O.decoder_layer_backward(cfg, W, x, dy)
        assert np.all(dx[0, e:] == 0.0)
        assert np.any(dx[0, :s] != 0.0) or s == 0


@pytest.mark.parametrize("D", [1, 2, 3, 5, 12])
def test_layer_chunked_equals_unchunked(D):
    """StreamBP's decomposition is exact: every gradient is the same at any D."""
    cfg = tiny_cfg()
    W = tiny_weights(cfg, seed=11)
    rng = np.random.default_rng(12)
    x = rng.standard_normal((2, 12, cfg.d_model))
    dy = rng.standard_normal((2, 12, cfg.d_model))
    dx0, g0 = O.decoder_layer_backward(cfg, W, x, dy)
    dx1, g1 = O.decoder_layer_backward_chunked(cfg, W, x, dy, D)
    rel = lambda a, b: np.linalg.norm(a - b) / max(np.linalg.norm(a), 1e-300)
    assert rel(dx0, dx1) <= 1e-12
    for k in g0:
        assert rel(g0[k], g1[k]) <= 1e-12, k


@pytest.mark.parametrize("D", [2, 3, 12])
def test_layer_reverse_order_rows_final_early(D):
    """The reading behind the reverse chunk order: visiting chunks D-1 .. 0, the input-gradient
    rows of chunk i (and so its dK/dV rows) are final as soon as chunk i is done, because only
    chunks j >= i attend to its keys.  Checked against the unchunked backward; the reverse sum
    itself equals it too."""
    cfg = tiny_cfg()
    W = tiny_weights(cfg, seed=21, bias=True)
    rng = np.random.default_rng(22)
    B, T = 2, 12
    x = rng.standard_normal((B, T, cfg.d_model))
    dy = rng.standard_normal((B, T, cfg.d_model))
    dx0, g0 = O.decoder_layer_backward(cfg, W, x, dy)
    rel = lambda a, b: np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
    for b in range(B):
        dx = np.zeros((T, cfg.d_model))
        for (s, e) in reversed(O.chunk_bounds(T, D)):
            _, cache = O.layer_forward_rows(cfg, W, x[b, :e], s)
            dxp, _ = O.layer_backward_rows(cfg, W, cache, dy[b, s:e])
            dx[:e] += dxp
            assert rel(dx[s:e], dx0[b, s:e]) <= 1e-12, (b, s, e)
        assert rel(dx, dx0[b]) <= 1e-12


# ------------------------------------------------------------------------------------------
# LM head + CE
# ------------------------------------------------------------------------------------------
def test_lmhead_loss_matches_library_cross_entropy():
    rng = np.random.default_rng(13)
    N, d, V = 11, 6, 17
    h = rng.standard_normal((N, d))
    W = rng.standard_normal((V, d))
    y = rng.integers(0, V, N)
    y[3] = -1
    w = rng.random(N)
    w[3] = 0.0
    loss, _, _, lse = O.lmhead_ce_forward_backward(h, W, y, w)
    z = torch.from_numpy(h @ W.T)
    ce = torch.nn.functional.cross_entropy(z, torch.from_numpy(y), reduction="none",
                                           ignore_index=-1).numpy()
    assert np.isclose(loss, np.sum(w * ce), rtol=1e-13)
    assert np.allclose(lse, torch.logsumexp(z, 1).numpy(), rtol=1e-14)


def test_lmhead_dlogits_closed_form():
    """With hidden = identity rows, d_weight^T is d loss / d logits = w (softmax - onehot)."""
    rng = np.random.default_rng(14)
    d = V = 9
    h = np.eye(d)
    W = rng.standard_normal((V, d))
    y = rng.integers(0, V, d)
    w = rng.random(d)
    _, _, dW, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    z = torch.from_numpy(h @ W.T)
    closed = (torch.softmax(z, 1) - torch.nn.functional.one_hot(torch.from_numpy(y), V)).numpy()
    assert np.allclose(dW.T, w[:, None] * closed, rtol=1e-13, atol=1e-15)


def test_lmhead_special_cases():
    rng = np.random.default_rng(15)
    N, d, V = 7, 5, 13
    h = rng.standard_normal((N, d))
    y = rng.integers(0, V, N)
    w = rng.random(N)
    loss, dH, dW, _ = O.lmhead_ce_forward_backward(h, np.zeros((V, d)), y, w)
    assert np.isclose(loss, math.log(V) * w.sum(), rtol=1e-14)
    assert np.all(dH == 0.0)
    onehot = np.eye(V)[y]
    assert np.allclose(dW, (w[:, None] * (1.0 / V - onehot)).T @ h, rtol=1e-13)
    loss1, dH1, dW1, _ = O.lmhead_ce_forward_backward(h, rng.standard_normal((1, d)),
                                                      np.zeros(N, int), w)
    assert loss1 == 0.0 and np.all(dH1 == 0) and np.all(dW1 == 0)


def test_lmhead_finite_differences_and_chunks():
    rng = np.random.default_rng(16)
    N, d, V = 10, 6, 11
    h = rng.standard_normal((N, d))
    W = rng.standard_normal((V, d))
    y = rng.integers(0, V, N)
    w = rng.standard_normal(N)            # GRPO-style weights may be negative
    loss, dH, dW, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    f = lambda: O.lmhead_ce_forward_backward(h, W, y, w)[0]
    _fd_check(f, h, [(i, j) for i in range(0, N, 3) for j in range(0, d, 2)], dH)
    _fd_check(f, W, [(i, j) for i in range(0, V, 3) for j in range(0, d, 2)], dW)
    for D in (1, 3, 10):
        l2, dH2, dW2 = O.lmhead_ce_backward_chunked(h, W, y, w, D)
        assert np.isclose(l2, loss, rtol=1e-13)
        assert np.allclose(dH2, dH, rtol=1e-13, atol=1e-15)
        assert np.allclose(dW2, dW, rtol=1e-13, atol=1e-15)
    with pytest.raises(ValueError):
        O.lmhead_ce_forward_backward(h, W, np.full(N, -1), w)


# ------------------------------------------------------------------------------------------
# Loss weights (objective normalisers folded into w) against library losses
# ------------------------------------------------------------------------------------------
def test_sft_and_grpo_weights_reproduce_library_objectives():
    rng = np.random.default_rng(17)
    B, T, V, d = 3, 20, 13, 5
    h = rng.standard_normal((B * T, d))
    W = rng.standard_normal((V, d))
    ids = rng.integers(0, V, (B, T))
    z = torch.from_numpy(h @ W.T)
    logp = torch.log_softmax(z, 1).numpy().reshape(B, T, V)
    # SFT, loss tokens t >= floor(0.3 T)
    y = rng.integers(0, V, (B, T))
    w = synth.loss_weights("sft_from", B, T, from_frac=0.3)
    loss, *_ = O.lmhead_ce_forward_backward(h, W, y.reshape(-1), w.reshape(-1).astype(np.float64))
    t0 = int(np.floor(0.3 * T))
    ref = torch.nn.functional.cross_entropy(z.reshape(B, T, V)[:, t0:].reshape(-1, V),
                                            torch.from_numpy(y[:, t0:].reshape(-1)))
    assert np.isclose(loss, ref.item(), rtol=1e-6)       # w is stored in fp32
    # GRPO: -mean over response tokens of A_s * log p(next token)
    A = rng.standard_normal(B)
    ys = synth.shifted_targets(ids)
    w = synth.loss_weights("grpo", B, T, prompt_len=6, advantages=A)
    loss, *_ = O.lmhead_ce_forward_backward(h, W, ys.reshape(-1), w.reshape(-1).astype(np.float64))
    terms = [A[b] * logp[b, t, ys[b, t]] for b in range(B) for t in range(5, T - 1)]
    assert np.isclose(loss, -np.mean(terms), rtol=1e-6)


# ------------------------------------------------------------------------------------------
# Stack
# ------------------------------------------------------------------------------------------
def test_stack_finite_differences_and_chunks():
    cfg = tiny_cfg(H=2, Hkv=1, hd=4, d=8, f=12)
    rng = np.random.default_rng(18)
    V, B, T = 10, 1, 6
    layers = [tiny_weights(cfg, seed=19 + i, std=0.4) for i in range(2)]
    E = rng.standard_normal((V, cfg.d_model))
    fg = 1 + 0.1 * rng.standard_normal(cfg.d_model)
    lm = 0.5 * rng.standard_normal((V, cfg.d_model))
    ids = rng.integers(0, V, (B, T))
    ys = synth.shifted_targets(ids)
    w = synth.loss_weights("shifted_tail", B, T, from_frac=0.25).astype(np.float64)
    f = lambda: O.stack_forward_backward(cfg, E, layers, fg, lm, ids, ys, w)[0]
    loss, g = O.stack_forward_backward(cfg, E, layers, fg, lm, ids, ys, w)
    _fd_check(f, lm, [(1, 2), (4, 0), (ys[0, 3], 5)], g["lm_head"])
    _fd_check(f, fg, [(0,), (3,)], g["final_g"])
    _fd_check(f, E, [(ids[0, 0], 1), (ids[0, 4], 6)], g["embed"])
    _fd_check(f, layers[0]["wq"], [(1, 1), (5, 3)], g["layers"][0]["wq"])
    _fd_check(f, layers[1]["w_down"], [(2, 2)], g["layers"][1]["w_down"])
    for D in (2, 3):
        loss2, g2 = O.stack_forward_backward(cfg, E, layers, fg, lm, ids, ys, w, num_chunks=D)
        assert np.isclose(loss2, loss, rtol=1e-13)
        assert np.allclose(g2["embed"], g["embed"], rtol=1e-11, atol=1e-14)
        assert np.allclose(g2["layers"][0]["wk"], g["layers"][0]["wk"], rtol=1e-11, atol=1e-14)


# ---------------------------------------------------------------------------------------------
# DPO (the third objective the pages name; the standard DPO loss is the reading taken)
def test_dpo_policy_equal_to_reference_closed_form():
    """Delta = 0 for every pair: loss = ln 2 and w = +-beta / (2P) on the response tokens."""
    rng = np.random.default_rng(40)
    P, T, beta = 3, 5, 0.3
    ce = np.abs(rng.standard_normal(2 * P * T))
    m = (rng.random(2 * P * T) > 0.3).astype(np.float64)
    ref = -(m * ce).reshape(2 * P, T).sum(1)
    loss, w, logp = O.dpo_objective(ce, m, ref, beta, P, T)
    assert np.isclose(loss, np.log(2.0), rtol=1e-15)
    sign = np.repeat(np.tile([1.0, -1.0], P), T)
    assert np.allclose(w, m * sign * beta / (2 * P), rtol=1e-15, atol=0)
    assert np.allclose(logp, ref, rtol=1e-15)


def test_dpo_swapping_roles_changes_loss_by_mean_beta_delta():
    """softplus(x) - softplus(-x) = x: exchanging chosen and rejected raises the loss by
    mean_p(beta Delta_p); sigmoid(x) + sigmoid(-x) = 1: the weights of a token before and after
    the exchange have opposite signs and magnitudes adding up to beta / P."""
    rng = np.random.default_rng(41)
    P, T, beta = 4, 3, 0.7
    ce = np.abs(rng.standard_normal(2 * P * T))
    m = np.ones(2 * P * T)
    ref = rng.standard_normal(2 * P) - 5.0
    loss, w, logp = O.dpo_objective(ce, m, ref, beta, P, T)
    perm = np.arange(2 * P).reshape(P, 2)[:, ::-1].reshape(-1)
    loss_s, w_s, _ = O.dpo_objective(ce.reshape(2 * P, T)[perm].reshape(-1), m,
                                     ref[perm], beta, P, T)
    delta = (logp[0::2] - ref[0::2]) - (logp[1::2] - ref[1::2])
    assert np.isclose(loss_s - loss, np.mean(beta * delta), rtol=1e-12)
    ws = w_s.reshape(2 * P, T)[perm]
    wo = w.reshape(2 * P, T)
    assert np.all(np.sign(ws) == -np.sign(wo))
    assert np.allclose(np.abs(ws) + np.abs(wo), beta / P, rtol=1e-14)


def test_dpo_gradient_finite_differences_through_lm_head():
    """The weights w_t = dloss/dCE_t turn the LM-head backward into the DPO gradient: dH and
    dW from lmhead_ce_forward_backward(h, W, y, w) match central differences of the DPO loss."""
    rng = np.random.default_rng(42)
    P, T, d, V, beta = 2, 3, 4, 7, 0.5
    N = 2 * P * T
    h = rng.standard_normal((N, d))
    W = rng.standard_normal((V, d))
    y = rng.integers(0, V, N)
    m = np.ones(N)
    m[0::T] = 0.0                                    # first token of each sequence: prompt
    ref = rng.standard_normal(2 * P) - 4.0

    def loss_of():
        return O.dpo_objective(O.lmhead_token_ce(h, W, y, m), m, ref, beta, P, T)[0]

    _, w, _ = O.dpo_objective(O.lmhead_token_ce(h, W, y, m), m, ref, beta, P, T)
    _, dH, dW, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    _fd_check(loss_of, h, [(1, 0), (4, 3), (7, 2), (11, 1)], dH)
    _fd_check(loss_of, W, [(y[2], 1), (0, 0), (5, 3)], dW)


def test_stack_dpo_finite_differences_and_chunks():
    cfg = tiny_cfg(H=2, Hkv=1, hd=4, d=8, f=12)
    rng = np.random.default_rng(43)
    V, P, T, beta = 10, 1, 6, 0.4
    layers = [tiny_weights(cfg, seed=44)]
    E = rng.standard_normal((V, cfg.d_model))
    fg = 1 + 0.1 * rng.standard_normal(cfg.d_model)
    lm = 0.5 * rng.standard_normal((V, cfg.d_model))
    ids = rng.integers(0, V, (2 * P, T))
    ys = synth.shifted_targets(ids)
    m = np.zeros((2 * P, T))
    m[:, 2:T - 1] = 1.0                              # response predictions (last has no target)
    ref = np.array([-9.0, -11.0])
    f = lambda: O.stack_dpo(cfg, E, layers, fg, lm, ids, ys, m, ref, beta)[0]
    loss, g, w = O.stack_dpo(cfg, E, layers, fg, lm, ids, ys, m, ref, beta)
    _fd_check(f, lm, [(ys[0, 3], 1), (2, 5)], g["lm_head"])
    _fd_check(f, layers[0]["wv"], [(1, 2), (3, 7)], g["layers"][0]["wv"])
    _fd_check(f, E, [(ids[1, 1], 0)], g["embed"])
    loss2, g2, _ = O.stack_dpo(cfg, E, layers, fg, lm, ids, ys, m, ref, beta, num_chunks=3)
    assert np.isclose(loss2, loss, rtol=1e-15)
    assert np.allclose(g2["layers"][0]["wq"], g["layers"][0]["wq"], rtol=1e-11, atol=1e-14)


# ------------------------------------------------------------------------------------------
# The hand-written chain rule against reverse-mode autograd: a torch fp64 forward written here
# from the definition (RMSNorm, projections with bias, rotate-half RoPE at absolute positions,
# causal GQA softmax attention, residual, SwiGLU MLP; embedding, final RMSNorm, untied LM head,
# sum_t w_t CE_t), differentiated by torch.autograd.  Agreement to 1e-10 catches terms too
# small for finite differences to see.
# ------------------------------------------------------------------------------------------
def _t(a):
    return None if a is None else torch.tensor(np.asarray(a, np.float64), requires_grad=True)


def _torch_layer(cfg, Wt, x):
    B, T, d = x.shape
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim

    def rms(v, g):
        return v * torch.rsqrt((v * v).mean(-1, keepdim=True) + cfg.rms_eps) * g

    def lin(v, w, b):
        out = v @ w.T
        return out if b is None else out + b

    n1 = rms(x, Wt["ln1_g"])
    q = lin(n1, Wt["wq"], Wt["bq"]).reshape(B, T, H, hd)
    k = lin(n1, Wt["wk"], Wt["bk"]).reshape(B, T, Hkv, hd)
    v = lin(n1, Wt["wv"], Wt["bv"]).reshape(B, T, Hkv, hd)
    half = hd // 2
    inv = cfg.rope_theta ** (-(2.0 * torch.arange(half, dtype=torch.float64)) / hd)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * inv[None, :]
    ang = torch.cat([ang, ang], dim=1)
    cos, sin = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]

    def rot(u):
        return u * cos + torch.cat([-u[..., half:], u[..., :half]], dim=-1) * sin

    q, k = rot(q), rot(k)
    k = k.repeat_interleave(H // Hkv, dim=2)
    v = v.repeat_interleave(H // Hkv, dim=2)
    s = torch.einsum("bthd,buhd->bhtu", q, k) / math.sqrt(hd)
    future = torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1)
    p = torch.softmax(s.masked_fill(future, float("-inf")), dim=-1)
    a = torch.einsum("bhtu,buhd->bthd", p, v).reshape(B, T, H * hd)
    h = x + a @ Wt["wo"].T
    n2 = rms(h, Wt["ln2_g"])
    g = n2 @ Wt["w_gate"].T
    return h + (g * torch.sigmoid(g) * (n2 @ Wt["w_up"].T)) @ Wt["w_down"].T


def _rel(a, b):
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("bias", [True, False])
def test_layer_backward_matches_autograd(bias):
    cfg = tiny_cfg(H=4, Hkv=2, hd=8, d=16, f=24)
    W = tiny_weights(cfg, seed=31, bias=bias)
    rng = np.random.default_rng(32)
    x = rng.standard_normal((2, 11, cfg.d_model))
    dy = rng.standard_normal((2, 11, cfg.d_model))
    dx0, g0 = O.decoder_layer_backward(cfg, W, x, dy)
    Wt = {n: _t(W.get(n)) for n in O.WEIGHT_NAMES}
    xt = _t(x)
    y = _torch_layer(cfg, Wt, xt)
    assert _rel(y.detach().numpy(), O.decoder_layer_forward(cfg, W, x)) <= 1e-12
    (y * torch.from_numpy(dy)).sum().backward()
    assert _rel(dx0, xt.grad.numpy()) <= 1e-10
    for n in O.WEIGHT_NAMES:
        if Wt[n] is not None:
            assert _rel(g0[n], Wt[n].grad.numpy()) <= 1e-10, n


def test_stack_backward_matches_autograd():
    cfg = tiny_cfg(H=4, Hkv=1, hd=4, d=16, f=20)
    rng = np.random.default_rng(33)
    B, T, V = 2, 9, 23
    layers = [tiny_weights(cfg, seed=34 + i, bias=(i == 0)) for i in range(2)]
    E = rng.standard_normal((V, cfg.d_model))
    fg = 1.0 + 0.2 * rng.standard_normal(cfg.d_model)
    lm = 0.5 * rng.standard_normal((V, cfg.d_model))
    ids = rng.integers(0, V, (B, T))
    targets = np.concatenate([ids[:, 1:], -np.ones((B, 1), np.int64)], axis=1)
    w = np.where(targets >= 0, rng.standard_normal((B, T)), 0.0)     # signed, GRPO-like
    loss0, g0 = O.stack_forward_backward(cfg, E, layers, fg, lm, ids, targets, w)
    Et, fgt, lmt = _t(E), _t(fg), _t(lm)
    Lt = [{n: _t(W.get(n)) for n in O.WEIGHT_NAMES} for W in layers]
    x = Et[torch.from_numpy(ids)]
    for Wt in Lt:
        x = _torch_layer(cfg, Wt, x)
    hf = x * torch.rsqrt((x * x).mean(-1, keepdim=True) + cfg.rms_eps) * fgt
    z = (hf @ lmt.T).reshape(B * T, V)
    y = torch.from_numpy(np.where(targets >= 0, targets, 0).reshape(-1))
    ce = torch.logsumexp(z, dim=-1) - z[torch.arange(B * T), y]
    loss = (torch.from_numpy(w.reshape(-1)) * ce).sum()
    loss.backward()
    lt = float(loss.detach())
    assert abs(loss0 - lt) <= 1e-12 * max(1.0, abs(lt))
    assert _rel(g0["lm_head"], lmt.grad.numpy()) <= 1e-10
    assert _rel(g0["final_g"], fgt.grad.numpy()) <= 1e-10
    assert _rel(g0["embed"], Et.grad.numpy()) <= 1e-10
    for i, Wt in enumerate(Lt):
        for n in O.WEIGHT_NAMES:
            if Wt[n] is not None:
                assert _rel(g0["layers"][i][n], Wt[n].grad.numpy()) <= 1e-10, (i, n)

"""fp64 CPU oracle for StreamBP's streamed exact backward (decoder layer + LM-head CE).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may call it.  It shares no code with the CUDA library (no kernels, headers,
tables or helpers); the two meet only through the seeded input generators, which hold none
of the method's arithmetic.

Sources (web pages on StreamBP, arXiv 2506.03077):
  [skill]  "StreamBP: Memory-Efficient Backpropagation" (skillsmp.com skill page), sections
           Core Concept, Architecture Overview, Implementation, Practical Guidance, Reference.
  [paper]  "StreamBP: Memory-Efficient Exact Backpropagation for Long Sequence Training of
           LLMs" (tomesphere.com), sections TL;DR, Findings, Abstract.

What is computed.  [paper] Abstract: StreamBP is an *exact* backward pass obtained by a
layer-wise linear decomposition of the chain rule along the sequence dimension.  Because the
method reaches, up to rounding order, the plain unchunked backward, the oracle is that plain
definition written out (functions without ``chunked`` in their name) plus a literal chunked
loop (``*_chunked``) that is used only to show that the decomposition changes nothing.

Readings of the pages where they are silent or garbled:
  * nn.Linear layout y = x W^T, W[out, in] ([skill] Implementation writes y = x W; the
    gradients are the same up to a transpose).
  * Rotate-half RoPE with absolute positions, inv_freq_j = theta^(-2j/hd); angles in fp64.
  * RMSNorm y = x / sqrt(mean(x^2) + eps) * gamma.  SiLU(x) = x * sigmoid(x).  Softmax scale
    1/sqrt(hd), no dropout.  GQA: query head h reads KV head floor(h / (H / Hkv)).
  * One global loss normaliser folded into per-token loss weights w_t (loss = sum_t w_t CE_t)
    instead of the sketch's per-chunk 1/(end - start) in its chunked CE ([skill]
    Implementation), which would contradict "identical to full BP" ([skill] Architecture
    Overview, Exact Gradients).
  * Chunk-i queries attend to the whole causal prefix [0, e_i) ([skill] Architecture Overview,
    Causal Structure Exploitation; Practical Guidance, Chunk Size Boundaries); the sketch's
    recompute of the layer on the chunk alone is right only for token-wise layers.

Everything here is float64 numpy; inputs given as bf16-rounded values are upcast exactly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------------------------
# A1: chunk decomposition.  [skill] Implementation, decompose_sequence: chunk = T // D,
# chunk i covers [i*chunk, (i+1)*chunk) and the last chunk takes the remainder.
# ----------------------------------------------------------------------------------------------
def chunk_bounds(seq_len: int, num_chunks: int) -> List[Tuple[int, int]]:
    if num_chunks < 1 or num_chunks > seq_len:
        raise ValueError("need 1 <= num_chunks <= seq_len")
    size = seq_len // num_chunks
    out = []
    for i in range(num_chunks):
        start = i * size
        end = (i + 1) * size if i < num_chunks - 1 else seq_len
        out.append((start, end))
    return out


# ----------------------------------------------------------------------------------------------
# Token-wise pieces of a Llama/Qwen decoder layer (the layer the pages train; [skill] Reference
# names Qwen 3, [paper] Abstract names transformer LLMs).  Each forward has a hand-derived
# backward; the pins in tests/ check them by central finite differences.
# ----------------------------------------------------------------------------------------------
def rmsnorm_forward(x: np.ndarray, gamma: np.ndarray, eps: float):
    """y = x * r * gamma with r = (mean_j x_j^2 + eps)^(-1/2) per row.  Returns (y, r)."""
    x = np.asarray(x, F64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(gamma, F64), r[..., 0]


def rmsnorm_backward(dy: np.ndarray, x: np.ndarray, gamma: np.ndarray, r: np.ndarray):
    """Chain rule of rmsnorm_forward.

    With u = gamma * dy and xhat = x * r:  dx = r * u - xhat * r * mean_j(xhat_j u_j),
    dgamma = sum over rows of dy * xhat.  Linear in dy.
    """
    x = np.asarray(x, F64)
    dy = np.asarray(dy, F64)
    r = np.asarray(r, F64)[..., None]
    xhat = x * r
    u = dy * np.asarray(gamma, F64)
    dx = r * u - xhat * r * np.mean(xhat * u, axis=-1, keepdims=True)
    dgamma = np.sum((dy * xhat).reshape(-1, x.shape[-1]), axis=0)
    return dx, dgamma


def rope_tables(positions: np.ndarray, head_dim: int, theta: float):
    """cos/sin tables [len(positions), head_dim] for rotate-half RoPE, angles in fp64."""
    half = head_dim // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=F64)) / head_dim)
    ang = np.asarray(positions, F64)[:, None] * inv_freq[None, :]
    ang = np.concatenate([ang, ang], axis=1)
    return np.cos(ang), np.sin(ang)


def _rotate_half(x):
    half = x.shape[-1] // 2
    return np.concatenate([-x[..., half:], x[..., :half]], axis=-1)


def rope_forward(x: np.ndarray, cos: np.ndarray, sin: np.ndarray):
    """x [..., T, heads, hd]; pair (j, j + hd/2) is rotated by angle pos * inv_freq_j."""
    c = cos[:, None, :]
    s = sin[:, None, :]
    return x * c + _rotate_half(x) * s


def rope_backward(dy: np.ndarray, cos: np.ndarray, sin: np.ndarray):
    """Transpose of rope_forward (the rotation is orthogonal, so this is also its inverse)."""
    c = cos[:, None, :]
    s = sin[:, None, :]
    t = dy * s
    half = dy.shape[-1] // 2
    rt = np.concatenate([t[..., half:], -t[..., :half]], axis=-1)
    return dy * c + rt


def silu(x):
    return x / (1.0 + np.exp(-x))


def swiglu_backward(dm, g, u):
    """m = silu(g) * u  ->  (dg, du)."""
    sg = 1.0 / (1.0 + np.exp(-g))
    dsilu = sg * (1.0 + g * (1.0 - sg))
    return dm * u * dsilu, dm * g * sg


# ----------------------------------------------------------------------------------------------
# Causal GQA attention over a key prefix.  Queries are rows [q_start, q_start + Tq) of the
# sequence, keys are rows [0, Tk).  Query at absolute position t sees keys u <= t.
# ----------------------------------------------------------------------------------------------
def attention_forward(q, k, v, q_start: int = 0):
    """q [Tq, H, hd], k/v [Tk, Hkv, hd] -> (out [Tq, H, hd], p [H, Tq, Tk])."""
    Tq, H, hd = q.shape
    Tk, Hkv, _ = k.shape
    group = H // Hkv
    kk = np.repeat(k, group, axis=1)          # head h -> kv head h // group
    vv = np.repeat(v, group, axis=1)
    s = np.einsum("thd,uhd->htu", q, kk) / math.sqrt(hd)
    tpos = q_start + np.arange(Tq)[:, None]
    upos = np.arange(Tk)[None, :]
    s = np.where(upos <= tpos, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    p = e / np.sum(e, axis=-1, keepdims=True)
    out = np.einsum("htu,uhd->thd", p, vv)
    return out, p


def attention_logsumexp(q, k, q_start: int = 0):
    """Log of the softmax normaliser of each causal score row, lse [Tq, H]:
    lse[t, h] = log sum_{u <= q_start + t} exp(q_t,h . k_u,g / sqrt(hd)), g = h // (H / Hkv).
    The statistic a flash-style attention keeps from its forward so that the backward can
    rebuild P = exp(S - lse) ([skill] Architecture Overview: the forward is recomputed per
    chunk and its statistics reused by that chunk's backward)."""
    Tq, H, hd = q.shape
    Tk, Hkv, _ = k.shape
    kk = np.repeat(k, H // Hkv, axis=1)
    s = np.einsum("thd,uhd->htu", q, kk) / math.sqrt(hd)
    s = np.where(np.arange(Tk)[None, :] <= q_start + np.arange(Tq)[:, None], s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    return (m[..., 0] + np.log(np.sum(np.exp(s - m), axis=-1))).T


def attention_backward(dout, q, k, v, p):
    """Chain rule of attention_forward.  Returns (dq, dk, dv) with dk/dv summed per KV head."""
    Tq, H, hd = q.shape
    Tk, Hkv, _ = k.shape
    group = H // Hkv
    kk = np.repeat(k, group, axis=1)
    vv = np.repeat(v, group, axis=1)
    dvv = np.einsum("htu,thd->uhd", p, dout)
    dp = np.einsum("thd,uhd->htu", dout, vv)
    ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
    scale = 1.0 / math.sqrt(hd)
    dq = np.einsum("htu,uhd->thd", ds, kk) * scale
    dkk = np.einsum("htu,thd->uhd", ds, q) * scale
    dk = dkk.reshape(Tk, Hkv, group, hd).sum(axis=2)
    dv = dvv.reshape(Tk, Hkv, group, hd).sum(axis=2)
    return dq, dk, dv


# ----------------------------------------------------------------------------------------------
# Decoder layer: pre-norm attention block + pre-norm SwiGLU MLP, nn.Linear weight layout.
# ----------------------------------------------------------------------------------------------
@dataclass
class LayerConfig:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    rms_eps: float
    rope_theta: float


WEIGHT_NAMES = ("ln1_g", "wq", "wk", "wv", "bq", "bk", "bv", "wo", "ln2_g", "w_gate", "w_up",
                "w_down")


def _lin(x, w, b=None):
    y = x @ np.asarray(w, F64).T
    if b is not None:
        y = y + np.asarray(b, F64)
    return y


def layer_forward_rows(cfg: LayerConfig, W: Dict[str, np.ndarray], x_prefix: np.ndarray,
                       q_start: int):
    """Forward of one sequence's layer for query rows [q_start, Tk) with keys/values from all
    rows [0, Tk) of ``x_prefix`` ([Tk, d]).  Returns (y_rows, cache)."""
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    Tk = x_prefix.shape[0]
    x_prefix = np.asarray(x_prefix, F64)
    n1, r1 = rmsnorm_forward(x_prefix, W["ln1_g"], cfg.rms_eps)
    cos, sin = rope_tables(np.arange(Tk), hd, cfg.rope_theta)
    k_pre = _lin(n1, W["wk"], W.get("bk")).reshape(Tk, Hkv, hd)
    v = _lin(n1, W["wv"], W.get("bv")).reshape(Tk, Hkv, hd)
    k = rope_forward(k_pre, cos, sin)
    rows = slice(q_start, Tk)
    x = x_prefix[rows]
    q_pre = _lin(n1[rows], W["wq"], W.get("bq")).reshape(Tk - q_start, H, hd)
    q = rope_forward(q_pre, cos[rows], sin[rows])
    a, p = attention_forward(q, k, v, q_start)
    a2 = a.reshape(Tk - q_start, H * hd)
    h = x + _lin(a2, W["wo"])
    n2, r2 = rmsnorm_forward(h, W["ln2_g"], cfg.rms_eps)
    g = _lin(n2, W["w_gate"])
    u = _lin(n2, W["w_up"])
    m = silu(g) * u
    y = h + _lin(m, W["w_down"])
    cache = dict(x_prefix=x_prefix, n1=n1, r1=r1, cos=cos, sin=sin, k=k, v=v, q=q, p=p, a2=a2,
                 h=h, n2=n2, r2=r2, g=g, u=u, m=m, q_start=q_start)
    return y, cache


def layer_backward_rows(cfg: LayerConfig, W: Dict[str, np.ndarray], cache, dy_rows: np.ndarray,
                        sum_scales: Optional[Dict[str, np.ndarray]] = None):
    """Backward of layer_forward_rows for upstream dy on the query rows.

    Returns (dx_prefix [Tk, d], grads dict).  Gradient flows to earlier rows only through the
    attention keys/values (the causal prefix).  If ``sum_scales`` is given, the column sums of
    the absolute summands of the bias gradients (sum_t |dq_pre|, |dk_pre|, |dv|) are added to
    it: the scale against which the rounding error of those sums is measured (the bias
    gradients are sums with heavy cancellation: without RoPE, sum_t dk_t is exactly 0 because
    softmax is invariant to a shift shared by all keys)."""
    H, Hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    c = cache
    Tk = c["x_prefix"].shape[0]
    qs = c["q_start"]
    rows = slice(qs, Tk)
    Tq = Tk - qs
    dy = np.asarray(dy_rows, F64)
    grads: Dict[str, np.ndarray] = {}
    # MLP: y = h + m W_d^T
    dm = dy @ np.asarray(W["w_down"], F64)
    grads["w_down"] = dy.T @ c["m"]
    dg, du = swiglu_backward(dm, c["g"], c["u"])
    dn2 = dg @ np.asarray(W["w_gate"], F64) + du @ np.asarray(W["w_up"], F64)
    grads["w_gate"] = dg.T @ c["n2"]
    grads["w_up"] = du.T @ c["n2"]
    dh_norm, grads["ln2_g"] = rmsnorm_backward(dn2, c["h"], W["ln2_g"], c["r2"])
    dh = dy + dh_norm
    # attention output projection: h = x + a W_o^T
    da2 = dh @ np.asarray(W["wo"], F64)
    grads["wo"] = dh.T @ c["a2"]
    da = da2.reshape(Tq, H, hd)
    dq, dk, dv = attention_backward(da, c["q"], c["k"], c["v"], c["p"])
    dq_pre = rope_backward(dq, c["cos"][rows], c["sin"][rows]).reshape(Tq, H * hd)
    dk_pre = rope_backward(dk, c["cos"], c["sin"]).reshape(Tk, Hkv * hd)
    dv = dv.reshape(Tk, Hkv * hd)
    n1 = c["n1"]
    dn1 = dk_pre @ np.asarray(W["wk"], F64) + dv @ np.asarray(W["wv"], F64)
    dn1[rows] += dq_pre @ np.asarray(W["wq"], F64)
    grads["wq"] = dq_pre.T @ n1[rows]
    grads["wk"] = dk_pre.T @ n1
    grads["wv"] = dv.T @ n1
    grads["bq"] = dq_pre.sum(axis=0)
    grads["bk"] = dk_pre.sum(axis=0)
    grads["bv"] = dv.sum(axis=0)
    if sum_scales is not None:
        for k, v in (("bq", dq_pre), ("bk", dk_pre), ("bv", dv)):
            sum_scales[k] = sum_scales.get(k, 0.0) + np.abs(v).sum(axis=0)
    dx, grads["ln1_g"] = rmsnorm_backward(dn1, c["x_prefix"], W["ln1_g"], c["r1"])
    dx[rows] += dh
    return dx, grads


def _zero_grads(cfg: LayerConfig, W) -> Dict[str, np.ndarray]:
    return {k: np.zeros(np.shape(W[k]) if W.get(k) is not None else _bias_shape(cfg, k), F64)
            for k in WEIGHT_NAMES}


def _bias_shape(cfg: LayerConfig, name: str):
    return {"bq": (cfg.n_heads * cfg.head_dim,), "bk": (cfg.n_kv_heads * cfg.head_dim,),
            "bv": (cfg.n_kv_heads * cfg.head_dim,)}[name]


def decoder_layer_forward(cfg: LayerConfig, W, x):
    """x [B, T, d] -> y [B, T, d] (plain, unchunked)."""
    x = np.asarray(x, F64)
    return np.stack([layer_forward_rows(cfg, W, x[b], 0)[0] for b in range(x.shape[0])])


def decoder_layer_backward(cfg: LayerConfig, W, x, dy, sum_scales=None):
    """Plain (unchunked) backward of the layer: returns (dx [B,T,d], grads).  This is the
    'full BP' that StreamBP must reproduce exactly ([skill] Architecture Overview, Exact
    Gradients; [paper] Abstract).  ``sum_scales``: see layer_backward_rows."""
    x = np.asarray(x, F64)
    dy = np.asarray(dy, F64)
    grads = _zero_grads(cfg, W)
    dx = np.zeros_like(x)
    for b in range(x.shape[0]):
        _, cache = layer_forward_rows(cfg, W, x[b], 0)
        dxb, gb = layer_backward_rows(cfg, W, cache, dy[b], sum_scales)
        dx[b] = dxb
        for k in grads:
            grads[k] += gb[k]
    return dx, grads


def decoder_layer_backward_chunked(cfg: LayerConfig, W, x, dy, num_chunks: int):
    """The StreamBP loop, written literally ([skill] Implementation, the streamed layer
    backward; [paper] Abstract, linear decomposition of the chain rule along the sequence).

    For each chunk i = [s_i, e_i): recompute the layer forward for query rows [s_i, e_i) over
    the causal prefix [0, e_i), backpropagate the chunk's slice of the upstream gradient, and
    add its contribution to every gradient (weights, and input rows of the whole prefix).
    Only the chunk's activations live at any time; gradients accumulate.  Used to show that
    the decomposition is exact (D-invariance), not by the product path."""
    x = np.asarray(x, F64)
    dy = np.asarray(dy, F64)
    grads = _zero_grads(cfg, W)
    dx = np.zeros_like(x)
    for b in range(x.shape[0]):
        for (s, e) in chunk_bounds(x.shape[1], num_chunks):
            _, cache = layer_forward_rows(cfg, W, x[b, :e], s)
            dxp, gb = layer_backward_rows(cfg, W, cache, dy[b, s:e])
            dx[b, :e] += dxp
            for k in grads:
                grads[k] += gb[k]
    return dx, grads


# ----------------------------------------------------------------------------------------------
# LM head + cross-entropy.  loss = sum_t w_t * (logsumexp(z_t) - z_t[y_t]), z = h W^T.
# [skill] Implementation, chunked CE gradient: d loss / d z_t = w_t * (softmax(z_t) - onehot(y_t)).
# ----------------------------------------------------------------------------------------------
def lmhead_ce_forward_backward(hidden, weight, targets, loss_weights):
    """hidden [N, d], weight [V, d], targets [N] (int; < 0 = ignored, needs w = 0),
    loss_weights [N].  Returns (loss, d_hidden [N, d], d_weight [V, d], lse [N])."""
    h = np.asarray(hidden, F64)
    W = np.asarray(weight, F64)
    y = np.asarray(targets, np.int64)
    w = np.asarray(loss_weights, F64)
    if np.any((y < 0) & (w != 0)):
        raise ValueError("ignored target with nonzero loss weight")
    z = h @ W.T
    zmax = np.max(z, axis=1, keepdims=True)
    lse = (zmax + np.log(np.sum(np.exp(z - zmax), axis=1, keepdims=True)))[:, 0]
    yy = np.where(y >= 0, y, 0)
    z_y = z[np.arange(len(y)), yy]
    ce = np.where(w != 0, lse - z_y, 0.0)
    loss = float(np.sum(w * ce))
    G = np.exp(z - lse[:, None])
    G[np.arange(len(y)), yy] -= 1.0
    G *= w[:, None]
    return loss, G @ W, G.T @ h, lse


def lmhead_ce_backward_chunked(hidden, weight, targets, loss_weights, num_chunks: int):
    """StreamBP's chunked LM-head backward: logits exist for one chunk of rows at a time and
    d_weight accumulates over chunks.  The normaliser is the global one carried in w."""
    N = np.shape(hidden)[0]
    loss = 0.0
    dH = np.zeros(np.shape(hidden), F64)
    dW = np.zeros(np.shape(weight), F64)
    for (s, e) in chunk_bounds(N, num_chunks):
        l_c, dh_c, dw_c, _ = lmhead_ce_forward_backward(hidden[s:e], weight, targets[s:e],
                                                        loss_weights[s:e])
        loss += l_c
        dH[s:e] = dh_c
        dW += dw_c
    return loss, dH, dW


# ----------------------------------------------------------------------------------------------
# A small stack: embedding -> L decoder layers -> final RMSNorm -> untied LM head -> sum w CE.
# ----------------------------------------------------------------------------------------------
def stack_forward_backward(cfg: LayerConfig, embed, layers, final_g, lm_w, ids, targets,
                           loss_weights, num_chunks: Optional[int] = None, store=None,
                           sum_scales: Optional[List[dict]] = None):
    """ids/targets/loss_weights [B, T].  Returns (loss, grads dict).  With ``num_chunks`` the
    layer and LM-head backwards use the chunked loops; otherwise the plain ones.  ``store``
    (optional): the storage format of the layer-input checkpoints and of the final-norm output
    (e.g. a rounding to bf16 when the model is kept in bf16), applied where they are stored;
    the arithmetic stays fp64.  ``sum_scales`` (optional list): receives one dict per layer
    with the absolute-summand scales of its bias gradients (unchunked mode; see
    layer_backward_rows)."""
    ids = np.asarray(ids, np.int64)
    B, T = ids.shape
    E = np.asarray(embed, F64)
    keep = store if store is not None else (lambda a: a)
    xs = [E[ids]]
    for W in layers:
        xs.append(keep(decoder_layer_forward(cfg, W, xs[-1])))
    hf, rf = rmsnorm_forward(xs[-1], final_g, cfg.rms_eps)
    hf = keep(hf)
    hflat = hf.reshape(B * T, -1)
    tflat = np.asarray(targets).reshape(-1)
    wflat = np.asarray(loss_weights, F64).reshape(-1)
    if num_chunks is None:
        loss, dhf, dlm, _ = lmhead_ce_forward_backward(hflat, lm_w, tflat, wflat)
    else:
        loss, dhf, dlm = 0.0, np.zeros_like(hflat), np.zeros(np.shape(lm_w), F64)
        for b in range(B):
            rs = slice(b * T, (b + 1) * T)
            l_b, dh_b, dw_b = lmhead_ce_backward_chunked(hflat[rs], lm_w, tflat[rs], wflat[rs],
                                                         num_chunks)
            loss += l_b
            dhf[rs] = dh_b
            dlm += dw_b
    grads = {"lm_head": dlm}
    dxl, grads["final_g"] = rmsnorm_backward(dhf.reshape(B, T, -1), xs[-1], final_g, rf)
    layer_grads = []
    for li in range(len(layers) - 1, -1, -1):
        if num_chunks is None:
            sc = {} if sum_scales is not None else None
            dxl, g = decoder_layer_backward(cfg, layers[li], xs[li], dxl, sc)
            if sum_scales is not None:
                sum_scales.insert(0, sc)
        else:
            dxl, g = decoder_layer_backward_chunked(cfg, layers[li], xs[li], dxl, num_chunks)
        layer_grads.append(g)
    grads["layers"] = layer_grads[::-1]
    dE = np.zeros_like(E)
    np.add.at(dE, ids.reshape(-1), dxl.reshape(B * T, -1))
    grads["embed"] = dE
    return loss, grads


# ----------------------------------------------------------------------------------------------
# DPO.  [paper] Abstract and [skill] Core Concept ("Multiple Objectives") and Practical
# Guidance ("Loss Objectives") name DPO among the objectives StreamBP serves; the pages give no
# formula.  Reading taken: the standard DPO objective on P pairs of sequences,
#     loss = (1/P) sum_p -log sigmoid(beta * Delta_p),
#     Delta_p = (logp(chosen_p) - ref(chosen_p)) - (logp(rejected_p) - ref(rejected_p)),
# where logp(seq) is the sum of the token log-probabilities (= -CE) over the response tokens
# (mask 1) and ref(.) are the reference model's sums, given.  Sequences are laid out
# [chosen_0, rejected_0, chosen_1, rejected_1, ...], seq_len tokens each.  Because loss depends
# on the network only through the per-token CE, its gradient is the gradient of sum_t w_t CE_t
# with w_t = dloss / dCE_t, which is what the streamed backward takes as loss weights.
# ----------------------------------------------------------------------------------------------
def lmhead_token_ce(hidden, weight, targets, mask):
    """Per-token cross-entropy lse(h W^T) - (h W^T)[y] [N]; 0 where mask == 0."""
    h = np.asarray(hidden, F64)
    W = np.asarray(weight, F64)
    y = np.asarray(targets, np.int64)
    m = np.asarray(mask, F64)
    if np.any((y < 0) & (m != 0)):
        raise ValueError("ignored target inside the mask")
    z = h @ W.T
    zmax = np.max(z, axis=1, keepdims=True)
    lse = (zmax + np.log(np.sum(np.exp(z - zmax), axis=1, keepdims=True)))[:, 0]
    z_y = z[np.arange(len(y)), np.where(y >= 0, y, 0)]
    return np.where(m != 0, lse - z_y, 0.0)


def _log_sigmoid(x):
    x = np.asarray(x, F64)
    return np.where(x >= 0, -np.log1p(np.exp(-x)), x - np.log1p(np.exp(x)))


def dpo_objective(token_ce, mask, ref_logp, beta: float, n_pairs: int, seq_len: int):
    """Returns (loss, w [2P*seq_len], seq_logp [2P]) with w_t = dloss / dCE_t."""
    ce = np.asarray(token_ce, F64).reshape(2 * n_pairs, seq_len)
    m = np.asarray(mask, F64).reshape(2 * n_pairs, seq_len)
    ref = np.asarray(ref_logp, F64).reshape(2 * n_pairs)
    logp = -np.sum(m * ce, axis=1)                       # sequence log-probabilities
    delta = (logp[0::2] - ref[0::2]) - (logp[1::2] - ref[1::2])
    loss = float(-np.mean(_log_sigmoid(beta * delta)))
    # d loss / d Delta_p = -(beta / P) sigmoid(-beta Delta_p); d Delta / d CE_t = -1 on the
    # chosen sequence's response tokens and +1 on the rejected one's
    coef = beta * np.exp(_log_sigmoid(-beta * delta)) / n_pairs
    sign = np.tile(np.array([1.0, -1.0]), n_pairs)       # chosen, rejected, ...
    w = m * (np.repeat(coef, 2) * sign)[:, None]
    return loss, w.reshape(-1), logp


def stack_dpo(cfg: LayerConfig, embed, layers, final_g, lm_w, ids, targets, mask, ref_logp,
              beta: float, num_chunks: Optional[int] = None, store=None):
    """DPO step on the small stack: forward for the sequence log-probabilities, the per-token
    weights, then the (optionally chunked) backward with those weights.  ids/targets/mask
    [2P, T].  ``store`` as in stack_forward_backward.  Returns (dpo loss, grads, w)."""
    ids = np.asarray(ids, np.int64)
    B, T = ids.shape
    E = np.asarray(embed, F64)
    keep = store if store is not None else (lambda a: a)
    x = E[ids]
    for W in layers:
        x = keep(decoder_layer_forward(cfg, W, x))
    hf, _ = rmsnorm_forward(x, final_g, cfg.rms_eps)
    hf = keep(hf)
    ce = lmhead_token_ce(hf.reshape(B * T, -1), lm_w, np.asarray(targets).reshape(-1),
                         np.asarray(mask).reshape(-1))
    loss, w, _ = dpo_objective(ce, mask, ref_logp, beta, B // 2, T)
    _, grads = stack_forward_backward(cfg, embed, layers, final_g, lm_w, ids, targets,
                                      w.reshape(B, T), num_chunks, store)
    return loss, grads, w

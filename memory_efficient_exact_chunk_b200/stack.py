"""Composition of a small decoder stack from libsbp calls: embedding -> L layers -> final
RMSNorm -> LM head + CE, then the streamed backward layer by layer.

The forward keeps only each layer's input (the layer-wise checkpoints StreamBP builds on;
skill page "StreamBP: Memory-Efficient Backpropagation", Core Concept and Architecture
Overview, Layer-Wise Application).  The backward runs the LM-head CE and every layer through
the streamed entry points with the same D.  Every arithmetic step runs in libsbp kernels; this
module only allocates buffers and orders the calls.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List

from . import sbp


@dataclass
class StackResult:
    loss: object                # device fp32 [1]
    grads: Dict[str, object]    # lm_head, final_g, embed, layers: List[dict]


class Workspaces:
    """Device buffers reused across calls (grown on demand)."""

    def __init__(self, device):
        self.device = device
        self.bufs = {}

    def get(self, name, nbytes):
        t = self.bufs.get(name)
        if t is None or t.numel() < nbytes:
            t = sbp.workspace(nbytes, self.device)
            self.bufs[name] = t
        return t


def stack_forward(cfg: sbp.LayerCfg, embed, layers: List[dict], final_g, ids, ws: Workspaces,
                  stream=None):
    """Embedding and L chunked layer forwards; returns the layer inputs (checkpoints), the
    final-norm output and its rstd."""
    import torch
    dev = embed.device
    N = cfg.batch * cfg.seq_len
    d = cfg.d_model
    xs = [torch.empty(N, d, dtype=embed.dtype, device=dev)]
    sbp.embedding_forward(ids, embed, xs[0], stream=stream)
    lws = ws.get("layer", sbp.layer_workspace_size(cfg))
    for W in layers:
        y = torch.empty(N, d, dtype=embed.dtype, device=dev)
        sbp.decoder_layer_forward(cfg, W, xs[-1], y, ws=lws, stream=stream)
        xs.append(y)
    hf = torch.empty(N, d, dtype=embed.dtype, device=dev)
    rstd = torch.empty(N, dtype=torch.float32, device=dev)
    sbp.rmsnorm_forward(xs[-1], final_g, cfg.rms_eps, hf, rstd, stream=stream)
    return xs, hf, rstd


def stack_backward_from(cfg: sbp.LayerCfg, layers: List[dict], final_g, lm_w, ids, targets,
                        loss_weights, xs, hf, rstd, ws: Workspaces, grads=None, stream=None,
                        on_final=None):
    """The streamed backward of the stack from its checkpoints.  `grads` (optional) holds fp32
    gradient buffers to accumulate into (the layout StackResult.grads uses); else fresh zeros.
    `on_final` (optional) is called with "head" once the LM-head and final-norm gradients are
    queued, "layer{l}" after layer l's backward and "embed" at the end: the points after which
    the work on the stream leaves that gradient unchanged."""
    import torch
    dev = hf.device
    N, d = hf.shape
    V = lm_w.shape[0]
    if grads is None:
        grads = zero_grads(layers, lm_w, final_g, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dhf = torch.empty(N, d, dtype=torch.float32, device=dev)
    cws = ws.get("lmhead", sbp.lmhead_ce_workspace_size(N, d, V, cfg.num_chunks,
                                                        sbp._dtype_code(hf)))
    sbp.lmhead_ce_backward(hf, lm_w, targets, loss_weights, cfg.num_chunks, loss, dhf,
                           grads["lm_head"], ws=cws, stream=stream)
    dx = torch.empty(N, d, dtype=torch.float32, device=dev)
    sbp.rmsnorm_backward(xs[-1], final_g, rstd, dhf, dx, grads["final_g"],
                         ws=ws.get("rms", 0), stream=stream)
    if on_final:
        on_final("head")
    lws = ws.get("layer", sbp.layer_workspace_size(cfg))
    dxn = dhf                                        # reuse the buffer: dhf is consumed
    for li in range(len(layers) - 1, -1, -1):
        sbp.decoder_layer_backward(cfg, layers[li], xs[li], dx, dxn, grads["layers"][li],
                                   ws=lws, stream=stream)
        if on_final:
            on_final(f"layer{li}")
        dx, dxn = dxn, dx
    sbp.embedding_backward(ids, dx, grads["embed"], ws=ws.get("embed", 0), stream=stream)
    if on_final:
        on_final("embed")
    return StackResult(loss, grads)


def zero_grads(layers, lm_w, final_g, dev, embed_shape=None):
    import torch
    g = {"lm_head": torch.zeros(lm_w.shape, dtype=torch.float32, device=dev),
         "final_g": torch.zeros(final_g.shape, dtype=torch.float32, device=dev),
         "layers": [{n: (torch.zeros(W[n].shape, dtype=torch.float32, device=dev)
                         if W.get(n) is not None else None) for n in sbp.WEIGHT_FIELDS}
                    for W in layers]}
    if embed_shape is not None:
        g["embed"] = torch.zeros(embed_shape, dtype=torch.float32, device=dev)
    return g


def stack_backward(cfg: sbp.LayerCfg, embed, layers: List[dict], final_g, lm_w, ids, targets,
                   loss_weights, stream=None, keep_workspace: dict | None = None) -> StackResult:
    """Forward (checkpoints only) and streamed backward of the whole stack.
    ids/targets int32 [B*T]; loss_weights fp32 [B*T]; weights on the device in cfg.dtype.
    Returns the loss and fp32 gradients (freshly zeroed, then accumulated by the library)."""
    ws = Workspaces(embed.device)
    if keep_workspace is not None:
        ws.bufs = keep_workspace
    xs, hf, rstd = stack_forward(cfg, embed, layers, final_g, ids, ws, stream=stream)
    grads = zero_grads(layers, lm_w, final_g, embed.device, embed_shape=embed.shape)
    return stack_backward_from(cfg, layers, final_g, lm_w, ids, targets, loss_weights, xs, hf,
                               rstd, ws, grads=grads, stream=stream)


def stack_dpo_step(cfg: sbp.LayerCfg, embed, layers: List[dict], final_g, lm_w, ids, targets,
                   response_mask, ref_logp, beta: float, ws: Workspaces, grads=None, stream=None):
    """One DPO step on 2P sequences laid out [chosen_0, rejected_0, ...] (include/sbp_dpo.h):
    the forward keeps the layer inputs, the streamed LM-head forward gives the per-token CE, the
    DPO loss and the per-token weights w_t = d loss / d CE_t follow, and the streamed backward
    runs with those weights.  response_mask [2P*T] fp32, ref_logp [2P] fp32 (device).  Returns
    the DPO loss (device [1]) and the fp32 gradients (accumulated into `grads` if given)."""
    import torch
    dev = embed.device
    B, T = cfg.batch, cfg.seq_len
    if B % 2:
        raise ValueError("DPO needs an even number of sequences (chosen, rejected pairs)")
    N = B * T
    xs, hf, rstd = stack_forward(cfg, embed, layers, final_g, ids, ws, stream=stream)
    V, d = lm_w.shape
    token_ce = torch.empty(N, dtype=torch.float32, device=dev)
    cws = ws.get("lmhead", sbp.lmhead_ce_workspace_size(N, d, V, cfg.num_chunks,
                                                        sbp._dtype_code(hf)))
    sbp.lmhead_ce_forward(hf, lm_w, targets, response_mask, cfg.num_chunks, token_ce, ws=cws,
                          stream=stream)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    w = torch.empty(N, dtype=torch.float32, device=dev)
    sbp.dpo_token_weights(B // 2, T, token_ce, response_mask, ref_logp, beta, loss, w,
                          ws=ws.get("dpo", sbp.dpo_workspace_size(B // 2)), stream=stream)
    if grads is None:
        grads = zero_grads(layers, lm_w, final_g, dev, embed_shape=embed.shape)
    r = stack_backward_from(cfg, layers, final_g, lm_w, ids, targets, w, xs, hf, rstd, ws,
                            grads=grads, stream=stream)
    return StackResult(loss, r.grads)

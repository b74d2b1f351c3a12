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


def stack_backward(cfg: sbp.LayerCfg, embed, layers: List[dict], final_g, lm_w, ids, targets,
                   loss_weights, stream=None, keep_workspace: dict | None = None) -> StackResult:
    """ids/targets int32 [B*T]; loss_weights fp32 [B*T]; weights on the device in cfg.dtype.
    Returns the loss and fp32 gradients (freshly zeroed, then accumulated by the library)."""
    import torch
    dev = embed.device
    B, T, d = cfg.batch, cfg.seq_len, cfg.d_model
    N = B * T
    V = lm_w.shape[0]
    wdt = embed.dtype
    ws_cache = keep_workspace if keep_workspace is not None else {}

    def ws(name, nbytes):
        t = ws_cache.get(name)
        if t is None or t.numel() < nbytes:
            t = sbp.workspace(nbytes, dev)
            ws_cache[name] = t
        return t

    lws = ws("layer", sbp.layer_workspace_size(cfg))
    # ---- forward: keep the input of every layer
    xs = [torch.empty(N, d, dtype=wdt, device=dev)]
    sbp.embedding_forward(ids, embed, xs[0], stream=stream)
    for W in layers:
        y = torch.empty(N, d, dtype=wdt, device=dev)
        sbp.decoder_layer_forward(cfg, W, xs[-1], y, ws=lws, stream=stream)
        xs.append(y)
    hf = torch.empty(N, d, dtype=wdt, device=dev)
    rstd = torch.empty(N, dtype=torch.float32, device=dev)
    sbp.rmsnorm_forward(xs[-1], final_g, cfg.rms_eps, hf, rstd, stream=stream)
    # ---- backward
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    dhf = torch.empty(N, d, dtype=torch.float32, device=dev)
    dlm = torch.zeros(V, d, dtype=torch.float32, device=dev)
    cws = ws("lmhead", sbp.lmhead_ce_workspace_size(N, d, V, cfg.num_chunks,
                                                    sbp._dtype_code(hf)))
    sbp.lmhead_ce_backward(hf, lm_w, targets, loss_weights, cfg.num_chunks, loss, dhf, dlm,
                           ws=cws, stream=stream)
    dfg = torch.zeros(d, dtype=torch.float32, device=dev)
    dx = torch.empty(N, d, dtype=torch.float32, device=dev)
    sbp.rmsnorm_backward(xs[-1], final_g, rstd, dhf, dx, dfg, ws=ws("rms", 0), stream=stream)
    layer_grads: List[dict] = [None] * len(layers)
    for li in range(len(layers) - 1, -1, -1):
        W = layers[li]
        g = {n: (torch.zeros(W[n].shape, dtype=torch.float32, device=dev)
                 if W.get(n) is not None else None) for n in sbp.WEIGHT_FIELDS}
        dxn = torch.empty(N, d, dtype=torch.float32, device=dev)
        sbp.decoder_layer_backward(cfg, W, xs[li], dx, dxn, g, ws=lws, stream=stream)
        layer_grads[li] = g
        dx = dxn
    dE = torch.zeros(embed.shape, dtype=torch.float32, device=dev)
    sbp.embedding_backward(ids, dx, dE, ws=ws("embed", 0), stream=stream)
    return StackResult(loss, {"lm_head": dlm, "final_g": dfg, "embed": dE,
                              "layers": layer_grads})

"""Device-memory model of a streamed training step of a decoder stack, and the longest sequence
that fits a memory budget at a given number of chunks D.

The pages' headline claim (paper page "StreamBP: Memory-Efficient Exact Backpropagation for
Long Sequence Training of LLMs", Abstract and Findings) is about memory: streaming the backward
over D sequence chunks lets backprop run on much longer sequences.  This module counts, byte by
byte, what stack.py keeps on the device during the streamed backward of an L-layer stack with
an untied LM head (one sequence of T tokens):

  resident, independent of T: bf16 weights and fp32 gradients (accumulated by the library);
  per token, independent of D: token ids, targets and loss weights, the layer-input
      checkpoints of the forward (L + 1 bf16 rows), the final-norm output (bf16) and its rstd,
      and the fp32 residual-stream gradients of the backward (two rows, dhf and dx);
  the library's workspaces, as the C ABI sizes them: the decoder layer's (per-chunk buffers,
      O(T / D), plus the K/V prefix and its fp32 gradient, O(T)), the LM head's (O(T / D):
      the logits never leave the chip), and the small ones of the embedding and RMSNorm
      backward.

Every workspace figure comes from the library's own *_workspace_size calls, which run on the
host (no GPU needed), so the model follows the library as it is built.  max_tokens() searches
the longest T whose total fits a budget.  The bench checks the model against
torch.cuda.max_memory_allocated on the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict

from . import sbp


@dataclass
class StackShape:
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 500000.0
    qkv_bias: bool = False

    @classmethod
    def from_workload(cls, wl):
        L = wl.layer
        return cls(wl.n_layers, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn, wl.vocab,
                   L.rms_eps, L.rope_theta, L.qkv_bias)

    def layer_params(self) -> int:
        d, dq, dkv, f = (self.d_model, self.n_heads * self.head_dim,
                         self.n_kv_heads * self.head_dim, self.ffn)
        p = 2 * d + dq * d + 2 * dkv * d + d * dq + 3 * f * d
        if self.qkv_bias:
            p += dq + 2 * dkv
        return p

    def params(self) -> int:
        return self.n_layers * self.layer_params() + 2 * self.vocab * self.d_model + self.d_model


def stack_step_bytes(shape: StackShape, T: int, D: int) -> Dict[str, int]:
    """Bytes live on the device during the streamed backward of one T-token sequence."""
    lib = sbp.load()
    d = shape.d_model
    cfg = sbp.layer_cfg(1, T, d, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.ffn,
                        shape.rms_eps, shape.rope_theta, sbp.SBP_BF16, D)
    layer_ws = sbp.layer_workspace_size(cfg)
    head_ws = sbp.lmhead_ce_workspace_size(T, d, shape.vocab, D, sbp.SBP_BF16)
    if layer_ws == 0 or head_ws == 0:
        raise ValueError(f"invalid sizes T={T} D={D}")
    out = {
        "weights_bf16": 2 * shape.params(),
        "grads_fp32": 4 * shape.params(),
        "inputs": 12 * T,                                     # ids, targets, loss weights
        "checkpoints": T * ((shape.n_layers + 2) * d * 2 + 4),  # layer inputs, final norm, rstd
        "residual_grads_fp32": 2 * T * d * 4,                  # dhf, dx
        "layer_workspace": layer_ws,
        "lmhead_workspace": head_ws,
        "small_workspaces": int(lib.sbp_embedding_backward_workspace_size(T, shape.vocab)) +
        int(lib.sbp_rmsnorm_backward_workspace_size(T, d)),
    }
    out["total"] = sum(out.values())
    return out


def transient_bytes(parts: Dict[str, int]) -> int:
    """What the streamed backward adds on top of weights, gradients, inputs and checkpoints."""
    return (parts["residual_grads_fp32"] + parts["layer_workspace"] + parts["lmhead_workspace"] +
            parts["small_workspaces"])


def max_tokens(shape: StackShape, D: int, budget_bytes: int, multiple: int = 128) -> int:
    """Longest T (a multiple of `multiple`, at least D) whose stack_step_bytes total fits the
    budget; 0 if none does.  The total grows with T, so a bisection finds it."""
    def fits(T):
        return stack_step_bytes(shape, T, D)["total"] <= budget_bytes

    lo = max(multiple, ((D + multiple - 1) // multiple) * multiple)
    if not fits(lo):
        return 0
    hi = lo
    while fits(hi):
        hi *= 2
        if hi > (1 << 31):
            return hi // 2
    while hi - lo > multiple:
        mid = ((lo + hi) // 2) // multiple * multiple
        if mid <= lo:
            break
        if fits(mid):
            lo = mid
        else:
            hi = mid
    return lo

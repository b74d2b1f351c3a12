"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds input generation only (random draws, bf16 rounding of those draws, loss
masks and per-token loss weights as the caller hands them to the library); none of the
backward arithmetic lives here.  Everything is numpy so that it imports without CUDA.

Workload shapes follow the long-sequence SFT / GRPO training runs of the StreamBP pages
(skill page "StreamBP: Memory-Efficient Backpropagation", Reference: Qwen models, long
sequences; paper page, Abstract: SFT and GRPO objectives).  The pages publish no dataset
items; these draws stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional

import numpy as np


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even), returned as fp32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of bf16-representable fp32 values (use after bf16_round)."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclass
class LayerShape:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    rms_eps: float
    rope_theta: float
    qkv_bias: bool = False


@dataclass
class Workload:
    name: str
    batch: int
    seq_len: int
    num_chunks: int
    dtype: str                      # "f32" or "bf16"
    layer: Optional[LayerShape] = None
    n_layers: int = 0
    vocab: int = 0
    hidden: int = 0                 # LM-head-only workloads
    loss: str = "sft_all"           # sft_all | sft_from | shifted_tail | grpo
    loss_from_frac: float = 0.0
    prompt_len: int = 0
    extra: Dict = field(default_factory=dict)


LLAMA3_8B = LayerShape(4096, 32, 8, 128, 14336, 1e-5, 500000.0)
QWEN25_7B = LayerShape(3584, 28, 4, 128, 18944, 1e-6, 1000000.0, qkv_bias=True)

WORKLOADS = {
    "tiny_stack_f32": Workload("tiny_stack_f32", 1, 256, 4, "f32",
                               LayerShape(64, 4, 4, 16, 172, 1e-6, 10000.0), 1, vocab=512,
                               loss="sft_all"),
    "lmhead_ce_32k": Workload("lmhead_ce_32k", 1, 32768, 8, "bf16", vocab=152064, hidden=3584,
                              loss="sft_from", loss_from_frac=0.3),
    "llama3_8b_layer_32k": Workload("llama3_8b_layer_32k", 1, 32768, 8, "bf16", LLAMA3_8B, 1),
    "llama3_8b_stack4_64k": Workload("llama3_8b_stack4_64k", 1, 65536, 16, "bf16", LLAMA3_8B,
                                     4, vocab=128256, loss="shifted_tail",
                                     loss_from_frac=0.25),
    "qwen25_7b_stack2_grpo": Workload("qwen25_7b_stack2_grpo", 8, 16384, 8, "bf16", QWEN25_7B,
                                      2, vocab=152064, loss="grpo", prompt_len=2048),
    # DPO on the same shapes: 4 (chosen, rejected) pairs of 16384 tokens, 2048-token prompts
    "qwen25_7b_stack2_dpo": Workload("qwen25_7b_stack2_dpo", 8, 16384, 8, "bf16", QWEN25_7B,
                                     2, vocab=152064, loss="dpo", prompt_len=2048,
                                     extra={"beta": 0.1}),
}


def normal(rng: np.random.Generator, shape, std: float, bf16: bool) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return bf16_round(a) if bf16 else a


def layer_weights(rng: np.random.Generator, L: LayerShape, bf16: bool, std: float = 0.02,
                  gamma_std: float = 0.0) -> Dict[str, Optional[np.ndarray]]:
    """Random-init weights in nn.Linear [out, in] layout; RMSNorm gains 1 (+ optional noise)."""
    d, dq, dkv, f = L.d_model, L.n_heads * L.head_dim, L.n_kv_heads * L.head_dim, L.ffn

    def gain():
        g = np.ones(d, np.float32)
        if gamma_std:
            g = g + rng.standard_normal(d, dtype=np.float32) * np.float32(gamma_std)
        return bf16_round(g) if bf16 else g

    W = {
        "ln1_g": gain(),
        "wq": normal(rng, (dq, d), std, bf16),
        "wk": normal(rng, (dkv, d), std, bf16),
        "wv": normal(rng, (dkv, d), std, bf16),
        "wo": normal(rng, (d, dq), std, bf16),
        "ln2_g": gain(),
        "w_gate": normal(rng, (f, d), std, bf16),
        "w_up": normal(rng, (f, d), std, bf16),
        "w_down": normal(rng, (d, f), std, bf16),
        "bq": None, "bk": None, "bv": None,
    }
    if L.qkv_bias:
        W["bq"] = normal(rng, (dq,), std, bf16)
        W["bk"] = normal(rng, (dkv,), std, bf16)
        W["bv"] = normal(rng, (dkv,), std, bf16)
    return W


def loss_weights(kind: str, batch: int, seq_len: int, *, from_frac: float = 0.0,
                 prompt_len: int = 0, advantages: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-token weights w [B, T] with the objective's normaliser folded in, so that the
    objective equals sum_t w_t * CE_t.

    sft_all      : mean CE over every token            w = 1 / (B T)
    sft_from     : mean CE over tokens t >= floor(from_frac T)  (prompt masked)
    shifted_tail : targets are the next token; loss tokens t in [floor(from_frac T), T - 2]
    grpo         : targets are the next token; response predictions t in [prompt_len - 1,
                   T - 2]; w = A_s / (number of response tokens in the batch), which makes
                   sum w CE = -mean(A * log p).
    """
    m = np.zeros((batch, seq_len), np.float64)
    if kind == "sft_all":
        m[:] = 1.0
    elif kind == "sft_from":
        m[:, int(np.floor(from_frac * seq_len)):] = 1.0
    elif kind == "shifted_tail":
        m[:, int(np.floor(from_frac * seq_len)):seq_len - 1] = 1.0
    elif kind == "grpo":
        m[:, prompt_len - 1:seq_len - 1] = 1.0
    else:
        raise ValueError(kind)
    n = m.sum()
    w = m / n
    if kind == "grpo":
        assert advantages is not None
        w = w * np.asarray(advantages, np.float64)[:, None]
    return w.astype(np.float32)


def token_ids(rng: np.random.Generator, batch: int, seq_len: int, vocab: int) -> np.ndarray:
    return rng.integers(0, vocab, size=(batch, seq_len), dtype=np.int64).astype(np.int32)


def shifted_targets(ids: np.ndarray) -> np.ndarray:
    """y_t = id_{t+1}; the last position has no target (-1)."""
    y = np.full_like(ids, -1)
    y[:, :-1] = ids[:, 1:]
    return y


def lmhead_inputs(seed: int, n_tokens: int, hidden: int, vocab: int, bf16: bool = True,
                  from_frac: float = 0.3, weight_std: float = 0.02):
    """Hidden states N(0,1) (an RMSNorm output), weight N(0, std), uniform targets, SFT mask."""
    rng = np.random.default_rng(seed)
    h = normal(rng, (n_tokens, hidden), 1.0, bf16)
    W = normal(rng, (vocab, hidden), weight_std, bf16)
    y = rng.integers(0, vocab, size=n_tokens, dtype=np.int64).astype(np.int32)
    w = loss_weights("sft_from", 1, n_tokens, from_frac=from_frac)[0]
    return h, W, y, w


def layer_inputs(seed: int, L: LayerShape, batch: int, seq_len: int, bf16: bool,
                 dy_std: float = 1e-3, gamma_std: float = 0.0):
    """Input hidden N(0,1), weights N(0,0.02), upstream gradient N(0, dy_std) (fp32)."""
    rng = np.random.default_rng(seed)
    W = layer_weights(rng, L, bf16, gamma_std=gamma_std)
    x = normal(rng, (batch, seq_len, L.d_model), 1.0, bf16)
    dy = rng.standard_normal((batch, seq_len, L.d_model), dtype=np.float32) * np.float32(dy_std)
    return W, x, dy

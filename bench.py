#!/usr/bin/env python
"""Benchmark of the streamed exact backward (StreamBP) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sbp|reference]
                    [--workload llama3_8b_stack4_64k|lmhead_ce_32k|llama3_8b_layer_32k]
                    [--chunks D] [--no-sweep] [--no-e2e] [--no-lmhead] [--no-layer] [--no-stack]

Default workload, the largest configuration that fits one GPU: a 4-layer Llama-3-8B-shaped
decoder stack (d 4096, 32 query / 8 KV heads of 128, SwiGLU 14336, RoPE theta 5e5) with an
untied LM head (vocabulary 128256), bf16 operands with fp32 accumulation, one 65536-token
sequence, next-token targets, mean CE over the last 75 % of tokens, D = 16.  One step = the
streamed backward of the whole stack from its layer-input checkpoints (LM-head CE, final norm,
four layers, embedding), all chunks.  Inputs are resident in HBM and larger than L2 (every
chunk re-reads each layer's weights and the LM-head weight), so no explicit L2 flush is used.
The line's `e2e` times the whole training step through the public API with the token data in
pinned host memory (copied in, forward + backward, loss read back).  Prints ONE JSON line on
rank 0; the LM-head workload (32K tokens, vocabulary 152064, D = 8), the single layer (32K
tokens, D = 8) and the GRPO / DPO stacks follow under `also`.

With N > 1 (torchrun, one process per GPU) every rank runs its own independent sequence
(weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "streamed backward tokens/s (1 B200) vs D; tensor-pipe % of peak; peak act. GB"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"sbp_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as fh:
            out = parse_clocks(fh)
        try:
            os.remove(self.path)
        except OSError:
            pass
        return out


def parse_clocks(lines):
    """Median SM clock, the maximum clock and the throttle reasons seen in nvidia-smi records
    of ClockSampler.FIELDS (csv, no header, no units); None without a usable record."""
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        f = [x.strip() for x in ln.split(",")]
        if len(f) < 9:
            continue
        try:
            clk, top = float(f[1]), float(f[2])
        except ValueError:
            continue
        sm.append(clk)
        mx = top
        for nm, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(nm)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


def fit_inverse_d(sweep):
    """Least-squares fit of the activation memory against D: workspace_gb ~ a / D + b.  a is
    the part that shrinks with the chunk (O(T/D)), b the part that does not (for the layer,
    the K/V prefix and the fp32 dK/dV accumulators)."""
    if not sweep or len(sweep) < 2:
        return None
    x = np.array([1.0 / r["D"] for r in sweep])
    y = np.array([r["workspace_gb"] for r in sweep])
    A = np.stack([x, np.ones_like(x)], 1)
    (a, b), *_ = np.linalg.lstsq(A, y, rcond=None)
    res = y - A @ np.array([a, b])
    return {"a_gb": float(a), "b_gb": float(b),
            "max_abs_residual_gb": float(np.max(np.abs(res)))}


# ----------------------------------------------------------------------------- workloads
def lmhead_workload(T):
    from memory_efficient_exact_chunk_b200 import synth
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    return wl, T or wl.seq_len


def sources_hash(rel_paths) -> str:
    """First 16 hex digits of the sha256 over the files (repo-relative paths, in order)."""
    h = hashlib.sha256()
    for rel in rel_paths:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(key: str):
    """DRAM bytes per launch of the kernel `key` recorded in profiles/traffic.json (the figure
    of an ncu capture summarised in profiles/), or None if the sources it was captured on have
    changed since (the entry stores their hash, and literal lines that fix the launch shapes,
    such as the vocabulary block of the LM head, which must still be present)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        ent = json.load(fh).get(key)
    if not ent:
        return None
    try:
        if sources_hash(ent["sources"]) != ent["sources_sha256_16"]:
            return None
        for rel, line in ent.get("requires", []):
            with open(os.path.join(ROOT, rel)) as fh:
                if line not in fh.read():
                    return None
    except OSError:
        return None
    return float(ent["dram_bytes_per_launch"])


def run_lmhead(args, rank, world, device):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, synth
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    T, d, V = (args.tokens or wl.seq_len), wl.hidden, wl.vocab
    D = (args.chunks if args.workload == "lmhead_ce_32k" else 0) or wl.num_chunks
    h, W, y, w = synth.lmhead_inputs(1000 + rank, T, d, V, bf16=True, from_frac=wl.loss_from_frac)
    n_valid = int(np.count_nonzero(w))
    hd = torch.from_numpy(h).to(torch.bfloat16).to(device)
    Wd = torch.from_numpy(W).to(torch.bfloat16).to(device)
    del W
    yd = torch.from_numpy(y).to(device)
    wd = torch.from_numpy(w).to(device)
    loss = torch.zeros(1, device=device)
    dH = torch.empty(T, d, device=device)
    dW = torch.zeros(V, d, device=device)
    torch.cuda.synchronize()
    resident = torch.cuda.memory_allocated(device)

    def make_ws(Dc):
        return sbp.workspace(sbp.lmhead_ce_workspace_size(T, d, V, Dc, sbp.SBP_BF16), device)

    ws = make_ws(D)
    step = lambda: sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW, ws=ws)
    flops_step = 8.0 * n_valid * d * V          # executed design: lse pass + 3 products
    flops_min = 6.0 * n_valid * d * V           # logits + dH + dW
    res = timed(args, step, world, device, profile=True)
    sbp.device_status(ws)
    torch.cuda.reset_peak_memory_stats(device)
    step()
    torch.cuda.synchronize()
    peak_alloc = torch.cuda.max_memory_allocated(device)
    out = {
        "tokens_per_step": T, "world": world, "n_loss_tokens": n_valid, "flops_step": flops_step,
        "flops_min_step": flops_min, "res": res, "ws_bytes": ws.numel(),
        "peak_act_gb": (peak_alloc - resident) / 1e9, "D": D,
        "config": {"workload": "lmhead_ce_32k" if T == wl.seq_len else f"lmhead_ce_{T}",
                   "batch": 1, "seq_len": T, "hidden": d,
                   "vocab": V, "num_chunks": D, "loss_mask": "first 30% of tokens",
                   "n_loss_tokens": n_valid,
                   "l2": "inputs larger than L2 (1.09 GB LM-head weight re-read per chunk)"},
    }
    # ---- D sweep (tokens/s and workspace vs D)
    if args.sweep and rank == 0 and world == 1:
        sweep = []
        for Dc in (1, 2, 4, 8, 16):
            wsc = make_ws(Dc)
            stepc = lambda: sbp.lmhead_ce_backward(hd, Wd, yd, wd, Dc, loss, dH, dW, ws=wsc)
            r = timed(argparse.Namespace(steps=2, warmup=1), stepc, 1, device, profile=False)
            sweep.append({"D": Dc, "tokens_per_s": T / (r["ms"] / 1e3),
                          "ms_per_step": r["ms"], "workspace_gb": wsc.numel() / 1e9})
            del wsc
        out["sweep"] = sweep
        out["memory_fit"] = fit_inverse_d(sweep)
    # ---- end to end through the C ABI from pinned host buffers
    if args.e2e:
        hh = torch.from_numpy(h).to(torch.bfloat16).pin_memory()
        yh = torch.from_numpy(y).pin_memory()
        wh = torch.from_numpy(w).pin_memory()
        lh = torch.zeros(1).pin_memory()
        stream = torch.cuda.current_stream(device)

        wsh = sbp.workspace(sbp.lmhead_ce_workspace_size_host(T, d, V, D, sbp.SBP_BF16), device)

        def e2e_step():
            # the public entry for host-resident inputs: the library stages each chunk's rows
            # while the previous chunk computes; the loss is read back
            sbp.lmhead_ce_backward_host(hh, Wd, yh, wh, D, loss, dH, dW, ws=wsh, stream=stream)
            lh.copy_(loss, non_blocking=True)

        r = timed(args, e2e_step, world, device, profile=False)
        out["e2e"] = {"value": T * world / (r["ms"] / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": hh.numel() * 2 + yh.numel() * 4 + wh.numel() * 4,
                      "d2h_bytes_per_step": 4}
    return out


def run_layer(args, rank, world, device, sweep=False):
    """One Llama-3-8B-shaped decoder layer (d 4096, 32/8 heads of 128, MLP 14336, theta 5e5),
    bf16, T = 32768, D = 8: one step = one sbp_decoder_layer_backward_stream call."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, synth
    wl = synth.WORKLOADS["llama3_8b_layer_32k"]
    L = wl.layer
    B, T = wl.batch, (args.layer_tokens or wl.seq_len)
    D = args.layer_chunks or wl.num_chunks
    W, x, dy = synth.layer_inputs(2000 + rank, L, B, T, bf16=True, dy_std=1e-3)
    names = sbp.WEIGHT_FIELDS
    Wd = {n: (torch.from_numpy(W[n]).to(torch.bfloat16).to(device) if W.get(n) is not None
              else None) for n in names}
    P = sum(int(np.prod(W[n].shape)) for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up",
                                              "w_down"))
    del W
    xd = torch.from_numpy(x).to(torch.bfloat16).to(device)
    dyd = torch.from_numpy(dy).to(device)
    del x, dy
    dx = torch.empty(B, T, L.d_model, device=device)
    grads = {n: (torch.zeros(Wd[n].shape, device=device) if Wd.get(n) is not None else None)
             for n in names}
    torch.cuda.synchronize()
    resident = torch.cuda.memory_allocated(device)

    def cfg_for(Dc):
        return sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn,
                             L.rms_eps, L.rope_theta, sbp.SBP_BF16, Dc)

    cfg = cfg_for(D)
    ws = sbp.workspace(sbp.layer_workspace_size(cfg), device)
    step = lambda: sbp.decoder_layer_backward(cfg, Wd, xd, dyd, dx, grads, ws=ws)
    lin_flops = 6.0 * P * B * T
    att_flops = 14.0 * L.head_dim * L.n_heads * B * T * (T + 1) / 2
    largs = argparse.Namespace(steps=max(1, min(args.steps, 3)), warmup=args.warmup)
    res = timed(largs, step, world, device, profile=True)
    sbp.device_status(ws)
    torch.cuda.reset_peak_memory_stats(device)
    step()
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated(device) - resident
    prof = res["prof"]
    k = largs.steps

    def tf(flops, ms):
        return flops * k / (ms / 1e3) / 1e12 if ms > 0 else None

    out = {
        "workload": "llama3_8b_layer_32k" if T == wl.seq_len else f"llama3_8b_layer_{T}",
        "value": B * T * world / (res["ms"] / 1e3), "unit": "tokens/s",
        "ms_per_step": res["ms"], "steps": k, "num_chunks": D,
        "config": {"batch": B, "seq_len": T, "d_model": L.d_model, "n_heads": L.n_heads,
                   "n_kv_heads": L.n_kv_heads, "head_dim": L.head_dim, "ffn": L.ffn,
                   "num_chunks": D, "linear_params": P},
        "flops_step": {"linear_6P": lin_flops, "attention_14hd": att_flops},
        "achieved_tflops_step": (lin_flops + att_flops) / (res["ms"] / 1e3) / 1e12,
        "kernels": {n: {"launches_per_step": v["launches"] / k, "ms_per_step": v["ms"] / k,
                        "busy_ms_per_step": v["busy_ms"] / k,
                        "share": v["busy_ms"] / res["ms_total"] if res["ms_total"] else None}
                    for n, v in prof.items() if v["launches"]},
        "gemm_tc_tflops": tf(lin_flops, prof["gemm_tc"]["busy_ms"]),
        "attn_tflops": tf(att_flops, prof["attn_fwd"]["busy_ms"] + prof["attn_bwd"]["busy_ms"]),
        "attn_fwd_tflops": tf(4.0 / 14.0 * att_flops, prof["attn_fwd"]["busy_ms"]),
        "attn_bwd_tflops": tf(10.0 / 14.0 * att_flops, prof["attn_bwd"]["busy_ms"]),
        "gpu_launches": res["launches"], "clocks": res["clocks"],
        "peak_act_gb": peak / 1e9, "workspace_gb": ws.numel() / 1e9,
    }
    # the same step with the chunks in reverse order (K/V prefix first, K/V projection
    # backward fused into each chunk's iteration)
    rstep = lambda: sbp.decoder_layer_backward_reverse(cfg, Wd, xd, dyd, dx, grads, ws=ws)
    rr = timed(largs, rstep, world, device, profile=True)
    sbp.device_status(ws)
    out["reverse_order"] = {
        "value": B * T * world / (rr["ms"] / 1e3), "unit": "tokens/s", "ms_per_step": rr["ms"],
        "steps": k, "num_chunks": D, "gpu_launches": rr["launches"], "clocks": rr["clocks"],
        "kernels": {n: {"launches_per_step": v["launches"] / k,
                        "busy_ms_per_step": v["busy_ms"] / k}
                    for n, v in rr["prof"].items() if v["launches"]},
    }
    if sweep and rank == 0 and world == 1:
        sw = []
        for Dc in (1, 2, 4, 8, 16):
            c2 = cfg_for(Dc)
            del ws
            torch.cuda.empty_cache()
            ws = sbp.workspace(sbp.layer_workspace_size(c2), device)
            st2 = lambda: sbp.decoder_layer_backward(c2, Wd, xd, dyd, dx, grads, ws=ws)
            r = timed(argparse.Namespace(steps=1, warmup=1), st2, 1, device, profile=False)
            sw.append({"D": Dc, "tokens_per_s": B * T / (r["ms"] / 1e3), "ms_per_step": r["ms"],
                       "workspace_gb": ws.numel() / 1e9})
        out["sweep"] = sw
        out["memory_fit"] = fit_inverse_d(sw)
    return out


def run_dpo_stack(args, rank, world, device, name="qwen25_7b_stack2_dpo"):
    """A DPO step on the Qwen2.5-7B-shaped 2-layer stack: 4 (chosen, rejected) pairs of 16384
    tokens (2048-token prompts), D = 8, beta 0.1.  One step = forward (layer-input checkpoints),
    streamed LM-head forward for the sequence log-probabilities, DPO loss and weights, streamed
    backward; all of it is timed.  The reference log-probabilities are the policy's own plus
    N(0, 1) per sequence (computed once before timing)."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, stack, synth
    wl = synth.WORKLOADS[name]
    L, B, T, V, D = wl.layer, wl.batch, wl.seq_len, wl.vocab, wl.num_chunks
    beta = float(wl.extra["beta"])
    gen = torch.Generator(device=device).manual_seed(4000 + rank)

    def rnd(*shape):
        return (torch.randn(*shape, generator=gen, device=device) * 0.02).to(torch.bfloat16)

    d, dq, dkv, f = L.d_model, L.n_heads * L.head_dim, L.n_kv_heads * L.head_dim, L.ffn
    layers = [{"ln1_g": torch.ones(d, dtype=torch.bfloat16, device=device),
               "wq": rnd(dq, d), "wk": rnd(dkv, d), "wv": rnd(dkv, d), "wo": rnd(d, dq),
               "ln2_g": torch.ones(d, dtype=torch.bfloat16, device=device),
               "w_gate": rnd(f, d), "w_up": rnd(f, d), "w_down": rnd(d, f),
               "bq": rnd(dq), "bk": rnd(dkv), "bv": rnd(dkv)} for _ in range(wl.n_layers)]
    embed, lm_w = rnd(V, d), rnd(V, d)
    final_g = torch.ones(d, dtype=torch.bfloat16, device=device)
    rng = np.random.default_rng(4000 + rank)
    ids = synth.token_ids(rng, B, T, V)
    y = synth.shifted_targets(ids)
    m = np.zeros((B, T), np.float32)
    m[:, wl.prompt_len - 1:T - 1] = 1.0
    ids_d = torch.from_numpy(ids.reshape(-1)).to(device)
    y_d = torch.from_numpy(y.reshape(-1)).to(device)
    m_d = torch.from_numpy(m.reshape(-1)).to(device)
    cfg = sbp.layer_cfg(B, T, d, L.n_heads, L.n_kv_heads, L.head_dim, f, L.rms_eps, L.rope_theta,
                        sbp.SBP_BF16, D)
    ws = stack.Workspaces(device)
    grads = stack.zero_grads(layers, lm_w, final_g, device, embed_shape=embed.shape)
    # reference = the policy's sequence log-probabilities + N(0, 1)
    xs, hf, _ = stack.stack_forward(cfg, embed, layers, final_g, ids_d, ws)
    ce = torch.empty(B * T, device=device)
    sbp.lmhead_ce_forward(hf, lm_w, y_d, m_d, D, ce)
    logp = -(m_d * ce).view(B, T).sum(1)
    ref = (logp + torch.randn(B, generator=gen, device=device)).float().contiguous()
    del xs, hf
    state = {}

    def step():
        state["r"] = stack.stack_dpo_step(cfg, embed, layers, final_g, lm_w, ids_d, y_d, m_d, ref,
                                          beta, ws, grads=grads)

    r = timed(argparse.Namespace(steps=1, warmup=args.warmup), step, world, device,
              profile=True)
    P = sum(int(layers[0][n].numel()) for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up",
                                                "w_down"))
    n_loss = int(m.sum())
    fwd_lin = 2.0 * P * B * T * wl.n_layers
    lin = 6.0 * P * B * T * wl.n_layers
    att = (14.0 + 4.0) * L.head_dim * L.n_heads * B * T * (T + 1) / 2 * wl.n_layers
    head = (8.0 + 2.0) * n_loss * d * V          # backward + the log-probability forward
    prof = r["prof"]
    return {
        "workload": wl.name, "value": B * T * world / (r["ms"] / 1e3), "unit": "tokens/s",
        "ms_per_step": r["ms"], "dpo_loss": float(state["r"].loss.item()),
        "config": {"batch": B, "pairs": B // 2, "seq_len": T, "n_layers": wl.n_layers,
                   "vocab": V, "num_chunks": D, "prompt_len": wl.prompt_len, "beta": beta,
                   "n_loss_tokens": n_loss},
        "flops_step": {"layers_forward_2P": fwd_lin, "layers_linear_6P": lin,
                       "layers_attention_18hd": att, "lmhead_10NdV": head},
        "achieved_tflops_step": (fwd_lin + lin + att + head) / (r["ms"] / 1e3) / 1e12,
        "kernels": {n: {"launches_per_step": v["launches"], "ms_per_step": v["ms"],
                        "busy_ms_per_step": v["busy_ms"],
                        "share": v["busy_ms"] / r["ms_total"] if r["ms_total"] else None}
                    for n, v in prof.items() if v["launches"]},
        "gpu_launches": r["launches"], "clocks": r["clocks"],
        "workspace_gb": sum(t.numel() for t in ws.bufs.values()) / 1e9,
    }


def run_stack(args, rank, world, device, name="llama3_8b_stack4_64k", steps=1, e2e=False):
    """A decoder stack + untied LM head, bf16, through the streamed entry points:
    llama3_8b_stack4_64k: four Llama-3-8B-shaped layers, vocabulary 128256, T = 65536, D = 16,
        targets = next token, mean CE over the last 75 % of tokens;
    qwen25_7b_stack2_grpo: two Qwen2.5-7B-shaped layers (QKV bias), vocabulary 152064,
        8 sequences of 16384 tokens, D = 8, GRPO loss (per-sequence advantage N(0, 1) over
        the response tokens after a 2048-token prompt).
    Weights are drawn on the device from a seeded generator (N(0, 0.02), gains 1).  The
    forward (layer-input checkpoints) and the streamed backward are timed separately; the
    metric is the backward (`steps` timed steps after args.warmup warm-ups).  With `e2e`, the
    whole training step is also timed through the public API from pinned host memory: the
    step's token ids, targets and loss weights are copied in, the forward and the streamed
    backward run, and the loss is read back."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp, stack, synth
    wl = synth.WORKLOADS[name]
    L, B, V = wl.layer, wl.batch, wl.vocab
    T = (args.stack_tokens or wl.seq_len) if name.startswith("llama") else wl.seq_len
    D = (args.chunks or wl.num_chunks) if args.workload == name else wl.num_chunks
    gen = torch.Generator(device=device).manual_seed(3000 + rank)

    def rnd(*shape):
        return (torch.randn(*shape, generator=gen, device=device) * 0.02).to(torch.bfloat16)

    d, dq, dkv, f = L.d_model, L.n_heads * L.head_dim, L.n_kv_heads * L.head_dim, L.ffn
    layers = []
    for _ in range(wl.n_layers):
        bias = L.qkv_bias
        layers.append({"ln1_g": torch.ones(d, dtype=torch.bfloat16, device=device),
                       "wq": rnd(dq, d), "wk": rnd(dkv, d), "wv": rnd(dkv, d), "wo": rnd(d, dq),
                       "ln2_g": torch.ones(d, dtype=torch.bfloat16, device=device),
                       "w_gate": rnd(f, d), "w_up": rnd(f, d), "w_down": rnd(d, f),
                       "bq": rnd(dq) if bias else None, "bk": rnd(dkv) if bias else None,
                       "bv": rnd(dkv) if bias else None})
    embed = rnd(V, d)
    lm_w = rnd(V, d)
    final_g = torch.ones(d, dtype=torch.bfloat16, device=device)
    rng = np.random.default_rng(3000 + rank)
    ids = synth.token_ids(rng, B, T, V)
    y = synth.shifted_targets(ids)
    if wl.loss == "grpo":
        adv = rng.standard_normal(B)
        w = synth.loss_weights("grpo", B, T, prompt_len=wl.prompt_len, advantages=adv)
    else:
        w = synth.loss_weights("shifted_tail", B, T, from_frac=wl.loss_from_frac)
    n_loss = int(np.count_nonzero(w))
    ids_d = torch.from_numpy(ids.reshape(-1)).to(device)
    y_d = torch.from_numpy(y.reshape(-1)).to(device)
    w_d = torch.from_numpy(w.reshape(-1)).to(device)
    cfg = sbp.layer_cfg(B, T, d, L.n_heads, L.n_kv_heads, L.head_dim, f, L.rms_eps,
                        L.rope_theta, sbp.SBP_BF16, D)
    ws = stack.Workspaces(device)
    grads = stack.zero_grads(layers, lm_w, final_g, device, embed_shape=embed.shape)
    state = {}

    def fwd():
        state["ck"] = stack.stack_forward(cfg, embed, layers, final_g, ids_d, ws)

    def bwd():
        xs, hf, rstd = state["ck"]
        state["r"] = stack.stack_backward_from(cfg, layers, final_g, lm_w, ids_d, y_d, w_d, xs,
                                               hf, rstd, ws, grads=grads)

    torch.cuda.synchronize(device)
    base = torch.cuda.memory_allocated(device)     # weights, gradients, inputs
    fwd()
    sargs = argparse.Namespace(steps=steps, warmup=args.warmup)
    rb = timed(sargs, bwd, world, device, profile=True)
    rf = timed(argparse.Namespace(steps=1, warmup=1), fwd, world, device, profile=False)
    torch.cuda.synchronize(device)
    torch.cuda.reset_peak_memory_stats(device)
    bwd()
    torch.cuda.synchronize(device)
    peak_total = torch.cuda.max_memory_allocated(device)
    xs, hf, rstd = state["ck"]
    ck = sum(t.numel() * t.element_size() for t in list(xs) + [hf, rstd])
    ws_gb = sum(t.numel() for t in ws.bufs.values()) / 1e9
    from memory_efficient_exact_chunk_b200 import memory_model as MM
    model = MM.stack_step_bytes(MM.StackShape.from_workload(wl), T, D) if B == 1 else None
    P = sum(int(layers[0][n].numel()) for n in ("wq", "wk", "wv", "wo", "w_gate", "w_up",
                                                "w_down"))
    pairs = B * T * (T + 1) / 2 * L.n_heads * wl.n_layers     # causal (query, key, head) pairs
    lin = 6.0 * P * B * T * wl.n_layers
    att = 14.0 * L.head_dim * pairs
    head = 8.0 * n_loss * d * V
    prof = rb["prof"]
    k = steps

    def tf(flops, ms):
        return flops * k / (ms / 1e3) / 1e12 if ms > 0 else None

    out = {
        "workload": wl.name if T == wl.seq_len and D == wl.num_chunks
        else f"{wl.name.rsplit('_', 1)[0]}_{T}_d{D}",
        "value": B * T * world / (rb["ms"] / 1e3), "unit": "tokens/s",
        "ms_per_step": rb["ms"], "steps": k, "forward_ms": rf["ms"],
        "fwd_bwd_tokens_per_s": B * T * world / ((rb["ms"] + rf["ms"]) / 1e3),
        "config": stack_config_dict(wl, T, D, n_loss),
        "flops_step": {"layers_linear_6P": lin, "layers_attention_14hd": att,
                       "lmhead_8NdV": head},
        "achieved_tflops_step": (lin + att + head) / (rb["ms"] / 1e3) / 1e12,
        "kernels": {n: {"launches_per_step": v["launches"] / k, "ms_per_step": v["ms"] / k,
                        "busy_ms_per_step": v["busy_ms"] / k,
                        "share": v["busy_ms"] / rb["ms_total"] if rb["ms_total"] else None}
                    for n, v in prof.items() if v["launches"]},
        "attn_bwd_flops_step": 10.0 * L.head_dim * pairs,
        "attn_fwd_flops_step": 4.0 * L.head_dim * pairs,
        "gemm_tc_tflops": tf(lin + head, prof["gemm_tc"]["busy_ms"]),
        "attn_fwd_tflops": tf(4.0 * L.head_dim * pairs, prof["attn_fwd"]["busy_ms"]),
        "attn_bwd_tflops": tf(10.0 * L.head_dim * pairs, prof["attn_bwd"]["busy_ms"]),
        "attn_bwd_busy_ms_total": prof["attn_bwd"]["busy_ms"],
        "attn_bwd_launches_per_step": prof["attn_bwd"]["launches"] / k,
        "gpu_launches": rb["launches"], "clocks": rb["clocks"],
        # transient memory of the streamed backward: its peak minus weights, gradients,
        # inputs and the forward's checkpoints
        "peak_act_gb": (peak_total - base - ck) / 1e9, "workspace_gb": ws_gb,
        "peak_total_gb": peak_total / 1e9, "checkpoints_gb": ck / 1e9,
        "model_total_gb": model["total"] / 1e9 if model else None,
        "model_transient_gb": MM.transient_bytes(model) / 1e9 if model else None,
    }
    if e2e:
        ids_h = torch.from_numpy(ids.reshape(-1)).pin_memory()
        y_h = torch.from_numpy(y.reshape(-1)).pin_memory()
        w_h = torch.from_numpy(w.reshape(-1)).pin_memory()
        loss_h = torch.zeros(1).pin_memory()

        def e2e_step():
            ids_d.copy_(ids_h, non_blocking=True)
            y_d.copy_(y_h, non_blocking=True)
            w_d.copy_(w_h, non_blocking=True)
            fwd()
            bwd()
            loss_h.copy_(state["r"].loss, non_blocking=True)

        # fewer timed steps than the device-resident timing: each e2e step also runs the
        # forward, and the whole bench should stay within a few minutes
        e2e_steps = min(steps, 8)
        re_ = timed(argparse.Namespace(steps=e2e_steps, warmup=args.warmup), e2e_step, world,
                    device, profile=False)
        out["e2e"] = {"value": B * T * world / (re_["ms"] / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": ids_h.numel() * 4 + y_h.numel() * 4 +
                      w_h.numel() * 4,
                      "d2h_bytes_per_step": 4,
                      "ms_per_step": re_["ms"], "steps": e2e_steps,
                      "what": "training step through the public API: token ids, targets and "
                              "loss weights copied from pinned host memory, forward "
                              "(layer-input checkpoints) + streamed backward on the device, "
                              "loss read back; weights and fp32 gradients stay resident in "
                              "HBM (a device-resident training step fed with host token data)"}
    return out


def max_over_ranks(ms: float, world: int) -> float:
    """The slowest rank's time (all ranks get it); plain value when there is one rank."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(args, step, world, device, profile):
    """W warm-up steps, then K timed steps between a barrier + synchronize on both sides;
    device time from CUDA events on the launching stream, max over ranks."""
    import torch
    import torch.distributed as dist
    from memory_efficient_exact_chunk_b200 import sbp
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    clk = ClockSampler(device.index or 0) if profile else None
    if clk:
        clk.start()
        time.sleep(0.3)
    n0 = sbp.launch_count()
    if profile:
        sbp.profile_begin()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        step()
    ev1.record()
    torch.cuda.synchronize(device)
    prof = sbp.profile_end() if profile else None
    launches = sbp.launch_count() - n0
    clocks = clk.stop() if clk else None
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        ms = max_over_ranks(ms, world)
        dist.barrier()
    return {"ms_total": ms, "ms": ms / args.steps, "prof": prof, "launches": launches,
            "clocks": clocks}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_lmhead_sample(n_rows: int, seed: int = 5):
    """The fp64 oracle on n_rows rows of the 32K workload's shapes (full hidden / vocab)."""
    from memory_efficient_exact_chunk_b200 import synth
    from oracle import sbp_oracle as O
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    h, W, y, w = synth.lmhead_inputs(seed, n_rows, wl.hidden, wl.vocab, bf16=True, from_frac=0.0)
    t0 = time.perf_counter()
    O.lmhead_ce_forward_backward(h, W, y, w)
    return time.perf_counter() - t0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(n_rows=2048):
    dt = sum(oracle_lmhead_sample(512, seed=5 + i) for i in range(n_rows // 512))
    return {"value": n_rows / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{n_rows} loss tokens of the 32K LM-head workload (hidden 3584, vocab "
                      f"152064), fp64 numpy, {dt:.1f} s"}


class OracleStackSample:
    """The fp64 oracle on a bounded sample of the 4-layer Llama-3-8B-shaped stack workload:
    one layer at full width (d 4096, 32/8 heads of 128, MLP 14336) on T_layer tokens (forward
    recompute + backward, as the streamed backward does per chunk), and the LM head at full
    width (vocabulary 128256) on `rows` loss rows.  Inputs are drawn once; run() times one pass
    and returns the stack's tokens/s implied by it: per token, four layers plus the LM head on
    the workload's share of loss tokens (75 %).  Attention is quadratic in T, so the reduced T
    understates the oracle's cost per token at 64K tokens."""

    def __init__(self, T_layer=512, rows=256, seed=7):
        from memory_efficient_exact_chunk_b200 import synth
        from oracle import sbp_oracle as O
        self.O = O
        wl = synth.WORKLOADS["llama3_8b_stack4_64k"]
        self.wl, L = wl, wl.layer
        self.T, self.rows = T_layer, rows
        W, x, dy = synth.layer_inputs(seed, L, 1, T_layer, bf16=True, dy_std=1e-3)
        self.W = {n: (None if v is None else v.astype(np.float64)) for n, v in W.items()}
        self.x, self.dy = x.astype(np.float64), dy.astype(np.float64)
        self.cfg = O.LayerConfig(L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn,
                                 L.rms_eps, L.rope_theta)
        self.h, self.Wh, self.y, self.w = synth.lmhead_inputs(seed, rows, L.d_model, wl.vocab,
                                                              bf16=True, from_frac=0.0)
        self.Wh = self.Wh.astype(np.float64)
        self.loss_share = 1.0 - wl.loss_from_frac

    def run(self):
        t0 = time.perf_counter()
        self.O.decoder_layer_backward(self.cfg, self.W, self.x, self.dy)
        t1 = time.perf_counter()
        self.O.lmhead_ce_forward_backward(self.h, self.Wh, self.y, self.w)
        t2 = time.perf_counter()
        per_token = (self.wl.n_layers * (t1 - t0) / self.T +
                     self.loss_share * (t2 - t1) / self.rows)
        return 1.0 / per_token, t2 - t0

    def describe(self):
        return (f"fp64 numpy oracle: one Llama-3-8B-shaped layer (forward + backward) on "
                f"{self.T} tokens and the 128256-word LM head on {self.rows} loss rows, both at "
                f"full width; tokens/s of the 4-layer stack + head implied per token "
                f"(4 x layer + {self.loss_share:.2f} x head)")


def cpu_baseline_stack():
    smp = OracleStackSample()
    smp.run()                                     # warm the BLAS threads
    vals, secs = [], 0.0
    while secs < 10.0 and len(vals) < 5:
        v, dt = smp.run()
        vals.append(v)
        secs += dt
    return {"value": statistics.median(vals), "unit": "tokens/s", "cores": cpu_cores(),
            "kind": "oracle", "sample": f"{smp.describe()}; median of {len(vals)} passes, "
                                        f"{secs:.1f} s"}


def stack_config_dict(wl, T, D, n_loss):
    """Shapes of a stack workload as the line's config reports them (both arms)."""
    L = wl.layer
    return {"batch": wl.batch, "seq_len": T, "n_layers": wl.n_layers, "d_model": L.d_model,
            "n_heads": L.n_heads, "n_kv_heads": L.n_kv_heads, "head_dim": L.head_dim,
            "ffn": L.ffn, "vocab": wl.vocab, "num_chunks": D, "n_loss_tokens": n_loss,
            "loss": wl.loss}


def stack_config(o):
    """The line's config for a stack workload (the same keys as the reference arm's)."""
    return dict(workload=o["workload"], **o["config"], l2=STACK_L2_NOTE)


STACK_L2_NOTE = ("inputs larger than L2 (each layer's 0.44 GB of weights and the 1.05 GB "
                 "LM-head weight are re-read per chunk)")


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores of rank 0, on a
    bounded sample of the 4-layer stack workload per step (the other ranks exit at once)."""
    if rank != 0:
        return 0
    from memory_efficient_exact_chunk_b200 import synth
    smp = OracleStackSample(T_layer=128, rows=64)
    wl = synth.WORKLOADS["llama3_8b_stack4_64k"]
    for _ in range(max(args.warmup, 1)):
        smp.run()
    t, vals = 0.0, []
    for _ in range(args.steps):
        v, dt = smp.run()
        vals.append(v)
        t += dt
    value = statistics.median(vals)
    w = synth.loss_weights("shifted_tail", wl.batch, wl.seq_len, from_frac=wl.loss_from_frac)
    cfg = dict(workload=wl.name, **stack_config_dict(wl, wl.seq_len, wl.num_chunks,
                                                     int(np.count_nonzero(w))), l2=STACK_L2_NOTE)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                         "kind": "oracle",
                         "sample": smp.describe() + " per step, on the host cores of rank 0 "
                                                    "(no GPU work)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def layer_main(args, rank, world, device):
    """The decoder-layer workload as the line's own workload (no LM head)."""
    import torch.distributed as dist
    peaks, peak_src = load_peaks()
    o = run_layer(args, rank, world, device, sweep=args.sweep)
    att = o["attn_tflops"] or 0.0
    line = {
        "metric": METRIC, "value": o["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": o["steps"], "warmup": args.warmup, "ms_per_step": o["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(workload=o["workload"], **o["config"]),
        "layer": o, "cpu_baseline": None,
        "roofline": {"bound": "tensor", "kernel": "attention backward + forward (tcgen05)",
                     "achieved": att, "peak": float(peaks["bf16_tflops_sustained"]),
                     "unit": "TFLOP/s", "frac": att / float(peaks["bf16_tflops_sustained"]),
                     "peak_source": f"{peak_src} bf16_tflops_sustained", "traffic": None},
        "gpu_launches": o["gpu_launches"], "clocks": o["clocks"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- memory
def maxlen_main(args, rank, world, device):
    """Longest sequence of the 4-layer Llama-3-8B-shaped stack + LM head that one GPU holds, by
    the library's memory model (memory_model.py) at D = 1, 2, 4, 8, 16, 32, with the budget =
    the device memory free after the CUDA context is up; then one streamed training step
    (forward + backward) at T = --stack-tokens and D = --chunks, whose
    torch.cuda.max_memory_allocated is compared with the model's prediction.  Prints one JSON
    line (not the bench contract's line)."""
    import torch
    from memory_efficient_exact_chunk_b200 import memory_model as MM
    from memory_efficient_exact_chunk_b200 import sbp, stack, synth
    wl = synth.WORKLOADS["llama3_8b_stack4_64k"]
    shape = MM.StackShape.from_workload(wl)
    free0, total = torch.cuda.mem_get_info(device)
    budget = free0 - (1 << 30)          # 1 GiB for torch's allocator slack and the kernels' own
    model = {D: MM.max_tokens(shape, D, budget) for D in (1, 2, 4, 8, 16, 32)}
    # by default 97 % of the model's longest sequence at this D (a margin for the allocator)
    T = args.stack_tokens or int(0.97 * model[args.chunks or 1])
    T = T // 128 * 128
    D = args.chunks or 1
    L = wl.layer
    gen = torch.Generator(device=device).manual_seed(5000 + rank)

    def rnd(*sh):
        return (torch.randn(*sh, generator=gen, device=device) * 0.02).to(torch.bfloat16)

    d, dq, dkv, f, V = (L.d_model, L.n_heads * L.head_dim, L.n_kv_heads * L.head_dim, L.ffn,
                        wl.vocab)
    layers = [{"ln1_g": torch.ones(d, dtype=torch.bfloat16, device=device),
               "wq": rnd(dq, d), "wk": rnd(dkv, d), "wv": rnd(dkv, d), "wo": rnd(d, dq),
               "ln2_g": torch.ones(d, dtype=torch.bfloat16, device=device),
               "w_gate": rnd(f, d), "w_up": rnd(f, d), "w_down": rnd(d, f),
               "bq": None, "bk": None, "bv": None} for _ in range(wl.n_layers)]
    embed, lm_w = rnd(V, d), rnd(V, d)
    final_g = torch.ones(d, dtype=torch.bfloat16, device=device)
    rng = np.random.default_rng(5000 + rank)
    ids = synth.token_ids(rng, 1, T, V)
    y = synth.shifted_targets(ids)
    w = synth.loss_weights("shifted_tail", 1, T, from_frac=wl.loss_from_frac)
    ids_d = torch.from_numpy(ids.reshape(-1)).to(device)
    y_d = torch.from_numpy(y.reshape(-1)).to(device)
    w_d = torch.from_numpy(w.reshape(-1)).to(device)
    cfg = sbp.layer_cfg(1, T, d, L.n_heads, L.n_kv_heads, L.head_dim, f, L.rms_eps,
                        L.rope_theta, sbp.SBP_BF16, D)
    grads = stack.zero_grads(layers, lm_w, final_g, device, embed_shape=embed.shape)
    ws = stack.Workspaces(device)
    torch.cuda.synchronize(device)
    torch.cuda.reset_peak_memory_stats(device)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record()
    xs, hf, rstd = stack.stack_forward(cfg, embed, layers, final_g, ids_d, ws)
    e1.record()
    r = stack.stack_backward_from(cfg, layers, final_g, lm_w, ids_d, y_d, w_d, xs, hf, rstd, ws,
                                  grads=grads)
    e2.record()
    torch.cuda.synchronize(device)
    peak = torch.cuda.max_memory_allocated(device)
    pred = MM.stack_step_bytes(shape, T, D)
    loss = float(r.loss.item())
    line = {
        "mode": "maxlen", "workload": "llama3_8b_stack4 + LM head 128256", "device_total_gb":
        total / 1e9, "budget_gb": budget / 1e9,
        "model_max_tokens": {str(k): v for k, v in model.items()},
        "run": {"seq_len": T, "num_chunks": D, "measured_peak_gb": peak / 1e9,
                "fraction_of_model_max": T / max(model.get(D, 0), 1) if D in model else None,
                "model_gb": pred["total"] / 1e9,
                "model_parts_gb": {k: v / 1e9 for k, v in pred.items()},
                "forward_ms": e0.elapsed_time(e1), "backward_ms": e1.elapsed_time(e2),
                "loss": loss, "finite": bool(np.isfinite(loss))},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- main
def lmhead_summary(out, args, peaks, peak_src):
    """The LM-head workload's numbers with the roofline of its dominant kernel, the tcgen05
    GEMM: all GEMM launches of a step, timed as the union of their CUDA-event intervals (the dH
    and dW products overlap on side streams)."""
    res = out["res"]
    prof = res["prof"]["gemm_tc"]
    tc_ms = prof["busy_ms"]
    n_l = max(prof["launches"], 1)
    achieved = (out["flops_step"] * args.steps) / (tc_ms / 1e3) / 1e12 if tc_ms > 0 else 0.0
    peak = float(peaks["bf16_tflops_sustained"])
    o = {
        "workload": out["config"]["workload"],
        "value": out["tokens_per_step"] * out["world"] / (res["ms"] / 1e3), "unit": "tokens/s",
        "ms_per_step": res["ms"], "steps": args.steps, "config": out["config"],
        "roofline": {
            "bound": "tensor", "kernel": "gemm_tc2_kernel (tcgen05, all GEMM launches of a step)",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak if peak else None,
            "peak_source": f"{peak_src} bf16_tflops_sustained",
            "flops_per_launch": out["flops_step"] / (n_l / args.steps),
            "launch_ms": prof["ms"] / n_l, "launches_per_step": n_l / args.steps,
            "gemm_busy_ms_per_step": tc_ms / args.steps,
            "share_of_step": tc_ms / res["ms_total"] if res["ms_total"] else None,
            "achieved_min_flops": (out["flops_min_step"] * args.steps) / (tc_ms / 1e3) / 1e12
            if tc_ms > 0 else 0.0,
            "traffic": traffic_from_profiles("gemm_tc2_kernel@lmhead_ce_32k"),
        },
        "gpu_launches": res["launches"], "clocks": res["clocks"],
        "peak_act_gb": out["peak_act_gb"], "workspace_gb": out["ws_bytes"] / 1e9,
    }
    for k in ("sweep", "memory_fit", "e2e"):
        if k in out:
            o[k] = out[k]
    return o


def base_line(world, args, o):
    return {"metric": METRIC, "value": o["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": o.get("steps", args.steps), "warmup": args.warmup,
            "ms_per_step": o["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}


def stack_main(args, rank, world, device):
    """Default line: the 4-layer Llama-3-8B-shaped stack + LM head (T = 65536, D = 16), the
    largest configuration that fits one GPU.  value = streamed-backward tokens/s."""
    import torch
    import torch.distributed as dist
    peaks, peak_src = load_peaks()
    o = run_stack(args, rank, world, device, "llama3_8b_stack4_64k", steps=args.steps,
                  e2e=args.e2e)
    peak = float(peaks["bf16_tflops_sustained"])
    k = o["steps"]
    busy = o["attn_bwd_busy_ms_total"]
    n_l = max(o["attn_bwd_launches_per_step"], 1)
    achieved = o["attn_bwd_tflops"] or 0.0
    line = base_line(world, args, o)
    line.update({
        "config": stack_config(o),
        "roofline": {
            "bound": "tensor",
            "kernel": "attention backward (attn_bwd_kv_kernel + attn_bwd_q_kernel, tcgen05; "
                      "one call per chunk and layer, its two kernels side by side)",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak if peak else None,
            "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long "
                           "step)",
            "frac_of_burst": achieved / float(peaks["bf16_tflops"]),
            "flops_per_unit": "10 * head_dim per causal (query, key, head) pair",
            "flops_per_launch": o["attn_bwd_flops_step"] / n_l,
            "launches_per_step": n_l,
            "launch_ms": busy / k / n_l,
            "share_of_step": o["kernels"]["attn_bwd"]["share"],
            "traffic": traffic_from_profiles("attn_bwd@llama3_8b_stack4_64k"),
        },
        "gpu_launches": o["gpu_launches"], "clocks": o["clocks"],
        "peak_act_gb": o["peak_act_gb"], "stack": o,
    })
    if "e2e" in o:
        line["e2e"] = o.pop("e2e")
    also = []
    if args.lmhead:
        torch.cuda.empty_cache()
        out = run_lmhead(args, rank, world, device)
        also.append(lmhead_summary(out, args, peaks, peak_src))
        del out
    if args.layer:
        torch.cuda.empty_cache()
        also.append(run_layer(args, rank, world, device, sweep=args.sweep))
    if args.stack:
        torch.cuda.empty_cache()
        also.append(run_stack(args, rank, world, device, "qwen25_7b_stack2_grpo"))
        torch.cuda.empty_cache()
        also.append(run_dpo_stack(args, rank, world, device))
    if also:
        line["also"] = also
    line["cpu_baseline"] = cpu_baseline_stack() if (args.cpu and rank == 0 and world == 1) \
        else None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def lmhead_main(args, rank, world, device):
    """The LM-head workload as the line's own workload."""
    import torch.distributed as dist
    peaks, peak_src = load_peaks()
    out = run_lmhead(args, rank, world, device)
    o = lmhead_summary(out, args, peaks, peak_src)
    line = base_line(world, args, o)
    line.update({k: o[k] for k in ("config", "roofline", "gpu_launches", "clocks",
                                   "peak_act_gb", "workspace_gb")})
    for k in ("sweep", "memory_fit", "e2e"):
        if k in o:
            line[k] = o[k]
    line["cpu_baseline"] = cpu_baseline() if (args.cpu and rank == 0 and world == 1) else None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sbp", choices=["sbp", "reference"])
    ap.add_argument("--workload", default="llama3_8b_stack4_64k",
                    choices=["llama3_8b_stack4_64k", "lmhead_ce_32k", "llama3_8b_layer_32k",
                             "maxlen"])
    ap.add_argument("--chunks", type=int, default=0,
                    help="override D of the line's own workload")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the LM head's sequence length (small cases for profiling)")
    ap.add_argument("--no-sweep", dest="sweep", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu", action="store_false")
    ap.add_argument("--no-lmhead", dest="lmhead", action="store_false",
                    help="skip the LM-head measurement added to the stack line")
    ap.add_argument("--no-layer", dest="layer", action="store_false",
                    help="skip the decoder-layer measurement added to the line")
    ap.add_argument("--layer-tokens", type=int, default=0)
    ap.add_argument("--no-stack", dest="stack", action="store_false",
                    help="skip the GRPO / DPO stack measurements added to the line")
    ap.add_argument("--stack-tokens", type=int, default=0,
                    help="override the 4-layer stack's sequence length (small cases)")
    ap.add_argument("--layer-chunks", type=int, default=0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from memory_efficient_exact_chunk_b200 import sbp
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    sbp.load()
    if args.workload == "llama3_8b_layer_32k":
        return layer_main(args, rank, world, device)
    if args.workload == "lmhead_ce_32k":
        return lmhead_main(args, rank, world, device)
    if args.workload == "maxlen":
        return maxlen_main(args, rank, world, device)
    return stack_main(args, rank, world, device)


if __name__ == "__main__":
    sys.exit(main())

"""Cycle accounting of the pair GEMM from the instrumented library (libsbp_timing.so, built
with SBP_GEMM_TIMING).

    python -m memory_efficient_exact_chunk_b200.build --timing
    python -m memory_efficient_exact_chunk_b200.timing lmhead > lmhead_timing.log
    python -m memory_efficient_exact_chunk_b200.timing layer > layer_timing.log
    python -m memory_efficient_exact_chunk_b200.timing summarize lmhead_timing.log
    python -m memory_efficient_exact_chunk_b200.timing summarize layer_timing.log

`lmhead` runs the LM-head CE backward twice (32768 tokens, D = 8, the bench's inputs); every
pair-GEMM launch prints, for CTA 0 (and CTA 1 for the producer): the producer's cycles waiting
for a free ring stage, the MMA issuer's cycles waiting for operands (full stage) and for a free
accumulator, and two epilogue warps' cycles waiting for a full accumulator and working.
`layer` runs the Llama-3-8B-shaped layer backward twice (16384 tokens, D = 2); the layer's
GEMMs print their accounts.  (The summary also reads the records of an attention dK/dV kernel
that prints "SBPT KV..." lines; the current attention kernels print none.)  `summarize` keeps
the second call (warm) of each kind and averages per launch shape.  Measurement only: the
product library is not involved.
"""
from __future__ import annotations

import collections
import os
import sys


def _load():
    from . import build, sbp
    if not os.path.exists(build.LIB_TIMING):
        raise RuntimeError("libsbp_timing.so missing: python -m "
                           "memory_efficient_exact_chunk_b200.build --timing")
    lib = sbp.load(build.LIB_TIMING)
    # load() keeps the first library a process opened: refuse to time the product one
    if os.path.realpath(lib._name) != os.path.realpath(build.LIB_TIMING):
        raise RuntimeError(f"{lib._name} is already loaded in this process; run the timing "
                           "workload in a fresh process")
    return lib


def run_lmhead(tokens: int = 0, chunks: int = 0):
    import torch
    from . import sbp, synth
    _load()
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    T, d, V = tokens or wl.seq_len, wl.hidden, wl.vocab
    D = chunks or wl.num_chunks
    h, W, y, w = synth.lmhead_inputs(1000, T, d, V, bf16=True, from_frac=wl.loss_from_frac)
    dev = "cuda"
    hd = torch.from_numpy(h).to(torch.bfloat16).to(dev)
    Wd = torch.from_numpy(W).to(torch.bfloat16).to(dev)
    yd, wd = torch.from_numpy(y).to(dev), torch.from_numpy(w).to(dev)
    loss = torch.zeros(1, device=dev)
    dH = torch.empty(T, d, device=dev)
    dW = torch.zeros(V, d, device=dev)
    ws = sbp.workspace(sbp.lmhead_ce_workspace_size(T, d, V, D, sbp.SBP_BF16), dev)
    for _ in range(2):
        sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW, ws=ws)
        torch.cuda.synchronize()
        sbp.device_status(ws)
    print(f"SBPT DONE T {T} D {D} loss {float(loss.item()):.6f}", flush=True)


def run_layer(tokens: int = 16384, chunks: int = 2):
    import torch
    from . import sbp, synth
    _load()
    wl = synth.WORKLOADS["llama3_8b_layer_32k"]
    L, B, T, D = wl.layer, wl.batch, tokens, chunks
    W, x, dy = synth.layer_inputs(2000, L, B, T, bf16=True, dy_std=1e-3)
    dev = "cuda"
    Wd = {n: (torch.from_numpy(W[n]).to(torch.bfloat16).to(dev) if W.get(n) is not None
              else None) for n in sbp.WEIGHT_FIELDS}
    xd = torch.from_numpy(x).to(torch.bfloat16).to(dev)
    dyd = torch.from_numpy(dy).to(dev)
    dx = torch.empty(B, T, L.d_model, device=dev)
    grads = {n: (torch.zeros(Wd[n].shape, device=dev) if Wd.get(n) is not None else None)
             for n in sbp.WEIGHT_FIELDS}
    cfg = sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn,
                        L.rms_eps, L.rope_theta, sbp.SBP_BF16, D)
    ws = sbp.workspace(sbp.layer_workspace_size(cfg), dev)
    for _ in range(2):
        sbp.decoder_layer_backward(cfg, Wd, xd, dyd, dx, grads, ws=ws)
        torch.cuda.synchronize()
        sbp.device_status(ws)
    print(f"SBPT DONE T {T} D {D}", flush=True)


def _fields(line):
    t = line.split()[2:]
    return dict(zip(t[0::2], t[1::2]))


def summarize(path: str) -> str:
    lines = [l.strip() for l in open(path) if l.startswith("SBPT ")]
    out = []
    kinds = {"ISSUE": [], "PROD": [], "EPI": [], "KVISSUE": [], "KVPROD": [], "KVEW": []}
    for l in lines:
        k = l.split()[1]
        if k in kinds:
            kinds[k].append(_fields(l))
    names = {"0": "store", "1": "accumulate", "2": "log-sum-exp", "3": "logit gradient"}
    # the run makes two identical calls: keep the second (warm) half of each kind
    for k in kinds:
        kinds[k] = kinds[k][len(kinds[k]) // 2:]
    agg = collections.defaultdict(lambda: [0, 0, 0, 0, 0])
    for f in kinds["ISSUE"]:
        if int(f["kblocks"]) == 0:
            continue
        a = agg[(int(f["M"]), int(f["N"]), int(f["K"]), f["epi"])]
        a[0] += 1
        a[1] += int(f["total"])
        a[2] += int(f["w_full"])
        a[3] += int(f["w_tempty"])
        a[4] += int(f["kblocks"])
    out.append("MMA issuer (CTA 0), per launch shape; a k-block is 64 deep, 512 cycles of "
               "tensor work at the nominal rate")
    out.append("| M | N | K | epilogue | launches | cycles/k-block | operand wait | "
               "accumulator wait | rest (issue, MMA back-pressure) cycles/k-block |")
    out.append("|---:|---:|---:|---|---:|---:|---:|---:|---:|")
    for key in sorted(agg):
        n, tot, wf, wt, kb = agg[key]
        out.append(f"| {key[0]} | {key[1]} | {key[2]} | {names.get(key[3], key[3])} | {n} | "
                   f"{tot / kb:.0f} | {100 * wf / tot:.0f} % | {100 * wt / tot:.0f} % | "
                   f"{(tot - wf - wt) / kb:.0f} |")
    pagg = collections.defaultdict(lambda: [0, 0, 0])
    for f in kinds["PROD"]:
        if int(f["tiles"]) == 0:
            continue
        a = pagg[(int(f["N"]), int(f["K"]), f["epi"])]
        a[0] += 1
        a[1] += int(f["total"])
        a[2] += int(f["w_empty"])
    out.append("")
    out.append("TMA producer (CTAs 0 and 1): share of its time spent waiting for a free stage")
    out.append("| N | K | epilogue | producer records | free-stage wait |")
    out.append("|---:|---:|---|---:|---:|")
    for key in sorted(pagg):
        n, tot, we = pagg[key]
        out.append(f"| {key[0]} | {key[1]} | {names.get(key[2], key[2])} | {n} | "
                   f"{100 * we / tot:.0f} % |")
    eagg = collections.defaultdict(lambda: [0, 0, 0, 0])
    for f in kinds["EPI"]:
        if int(f["M"]) == 0:
            continue
        a = eagg[(int(f["N"]), int(f["K"]), f["epi"])]
        a[0] += 1
        a[1] += int(f["total"])
        a[2] += int(f["w_tfull"])
        a[3] += int(f["work"])
    out.append("")
    out.append("Epilogue warps 2 and 9 of CTA 0: share of time working (the rest waits for a "
               "full accumulator)")
    out.append("| N | K | epilogue | warp records | working |")
    out.append("|---:|---:|---|---:|---:|")
    for key in sorted(eagg):
        n, tot, wt, wk = eagg[key]
        out.append(f"| {key[0]} | {key[1]} | {names.get(key[2], key[2])} | {n} | "
                   f"{100 * wk / tot:.0f} % |")
    if kinds["KVISSUE"]:
        out.append("")
        out.extend(_summarize_kv(kinds))
    return "\n".join(out)


def _summarize_kv(kinds) -> list:
    """Per (head, 128-query tile) pair averages of the dK/dV kernel's CTA 0, per launch."""
    out = ["Attention dK/dV kernel, CTA 0 (one 128-key tile of one KV head), cycles per "
           "(query head, 128-query tile) pair",
           "| chunk start | Tc | pairs | total | MMA issuer: wait dS | wait Q/dO | wait flush | "
           "issuing | element-wise: wait scores | working | flushing | producer: wait stage |",
           "|---:|---:|---:|---:|---:|---:|---:|---:|---:|---:|---:|---:|"]
    ew = collections.defaultdict(list)
    for f in kinds["KVEW"]:
        ew[(f["s"], f["Tc"])].append(f)
    prod = {(f["s"], f["Tc"]): f for f in kinds["KVPROD"]}
    for f in kinds["KVISSUE"]:
        n = int(f["pairs"])
        if n == 0:
            continue
        key = (f["s"], f["Tc"])
        e = ew.get(key, [])
        avg = lambda name: sum(int(x[name]) for x in e) / max(1, len(e)) / n
        p = prod.get(key)
        out.append(f"| {f['s']} | {f['Tc']} | {n} | {int(f['total']) / n:.0f} | "
                   f"{int(f['w_ds']) / n:.0f} | {int(f['w_qd']) / n:.0f} | "
                   f"{int(f['w_free']) / n:.0f} | {int(f['issue']) / n:.0f} | "
                   f"{avg('w_sdp'):.0f} | {avg('work'):.0f} | {avg('flush'):.0f} | "
                   f"{(int(p['w_empty']) / n if p else float('nan')):.0f} |")
    return out


if __name__ == "__main__":
    if len(sys.argv) >= 2 and sys.argv[1] == "lmhead":
        run_lmhead()
    elif len(sys.argv) >= 2 and sys.argv[1] == "layer":
        run_layer()
    elif len(sys.argv) == 3 and sys.argv[1] == "summarize":
        print(summarize(sys.argv[2]))
    else:
        print(__doc__)
        sys.exit(2)

"""Cycle accounting of the pair GEMM on the LM-head CE backward, from the instrumented library.

    python -m memory_efficient_exact_chunk_b200.build --timing
    python -m memory_efficient_exact_chunk_b200.gemm_timing run > timing.log
    python -m memory_efficient_exact_chunk_b200.gemm_timing summarize timing.log

`run` loads libsbp_timing.so (the pair kernel built with SBP_GEMM_TIMING) and runs the LM-head
CE backward twice (32768 tokens, D = 8, the bench's inputs); every pair-GEMM launch prints, for
CTA 0 (and CTA 1 for the producer): the producer's cycles waiting for a free ring stage, the MMA
issuer's cycles waiting for operands (full stage) and for a free accumulator, and two epilogue
warps' cycles waiting for a full accumulator and working.  `summarize` keeps the second call
(warm) and averages per launch shape.  Measurement only: the product library is not involved.
"""
from __future__ import annotations

import collections
import os
import sys


def run(tokens: int = 0, chunks: int = 0):
    import torch
    from . import build, sbp, synth
    if not os.path.exists(build.LIB_TIMING):
        raise RuntimeError("libsbp_timing.so missing: python -m "
                           "memory_efficient_exact_chunk_b200.build --timing")
    sbp.load(build.LIB_TIMING)
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


def _fields(line):
    t = line.split()[2:]
    return dict(zip(t[0::2], t[1::2]))


def summarize(path: str) -> str:
    lines = [l.strip() for l in open(path) if l.startswith("SBPT ")]
    out = []
    kinds = {"ISSUE": [], "PROD": [], "EPI": []}
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
    return "\n".join(out)


if __name__ == "__main__":
    if len(sys.argv) >= 2 and sys.argv[1] == "run":
        run()
    elif len(sys.argv) == 3 and sys.argv[1] == "summarize":
        print(summarize(sys.argv[2]))
    else:
        print(__doc__)
        sys.exit(2)

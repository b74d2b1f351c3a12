"""Checks at the full sizes the bench times (32K-token LM head, 32K-token Llama-3-8B layer), in
the bench's launch configuration.  The oracle cannot run these sizes whole, so the checks are:
sampled rows of d_hidden (each row depends only on its own hidden state) against the oracle,
and D = 1 vs D = 8 agreement within 1e-5 for every output (the exactness of the chunking)."""
import numpy as np
import pytest

from oracle import sbp_oracle as O
from memory_efficient_exact_chunk_b200 import synth

pytestmark = pytest.mark.gpu


def _rel(a, b):
    import torch
    return ((a.double() - b.double()).norm() / b.double().norm().clamp_min(1e-300)).item()


def test_lmhead_full_size():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    T, d, V = wl.seq_len, wl.hidden, wl.vocab
    h, W, y, w = synth.lmhead_inputs(77, T, d, V, bf16=True, from_frac=wl.loss_from_frac)
    hd = torch.from_numpy(h).to(torch.bfloat16).cuda()
    Wd = torch.from_numpy(W).to(torch.bfloat16).cuda()
    yd = torch.from_numpy(y).cuda()
    wd = torch.from_numpy(w).cuda()
    out = {}
    for D in (wl.num_chunks, 2 * wl.num_chunks, 1):
        loss = torch.zeros(1, device="cuda")
        dH = torch.full((T, d), float("nan"), device="cuda")
        dW = torch.zeros(V, d, device="cuda")
        ws = sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW)
        sbp.device_status(ws)
        out[D] = (loss, dH, dW)
        del ws
    l1, dH1, dW1 = out[1]
    for D in (wl.num_chunks, 2 * wl.num_chunks):
        lD, dHD, dWD = out[D]
        errs = {"loss": abs(lD.item() - l1.item()) / abs(l1.item()), "dH": _rel(dHD, dH1),
                "dW": _rel(dWD, dW1)}
        print(f"lmhead D={D} vs D=1:", errs)
        assert all(v <= 1e-5 for v in errs.values()), (D, errs)
    l8, dH8, dW8 = out[wl.num_chunks]
    # sampled rows against the oracle (masked rows must be exactly zero)
    masked = np.flatnonzero(w == 0)
    live = np.flatnonzero(w != 0)
    rng = np.random.default_rng(0)
    rows = list(rng.choice(live, 5, replace=False)) + [int(live[0]), int(live[-1])]
    W64 = W.astype(np.float64)
    for r in rows:
        _, dh0, _, _ = O.lmhead_ce_forward_backward(h[r:r + 1], W64, y[r:r + 1], w[r:r + 1])
        got = dH8[r].double().cpu().numpy()
        err = np.linalg.norm(got - dh0[0]) / np.linalg.norm(dh0[0])
        assert err <= 1e-2, (r, err)
    assert torch.all(dH8[torch.from_numpy(masked[:1000]).cuda()] == 0)


def test_llama_layer_full_size_chunk_invariance():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    wl = synth.WORKLOADS["llama3_8b_layer_32k"]
    L, B, T = wl.layer, wl.batch, wl.seq_len
    W, x, dy = synth.layer_inputs(78, L, B, T, bf16=True, dy_std=1e-3)
    names = sbp.WEIGHT_FIELDS
    Wd = {n: (torch.from_numpy(W[n]).to(torch.bfloat16).cuda() if W.get(n) is not None else None)
          for n in names}
    xd = torch.from_numpy(x).to(torch.bfloat16).cuda()
    dyd = torch.from_numpy(dy).cuda()
    res = {}
    for D in (wl.num_chunks, 2 * wl.num_chunks, 1, -wl.num_chunks):
        # D < 0: |D| chunks in reverse order
        cfg = sbp.layer_cfg(B, T, L.d_model, L.n_heads, L.n_kv_heads, L.head_dim, L.ffn,
                            L.rms_eps, L.rope_theta, sbp.SBP_BF16, abs(D))
        dx = torch.full((B, T, L.d_model), float("nan"), device="cuda")
        g = {n: (torch.zeros(Wd[n].shape, device="cuda") if Wd.get(n) is not None else None)
             for n in names}
        run = sbp.decoder_layer_backward_reverse if D < 0 else sbp.decoder_layer_backward
        ws = run(cfg, Wd, xd, dyd, dx, g)
        sbp.device_status(ws)
        res[D] = (dx, g)
        del ws
        torch.cuda.empty_cache()
    dx1, g1 = res[1]
    for D in (wl.num_chunks, 2 * wl.num_chunks, -wl.num_chunks):
        dxD, gD = res[D]
        assert torch.isfinite(dxD).all()
        errs = {"dx": _rel(dxD, dx1)}
        for n, v in g1.items():
            if v is not None:
                errs[n] = _rel(gD[n], v)
        print(f"layer D={D} vs D=1:", errs)
        bad = {k: v for k, v in errs.items() if not v <= 1e-5}
        assert not bad, (D, errs)

"""GPU check of the chunk attention forward (tensor-core kernel, head_dim 128) against a plain
PyTorch fp64 causal attention of the same bf16 operands, and against the CUDA-core kernel."""
import math

import pytest

pytestmark = pytest.mark.gpu


def _reference(q, Kp, Vp, s):
    """fp64 causal GQA attention of chunk queries (positions s..s+Tc) over keys [0, s+Tc)."""
    import torch
    B, T, Hkv, hd = Kp.shape
    R, H, _ = q.shape
    Tc = R // B
    grp = H // Hkv
    out = torch.empty(R, H, hd, dtype=torch.float64)
    lse = torch.empty(R, H, dtype=torch.float64)
    for b in range(B):
        qb = q[b * Tc:(b + 1) * Tc].double().cpu()                     # [Tc, H, hd]
        kb = Kp[b, :s + Tc].double().cpu().repeat_interleave(grp, 1)   # [e, H, hd]
        vb = Vp[b, :s + Tc].double().cpu().repeat_interleave(grp, 1)
        sc = torch.einsum("thd,uhd->htu", qb, kb) / math.sqrt(hd)
        tpos = torch.arange(s, s + Tc)[:, None]
        upos = torch.arange(s + Tc)[None, :]
        sc = sc.masked_fill(upos > tpos, float("-inf"))
        lse[b * Tc:(b + 1) * Tc] = torch.logsumexp(sc, -1).t()
        out[b * Tc:(b + 1) * Tc] = torch.einsum("htu,uhd->thd", torch.softmax(sc, -1), vb)
    return out, lse


@pytest.mark.parametrize("B,T,s,Tc,H,Hkv,qscale", [
    (1, 256, 0, 256, 2, 1, 1.0),
    (2, 384, 128, 128, 4, 2, 1.0),
    (1, 300, 100, 150, 2, 2, 1.0),      # ragged chunk and sequence
    (1, 1024, 512, 512, 8, 2, 1.0),
    (1, 512, 128, 256, 2, 1, 12.0),     # peaked softmax: exercises the output rescale
    # the key range split at a quarter of the sequence (key tile ceil(ceil(T / 128) / 4)):
    (2, 512, 256, 256, 4, 2, 1.0),      # two sequences, every pair split
    (1, 600, 250, 350, 2, 1, 1.0),      # unaligned chunk: a tile straddles the split (rows
                                        # before it see no key in the second segment) and a
                                        # split pair with one tile
])
def test_attention_forward_tc(B, T, s, Tc, H, Hkv, qscale):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(T + s + H)
    hd = 128
    q = (torch.randn(B * Tc, H, hd, generator=g) * qscale).to(torch.bfloat16).cuda()
    Kp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    Vp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    ref_o, ref_l = _reference(q, Kp, Vp, s)
    for path in (2, 1):
        o = torch.full((B * Tc, H, hd), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B * Tc, H), float("nan"), device="cuda")
        ws = sbp.debug_attn_fwd_bf16(q, Kp, Vp, o, lse, s, path=path)
        sbp.device_status(ws)
        eo = ((o.double().cpu() - ref_o).norm() / ref_o.norm()).item()
        el = (lse.double().cpu() - ref_l).abs().max().item()
        assert eo <= 1e-2, (path, eo)
        assert el <= 2e-3 * max(1.0, qscale), (path, el)


def test_attention_forward_tc_chunking_is_bitwise_neutral():
    """A query row's output does not depend on which chunk it is computed in."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(5)
    B, T, H, Hkv, hd = 1, 512, 4, 2, 128
    q = torch.randn(T, H, hd, generator=g).to(torch.bfloat16).cuda()
    Kp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    Vp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    o_full = torch.empty(T, H, hd, dtype=torch.bfloat16, device="cuda")
    l_full = torch.empty(T, H, device="cuda")
    sbp.debug_attn_fwd_bf16(q, Kp, Vp, o_full, l_full, 0, path=2)
    for s, e in ((0, 128), (128, 384), (384, 512), (100, 300)):
        o = torch.empty(e - s, H, hd, dtype=torch.bfloat16, device="cuda")
        l = torch.empty(e - s, H, device="cuda")
        sbp.debug_attn_fwd_bf16(q[s:e].contiguous(), Kp, Vp, o, l, s, path=2)
        torch.cuda.synchronize()
        assert torch.equal(o, o_full[s:e]) and torch.equal(l, l_full[s:e]), (s, e)


@pytest.mark.parametrize("B,T,s,Tc,H,Hkv", [
    (1, 256, 0, 256, 2, 1),
    (2, 384, 128, 128, 4, 2),
    (1, 300, 100, 150, 2, 2),      # ragged chunk and sequence
    (1, 640, 256, 384, 4, 1),
])
def test_attention_backward_tc(B, T, s, Tc, H, Hkv):
    """dQ, dK, dV of the chunk queries against fp64 autograd of the same bf16 operands."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(7 * T + s + H)
    hd = 128
    q = torch.randn(B * Tc, H, hd, generator=g).to(torch.bfloat16).cuda()
    Kp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    Vp = torch.randn(B, T, Hkv, hd, generator=g).to(torch.bfloat16).cuda()
    dO = torch.randn(B * Tc, H, hd, generator=g).to(torch.bfloat16).cuda()
    o = torch.empty(B * Tc, H, hd, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B * Tc, H, device="cuda")
    sbp.debug_attn_fwd_bf16(q, Kp, Vp, o, lse, s, path=2)
    # fp64 autograd reference
    qr = q.double().cpu().requires_grad_()
    kr = Kp.double().cpu().requires_grad_()
    vr = Vp.double().cpu().requires_grad_()
    out, _ = _reference_autograd(qr, kr, vr, s)
    out.backward(dO.double().cpu())
    for path in (2, 1):
        dq = torch.full((B * Tc, H, hd), float("nan"), device="cuda")
        dK = torch.zeros(B, T, Hkv, hd, device="cuda")
        dV = torch.zeros(B, T, Hkv, hd, device="cuda")
        ws = sbp.debug_attn_bwd_bf16(q, Kp, Vp, o, dO, lse, dq, dK, dV, s, path=path)
        sbp.device_status(ws)
        for got, want, name in ((dq, qr.grad, "dq"), (dK, kr.grad, "dK"), (dV, vr.grad, "dV")):
            err = ((got.double().cpu() - want).norm() / want.norm()).item()
            assert err <= 1e-2, (path, name, err)
        assert torch.all(dK[:, s + Tc:] == 0) and torch.all(dV[:, s + Tc:] == 0)


def _reference_autograd(q, Kp, Vp, s):
    import torch
    B, T, Hkv, hd = Kp.shape
    R, H, _ = q.shape
    Tc = R // B
    grp = H // Hkv
    outs = []
    for b in range(B):
        qb = q[b * Tc:(b + 1) * Tc]
        kb = Kp[b, :s + Tc].repeat_interleave(grp, 1)
        vb = Vp[b, :s + Tc].repeat_interleave(grp, 1)
        sc = torch.einsum("thd,uhd->htu", qb, kb) / math.sqrt(hd)
        tpos = torch.arange(s, s + Tc)[:, None]
        upos = torch.arange(s + Tc)[None, :]
        sc = sc.masked_fill(upos > tpos, float("-inf"))
        outs.append(torch.einsum("htu,uhd->thd", torch.softmax(sc, -1), vb))
    return torch.cat(outs), None

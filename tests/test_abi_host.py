"""Host-side checks of the C ABI (no kernel launch): the library loads, exports every symbol
that include/sbp.h declares, and rejects bad arguments before queueing any work."""
import ctypes as C
import os
import re

import pytest

from memory_efficient_exact_chunk_b200 import build as sbp_build
from memory_efficient_exact_chunk_b200 import sbp
from oracle import sbp_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x100000  # an aligned address that is never dereferenced (argument checks fail first)


@pytest.fixture(scope="module")
def lib():
    sbp_build.build()
    return sbp.load()


def header_symbols():
    txt = "".join(open(os.path.join(ROOT, "include", f)).read()
                  for f in sorted(os.listdir(os.path.join(ROOT, "include"))) if f.endswith(".h"))
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sbp_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(lib):
    syms = header_symbols()
    assert "sbp_lmhead_ce_backward_stream" in syms and "sbp_decoder_layer_backward_stream" in syms
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(sbp.EXPORTS) | set(syms)
    assert lib.sbp_version().decode().startswith("sbp")


def test_chunk_bounds_matches_oracle(lib):
    for T in (1, 7, 10, 256, 32768, 65536):
        for D in (1, 2, 3, 7, 8, 16):
            if D > T:
                with pytest.raises(sbp.SbpError):
                    sbp.chunk_bounds(T, D)
                continue
            assert sbp.chunk_bounds(T, D) == O.chunk_bounds(T, D)


def test_workspace_sizes(lib):
    assert sbp.lmhead_ce_workspace_size(1024, 64, 1000, 4, sbp.SBP_BF16) > 0
    assert sbp.lmhead_ce_workspace_size(1024, 64, 1000, 0, sbp.SBP_BF16) == 0
    assert sbp.lmhead_ce_workspace_size(4, 64, 1000, 5, sbp.SBP_BF16) == 0
    cfg = sbp.layer_cfg(1, 256, 64, 4, 4, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 4)
    w4 = sbp.layer_workspace_size(cfg)
    assert w4 > 0
    cfg1 = sbp.layer_cfg(1, 256, 64, 4, 4, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 1)
    assert sbp.layer_workspace_size(cfg1) > w4          # per-chunk buffers scale with T / D
    bad = sbp.layer_cfg(1, 256, 64, 4, 3, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 4)
    assert sbp.layer_workspace_size(bad) == 0


def _lm_call(lib, **kw):
    a = dict(N=64, d=64, V=100, D=2, dt=sbp.SBP_F32, h=FAKE, W=FAKE, y=FAKE, w=FAKE, loss=FAKE,
             dH=FAKE, dW=FAKE, ws=FAKE, wsb=1 << 40)
    a.update(kw)
    return lib.sbp_lmhead_ce_backward_stream(a["N"], a["d"], a["V"], a["D"], a["dt"], a["h"],
                                             a["W"], a["y"], a["w"], a["loss"], a["dH"], a["dW"],
                                             a["ws"], a["wsb"], None)


def test_lmhead_argument_errors(lib):
    assert _lm_call(lib, h=None) == 1
    assert _lm_call(lib, dW=None) == 1
    assert _lm_call(lib, D=0) == 1
    assert _lm_call(lib, D=65) == 1
    assert _lm_call(lib, N=0) == 1
    assert _lm_call(lib, dt=7) == 1
    assert _lm_call(lib, h=FAKE + 4) == 1                      # misaligned
    assert _lm_call(lib, dt=sbp.SBP_BF16, d=60) == 2            # unsupported width
    assert _lm_call(lib, wsb=16) == 3                            # workspace too small
    assert _lm_call(lib, ws=FAKE + 16) == 1                      # workspace misaligned
    assert "workspace" in lib.sbp_last_error().decode()


@pytest.mark.parametrize("entry", ["sbp_decoder_layer_backward_stream",
                                   "sbp_decoder_layer_backward_stream_reverse"])
def test_layer_argument_errors(lib, entry):
    cfg = sbp.layer_cfg(1, 256, 64, 4, 4, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 4)
    names = sbp.WEIGHT_FIELDS
    w = sbp.LayerWeights(**{n: (FAKE if n not in ("bq", "bk", "bv") else None) for n in names})
    g = sbp.LayerGrads(**{n: (FAKE if n not in ("bq", "bk", "bv") else None) for n in names})
    fn = getattr(lib, entry)

    def call(c=cfg, w=w, g=g, x=FAKE, dy=FAKE, dx=FAKE, ws=FAKE, wsb=1 << 40):
        return fn(C.byref(c), C.byref(w), x, dy, dx, C.byref(g), ws, wsb, None)

    assert call(x=None) == 1
    assert call(wsb=1024) == 3
    bad = sbp.layer_cfg(1, 256, 64, 4, 3, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 4)
    assert call(c=bad) == 1                                      # n_heads % n_kv_heads
    assert call(c=sbp.layer_cfg(1, 256, 64, 4, 4, 16, 172, 1e-6, 1e4, sbp.SBP_F32, 257)) == 1
    assert call(c=sbp.layer_cfg(1, 256, 64, 4, 4, 15, 172, 1e-6, 1e4, sbp.SBP_F32, 4)) == 2
    assert call(c=sbp.layer_cfg(1, 256, 64, 4, 4, 16, 172, 1e-6, 1e4, sbp.SBP_BF16, 4)) == 2
    wb = sbp.LayerWeights(**{n: FAKE for n in names})
    assert call(w=wb) == 1                                        # biases without bias grads
    w1 = sbp.LayerWeights(**{n: (FAKE if n != "bk" else None) for n in names})
    assert call(w=w1) == 1                                        # partial bias set


def test_lmhead_forward_and_dpo_argument_errors(lib):
    """Checked on the host before anything is queued (no GPU needed)."""
    def fwd(N=1024, d=64, V=1000, D=4, dt=sbp.SBP_F32, h=FAKE, W=FAKE, y=FAKE, w=FAKE, ce=FAKE,
            ws=FAKE, wsb=1 << 40):
        return lib.sbp_lmhead_ce_forward_stream(N, d, V, D, dt, h, W, y, w, ce, None, ws, wsb,
                                                None)
    assert fwd(ce=None) == 1
    assert fwd(N=0) == 1
    assert fwd(D=2000) == 1
    assert fwd(dt=sbp.SBP_BF16, d=60) == 2
    assert fwd(wsb=16) == 3
    assert sbp.dpo_workspace_size(0) == 0 and sbp.dpo_workspace_size(4) >= 256

    def dpo(P=2, T=8, ce=FAKE, m=FAKE, ref=FAKE, beta=0.1, loss=FAKE, w=FAKE, ws=FAKE,
            wsb=1 << 20):
        return lib.sbp_dpo_token_weights(P, T, ce, m, ref, beta, loss, None, w, ws, wsb, None)
    assert dpo(P=0) == 1
    assert dpo(T=0) == 1
    assert dpo(beta=0.0) == 1
    assert dpo(beta=-1.0) == 1
    assert dpo(ref=None) == 1
    assert dpo(w=None) == 1
    assert dpo(wsb=8) == 3


def test_lmhead_host_entry_argument_errors(lib):
    def call(N=1024, d=64, V=1000, D=4, dt=sbp.SBP_BF16, h=FAKE, W=FAKE, y=FAKE, w=FAKE,
             loss=FAKE, dH=FAKE, dW=FAKE, ws=FAKE, wsb=1 << 40):
        return lib.sbp_lmhead_ce_backward_stream_host(N, d, V, D, dt, h, W, y, w, loss, dH, dW, ws,
                                                      wsb, None)
    assert call(h=None) == 1
    assert call(N=0) == 1
    assert call(D=0) == 1
    assert call(d=60) == 2
    assert call(wsb=64) == 3
    assert (sbp.lmhead_ce_workspace_size_host(1024, 64, 1000, 4, sbp.SBP_BF16) >
            sbp.lmhead_ce_workspace_size(1024, 64, 1000, 4, sbp.SBP_BF16) > 0)


def test_workspace_falls_as_one_over_d_at_bench_shapes(lib):
    """The O(T/D) claim, from the library's own sizing at the bench's full shapes (no GPU):
    the LM head's workspace is a / D (everything in it is per chunk), the layer's a / D + b with
    b the O(T d_kv) K/V prefix and fp32 dK/dV (R13)."""
    import numpy as np
    from memory_efficient_exact_chunk_b200 import synth
    Ds = (1, 2, 4, 8, 16)
    wl = synth.WORKLOADS["lmhead_ce_32k"]
    lm = [sbp.lmhead_ce_workspace_size(wl.seq_len, wl.hidden, wl.vocab, D, sbp.SBP_BF16)
          for D in Ds]
    prod = [w * D for w, D in zip(lm, Ds)]
    assert max(prod) / min(prod) < 1.001, prod
    wl = synth.WORKLOADS["llama3_8b_layer_32k"]
    L = wl.layer
    lay = [sbp.layer_workspace_size(sbp.layer_cfg(wl.batch, wl.seq_len, L.d_model, L.n_heads,
                                                  L.n_kv_heads, L.head_dim, L.ffn, L.rms_eps,
                                                  L.rope_theta, sbp.SBP_BF16, D)) for D in Ds]
    A = np.array([[1.0 / D, 1.0] for D in Ds])
    (a, b), *_ = np.linalg.lstsq(A, np.array(lay, dtype=np.float64), rcond=None)
    assert np.max(np.abs(A @ np.array([a, b]) - lay)) < 1e-6 * lay[0]
    # b is the whole-sequence part: bf16 K/V prefix plus fp32 dK/dV, 12 bytes per K/V element
    kv = wl.batch * wl.seq_len * L.n_kv_heads * L.head_dim
    assert 12 * kv <= b < 12 * kv * 1.1, (b, 12 * kv)


def test_noalloc_invalid_sizes_are_argument_errors(lib):
    """Invalid sizes reach the caller as SBP_ERR_INVALID_ARG before any device or symbol
    lookup (this host has no GPU, so a lookup would fail with SBP_ERR_CUDA instead)."""
    for n, d, V, D in ((0, 64, 100, 1), (10, 0, 100, 1), (10, 64, 0, 1), (10, 64, 100, 0),
                       (10, 64, 100, 11)):
        rc = lib.sbp_lmhead_ce_backward_noalloc(n, d, V, D, sbp.SBP_BF16, *([None] * 8))
        assert rc == 1, (n, d, V, D, rc)
        assert "invalid sizes" in lib.sbp_last_error().decode()


def test_stall_hook_argument_errors(lib):
    f = lib.sbp_debug_gemm_stall_bf16
    assert f(0, 256, 64, FAKE, FAKE, FAKE, 10**6, FAKE, None) == 1
    assert f(128, 256, 64, None, FAKE, FAKE, 10**6, FAKE, None) == 1
    assert f(128, 256, 64, FAKE, FAKE, FAKE, 10**4, FAKE, None) == 1
    assert f(128, 256, 64, FAKE, FAKE, FAKE, 3 * 10**9, FAKE, None) == 1


def test_attention_forward_workspace_size_is_checked_before_any_call():
    """The debug attention forward's workspace holds the status word and the key-range split's
    scratch (partial O, maxima and sums, two flags per query-tile pair); a smaller buffer is
    refused on the host, before the library is called."""
    import torch
    B, T, Tc, H, Hkv, hd = 2, 1024, 384, 4, 2, 128
    pairs = ((Tc + 127) // 128 + 1) // 2
    need = sbp.debug_attn_fwd_workspace_bytes(B, Tc, H, hd)
    assert need == 256 + 4 * B * Tc * H * hd + 8 * B * Tc * H + 8 * B * H * pairs
    q = torch.empty(B * Tc, H, hd, dtype=torch.bfloat16)
    Kp = torch.empty(B, T, Hkv, hd, dtype=torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty(B * Tc, H)
    small = torch.empty(need - 16, dtype=torch.uint8)
    with pytest.raises(ValueError):
        sbp.debug_attn_fwd_bf16(q, Kp, Kp, o, lse, 0, path=2, ws=small)

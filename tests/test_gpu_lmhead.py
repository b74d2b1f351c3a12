"""GPU parity of sbp_lmhead_ce_backward_stream against the fp64 oracle (called through the C
ABI).  Tolerances: max relative Frobenius error 1e-5 (fp32 path) and 1e-2 (bf16 operands,
fp32 accumulation) per tensor; D = 1 vs D > 1 within 1e-5."""
import numpy as np
import pytest

from oracle import sbp_oracle as O
from memory_efficient_exact_chunk_b200 import synth
from tests.helpers import f64, rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}


def _run(h, W, y, w, D, dtype, dW0=None):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    hd, Wd = to_dev(h, dtype), to_dev(W, dtype)
    yd = torch.from_numpy(np.asarray(y, np.int32)).cuda()
    wd = torch.from_numpy(np.asarray(w, np.float32)).cuda()
    loss = torch.full((1,), float("nan"), device="cuda")
    dH = torch.full(hd.shape, float("nan"), device="cuda")
    dW = torch.zeros(Wd.shape, device="cuda") if dW0 is None else to_dev(dW0, "f32")
    ws = sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW)
    sbp.device_status(ws)
    torch.cuda.synchronize()
    return to_np(loss)[0], to_np(dH), to_np(dW)


def _inputs(seed, N, d, V, dtype, frac=0.3, neg=False):
    h, W, y, w = synth.lmhead_inputs(seed, N, d, V, bf16=(dtype == "bf16"), from_frac=frac)
    if neg:
        rng = np.random.default_rng(seed + 1)
        w = (w * rng.standard_normal(N)).astype(np.float32)
    return h, W, y, w


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,d,V,D", [(300, 64, 1000, 1), (300, 64, 1000, 3), (257, 128, 9000, 4),
                                     (512, 96, 8192 + 100, 8)])
def test_lmhead_parity(dtype, N, d, V, D):
    h, W, y, w = _inputs(N + V, N, d, V, dtype, neg=(D == 3))
    loss, dH, dW = _run(h, W, y, w, D, dtype)
    l0, dH0, dW0, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    assert abs(loss - l0) <= TOL[dtype] * abs(l0)
    assert rel_fro(dH, dH0) <= TOL[dtype]
    assert rel_fro(dW, dW0) <= TOL[dtype]
    masked = np.asarray(w) == 0
    assert np.all(dH[masked] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lmhead_d_invariance_and_accumulate(dtype):
    N, d, V = 1024, 128, 5000
    h, W, y, w = _inputs(7, N, d, V, dtype)
    base = _run(h, W, y, w, 1, dtype)
    for D in (2, 4, 8, 13):
        got = _run(h, W, y, w, D, dtype)
        assert abs(got[0] - base[0]) <= 1e-5 * abs(base[0])
        assert rel_fro(got[1], base[1]) <= 1e-5
        assert rel_fro(got[2], base[2]) <= 1e-5
    # d_weight accumulates onto what the caller passes in
    scale = np.float32(np.std(base[2]))
    prior = (np.random.default_rng(3).standard_normal((V, d)) * scale).astype(np.float32)
    got = _run(h, W, y, w, 4, dtype, dW0=prior)
    assert rel_fro(got[2] - prior, base[2]) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lmhead_masked_chunks_keep_prior_dw(dtype):
    """Chunks without loss rows launch products with no live rows and a dW product over an
    empty K range; those return at once and must leave the caller's d_weight as it is."""
    N, d, V = 2048, 256, 5000
    h, W, y, w = _inputs(12, N, d, V, dtype, frac=0.6)    # chunks 0 and 1 fully masked at D=4
    assert not np.any(w[:1024]) and np.any(w[1024:1536])
    prior = (np.random.default_rng(4).standard_normal((V, d)) * 1e-3).astype(np.float32)
    loss1, dH1, dW1 = _run(h, W, y, w, 1, dtype, dW0=prior)
    loss4, dH4, dW4 = _run(h, W, y, w, 4, dtype, dW0=prior)
    l0, dH0, dW0, _ = O.lmhead_ce_forward_backward(f64(h), f64(W), y, w)
    assert rel_fro(dW4 - prior, dW0) <= TOL[dtype] and rel_fro(dH4, dH0) <= TOL[dtype]
    assert rel_fro(dW4, dW1) <= 1e-5 and rel_fro(dH4, dH1) <= 1e-5
    assert abs(loss4 - loss1) <= 1e-5 * abs(loss1)
    # a fully masked input: nothing but the loss (0) and dH (0) is written
    z = np.zeros_like(w)
    lz, dHz, dWz = _run(h, W, y, z, 4, dtype, dW0=prior)
    assert lz == 0.0 and np.all(dHz == 0.0) and np.array_equal(dWz, prior)


def test_lmhead_all_masked_chunk_and_bad_target():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    N, d, V = 256, 64, 300
    h, W, y, w = _inputs(11, N, d, V, "f32", frac=0.6)   # chunks 0 and 1 fully masked at D=4
    loss, dH, dW = _run(h, W, y, w, 4, "f32")
    l0, dH0, dW0, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    assert rel_fro(dH, dH0) <= 1e-5 and rel_fro(dW, dW0) <= 1e-5
    # a target outside [0, V) with a nonzero weight raises the device status
    y_bad = y.copy()
    y_bad[-1] = V + 5
    hd, Wd = to_dev(h, "f32"), to_dev(W, "f32")
    loss_t = torch.zeros(1, device="cuda")
    dH_t = torch.zeros(N, d, device="cuda")
    dW_t = torch.zeros(V, d, device="cuda")
    ws = sbp.lmhead_ce_backward(hd, Wd, torch.from_numpy(y_bad.astype(np.int32)).cuda(),
                                torch.from_numpy(w).cuda(), 4, loss_t, dH_t, dW_t)
    with pytest.raises(sbp.SbpError) as ei:
        sbp.device_status(ws)
    assert ei.value.code == 6
    sbp.device_status(ws)   # cleared by the read


def test_lmhead_full_width_reduced_rows():
    """Hidden 3584 and vocabulary 152064 (the 32K-token SFT workload's widths) on 192 rows."""
    N, d, V = 192, 3584, 152064
    h, W, y, w = _inputs(2, N, d, V, "bf16")
    loss, dH, dW = _run(h, W, y, w, 2, "bf16")
    l0, dH0, dW0, _ = O.lmhead_ce_forward_backward(h, W, y, w)
    assert abs(loss - l0) <= 1e-2 * abs(l0)
    assert rel_fro(dH, dH0) <= 1e-2
    assert rel_fro(dW, dW0) <= 1e-2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lmhead_one_row_chunks(dtype):
    """D = N: one row per chunk (the degenerate decomposition) equals the oracle and D = 1."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    N, d, V = 45, 64, 700
    h, W, y, w = synth.lmhead_inputs(46, N, d, V, bf16=(dtype == "bf16"), from_frac=0.3)
    hd, Wd = to_dev(h, dtype), to_dev(W, dtype)
    yd, wd = torch.from_numpy(y).cuda(), torch.from_numpy(w).cuda()
    out = {}
    for D in (N, 1):
        loss = torch.zeros(1, device="cuda")
        dH = torch.full((N, d), float("nan"), device="cuda")
        dW = torch.zeros(V, d, device="cuda")
        ws = sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW)
        sbp.device_status(ws)
        out[D] = (to_np(loss)[0], to_np(dH), to_np(dW))
    l0, dH0, dW0, _ = O.lmhead_ce_forward_backward(f64(h), f64(W), y, w)
    tol = 1e-5 if dtype == "f32" else 1e-2
    lN, dHN, dWN = out[N]
    assert abs(lN - l0) <= tol * abs(l0)
    assert rel_fro(dHN, dH0) <= tol and rel_fro(dWN, dW0) <= tol
    l1, dH1, dW1 = out[1]
    assert abs(lN - l1) <= 1e-6 * abs(l1)
    assert rel_fro(dHN, dH1) <= 1e-5 and rel_fro(dWN, dW1) <= 1e-5


@pytest.mark.parametrize("D", [1, 3, 8])
def test_lmhead_host_inputs_match_device_entry(D):
    """sbp_lmhead_ce_backward_stream_host (inputs in pinned host memory, staged by chunk on a
    side stream) gives bit for bit the results of the device-input entry."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    N, d, V = 1500, 128, 3000
    h, W, y, w = synth.lmhead_inputs(47, N, d, V, bf16=True, from_frac=0.25)
    hd, Wd = to_dev(h, "bf16"), to_dev(W, "bf16")
    yd, wd = torch.from_numpy(y).cuda(), torch.from_numpy(w).cuda()
    hh = hd.cpu().pin_memory()
    yh, wh = torch.from_numpy(y).pin_memory(), torch.from_numpy(w).pin_memory()
    res = []
    for host in (False, True):
        loss = torch.zeros(1, device="cuda")
        dH = torch.full((N, d), float("nan"), device="cuda")
        dW = torch.zeros(V, d, device="cuda")
        if host:
            ws = sbp.lmhead_ce_backward_host(hh, Wd, yh, wh, D, loss, dH, dW)
        else:
            ws = sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss, dH, dW)
        sbp.device_status(ws)
        res.append((loss.cpu(), dH.cpu(), dW.cpu()))
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)

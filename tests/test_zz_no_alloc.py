"""GPU test of sbp_lmhead_ce_backward_noalloc, the LM-head CE backward for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the library).

It is called through the C ABI and must give what the workspace entry point gives, on two calls
in a row (the shared scratch keeps the previous call's contents, which must not leak into the
next result).  Tolerance: relative Frobenius 1e-5, the bar used for D = 1 vs D > 1."""
import numpy as np
import pytest

from memory_efficient_exact_chunk_b200 import synth
from tests.helpers import rel_fro, to_dev, to_np

pytestmark = pytest.mark.gpu


def _buffers(h, W, y, w, dtype):
    import torch
    return (to_dev(h, dtype), to_dev(W, dtype), torch.from_numpy(y.astype(np.int32)).cuda(),
            torch.from_numpy(w.astype(np.float32)).cuda())


def _outputs(N, d, V):
    import torch
    return (torch.full((1,), float("nan"), device="cuda"),
            torch.full((N, d), float("nan"), device="cuda"), torch.zeros(V, d, device="cuda"))


@pytest.mark.parametrize("dtype,N,d,V,D", [("bf16", 640, 128, 3000, 4), ("f32", 300, 64, 1000, 3)])
def test_noalloc_matches_workspace_entry_twice(dtype, N, d, V, D):
    """Two calls in a row match the workspace entry point, and the calls allocate no device
    memory: after the first call (which may do the per-device set-up) the driver's free memory
    and torch's allocated bytes stay the same across the second call."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    h, W, y, w = synth.lmhead_inputs(21, N, d, V, bf16=(dtype == "bf16"))
    hd, Wd, yd, wd = _buffers(h, W, y, w, dtype)
    loss0, dH0, dW0 = _outputs(N, d, V)
    sbp.lmhead_ce_backward(hd, Wd, yd, wd, D, loss0, dH0, dW0)
    torch.cuda.synchronize()
    outs = [_outputs(N, d, V) for _ in range(2)]
    free_before = alloc_before = None
    for i, (loss, dH, dW) in enumerate(outs):
        if i == 1:
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info()[0]
            alloc_before = torch.cuda.memory_allocated()
        sbp.lmhead_ce_backward_noalloc(hd, Wd, yd, wd, D, loss, dH, dW)
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.mem_get_info()[0] == free_before
            assert torch.cuda.memory_allocated() == alloc_before
        assert abs(loss.item() - loss0.item()) <= 1e-5 * abs(loss0.item())
        assert rel_fro(to_np(dH), to_np(dH0)) <= 1e-5
        assert rel_fro(to_np(dW), to_np(dW0)) <= 1e-5


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from memory_efficient_exact_chunk_b200 import sbp
    lib = sbp.load()
    rc = lib.sbp_lmhead_ce_backward_noalloc(32768, 3584, 152064, 8, sbp.SBP_BF16, *([None] * 8))
    assert rc == 3
    assert "scratch" in lib.sbp_last_error().decode()

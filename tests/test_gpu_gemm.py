"""GPU check of the GEMM engine (tensor-core tcgen05 kernel and CUDA-core kernel) against a
plain PyTorch fp64 product of the same bf16 operands, for every operand layout."""
import pytest

pytestmark = pytest.mark.gpu


def _ref(A, at, B, bt):
    a = A.double().cpu()
    b = B.double().cpu()
    a = a.t() if at else a
    b = b.t() if bt else b
    return a @ b


@pytest.mark.parametrize("path", [1, 3, 4])
@pytest.mark.parametrize("at,bt", [(0, 1), (0, 0), (1, 1), (1, 0)])
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 328, 136), (64, 8, 520), (392, 1032, 3584),
                                   (8, 512, 8), (1000, 776, 520)])
def test_gemm_layouts(path, at, bt, M, N, K):
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A = torch.randn((K, M) if at else (M, K), generator=g).to(torch.bfloat16).cuda()
    B = torch.randn((N, K) if bt else (K, N), generator=g).to(torch.bfloat16).cuda()
    C0 = torch.randn(M, N, generator=g).cuda()
    C = torch.full((M, N), float("nan"), device="cuda")
    ws = sbp.debug_gemm_bf16(A, at, B, bt, C, path=path)
    sbp.device_status(ws)
    ref = _ref(A, at, B, bt)
    err = ((C.double().cpu() - ref).norm() / ref.norm()).item()
    assert err <= 1e-5, err
    C1 = C0.clone()
    sbp.debug_gemm_bf16(A, at, B, bt, C1, accumulate=True, path=path, ws=ws)
    sbp.device_status(ws)
    ref1 = ref + C0.double().cpu()
    err = ((C1.double().cpu() - ref1).norm() / ref1.norm()).item()
    assert err <= 1e-5, err


def test_gemm_tensor_core_rejects_unaligned_layout():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    A = torch.randn(64, 20).to(torch.bfloat16).cuda()     # leading dimension 20: not a multiple of 8
    B = torch.randn(20, 64).to(torch.bfloat16).cuda()
    C = torch.zeros(64, 64, device="cuda")
    for path in (2, 3, 4):
        with pytest.raises(sbp.SbpError) as ei:
            sbp.debug_gemm_bf16(A, 0, B, 0, C, path=path)
        assert ei.value.code == 2
    sbp.debug_gemm_bf16(A, 0, B, 0, C, path=0)               # automatic: CUDA cores
    ref = _ref(A, 0, B, 0)
    assert ((C.double().cpu() - ref).norm() / ref.norm()).item() <= 1e-5


def test_gemm_pair_kernel_large_ragged_accumulate():
    """A product big enough for the automatic choice of the CTA-pair kernel, ragged edges."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(11)
    M, N, K = 4000, 4616, 1032
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(K, N, generator=g).to(torch.bfloat16).cuda()
    ref = _ref(A, 0, B, 0)
    for path in (0, 4):
        C = torch.full((M, N), float("nan"), device="cuda")
        ws = sbp.debug_gemm_bf16(A, 0, B, 0, C, path=path)
        sbp.device_status(ws)
        err = ((C.double().cpu() - ref).norm() / ref.norm()).item()
        assert err <= 1e-5, (path, err)


@pytest.mark.parametrize("path", [1, 3, 4])
@pytest.mark.parametrize("at", [0, 1])
@pytest.mark.parametrize("K", [3072, 2504])
def test_gemm_k_blocks_match_sliced_products(path, at, K):
    """kblk: C equals, bit for bit, the same product taken as consecutive K slices of kblk
    rows added into C one after another (the rounding a chunked token sum sees), and stays
    within the fp32 bound of the exact product."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(K + at)
    M, N, kb = 264, 520, 1024
    A = torch.randn((K, M) if at else (M, K), generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(K, N, generator=g).to(torch.bfloat16).cuda()
    C = torch.full((M, N), float("nan"), device="cuda")
    ws = sbp.debug_gemm_bf16(A, at, B, 0, C, path=path, kblk=kb)
    sbp.device_status(ws)
    Cs = torch.full((M, N), float("nan"), device="cuda")
    for k0 in range(0, K, kb):
        k1 = min(K, k0 + kb)
        As = A[k0:k1] if at else A[:, k0:k1]
        sbp.debug_gemm_bf16(As, at, B[k0:k1], 0, Cs, accumulate=k0 > 0, path=path, ws=ws)
    sbp.device_status(ws)
    assert torch.equal(C, Cs)
    ref = _ref(A, at, B, 0)
    assert ((C.double().cpu() - ref).norm() / ref.norm()).item() <= 1e-5


def test_gemm_k_blocks_of_half_a_pair_stage():
    """kblk = 320 (a multiple of 64, not of the pair kernel's 128-column stage): the automatic
    choice takes the single-CTA kernel for a product the pair kernel would otherwise take, the
    result equals the sliced products bit for bit, and an explicit pair request is refused."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(5)
    M, N, K, kb = 2048, 2560, 1000, 320
    A = torch.randn(K, M, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(K, N, generator=g).to(torch.bfloat16).cuda()
    C = torch.full((M, N), float("nan"), device="cuda")
    ws = sbp.debug_gemm_bf16(A, 1, B, 0, C, path=0, kblk=kb)
    sbp.device_status(ws)
    Cs = torch.full((M, N), float("nan"), device="cuda")
    for k0 in range(0, K, kb):
        k1 = min(K, k0 + kb)
        sbp.debug_gemm_bf16(A[k0:k1], 1, B[k0:k1], 0, Cs, accumulate=k0 > 0, path=3, ws=ws)
    sbp.device_status(ws)
    assert torch.equal(C, Cs)
    with pytest.raises(sbp.SbpError) as ei:
        sbp.debug_gemm_bf16(A, 1, B, 0, C, path=4, kblk=kb)
    assert ei.value.code == 2


def test_gemm_k_block_argument_checked():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    A = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(64, 64, device="cuda")
    with pytest.raises(sbp.SbpError) as ei:
        sbp.debug_gemm_bf16(A, 0, B, 0, C, kblk=100)
    assert ei.value.code == 1


@pytest.mark.parametrize("wait_ms", [2, 20])
def test_bounded_wait_times_out_and_context_survives(wait_ms):
    """Failure detection without a GPU fault: the single-CTA GEMM launched with a producer that
    issues no copy, so its MMA issuer's operand wait can never complete.  The bounded wait must
    give up after the stated limit with nothing in flight, every role must wind down and free
    TMEM, the status word must report SBP_ERR_DEVICE_TIMEOUT (and be cleared by the read), C
    must be left untouched, and a normal GEMM on the same device and workspace right after
    must still match fp64."""
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    g = torch.Generator().manual_seed(wait_ms)
    A = torch.randn(256, 128, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(512, 128, generator=g).to(torch.bfloat16).cuda()
    C = torch.full((256, 512), float("nan"), device="cuda")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    ws = sbp.debug_gemm_stall_bf16(A, B, C, wait_ms * 1_000_000)
    t1.record()
    with pytest.raises(sbp.SbpError) as e:
        sbp.device_status(ws)
    assert e.value.code == 5, e.value
    elapsed = t0.elapsed_time(t1)
    assert 0.9 * wait_ms <= elapsed <= wait_ms + 500.0, elapsed
    assert torch.isnan(C).all()
    sbp.device_status(ws)                       # the read cleared the word
    sbp.debug_gemm_bf16(A, 0, B, 1, C, path=3, ws=ws)
    sbp.device_status(ws)
    ref = A.double().cpu() @ B.double().cpu().t()
    err = ((C.double().cpu() - ref).norm() / ref.norm()).item()
    assert err <= 1e-5, err


def test_stall_entry_rejects_bad_limits():
    import torch
    from memory_efficient_exact_chunk_b200 import sbp
    A = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    C = torch.zeros(128, 256, device="cuda")
    for bad in (0, 99_999, 2_000_000_001):
        with pytest.raises(sbp.SbpError) as e:
            sbp.debug_gemm_stall_bf16(A, B, C, bad)
        assert e.value.code == 1

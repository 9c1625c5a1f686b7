"""tcgen05 GEMM building block (jolt_gemm_bf16) vs a float64 product of the same bf16 inputs."""
import pytest
import torch

from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def ref_mm(A, B, a_mn, b_mn):
    A64 = A.double()
    B64 = B.double()
    Al = A64.transpose(-1, -2) if a_mn else A64       # [.., M, K]
    Bl = B64 if b_mn else B64.transpose(-1, -2)       # [.., K, N]
    return Al @ Bl


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(128, 128, 64), (1000, 1152, 1000), (304, 96, 4160),
                                   (4096, 256, 128), (64, 384, 200),
                                   # grids large enough for two 128-row tiles per CTA, ragged M/N/K
                                   (16000, 1152, 192), (80000, 200, 72)])
@pytest.mark.parametrize("plan", ["default", "perchunk", "persistent", "pairs"])
def test_gemm_majors_and_ragged(cuda_ok, plan, a_mn, b_mn, M, N, K):
    # every kernel form: the one-tile kernel (multi-chunk or per-chunk copies of MN-major operands)
    # and the persistent single-CTA / CTA-pair forms
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N * 3 + K + a_mn * 2 + b_mn)
    A = torch.randn((K, M) if a_mn else (M, K), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((K, N) if b_mn else (N, K), generator=g, device="cuda").to(torch.bfloat16)
    C = api.gemm_bf16(A, B, a_mn, b_mn, plan=plan)
    torch.cuda.synchronize()
    R = ref_mm(A, B, a_mn, b_mn)
    err = (C.double() - R).abs().max().item() / R.abs().max().item()
    assert err < tol(K), err


def tol(K):
    # fp32 accumulation of exact bf16 products: relative error grows like sqrt(K) * 2^-24
    return 2e-7 * K ** 0.5 + 1e-6


@pytest.mark.parametrize("plan", ["default", "persistent", "pairs"])
def test_gemm_split_k_and_batch(cuda_ok, plan):
    g = torch.Generator(device="cuda").manual_seed(1)
    bt, M, N, K = 3, 384, 256, 8192
    A = torch.randn(bt, K, M, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(bt, K, N, generator=g, device="cuda").to(torch.bfloat16)
    C = torch.zeros(bt, M, N, device="cuda")
    api.gemm_bf16(A, B, True, True, C=C, k_split=8, accumulate=True, plan=plan)
    torch.cuda.synchronize()
    R = ref_mm(A, B, True, True)
    err = (C.double() - R).abs().max().item() / R.abs().max().item()
    assert err < tol(K), err


@pytest.mark.parametrize("a_mn,b_mn", [(0, 0), (0, 1), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(1000, 1152, 1000), (16000, 1152, 192), (304, 200, 72), (4096, 96, 640)])
def test_gemm_hilo_outputs_split_the_fp32_result(cuda_ok, a_mn, b_mn, M, N, K):
    """The epilogue's bf16 hi / lo outputs are exactly the split of the fp32 result the same
    kernel stores (same tile plan, same accumulation order)."""
    g = torch.Generator(device="cuda").manual_seed(M + 5 * N + 7 * K + a_mn + 2 * b_mn)
    A = torch.randn((K, M) if a_mn else (M, K), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((K, N) if b_mn else (N, K), generator=g, device="cuda").to(torch.bfloat16)
    C = api.gemm_bf16(A, B, a_mn, b_mn)
    hi, lo = api.gemm_bf16_hilo(A, B, a_mn, b_mn)
    hi_only, none = api.gemm_bf16_hilo(A, B, a_mn, b_mn, lo=False)
    torch.cuda.synchronize()
    h_ref = C.to(torch.bfloat16)
    l_ref = (C - h_ref.float()).to(torch.bfloat16)
    assert none is None
    assert torch.equal(hi.view(torch.int16), h_ref.view(torch.int16))
    assert torch.equal(hi_only.view(torch.int16), h_ref.view(torch.int16))
    assert torch.equal(lo.view(torch.int16), l_ref.view(torch.int16))


@pytest.mark.parametrize("b", [2, 4, 8])
@pytest.mark.parametrize("M,K,bt,xf32", [(1000, 448, 2, False), (333, 1344, 1, True), (4096, 96, 3, False)])
def test_gemm_residual_epilogue_matches_standalone_coder(cuda_ok, M, K, bt, xf32, b):
    """The fused epilogue codes X - A @ B exactly as the stand-alone path does: the fp32 product
    stored by the same kernel, subtracted, rotated (jolt_rotate_rows) and quantised
    (jolt_quantize_pack)."""
    g = torch.Generator(device="cuda").manual_seed(M + K + 11 * b + bt)
    A = torch.randn(bt, M, K, generator=g, device="cuda").to(torch.bfloat16)
    B = (0.05 * torch.randn(bt, K, 128, generator=g, device="cuda")).to(torch.bfloat16)
    X = torch.randn(bt, M, 128, generator=g, device="cuda")
    X = X if xf32 else X.to(torch.bfloat16)
    seed = 0x1234ABCD + b
    codes, sz, err = api.gemm_bf16_residual(A, B, X, seed, b)
    C = api.gemm_bf16(A, B, False, True)
    x = (X.float() - C).reshape(bt * M, 128)
    rc, rsz, rerr = api.quantize_pack(api.rotate_rows(x, seed), b)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and int(rerr.item()) == 0
    assert torch.equal(codes, rc)
    assert torch.equal(sz.view(torch.int16), rsz.view(torch.int16))

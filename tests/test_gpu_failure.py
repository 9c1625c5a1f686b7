"""Failure detection on the GPU without a fault: a wait that nothing will end gives up after its
bound, the kernel returns, the host reads JOLT_ERR_TIMEOUT from the workspace's error word, and
the context stays usable (a GEMM afterwards is still exact)."""
import pytest
import torch

from long_context_st_b200 import api
from long_context_st_b200._lib import lib, JoltError

pytestmark = pytest.mark.gpu

JOLT_ERR_TIMEOUT = -3


@pytest.mark.parametrize("which", [0, 1], ids=["mbarrier", "grid_barrier"])
def test_bounded_wait_reports_timeout_and_context_survives(cuda_ok, which):
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib().jolt_selftest_timeout(which, 1_000_000, ws.data_ptr(), 512, st) == 0
    with pytest.raises(JoltError) as e:
        api.check_ws(ws)
    assert e.value.status == JOLT_ERR_TIMEOUT
    api.check_ws(ws)  # the error word was cleared by the read
    g = torch.Generator(device="cuda").manual_seed(3)
    A = torch.randn(300, 256, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(200, 256, generator=g, device="cuda").to(torch.bfloat16)
    C = api.gemm_bf16(A, B)
    torch.cuda.synchronize()
    R = A.double() @ B.double().T
    assert (C.double() - R).abs().max().item() <= 1e-5 * R.abs().max().item()


def test_selftest_rejects_unbounded_limits(cuda_ok):
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib().jolt_selftest_timeout(0, 0, ws.data_ptr(), 512, st) == -1
    assert lib().jolt_selftest_timeout(0, 5_000_000_000, ws.data_ptr(), 512, st) == -1
    assert lib().jolt_selftest_timeout(2, 1000, ws.data_ptr(), 512, st) == -1

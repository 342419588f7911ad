"""Failure detection on the GPU without a GPU fault: the GEMM kernels' bounded
mbarrier waits are given a 1 ns limit so that they run out on purpose. The
kernels must record the timeout, drain their own copies and MMAs, free TMEM and
return; the host reads MOE_ERR_DEVICE_TIMEOUT, and the next call on the same
context and workspace computes the right answer."""
import pytest
import torch

from sparse_mixture_experts_aux_b200 import Workspace, _lib, forward, moe_get_device_status
from sparse_mixture_experts_aux_b200.inputs import Workload, make_inputs
from tests.parity_util import compare, oracle_quantized_weights, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("w", [
    Workload("timeout routed", 1000, 512, 4, 320, 2, seed=41),
    Workload("timeout shared", 300, 256, 16, 128, 4, d_s=192, seed=42),
    Workload("timeout pair kernels", 4200, 256, 2, 256, 1, d_s=128, seed=43),
], ids=lambda w: w.name)
def test_expired_waits_are_reported_and_the_context_survives(w):
    inp = make_inputs(w, device="cuda")
    ws = Workspace()
    assert moe_get_device_status() == _lib.MOE_OK
    for _ in range(3):
        forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], inp["W_shared"], k=w.k,
                d_s=w.d_s, workspace=ws, wait_timeout_ns=1)
        torch.cuda.synchronize()
        assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT
        assert moe_get_device_status() == _lib.MOE_OK  # reading it resets it
    gpu = run_gpu(w, inp, ws)  # default limit: completes and matches the oracle
    compare(w, gpu, run_oracle(w, inp))


@pytest.mark.parametrize("w", [
    Workload("timeout fp8 32-row box", 20, 256, 4, 320, 2, seed=44),
    Workload("timeout fp8 128-row box", 700, 256, 4, 320, 2, seed=45),
], ids=lambda w: w.name)
def test_expired_waits_fp8_kernels(w):
    inp = make_inputs(w, device="cuda")
    fp8 = oracle_quantized_weights(inp)
    ws = Workspace()
    for _ in range(3):
        forward(inp["x"], inp["W_r"], fp8["W_g"], fp8["W_u"], fp8["W_d"], None, k=w.k,
                workspace=ws, weight_scales=fp8["weight_scales"], wait_timeout_ns=1)
        torch.cuda.synchronize()
        assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT
        assert moe_get_device_status() == _lib.MOE_OK
    gpu = run_gpu(w, inp, ws, fp8=fp8)
    compare(w, gpu, run_oracle(w, inp, fp8=fp8))

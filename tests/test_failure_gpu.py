"""Failure detection on the GPU without a GPU fault: the GEMM kernels' bounded
mbarrier waits are given a 1 ns limit so that they run out on purpose. The
kernels must record the timeout, drain their own copies and MMAs, free TMEM and
return; the host reads MOE_ERR_DEVICE_TIMEOUT, and the next call on the same
context and workspace computes the right answer."""
import pytest
import torch

from sparse_mixture_experts_aux_b200 import (Workspace, _lib, forward, moe_get_device_status,
                                             routing_views)
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
    Workload("timeout token-major 32-row box", 20, 256, 4, 256, 2, seed=47),
], ids=lambda w: w.name)
def test_expired_waits_are_reported_and_the_context_survives(w):
    inp = make_inputs(w, device="cuda")
    ws = Workspace()
    assert moe_get_device_status() == _lib.MOE_OK
    for _ in range(3):
        forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], inp["W_shared"], k=w.k,
                d_s=w.d_s, workspace=ws, wait_timeout_ns=1)
        torch.cuda.synchronize()
        # the call's own status word records it, and so does the device-wide word
        status = routing_views(ws.buf, inp["x"], inp["W_g"], w.E, w.k, 0.0, w.d_s)["status"]
        assert int(status[0]) != 0
        assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT
        assert moe_get_device_status() == _lib.MOE_OK  # reading it resets it
    gpu = run_gpu(w, inp, ws)  # default limit: completes and matches the oracle
    assert int(gpu[3]["status"][0]) == 0  # cleared by the next call
    compare(w, gpu, run_oracle(w, inp))


def test_host_io_reports_its_own_timeout_only():
    # two calls through the host-buffer entry point on two streams, one with
    # waits that expire: only that call reports the timeout
    w = Workload("timeout host io", 300, 256, 4, 320, 2, seed=46)
    inp = make_inputs(w, device="cuda")
    out = {}
    for name, tmo in (("bad", 1), ("good", 0)):
        ws = Workspace()
        ws.get(_lib.moe_workspace_size(_lib.make_dims(w.T, w.d, w.d_e), w.E, w.k, 0.0), "cuda")
        stream = torch.cuda.Stream()
        dims = _lib.make_dims(w.T, w.d, w.d_e, 0, _lib.MOE_BF16, None, ws.buf, ws.buf.numel(),
                              stream.cuda_stream, wait_timeout_ns=tmo)
        x_host = inp["x"].cpu().pin_memory()
        y_host = torch.empty_like(x_host).pin_memory()
        st = _lib.moe_forward_host_io(
            dims, x_host, torch.empty_like(inp["x"]), inp["W_r"], inp["W_g"], inp["W_u"],
            inp["W_d"], None, w.E, w.k, 0.0, torch.empty_like(inp["x"]), y_host,
            torch.empty(1, device="cuda"), torch.empty(1).pin_memory(),
            torch.empty(w.E, dtype=torch.int32, device="cuda"),
            torch.empty(w.E, dtype=torch.int32).pin_memory(), check=False)
        out[name] = st
    assert out == {"bad": _lib.MOE_ERR_DEVICE_TIMEOUT, "good": _lib.MOE_OK}
    torch.cuda.synchronize()
    assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT  # the device-wide word too
    assert moe_get_device_status() == _lib.MOE_OK


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

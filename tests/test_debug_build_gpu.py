"""The MOE_DEBUG build (libmoe_debug.so) on the GPU.

Its kernels check every permuted row (scatter, combine), the segment total
(scan) and every GEMM tile's expert and row coordinates against the buffers
they address; a failed check sets a bit in the device error word and skips
the access instead of trapping. On correct inputs no check may fire, and the
checks change no arithmetic: the outputs must equal the release library's
bit for bit and match the oracle. Covered: the 1-CTA and CTA-pair GEMMs, the
shared expert, capacity, and both FP8 weight paths."""
import ctypes

import pytest
import torch

from sparse_mixture_experts_aux_b200 import Workspace, _lib, forward, moe_get_device_status
from sparse_mixture_experts_aux_b200.inputs import Workload, make_inputs
from tests.parity_util import compare, oracle_quantized_weights, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _debug_forward(w, inp, ws, W, scales=None, act_fp8=False):
    dbg = _lib.load_debug()
    fmt = _lib.MOE_WEIGHTS_DTYPE
    if scales is not None:
        fmt = _lib.MOE_WEIGHTS_FP8_W8A8 if act_fp8 else _lib.MOE_WEIGHTS_FP8
    dims = _lib.make_dims(w.T, w.d, w.d_e, w.d_s, _lib.MOE_BF16, inp["router_bias"], ws,
                          ws.numel(), torch.cuda.current_stream().cuda_stream,
                          weight_format=fmt, weight_scales=scales)
    y = torch.empty_like(inp["x"])
    aux = torch.empty(1, dtype=torch.float32, device="cuda")
    counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
    p = _lib._ptr
    st = dbg.moe_forward(ctypes.byref(dims), p(inp["x"]), p(inp["W_r"]), p(W["W_g"]),
                         p(W["W_u"]), p(W["W_d"]), p(inp["W_shared"]), w.E, w.k,
                         w.capacity_factor, p(y), p(aux), p(counts))
    assert st == _lib.MOE_OK, _lib.status_string(st)
    torch.cuda.synchronize()
    assert dbg.moe_get_device_status() == _lib.MOE_OK, "a debug bounds check or wait fired"
    return y, aux, counts


CASES = [
    (Workload("debug shared+capacity", 700, 256, 8, 256, 2, d_s=256, capacity_factor=0.8,
              seed=71), None),
    (Workload("debug pair kernels odd tiles", 4300, 256, 2, 320, 1, d_s=128, seed=72), None),
    (Workload("debug fp8 weights, 32-row box", 20, 256, 4, 320, 2, seed=73), "fp8"),
    (Workload("debug w8a8", 300, 256, 8, 256, 2, seed=74), "w8a8"),
]


@pytest.mark.parametrize("w,fmt", CASES, ids=[c[0].name for c in CASES])
def test_debug_build_is_silent_and_bit_identical(w, fmt):
    inp = make_inputs(w, device="cuda")
    W, scales, act = inp, None, fmt == "w8a8"
    if fmt is not None:
        W = oracle_quantized_weights(inp)
        scales = W["weight_scales"]
    ws = Workspace()
    y_rel, aux_rel, counts_rel = forward(inp["x"], inp["W_r"], W["W_g"], W["W_u"], W["W_d"],
                                         inp["W_shared"], k=w.k,
                                         capacity_factor=w.capacity_factor, d_s=w.d_s,
                                         workspace=ws, weight_scales=scales, act_fp8=act)
    torch.cuda.synchronize()
    assert moe_get_device_status() == _lib.MOE_OK
    ws_dbg = torch.empty_like(ws.buf)
    y, aux, counts = _debug_forward(w, inp, ws_dbg, W, scales, act)
    assert torch.equal(y, y_rel) and torch.equal(aux, aux_rel) and torch.equal(counts, counts_rel)
    from sparse_mixture_experts_aux_b200 import routing_views
    views = routing_views(ws_dbg, inp["x"], W["W_g"], w.E, w.k, w.capacity_factor, w.d_s,
                          act_fp8=act)
    assert int(views["status"][0]) == 0
    compare(w, (y, aux, counts, views), run_oracle(w, inp, fp8=W if fmt else None,
                                                    act_fp8=act))

"""moe_forward_no_alloc: the forward pass for callers that cannot allocate
device memory (for example a plugin inside a host that has reserved all free
device memory for its own pool). It runs on the library's own statically
sized scratch array instead of a caller-provided workspace.

Checked here through the C ABI: its results match moe_forward's (given a
torch-allocated workspace) on two calls in a row, and after calls of layers
with another layout that leave different stale contents in the shared
array; a layer that needs more scratch than the fixed maximum is refused
before anything is enqueued. This
file is collected last on purpose, so that a stop-at-first-failure run has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_aux_b200 import Workspace, _lib, forward, moe_get_device_status
from sparse_mixture_experts_aux_b200.inputs import MIXTRAL, MIXTRAL_DECODE, Workload, make_inputs
from tests.parity_util import Y_TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


CASES = [
    MIXTRAL_DECODE,
    Workload("no-alloc shared expert + capacity", 700, 256, 8, 256, 2, d_s=256,
             capacity_factor=0.8, seed=51),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_no_alloc_matches_workspace_entry_point_on_two_calls(w):
    inp = make_inputs(w, device="cuda")
    y_ref, aux_ref, counts_ref = forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"],
                                         inp["W_shared"], k=w.k,
                                         capacity_factor=w.capacity_factor,
                                         router_bias=inp["router_bias"], d_s=w.d_s,
                                         workspace=Workspace())
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    dt = _lib.MOE_BF16 if w.dtype == "bf16" else _lib.MOE_F32
    dims = _lib.make_dims(w.T, w.d, w.d_e, w.d_s, dt, inp["router_bias"], None, 0, stream)
    assert _lib.moe_workspace_size(dims, w.E, w.k, w.capacity_factor) <= \
        _lib.MOE_NO_ALLOC_WORKSPACE_BYTES
    tol = Y_TOL[w.dtype]
    ref = y_ref.float().cpu().numpy()
    for _ in range(2):
        y = torch.full_like(inp["x"], float("nan"))
        aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        counts = torch.full((w.E,), -1, dtype=torch.int32, device="cuda")
        st = _lib.moe_forward_no_alloc(dims, inp["x"], inp["W_r"], inp["W_g"], inp["W_u"],
                                       inp["W_d"], inp["W_shared"], w.E, w.k, w.capacity_factor,
                                       y, aux, counts, check=False)
        assert st == _lib.MOE_OK, _lib.status_string(st)
        torch.cuda.synchronize()
        assert moe_get_device_status() == _lib.MOE_OK
        got = y.float().cpu().numpy()
        assert np.all(np.abs(got - ref) <= tol * np.maximum(1.0, np.abs(ref)))
        assert torch.equal(counts.cpu(), counts_ref.cpu())
        assert float(aux.cpu()[0]) == pytest.approx(float(aux_ref.cpu()[0]), rel=1e-6)


def _no_alloc_call(w, inp):
    stream = torch.cuda.current_stream().cuda_stream
    dt = _lib.MOE_BF16 if w.dtype == "bf16" else _lib.MOE_F32
    dims = _lib.make_dims(w.T, w.d, w.d_e, w.d_s, dt, inp["router_bias"], None, 0, stream)
    y = torch.full_like(inp["x"], float("nan"))
    aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    counts = torch.full((w.E,), -1, dtype=torch.int32, device="cuda")
    st = _lib.moe_forward_no_alloc(dims, inp["x"], inp["W_r"], inp["W_g"], inp["W_u"],
                                   inp["W_d"], inp["W_shared"], w.E, w.k, w.capacity_factor,
                                   y, aux, counts, check=False)
    assert st == _lib.MOE_OK, _lib.status_string(st)
    torch.cuda.synchronize()
    assert moe_get_device_status() == _lib.MOE_OK
    return y, aux, counts


def test_no_alloc_after_a_different_layout():
    # Every call shares the scratch array and finds what the previous call left:
    # here each call follows a layer with another E, capacity cut, shared expert
    # and row layout, so stale segment starts, row gates, logits splits and rows
    # of the other layout sit in the array when it starts.
    layers = [CASES[1], MIXTRAL_DECODE, CASES[1], MIXTRAL_DECODE]
    inputs = {w.name: make_inputs(w, device="cuda") for w in layers[:2]}
    refs = {}
    for w in layers[:2]:
        inp = inputs[w.name]
        refs[w.name] = forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"],
                               inp["W_shared"], k=w.k, capacity_factor=w.capacity_factor,
                               router_bias=inp["router_bias"], d_s=w.d_s, workspace=Workspace())
    torch.cuda.synchronize()
    for w in layers:
        y, aux, counts = _no_alloc_call(w, inputs[w.name])
        y_ref, aux_ref, counts_ref = refs[w.name]
        ref = y_ref.float().cpu().numpy()
        got = y.float().cpu().numpy()
        assert np.all(np.abs(got - ref) <= Y_TOL[w.dtype] * np.maximum(1.0, np.abs(ref))), w.name
        assert torch.equal(counts.cpu(), counts_ref.cpu())
        assert float(aux.cpu()[0]) == pytest.approx(float(aux_ref.cpu()[0]), rel=1e-6)


def test_no_alloc_refuses_layers_beyond_its_scratch():
    w = MIXTRAL  # T=4096: the workspace is several hundred MiB
    dims = _lib.make_dims(w.T, w.d, w.d_e, 0, _lib.MOE_BF16, None, None, 0, 0)
    need = _lib.moe_workspace_size(dims, w.E, w.k, 0.0)
    assert need > _lib.MOE_NO_ALLOC_WORKSPACE_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes before any launch
    st = _lib.moe_forward_no_alloc(dims, fake, fake, fake, fake, fake, None, w.E, w.k, 0.0, fake,
                                   fake, fake, check=False)
    assert st == _lib.MOE_ERR_SCRATCH_LIMIT
    assert _lib.status_string(st) == "MOE_ERR_SCRATCH_LIMIT"

"""GPU parity: moe_forward (through the C ABI) against the fp64 oracle.

Small cases span several 128-row tiles, N tails and ragged row counts; the
full-size workloads are compared on every routing result and on a seeded
sample of 256 output rows (the oracle evaluates those one by one)."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_aux_b200 import Workspace, forward, moe_get_device_status
from sparse_mixture_experts_aux_b200.inputs import (DEEPSEEK_V3, MIXTRAL, MIXTRAL_DECODE,
                                                    SWITCH_ZIPF, TINY_F32, Workload, make_inputs)
from tests.parity_util import check_workload, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

SMALL = [
    Workload("bf16 ragged rows, N tail", 1000, 512, 4, 320, 2, seed=11),
    Workload("bf16 many experts", 777, 256, 32, 256, 4, seed=12),
    Workload("bf16 shared expert", 300, 256, 16, 128, 4, d_s=192, seed=13),
    Workload("bf16 capacity zipf top1", 2048, 256, 16, 256, 1, capacity_factor=1.25,
             zipf_bias=True, seed=14),
    Workload("bf16 capacity top2", 600, 192, 8, 192, 2, capacity_factor=0.5, seed=15),
    Workload("bf16 down N tail d=320", 513, 320, 8, 256, 2, seed=16),
    Workload("bf16 k=E", 200, 128, 4, 128, 4, seed=17),
    Workload("bf16 single expert", 130, 128, 1, 128, 1, seed=18),
    Workload("bf16 E=1024 k=32", 64, 64, 1024, 64, 32, seed=19),
    Workload("bf16 one token", 1, 256, 8, 256, 2, seed=20),
    # batches of <= 64 / <= 32 tokens use the short activation boxes
    Workload("bf16 T=48 shared expert, 64-row box", 48, 256, 8, 256, 2, d_s=128, seed=33),
    Workload("bf16 T=20 capacity, 32-row box", 20, 192, 4, 192, 2, capacity_factor=1.5, seed=34),
    Workload("bf16 shared+capacity", 700, 256, 8, 256, 2, d_s=256, capacity_factor=0.8, seed=21),
    Workload("fp32 shared+capacity", 333, 128, 8, 96, 2, "f32", d_s=64, capacity_factor=0.7, seed=22),
    Workload("fp32 ragged", 257, 96, 5, 160, 3, "f32", seed=23),
    # more than 64 tokens and up to 2048 (gate/up) or 512 (down) routed rows per
    # expert: the swapped-operand kernels, token tiles sized to their valid rows
    Workload("bf16 T=65, smallest swapped batch", 65, 256, 8, 256, 2, seed=35),
    Workload("bf16 about 3 rows per expert (N=16 tiles), shared", 100, 256, 64, 128, 2, d_s=64,
             seed=36),
    # > 512 routed rows per expert run the down GEMM on CTA pairs (cta_group::2),
    # > 2048 the gate/up GEMM as well
    Workload("pair odd tile counts", 4300, 256, 2, 320, 1, seed=24),
    Workload("pair shared expert", 4200, 256, 2, 256, 1, d_s=128, seed=25),
    Workload("pair both GEMMs k=2", 2200, 256, 2, 192, 2, seed=28),
    Workload("pair down only", 1100, 256, 2, 320, 1, seed=29),
    Workload("pair down N tail d=320", 1300, 320, 2, 256, 2, seed=26),
    Workload("pair capacity", 2600, 256, 4, 192, 1, capacity_factor=0.9, zipf_bias=True, seed=27),
]


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_parity(w):
    check_workload(w)


def test_tiny_fp32_workload_full():
    r = check_workload(TINY_F32)
    assert r["near_ties"] == 0


def test_decode_workload_full():
    check_workload(MIXTRAL_DECODE)


def test_mixtral_workload_sampled():
    check_workload(MIXTRAL, sample=256)


def test_switch_zipf_workload_sampled():
    r = check_workload(SWITCH_ZIPF, sample=256)
    print(f"switch: {r['rows_compared']} of {r['rows_sampled']} sampled rows compared, "
          f"{r['near_ties']} near-tie tokens, {r['excluded']} tokens excluded")
    assert r["rows_compared"] >= 200


def test_deepseek_v3_workload_sampled():
    check_workload(DEEPSEEK_V3, sample=256)


def test_uniform_router_ties_and_aux_exactly_one():
    w = Workload("uniform router", 256, 128, 8, 128, 2, seed=30)
    inp = make_inputs(w, device="cuda")
    inp["W_r"].zero_()
    y, aux, counts, views = run_gpu(w, inp)
    idx = views["topk_idx"].cpu().numpy()
    assert (idx == np.array([0, 1])).all()
    assert counts.cpu().tolist() == [256, 256, 0, 0, 0, 0, 0, 0]
    assert float(aux.cpu()[0]) == 1.0
    assert torch.allclose(views["gates"].cpu(), torch.full((256, 2), 0.5))


def test_empty_batch():
    w = Workload("empty", 0, 128, 8, 128, 2, seed=31)
    inp = make_inputs(w, device="cuda")
    aux = torch.full((1,), 7.0, device="cuda")
    counts = torch.full((8,), 7, dtype=torch.int32, device="cuda")
    y, aux, counts = forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"], k=2,
                             aux=aux, counts=counts)
    torch.cuda.synchronize()
    assert float(aux[0]) == 0.0 and counts.cpu().tolist() == [0] * 8 and y.shape == (0, 128)


def test_deterministic_bits():
    w = SMALL[1]
    inp = make_inputs(w, device="cuda")
    a = run_gpu(w, inp)
    b = run_gpu(w, inp)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_every_assignment_dropped_gives_zero():
    w = Workload("all dropped", 128, 128, 8, 128, 1, capacity_factor=1e-6, seed=32)
    inp = make_inputs(w, device="cuda")
    y, aux, counts, views = run_gpu(w, inp)
    assert (views["slot_pos"] == -1).all()
    assert torch.count_nonzero(y) == 0
    assert int(counts.sum()) == 128


def test_workspace_reuse_across_shapes():
    ws = Workspace()
    for w in (SMALL[0], SMALL[2], SMALL[0]):
        inp = make_inputs(w, device="cuda")
        gpu = run_gpu(w, inp, ws)
        compare(w, gpu, run_oracle(w, inp))


def test_host_io_entry_point_matches_device_entry_point():
    from sparse_mixture_experts_aux_b200 import _lib
    w = SMALL[0]
    inp = make_inputs(w, device="cuda")
    ws = Workspace()
    y_ref, aux_ref, counts_ref = forward(inp["x"], inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"],
                                         k=w.k, workspace=ws)
    torch.cuda.synchronize()
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty_like(x_host).pin_memory()
    aux_host = torch.empty(1, dtype=torch.float32).pin_memory()
    counts_host = torch.empty(w.E, dtype=torch.int32).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    y_dev = torch.empty_like(inp["x"])
    aux_dev = torch.empty(1, dtype=torch.float32, device="cuda")
    counts_dev = torch.empty(w.E, dtype=torch.int32, device="cuda")
    dims = _lib.make_dims(w.T, w.d, w.d_e, 0, _lib.MOE_BF16, None, ws.buf, ws.buf.numel(),
                          torch.cuda.current_stream().cuda_stream)
    _lib.moe_forward_host_io(dims, x_host, x_dev, inp["W_r"], inp["W_g"], inp["W_u"], inp["W_d"],
                             None, w.E, w.k, 0.0, y_dev, y_host, aux_dev, aux_host, counts_dev,
                             counts_host)
    assert torch.equal(y_host, y_ref.cpu())
    assert torch.equal(aux_host, aux_ref.cpu()) and torch.equal(counts_host, counts_ref.cpu())
    assert moe_get_device_status() == 0

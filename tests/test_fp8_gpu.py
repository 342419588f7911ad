"""GPU parity of the FP8 (E4M3) expert-weight path against the oracle.

* moe_quantize_fp8: codes and scales bit-exact against the oracle's quantiser
  (bf16 and fp32 weights, zero rows, exact rounding ties, grid-stride sizes).
* moe_dequantize_fp8: every finite code, times several scales (subnormal fp32
  products included), bit-exact against the oracle's exact value rounded once
  to fp32: this pins the on-chip decode the GEMM converters share.
* moe_forward with FP8 weights: routing exactly as in the bf16 path, y within
  the bf16 tolerance of the oracle computing with code * scale in fp64; small
  cases over the three activation-box sizes and N tails (weights quantised by
  the oracle), random codes, and the full-size Mixtral decode shape.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_aux_b200 import dequantize_fp8, quantize_fp8
from sparse_mixture_experts_aux_b200.inputs import (MIXTRAL_DECODE, Workload, make_fp8_weights,
                                                    make_inputs)
from tests.parity_util import compare, oracle_quantized_weights, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _finite_codes() -> np.ndarray:
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def _tie_row(cols: int) -> np.ndarray:
    """448 (so the row scale is exactly 1) followed by midpoints between
    neighbouring E4M3 values of both signs: every entry is a rounding tie."""
    vals = np.sort(np.unique(np.abs(O.e4m3_decode(_finite_codes()))))
    mids = (vals[:-1] + vals[1:]) / 2
    row = np.concatenate([[448.0], mids, -mids])
    return np.resize(row, cols)


@pytest.mark.parametrize("dtype,rows,cols", [
    (torch.bfloat16, 100, 4096),
    (torch.float32, 9000, 32),      # more rows than the quantiser's grid
    (torch.float32, 17, 1008),      # columns not a multiple of the block
    (torch.bfloat16, 1, 16),
])
def test_quantizer_bit_exact(dtype, rows, cols):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    w = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    if rows > 3:
        w[1] = 0.0                                   # all-zero row: scale 1, codes 0
        w[2] = 0.0
        w[2, cols // 2] = -3.5                       # one non-zero entry
        w[3] = torch.from_numpy(_tie_row(cols)).float()
    w = w.to(dtype)
    codes, scales = quantize_fp8(w.cuda())
    torch.cuda.synchronize()
    ref_codes, ref_scales = O.quantize_rows_fp8(w.float().numpy())
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


def test_dequantizer_covers_every_code_bit_exact():
    codes = np.zeros(256, dtype=np.uint8)
    fc = _finite_codes()
    codes[:fc.size] = fc
    scales = np.array([1.0, 2.0 ** -20, 0.0037, 3e30, 1e-38, 7.25], dtype=np.float32)
    cm = np.tile(codes, (scales.size, 1))
    out = dequantize_fp8(torch.from_numpy(cm).cuda(), torch.from_numpy(scales).cuda())
    torch.cuda.synchronize()
    ref = O.dequantize_rows_fp8(cm, scales).astype(np.float32)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


SMALL_FP8 = [
    Workload("fp8 one token, 32-row box", 1, 256, 8, 256, 2, seed=40),
    Workload("fp8 T=20 capacity, 32-row box", 20, 192, 4, 192, 2, capacity_factor=1.5, seed=41),
    Workload("fp8 T=48 N tail, 64-row box", 48, 256, 8, 320, 2, seed=42),
    Workload("fp8 ragged rows, 128-row box", 1000, 512, 4, 320, 2, seed=43),
    Workload("fp8 many experts", 777, 256, 32, 256, 4, seed=44),
    Workload("fp8 down N tail d=320", 513, 320, 8, 256, 2, seed=45),
    Workload("fp8 sigmoid groups selection bias", 300, 256, 16, 128, 4, gate_mode=2, n_group=4,
             topk_group=2, selection_bias=True, seed=46),
]


@pytest.mark.parametrize("w", SMALL_FP8, ids=[w.name for w in SMALL_FP8])
def test_fp8_forward_small(w):
    inp = make_inputs(w, device="cuda")
    fp8 = oracle_quantized_weights(inp)
    gpu = run_gpu(w, inp, fp8=fp8)
    ref = run_oracle(w, inp, fp8=fp8)
    compare(w, gpu, ref)


def test_fp8_forward_random_codes():
    w = Workload("fp8 random codes", 600, 384, 8, 448, 2, seed=47)
    inp = make_inputs(w, device="cuda")
    fp8 = make_fp8_weights(w, device="cuda")
    compare(w, run_gpu(w, inp, fp8=fp8), run_oracle(w, inp, fp8=fp8))


def test_fp8_forward_mixtral_decode_full_size():
    w = MIXTRAL_DECODE
    inp = make_inputs(w, device="cuda")
    fp8 = make_fp8_weights(w, device="cuda")
    gpu = run_gpu(w, inp, fp8=fp8)
    inp.pop("W_g"), inp.pop("W_u"), inp.pop("W_d")
    compare(w, gpu, run_oracle(w, inp, fp8=fp8))

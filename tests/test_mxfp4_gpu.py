"""GPU parity of the MXFP4 expert-weight path (MOE_WEIGHTS_MXFP4) against the oracle.

* moe_quantize_mxfp4: codes (two per byte), E8M0 block scales and row factors
  bit-exact against the oracle's block quantiser (bf16 and fp32 weights, zero
  blocks and rows, exact rounding ties, saturation, grid-stride sizes).
* moe_dequantize_mxfp4: every code at several block exponents, bit-exact
  against the oracle's exact value: this pins the on-chip decode the GEMM
  converters share (including the nibble order of the hardware conversion).
* moe_forward with MXFP4 weights: routing exactly as in the bf16 path, y within
  the bf16 tolerance of the oracle computing with code * 2^X in fp64, over the
  three activation-box sizes, many experts, capacity and the full-size decode
  shape; and the bounded waits' timeout path.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_aux_b200 import (Workspace, _lib, dequantize_mxfp4, forward,
                                             moe_get_device_status, quantize_mxfp4)
from sparse_mixture_experts_aux_b200.inputs import MIXTRAL_DECODE, Workload, make_inputs
from tests.parity_util import (compare, oracle_mxfp4_weights, pack_e2m1, row_factors_of,
                               run_gpu, run_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _unpack(packed: np.ndarray) -> np.ndarray:
    lo, hi = packed & 0xF, packed >> 4
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2], out[..., 1::2] = lo, hi
    return out


def _tie_block(X: int) -> np.ndarray:
    """A block whose absmax gives exponent X and whose other entries sit exactly
    on midpoints between neighbouring E2M1 values (scaled by 2^X), both signs."""
    vals = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (vals[:-1] + vals[1:]) / 2
    b = np.resize(np.concatenate([mids, -mids, [7.5, -6.5]]), 32)
    b[0] = 7.0  # absmax in [4, 8): exponent X; 7 saturates to 6
    return b * 2.0 ** X


@pytest.mark.parametrize("dtype,rows,cols", [
    (torch.bfloat16, 100, 4096),
    (torch.float32, 9000, 64),      # more rows than the quantiser's grid
    (torch.float32, 17, 1024),
    (torch.bfloat16, 1, 32),
])
def test_quantizer_bit_exact(dtype, rows, cols):
    g = torch.Generator().manual_seed(rows * 7 + cols)
    w = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    w *= torch.exp2(torch.randint(-12, 4, (rows, cols // 32), generator=g).float()).repeat_interleave(32, 1)
    if rows > 3:
        w[1] = 0.0                                             # all-zero row: factor 1
        w[2, :32] = 0.0                                        # one all-zero block
        w[3, :32] = torch.from_numpy(_tie_block(-3)).float()   # ties and saturation
    w = w.to(dtype)
    codes, bsc, rf = quantize_mxfp4(w.cuda())
    torch.cuda.synchronize()
    rc, rx = O.quantize_rows_mxfp4(w.float().numpy())
    assert np.array_equal(_unpack(codes.cpu().numpy()), rc), "E2M1 codes differ"
    assert np.array_equal(bsc.cpu().numpy().astype(np.int64) - 127, rx), "block exponents differ"
    assert np.array_equal(rf.cpu().numpy(), row_factors_of(rc, rx)), "row factors differ"


def test_dequantizer_every_code_bit_exact():
    # rows of all 16 codes (twice) in blocks whose exponents lie within 23 of the
    # row's largest: the layer's decode is exact there
    codes = np.resize(np.arange(16, dtype=np.uint8), (6, 32 * 4))
    exps = np.array([[0, -5, -23, -1], [7, 7, 7, 7], [-40, -44, -63, -50],
                     [20, 0, 12, 1], [0, 0, 0, 0], [-1, -2, -3, -4]], dtype=np.int64)
    rf = row_factors_of(codes, exps)
    packed = torch.from_numpy(pack_e2m1(codes)).cuda()
    bsc = torch.from_numpy((exps + 127).astype(np.uint8)).cuda()
    out = dequantize_mxfp4(packed, bsc, torch.from_numpy(rf).cuda())
    torch.cuda.synchronize()
    want = O.dequantize_rows_mxfp4(codes, exps).astype(np.float32)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), want.view(np.uint32))


SMALL_MX = [
    Workload("mxfp4 one token, 32-row box", 1, 256, 8, 256, 2, seed=80),
    Workload("mxfp4 T=20 capacity, 32-row box", 20, 256, 4, 512, 2, capacity_factor=1.5, seed=81),
    Workload("mxfp4 T=48, 64-row box", 48, 512, 8, 256, 2, seed=82),
    Workload("mxfp4 ragged rows, 128-row box", 1000, 256, 4, 768, 2, seed=83),
    Workload("mxfp4 many experts", 777, 256, 32, 256, 4, seed=84),
]


@pytest.mark.parametrize("w", SMALL_MX, ids=[w.name for w in SMALL_MX])
def test_mxfp4_forward_small(w):
    inp = make_inputs(w, device="cuda")
    mx = oracle_mxfp4_weights(inp)
    compare(w, run_gpu(w, inp, fp8=mx), run_oracle(w, inp, fp8=mx))


def test_library_quantised_layer_matches_oracle_quantised_layer():
    # the same weights quantised by the library give the same codes, so the same layer
    w = SMALL_MX[3]
    inp = make_inputs(w, device="cuda")
    mx = oracle_mxfp4_weights(inp)
    lib = {}
    parts_b, parts_r = [], []
    for name in ("W_g", "W_u", "W_d"):
        lib[name], b, r = quantize_mxfp4(inp[name])
        parts_b.append(b.reshape(-1))
        parts_r.append(r.reshape(-1))
        assert torch.equal(lib[name], mx[name])
    assert torch.equal(torch.cat(parts_b), mx["block_scales"])
    assert torch.equal(torch.cat(parts_r), mx["weight_scales"])


def test_mxfp4_decode_full_size():
    w = MIXTRAL_DECODE
    inp = make_inputs(w, device="cuda")
    mx = oracle_mxfp4_weights(inp)
    gpu = run_gpu(w, inp, fp8=mx)
    inp.pop("W_g"), inp.pop("W_u"), inp.pop("W_d")
    compare(w, gpu, run_oracle(w, inp, fp8=mx))


@pytest.mark.parametrize("w", [
    Workload("timeout mxfp4 32-row box", 20, 256, 4, 256, 2, seed=85),
    Workload("timeout mxfp4 128-row box", 700, 256, 4, 512, 2, seed=86),
], ids=lambda w: w.name)
def test_mxfp4_expired_waits(w):
    inp = make_inputs(w, device="cuda")
    mx = oracle_mxfp4_weights(inp)
    ws = Workspace()
    for _ in range(2):
        forward(inp["x"], inp["W_r"], mx["W_g"], mx["W_u"], mx["W_d"], None, k=w.k, workspace=ws,
                weight_scales=mx["weight_scales"], weight_block_scales=mx["block_scales"],
                wait_timeout_ns=1)
        torch.cuda.synchronize()
        assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT
        assert moe_get_device_status() == _lib.MOE_OK
    compare(w, run_gpu(w, inp, ws, fp8=mx), run_oracle(w, inp, fp8=mx))

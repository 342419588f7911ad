"""GPU parity of the FP8-on-both-operands path (MOE_WEIGHTS_FP8_W8A8).

* The E4M3 activation rows the layer builds: the codes and scales of every
  kept x row bit-exact against the oracle's per-row quantiser (both decide in
  fp32 from the same bf16 values).
* The hidden rows' codes: the layer decides them from its own fp32 H, the
  oracle from its fp64 H, so a code may flip where H sits within fp32
  accumulation error of a rounding boundary; almost all must agree.
* y against the oracle's W8A8 expert within the bf16 tolerance, routing exact,
  over the three activation-box sizes, N and K tails, many experts, capacity,
  random codes, and the full-size decode and (sampled) Mixtral shapes.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_aux_b200 import Workspace, _lib, forward, moe_get_device_status
from sparse_mixture_experts_aux_b200.inputs import (MIXTRAL, MIXTRAL_DECODE, Workload,
                                                    make_fp8_weights, make_inputs)
from tests.parity_util import compare, oracle_quantized_weights, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check_activation_codes(w, inp, gpu, ref):
    views = gpu[3]
    slot = views["slot_pos"].cpu().numpy()
    codes, scales = O.quantize_rows_fp8(inp["x"].float().cpu().numpy())
    xq = views["xq"].cpu().numpy()
    xs = views["xscale"].cpu().numpy()
    t, s = np.nonzero(slot >= 0)
    pos = slot[t, s]
    assert np.array_equal(xq[pos], codes[t]), "E4M3 activation codes differ"
    assert np.array_equal(xs[pos].view(np.uint32), scales[t].view(np.uint32))


SMALL_W8A8 = [
    Workload("w8a8 one token, 32-row box", 1, 256, 8, 256, 2, seed=60),
    Workload("w8a8 T=20 capacity, 32-row box", 20, 192, 4, 192, 2, capacity_factor=1.5, seed=61),
    Workload("w8a8 T=48 N tail, 64-row box", 48, 256, 8, 320, 2, seed=62),
    Workload("w8a8 ragged rows, K tail, 128-row box", 1000, 320, 4, 448, 2, seed=63),
    Workload("w8a8 many experts", 777, 256, 32, 256, 4, seed=64),
    Workload("w8a8 sigmoid groups selection bias", 300, 256, 16, 128, 4, gate_mode=2, n_group=4,
             topk_group=2, selection_bias=True, seed=65),
]


@pytest.mark.parametrize("w", SMALL_W8A8, ids=[w.name for w in SMALL_W8A8])
def test_w8a8_small(w):
    inp = make_inputs(w, device="cuda")
    fp8 = oracle_quantized_weights(inp)
    gpu = run_gpu(w, inp, fp8=fp8, act_fp8=True)
    ref = run_oracle(w, inp, fp8=fp8, act_fp8=True)
    _check_activation_codes(w, inp, gpu, ref)
    compare(w, gpu, ref)


def test_w8a8_hidden_codes_mostly_agree():
    w = Workload("w8a8 hidden codes", 64, 256, 4, 256, 1, seed=66)
    inp = make_inputs(w, device="cuda")
    fp8 = oracle_quantized_weights(inp)
    gpu = run_gpu(w, inp, fp8=fp8, act_fp8=True)
    views = gpu[3]
    ref = run_oracle(w, inp, fp8=fp8, act_fp8=True)
    slot = views["slot_pos"].cpu().numpy()
    hq = views["hq"].cpu().numpy()
    x = inp["x"].float().cpu().numpy()
    agree = total = 0
    E, de = w.E, w.d_e
    sc = fp8["weight_scales"].cpu().numpy()
    for e in range(E):
        toks = np.nonzero((ref.idx[:, 0] == e) & ref.keep[:, 0])[0]
        if toks.size == 0:
            continue
        Wg = O.dequantize_rows_fp8(fp8["W_g"][e].cpu().numpy(), sc[e * de:(e + 1) * de])
        Wu = O.dequantize_rows_fp8(fp8["W_u"][e].cpu().numpy(), sc[E * de + e * de:E * de + (e + 1) * de])
        xq = O.fake_quant_rows_fp8(x[toks])
        h = O.silu(xq @ Wg.T) * (xq @ Wu.T)
        codes, _ = O.quantize_rows_fp8(h)
        got = hq[slot[toks, 0]]
        agree += int((got == codes).sum())
        total += codes.size
    assert total > 0 and agree / total > 0.999, agree / total


def test_w8a8_random_codes():
    w = Workload("w8a8 random codes", 600, 384, 8, 448, 2, seed=67)
    inp = make_inputs(w, device="cuda")
    fp8 = make_fp8_weights(w, device="cuda")
    compare(w, run_gpu(w, inp, fp8=fp8, act_fp8=True), run_oracle(w, inp, fp8=fp8, act_fp8=True))


def test_w8a8_decode_full_size():
    w = MIXTRAL_DECODE
    inp = make_inputs(w, device="cuda")
    fp8 = make_fp8_weights(w, device="cuda")
    gpu = run_gpu(w, inp, fp8=fp8, act_fp8=True)
    inp.pop("W_g"), inp.pop("W_u"), inp.pop("W_d")
    compare(w, gpu, run_oracle(w, inp, fp8=fp8, act_fp8=True))


def test_w8a8_mixtral_sampled_rows():
    w = MIXTRAL
    inp = make_inputs(w, device="cuda")
    fp8 = make_fp8_weights(w, device="cuda")
    gpu = run_gpu(w, inp, fp8=fp8, act_fp8=True)
    inp.pop("W_g"), inp.pop("W_u"), inp.pop("W_d")
    rows = np.sort(np.random.default_rng(5).choice(w.T, size=256, replace=False))
    compare(w, gpu, run_oracle(w, inp, rows=rows, fp8=fp8, act_fp8=True))


def test_w8a8_expired_waits_are_reported():
    w = Workload("w8a8 timeout", 300, 256, 4, 320, 2, seed=68)
    inp = make_inputs(w, device="cuda")
    fp8 = oracle_quantized_weights(inp)
    ws = Workspace()
    for _ in range(2):
        forward(inp["x"], inp["W_r"], fp8["W_g"], fp8["W_u"], fp8["W_d"], None, k=w.k,
                workspace=ws, weight_scales=fp8["weight_scales"], act_fp8=True, wait_timeout_ns=1)
        torch.cuda.synchronize()
        assert moe_get_device_status() == _lib.MOE_ERR_DEVICE_TIMEOUT
        assert moe_get_device_status() == _lib.MOE_OK
    gpu = run_gpu(w, inp, ws, fp8=fp8, act_fp8=True)
    compare(w, gpu, run_oracle(w, inp, fp8=fp8, act_fp8=True))

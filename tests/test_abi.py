"""The C ABI library loads, exports every symbol include/moe.h declares, and
rejects bad arguments on the host before touching a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_aux_b200 import _lib
from sparse_mixture_experts_aux_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return _lib.load()


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "moe.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", hdr)


def test_header_declares_the_binding_surface():
    names = declared_symbols()
    assert sorted(names) == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # and nothing that is not declared is exported under the moe_ prefix
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert exported == set(declared_symbols())


def test_debug_library_exports_the_same_symbols():
    B.build(debug=True)
    dbg = _lib.load_debug()
    for name in declared_symbols():
        assert hasattr(dbg, name), name
    out = os.popen(f"nm -D --defined-only {_lib.DEBUG_LIB_PATH}").read()
    assert set(re.findall(r"\bT (moe_\w+)", out)) == set(declared_symbols())


def test_status_strings(lib):
    assert _lib.status_string(0) == "MOE_OK"
    assert _lib.status_string(5) == "MOE_ERR_DEVICE_TIMEOUT"
    assert _lib.status_string(7) == "MOE_ERR_DEVICE_BOUNDS"
    assert _lib.status_string(99) == "MOE_STATUS_UNKNOWN"


def test_capacity_matches_page_example(lib):
    # kevinluzbetak capacity example: 4096 tokens, 4 experts, top-2, factor 1.25 -> 2560
    assert _lib.moe_capacity(4096, 4, 2, 1.25) == 2560
    assert _lib.moe_capacity(16384, 64, 1, 1.25) == 320
    assert _lib.moe_capacity(100, 4, 2, 0.0) == -1
    assert _lib.moe_capacity(100, 4, 2, -1.0) == -1
    assert _lib.moe_capacity(8, 2, 1, 0.5) == 2
    # a factor so large that no expert can overflow is clamped to T*k
    assert _lib.moe_capacity(10, 2, 1, 1e30) == 10


def test_capacity_agrees_with_oracle_formula(lib):
    from oracle import moe_oracle as O
    import numpy as np
    # the layer takes the factor as an fp32; the oracle is given that same value
    for T, E, k, cf in [(1000, 7, 3, 1.1), (333, 5, 2, 0.37), (4096, 64, 1, 2.0), (17, 3, 1, 0.99),
                        (2600, 4, 1, 0.9)]:
        cf32 = float(np.float32(cf))
        assert _lib.moe_capacity(T, E, k, cf) == O.capacity_limit(cf32, T, k, E)


def _dims(**kw):
    base = dict(T=128, d=256, d_e=256, d_s=0, dtype=_lib.MOE_BF16)
    base.update(kw)
    return _lib.make_dims(**base)


def test_workspace_size_and_layout(lib):
    d = _dims()
    n = _lib.moe_workspace_size(d, 8, 2, 0.0)
    assert n > 0
    L = _lib.moe_workspace_layout(d, 8, 2, 0.0)
    # rows reserved cover T*k assignments plus per-expert padding to 128 rows
    assert L.rows_max >= 128 * 2 + 127 * 8 and L.rows_max % 128 == 0
    offs = [L.logits, L.topk_idx, L.gates, L.slot_pos, L.probsum, L.tile_start, L.xp, L.h, L.yrows]
    assert all(o % 256 == 0 for o in offs)
    assert max(offs) < n
    assert L.capacity == -1
    # a shared expert needs more scratch
    assert _lib.moe_workspace_size(_dims(d_s=128), 8, 2, 0.0) > n


@pytest.mark.parametrize("E,k,kw,want", [
    (8, 0, {}, _lib.MOE_ERR_INVALID_ARG),          # k < 1
    (8, 9, {}, _lib.MOE_ERR_INVALID_ARG),          # k > E
    (0, 1, {}, _lib.MOE_ERR_INVALID_ARG),          # no experts
    (2048, 2, {}, _lib.MOE_ERR_UNSUPPORTED),       # E above the build limit
    (64, 33, {}, _lib.MOE_ERR_UNSUPPORTED),        # k above the build limit
    (8, 2, dict(d=100), _lib.MOE_ERR_UNSUPPORTED),  # bf16 width not a multiple of 64
    (8, 2, dict(d_e=96), _lib.MOE_ERR_UNSUPPORTED),
    (8, 2, dict(d_s=32), _lib.MOE_ERR_UNSUPPORTED),
    (8, 2, dict(dtype=_lib.MOE_F32, d=48), _lib.MOE_ERR_UNSUPPORTED),
    (8, 2, dict(T=-1), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(d=0), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(dtype=7), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(gate_mode=7), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(n_group=3, topk_group=1), _lib.MOE_ERR_INVALID_ARG),   # 3 does not divide E
    (8, 2, dict(n_group=4, topk_group=5), _lib.MOE_ERR_INVALID_ARG),   # more groups than exist
    (8, 4, dict(n_group=4, topk_group=1), _lib.MOE_ERR_INVALID_ARG),   # k > experts in 1 group
    (64, 2, dict(n_group=64, topk_group=2), _lib.MOE_ERR_UNSUPPORTED),  # n_group above 32
    (8, 2, dict(n_group=-1), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(weight_format=5), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(weight_format=1, dtype=_lib.MOE_F32), _lib.MOE_ERR_UNSUPPORTED),  # FP8: bf16 x
    (8, 2, dict(weight_format=1, d_s=128), _lib.MOE_ERR_UNSUPPORTED),  # FP8: no shared expert
    (8, 2, dict(weight_format=2, dtype=_lib.MOE_F32), _lib.MOE_ERR_UNSUPPORTED),  # W8A8: bf16 x
    (8, 2, dict(weight_format=4), _lib.MOE_ERR_INVALID_ARG),
    (8, 2, dict(weight_format=3, d=320), _lib.MOE_ERR_UNSUPPORTED),    # MXFP4: d % 256
    (8, 2, dict(weight_format=3, d_e=192), _lib.MOE_ERR_UNSUPPORTED),  # MXFP4: d_e % 256
    (8, 2, dict(weight_format=3, d_s=256), _lib.MOE_ERR_UNSUPPORTED),  # MXFP4: no shared
])
def test_forward_rejects_bad_shapes_on_host(lib, E, k, kw, want):
    d = _dims(**kw)
    st = _lib.moe_forward(d, 16, 16, 16, 16, 16, None, E, k, 0.0, 16, 16, 16, check=False)
    assert st == want
    assert _lib.moe_workspace_size(d, E, k, 0.0) == 0


def test_forward_rejects_bad_pointers_on_host(lib):
    d = _dims()
    ws_bytes = _lib.moe_workspace_size(d, 8, 2, 0.0)
    good = 1 << 20  # never dereferenced: every case below fails validation first
    args = dict(x=good, W_r=good, W_g=good, W_u=good, W_d=good, W_shared=None, y=good, aux=good,
                counts=good)

    def call(dims=d, cf=0.0, **over):
        a = dict(args, **over)
        return _lib.moe_forward(dims, a["x"], a["W_r"], a["W_g"], a["W_u"], a["W_d"],
                                a["W_shared"], 8, 2, cf, a["y"], a["aux"], a["counts"], check=False)

    for name in ("x", "W_r", "W_g", "W_u", "W_d", "y", "aux", "counts"):
        assert call(**{name: 0}) == _lib.MOE_ERR_INVALID_ARG, name
    for name in ("x", "W_r", "W_g", "W_u", "W_d", "y"):
        assert call(**{name: good + 8}) == _lib.MOE_ERR_INVALID_ARG, name  # misaligned
    assert call(aux=good + 2) == _lib.MOE_ERR_INVALID_ARG
    assert call(cf=float("nan")) == _lib.MOE_ERR_INVALID_ARG
    # shared expert requested without its weights
    assert call(dims=_dims(d_s=128)) == _lib.MOE_ERR_INVALID_ARG
    # workspace missing, too small, misaligned
    assert call() == _lib.MOE_ERR_WORKSPACE
    small = _dims(workspace=good, workspace_bytes=ws_bytes - 1)
    assert call(dims=small) == _lib.MOE_ERR_WORKSPACE
    skew = _dims(workspace=good + 16, workspace_bytes=ws_bytes)
    assert call(dims=skew) == _lib.MOE_ERR_WORKSPACE
    assert _lib.moe_forward(None, good, good, good, good, good, None, 8, 2, 0.0, good, good, good,
                            check=False) == _lib.MOE_ERR_INVALID_ARG


def test_routing_variants_are_accepted_on_host(lib):
    for kw in (dict(gate_mode=1), dict(gate_mode=2), dict(gate_mode=2, n_group=4, topk_group=2),
               dict(n_group=8, topk_group=8)):
        d = _dims(**kw)
        assert _lib.moe_workspace_size(d, 8, 2, 0.0) > 0, kw
        st = _lib.moe_forward(d, 16, 16, 16, 16, 16, None, 8, 2, 0.0, 16, 16, 16, check=False)
        assert st == _lib.MOE_ERR_WORKSPACE, kw  # valid; only the workspace is missing
    assert _lib.moe_forward(_dims(selection_bias=(1 << 20) + 4), 1 << 20, 1 << 20, 1 << 20,
                            1 << 20, 1 << 20, None, 8, 2, 0.0, 1 << 20, 1 << 20, 1 << 20,
                            check=False) == _lib.MOE_ERR_INVALID_ARG  # misaligned bias


def test_fp8_weights_validated_on_host(lib):
    g = 1 << 20
    fwd = lambda d: _lib.moe_forward(d, g, g, g, g, g, None, 8, 2, 0.0, g, g, g, check=False)
    assert fwd(_dims(weight_format=1)) == _lib.MOE_ERR_INVALID_ARG          # scales missing
    assert fwd(_dims(weight_format=1, weight_scales=g + 2)) == _lib.MOE_ERR_INVALID_ARG
    assert _lib.moe_workspace_size(_dims(weight_format=1, weight_scales=g), 8, 2, 0.0) > 0
    assert fwd(_dims(weight_format=1, weight_scales=g)) == _lib.MOE_ERR_WORKSPACE  # valid
    assert fwd(_dims(weight_format=2, weight_scales=g)) == _lib.MOE_ERR_WORKSPACE  # valid
    assert fwd(_dims(weight_format=2)) == _lib.MOE_ERR_INVALID_ARG  # scales missing
    # W8A8 needs more workspace (activation codes and scales) and reports where they are
    n1 = _lib.moe_workspace_size(_dims(weight_format=1), 8, 2, 0.0)
    n2 = _lib.moe_workspace_size(_dims(weight_format=2), 8, 2, 0.0)
    assert n2 > n1
    L = _lib.moe_workspace_layout(_dims(weight_format=2), 8, 2, 0.0)
    assert 0 < L.xscale < n2 and 0 < L.hq < n2 and 0 < L.hscale < n2
    assert L.hq + L.rows_max * 256 <= n2
    # quantiser and dequantiser: argument checks on the host, nothing launched
    for args in [(0, 1, 4, 64, g, g), (g, 1, 4, 64, 0, g), (g, 1, 4, 64, g, 0), (g, 1, 4, 24, g, g),
                 (g, 1, -1, 64, g, g), (g, 9, 4, 64, g, g), (g, 1, 4, 0, g, g)]:
        assert _lib.moe_quantize_fp8(*args) == _lib.MOE_ERR_INVALID_ARG, args
    assert _lib.moe_quantize_fp8(g, 1, 0, 64, g, g) == _lib.MOE_OK  # no rows: nothing to do
    for args in [(0, g, 4, 64, g), (g, 0, 4, 64, g), (g, g, 4, 64, 0), (g, g, 4, 40, g),
                 (g + 8, g, 4, 64, g), (g, g, 4, 64, g + 4), (g, g, -2, 64, g)]:
        assert _lib.moe_dequantize_fp8(*args) == _lib.MOE_ERR_INVALID_ARG, args
    assert _lib.moe_dequantize_fp8(g, g, 0, 64, g) == _lib.MOE_OK


def test_mxfp4_weights_validated_on_host(lib):
    g = 1 << 20
    fwd = lambda d: _lib.moe_forward(d, g, g, g, g, g, None, 8, 2, 0.0, g, g, g, check=False)
    mx = dict(weight_format=3, weight_scales=g, weight_block_scales=g)
    assert fwd(_dims(**mx)) == _lib.MOE_ERR_WORKSPACE                     # valid
    assert fwd(_dims(**dict(mx, weight_block_scales=None))) == _lib.MOE_ERR_INVALID_ARG
    assert fwd(_dims(**dict(mx, weight_block_scales=g + 8))) == _lib.MOE_ERR_INVALID_ARG
    assert fwd(_dims(**dict(mx, weight_scales=None))) == _lib.MOE_ERR_INVALID_ARG
    assert fwd(_dims(**dict(mx, dtype=_lib.MOE_F32))) == _lib.MOE_ERR_UNSUPPORTED
    # the same workspace as FP8 weight-only (no activation codes)
    assert _lib.moe_workspace_size(_dims(**mx), 8, 2, 0.0) == \
        _lib.moe_workspace_size(_dims(weight_format=1), 8, 2, 0.0)
    for args in [(0, 1, 4, 64, g, g, g), (g, 1, 4, 64, 0, g, g), (g, 1, 4, 64, g, 0, g),
                 (g, 1, 4, 64, g, g, 0), (g, 1, 4, 48, g, g, g), (g, 1, -1, 64, g, g, g),
                 (g, 9, 4, 64, g, g, g), (g + 8, 1, 4, 64, g, g, g), (g, 1, 4, 64, g + 8, g, g)]:
        assert _lib.moe_quantize_mxfp4(*args) == _lib.MOE_ERR_INVALID_ARG, args
    assert _lib.moe_quantize_mxfp4(g, 1, 0, 64, g, g, g) == _lib.MOE_OK
    for args in [(0, g, g, 4, 64, g), (g, 0, g, 4, 64, g), (g, g, 0, 4, 64, g),
                 (g, g, g, 4, 64, 0), (g, g, g, 4, 40, g), (g + 8, g, g, 4, 64, g),
                 (g, g, g, 4, 64, g + 4), (g, g, g, -1, 64, g)]:
        assert _lib.moe_dequantize_mxfp4(*args) == _lib.MOE_ERR_INVALID_ARG, args
    assert _lib.moe_dequantize_mxfp4(g, g, g, 0, 64, g) == _lib.MOE_OK


def test_binding_refuses_cpu_tensors():
    import torch
    from sparse_mixture_experts_aux_b200 import forward
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    w = torch.zeros(2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError, match="CUDA"):
        forward(x, torch.zeros(2, 64), w, w, w, k=1)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not found"):
        _lib.load.__wrapped__(str(tmp_path / "nope.so")) if hasattr(_lib.load, "__wrapped__") \
            else _load_fresh(str(tmp_path / "nope.so"))


def _load_fresh(path):
    saved = _lib._lib
    _lib._lib = None
    try:
        return _lib.load(path)
    finally:
        _lib._lib = saved

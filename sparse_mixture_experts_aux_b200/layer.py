"""Torch-facing wrapper of moe_forward: torch supplies device memory and the
stream, the library does every step of the layer. Marshalling only."""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return _lib.MOE_BF16
    if dt == torch.float32:
        return _lib.MOE_F32
    raise TypeError(f"unsupported activation dtype {dt}; expected bfloat16 or float32")


class Workspace:
    """A reusable device scratch buffer (torch-allocated, 512-byte aligned)."""

    def __init__(self, device=None):
        self.buf: Optional[torch.Tensor] = None
        self.device = device

    def get(self, nbytes: int, device) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != torch.device(device):
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        return self.buf


def _dims_for(x: torch.Tensor, W_g: torch.Tensor, d_s: int, router_bias, ws, stream, events,
              wait_timeout_ns: int = 0, routing: Optional[dict] = None, weight_scales=None,
              act_fp8: bool = False, weight_block_scales=None):
    T, d = x.shape
    d_e = W_g.shape[1]
    routing = routing or {}
    fmt = _lib.MOE_WEIGHTS_DTYPE
    if W_g.dtype == torch.uint8:
        fmt = _lib.MOE_WEIGHTS_FP8_W8A8 if act_fp8 else _lib.MOE_WEIGHTS_FP8
        if weight_block_scales is not None:
            fmt = _lib.MOE_WEIGHTS_MXFP4
    return _lib.make_dims(T, d, d_e, d_s, dtype_code(x.dtype), router_bias, ws,
                          ws.numel() if ws is not None else 0, stream, events,
                          wait_timeout_ns=wait_timeout_ns,
                          gate_mode=routing.get("gate_mode", 0),
                          selection_bias=routing.get("selection_bias"),
                          n_group=routing.get("n_group", 0),
                          topk_group=routing.get("topk_group", 0),
                          weight_format=fmt, weight_scales=weight_scales,
                          weight_block_scales=weight_block_scales)


def forward(x: torch.Tensor, W_r: torch.Tensor, W_g: torch.Tensor, W_u: torch.Tensor,
            W_d: torch.Tensor, W_shared: Optional[torch.Tensor] = None, k: int = 2,
            capacity_factor: float = 0.0, router_bias: Optional[torch.Tensor] = None,
            d_s: int = 0, workspace: Optional[Workspace] = None, stream=None, events=None,
            y: Optional[torch.Tensor] = None, aux: Optional[torch.Tensor] = None,
            counts: Optional[torch.Tensor] = None, wait_timeout_ns: int = 0,
            gate_mode: int = 0, selection_bias: Optional[torch.Tensor] = None,
            n_group: int = 0, topk_group: int = 0, weight_scales: Optional[torch.Tensor] = None,
            act_fp8: bool = False, weight_block_scales: Optional[torch.Tensor] = None):
    """Run the routed MoE FFN layer; returns (y, aux[1] fp32, counts[E] int32) on x's device.

    Shapes: x [T, d]; W_r [E, d] fp32; W_g, W_u [E, d_e, d]; W_d [E, d, d_e];
    W_shared packed [gate d_s*d | up d_s*d | down d*d_s] when d_s > 0.
    FP8 expert weights: W_g, W_u, W_d as uint8 E4M3 codes (quantize_fp8) and
    weight_scales = their per-row scales concatenated [W_g | W_u | W_d] (bf16 x).
    act_fp8 (with FP8 weights): E4M3 activations inside the experts as well
    (MOE_WEIGHTS_FP8_W8A8 in include/moe.h).
    MXFP4 expert weights: W_g, W_u, W_d as packed uint8 E2M1 codes [.., K / 2]
    (quantize_mxfp4), weight_block_scales = their E8M0 block scales and
    weight_scales = their row factors, each concatenated [W_g | W_u | W_d].
    wait_timeout_ns: limit of the GEMM kernels' device-side waits (0 = library default).
    gate_mode / selection_bias / n_group / topk_group: routing variants (include/moe.h).
    """
    for name, t in (("x", x), ("W_r", W_r), ("W_g", W_g), ("W_u", W_u), ("W_d", W_d)):
        if not t.is_cuda:
            raise RuntimeError(f"{name} must be a CUDA tensor (the layer has no CPU path)")
        if not t.is_contiguous():
            raise RuntimeError(f"{name} must be contiguous")
    E = W_r.shape[0]
    dev = x.device
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    elif isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    workspace = workspace or Workspace()
    routing = dict(gate_mode=gate_mode, selection_bias=selection_bias, n_group=n_group,
                   topk_group=topk_group)
    if W_g.dtype == torch.uint8:
        if weight_scales is None or not weight_scales.is_cuda or weight_scales.dtype != torch.float32:
            raise RuntimeError("FP8 weights need weight_scales: a CUDA fp32 tensor")
    elif act_fp8:
        raise RuntimeError("act_fp8 needs FP8 (uint8) weights")
    if weight_block_scales is not None and (act_fp8 or W_g.dtype != torch.uint8):
        raise RuntimeError("weight_block_scales go with MXFP4 (uint8) weights, without act_fp8")
    probe = _dims_for(x, W_g, d_s, router_bias, None, stream, events, routing=routing,
                      weight_scales=weight_scales, act_fp8=act_fp8,
                      weight_block_scales=weight_block_scales)
    nbytes = _lib.moe_workspace_size(probe, E, k, capacity_factor)
    if nbytes == 0:
        raise _lib.MoeError(_lib.MOE_ERR_INVALID_ARG, "moe_workspace_size")
    ws = workspace.get(nbytes, dev)
    dims = _dims_for(x, W_g, d_s, router_bias, ws, stream, events, wait_timeout_ns, routing,
                     weight_scales, act_fp8, weight_block_scales)
    y = torch.empty_like(x) if y is None else y
    aux = torch.empty(1, dtype=torch.float32, device=dev) if aux is None else aux
    counts = torch.empty(E, dtype=torch.int32, device=dev) if counts is None else counts
    _lib.moe_forward(dims, x, W_r, W_g, W_u, W_d, W_shared, E, k, capacity_factor, y, aux, counts)
    return y, aux, counts


def quantize_fp8(w: torch.Tensor, stream=None):
    """E4M3 codes (uint8, w's shape) and per-row fp32 scales of a CUDA weight
    tensor whose last dimension is the row (include/moe.h, moe_quantize_fp8)."""
    if not w.is_cuda or not w.is_contiguous():
        raise RuntimeError("w must be a contiguous CUDA tensor")
    cols = w.shape[-1]
    rows = w.numel() // cols
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    st = torch.cuda.current_stream(w.device).cuda_stream if stream is None else stream
    rc = _lib.moe_quantize_fp8(w, dtype_code(w.dtype), rows, cols, codes, scales, st)
    if rc != _lib.MOE_OK:
        raise _lib.MoeError(rc, "moe_quantize_fp8")
    return codes, scales


def dequantize_fp8(codes: torch.Tensor, scales: torch.Tensor, stream=None) -> torch.Tensor:
    """fp32 weights code * scale, as the FP8 layer computes with them (moe_dequantize_fp8)."""
    cols = codes.shape[-1]
    rows = codes.numel() // cols
    out = torch.empty(codes.shape, dtype=torch.float32, device=codes.device)
    st = torch.cuda.current_stream(codes.device).cuda_stream if stream is None else stream
    rc = _lib.moe_dequantize_fp8(codes, scales, rows, cols, out, st)
    if rc != _lib.MOE_OK:
        raise _lib.MoeError(rc, "moe_dequantize_fp8")
    return out


def quantize_mxfp4(w: torch.Tensor, stream=None):
    """MXFP4 codes (uint8, w's shape with the last dimension halved), E8M0 block
    scales (uint8, last dimension / 32) and fp32 row factors (w's shape without
    the last dimension) of a CUDA weight tensor whose last dimension is the row
    (include/moe.h, moe_quantize_mxfp4)."""
    if not w.is_cuda or not w.is_contiguous():
        raise RuntimeError("w must be a contiguous CUDA tensor")
    cols = w.shape[-1]
    rows = w.numel() // cols
    codes = torch.empty(*w.shape[:-1], cols // 2, dtype=torch.uint8, device=w.device)
    bscales = torch.empty(*w.shape[:-1], cols // 32, dtype=torch.uint8, device=w.device)
    factors = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    st = torch.cuda.current_stream(w.device).cuda_stream if stream is None else stream
    rc = _lib.moe_quantize_mxfp4(w, dtype_code(w.dtype), rows, cols, codes, bscales, factors, st)
    if rc != _lib.MOE_OK:
        raise _lib.MoeError(rc, "moe_quantize_mxfp4")
    return codes, bscales, factors


def dequantize_mxfp4(codes: torch.Tensor, bscales: torch.Tensor, factors: torch.Tensor,
                     stream=None) -> torch.Tensor:
    """fp32 weights code * 2^X, as the MXFP4 layer computes with them (moe_dequantize_mxfp4)."""
    cols = codes.shape[-1] * 2
    rows = codes.numel() * 2 // cols
    out = torch.empty(*codes.shape[:-1], cols, dtype=torch.float32, device=codes.device)
    st = torch.cuda.current_stream(codes.device).cuda_stream if stream is None else stream
    rc = _lib.moe_dequantize_mxfp4(codes, bscales, factors, rows, cols, out, st)
    if rc != _lib.MOE_OK:
        raise _lib.MoeError(rc, "moe_dequantize_mxfp4")
    return out


def routing_views(ws: torch.Tensor, x: torch.Tensor, W_g: torch.Tensor, E: int, k: int,
                  capacity_factor: float = 0.0, d_s: int = 0, act_fp8: bool = False) -> dict:
    """Views of the routing results moe_forward left in workspace `ws` (with
    act_fp8 and FP8 weights, also the E4M3 activation rows and their scales)."""
    T, d = x.shape
    dims = _dims_for(x, W_g, d_s, None, ws, 0, None, act_fp8=act_fp8)
    L = _lib.moe_workspace_layout(dims, E, k, capacity_factor)
    b = ws

    def view(off, n, dt):
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        return b[off:off + nbytes].view(dt)

    d_e = W_g.shape[1]
    return dict(
        logits=view(L.logits, T * E, torch.float32).view(T, E),
        topk_idx=view(L.topk_idx, T * k, torch.int32).view(T, k),
        gates=view(L.gates, T * k, torch.float32).view(T, k),
        slot_pos=view(L.slot_pos, T * k, torch.int32).view(T, k),
        probsum=view(L.probsum, E, torch.float64),
        tile_start=view(L.tile_start, E + 1, torch.int32),
        xp=view(L.xp, L.rows_max * d, x.dtype).view(L.rows_max, d),
        h=view(L.h, L.rows_max * d_e, x.dtype).view(L.rows_max, d_e),
        yrows=view(L.yrows, L.rows_max * d, x.dtype).view(L.rows_max, d),
        rows_max=L.rows_max, capacity=L.capacity,
        status=view(L.status, 1, torch.int32),
        **(dict(xq=view(L.xp, L.rows_max * d, torch.uint8).view(L.rows_max, d),
                xscale=view(L.xscale, L.rows_max, torch.float32),
                hq=view(L.hq, L.rows_max * d_e, torch.uint8).view(L.rows_max, d_e),
                hscale=view(L.hscale, L.rows_max, torch.float32)) if act_fp8 else {}),
    )

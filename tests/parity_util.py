"""Helpers for the GPU-vs-oracle parity tests: run both sides on the same seeded
inputs and compare element by element at the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_aux_b200 import (Workspace, forward, moe_get_device_status,
                                             routing_views)
from sparse_mixture_experts_aux_b200.inputs import Workload, make_inputs, split_shared

MARGIN = 1e-5        # routing decisions are compared where the k-th/(k+1)-th gap exceeds this
GATE_TOL = 1e-6      # absolute, on gates
Y_TOL = {"f32": 1e-4, "bf16": 2e-2}  # max|err| <= tol * max(1, |ref|)


def run_gpu(w: Workload, inp: dict, ws: Workspace | None = None, fp8: dict | None = None,
            act_fp8: bool = False):
    """fp8: E4M3 codes W_g, W_u, W_d and weight_scales (device) to use instead of
    the dtype weights in `inp`; act_fp8: E4M3 activations too (W8A8)."""
    ws = ws or Workspace()
    src = fp8 if fp8 is not None else inp
    y, aux, counts = forward(inp["x"], inp["W_r"], src["W_g"], src["W_u"], src["W_d"],
                             inp["W_shared"], k=w.k, capacity_factor=w.capacity_factor,
                             router_bias=inp["router_bias"], d_s=w.d_s, workspace=ws,
                             gate_mode=w.gate_mode, selection_bias=inp.get("selection_bias"),
                             n_group=w.n_group, topk_group=w.topk_group,
                             weight_scales=fp8["weight_scales"] if fp8 is not None else None,
                             act_fp8=act_fp8,
                             weight_block_scales=fp8.get("block_scales") if fp8 else None)
    torch.cuda.synchronize()
    assert moe_get_device_status() == 0, "a device-side wait timed out"
    views = routing_views(ws.buf, inp["x"], src["W_g"], w.E, w.k, w.capacity_factor, w.d_s,
                          act_fp8=act_fp8)
    return y, aux, counts, views


def run_oracle(w: Workload, inp: dict, rows=None, fp8: dict | None = None,
               act_fp8: bool = False) -> O.OracleResult:
    """fp8: as in run_gpu; the oracle then computes with code * scale (its own
    dequantisation, fp64)."""
    x = inp["x"].cpu()
    bias = inp["router_bias"].cpu() if inp["router_bias"] is not None else None

    def expert(e):
        if fp8 is None:
            return inp["W_g"][e].cpu(), inp["W_u"][e].cpu(), inp["W_d"][e].cpu()
        if "oracle_mx" in fp8:  # MXFP4: the oracle's own codes and block exponents
            return tuple(O.dequantize_rows_mxfp4(c[e], x[e]) for c, x in fp8["oracle_mx"])
        E, de, d = w.E, w.d_e, w.d
        sc = fp8["weight_scales"]
        parts = ((fp8["W_g"][e], sc[e * de:(e + 1) * de]),
                 (fp8["W_u"][e], sc[E * de + e * de:E * de + (e + 1) * de]),
                 (fp8["W_d"][e], sc[2 * E * de + e * d:2 * E * de + (e + 1) * d]))
        return tuple(O.dequantize_rows_fp8(c.cpu().numpy(), s.cpu().numpy()) for c, s in parts)

    shared = None
    if w.d_s:
        shared = tuple(t.cpu() for t in split_shared(inp["W_shared"], w.d, w.d_s))
    sel = inp.get("selection_bias")
    sel = sel.cpu() if sel is not None else None
    ref = O.moe_forward(x, inp["W_r"].cpu(), expert, w.k, layer_capacity_factor(w), bias, shared,
                        rows, gate_mode=w.gate_mode, selection_bias=sel,
                        n_group=max(w.n_group, 1), topk_group=max(w.topk_group, 1),
                        act_fp8=act_fp8)
    ref.selection_bias = sel  # for the near-tie bookkeeping of compare()
    return ref


def layer_capacity_factor(w: Workload) -> float:
    """The capacity factor as the layer receives it: the C ABI takes an fp32."""
    return float(np.float32(w.capacity_factor))


def expected_slot_pos(ref: O.OracleResult, E: int) -> tuple:
    """Row of each kept assignment in the expert-grouped buffers, from the
    oracle's routing: experts in order, each segment padded to 128 rows, tokens
    in index order inside a segment; -1 for dropped assignments."""
    T, k = ref.idx.shape
    kept = np.zeros(E, dtype=np.int64)
    for e in range(E):
        kept[e] = int(((ref.idx == e) & ref.keep).sum())
    tiles = (kept + 127) // 128
    start = np.concatenate([[0], np.cumsum(tiles)]) * 128
    pos = np.full((T, k), -1, dtype=np.int64)
    seen = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            if ref.keep[t, s]:
                e = ref.idx[t, s]
                pos[t, s] = start[e] + seen[e]
                seen[e] += 1
    return pos, np.concatenate([[0], np.cumsum(tiles)])


def contested_experts(ref: O.OracleResult, w: Workload, sel_bias=None) -> dict:
    """For each near-tie token (margin <= MARGIN), the experts whose choice it
    may legitimately flip: those whose selection score lies in the band around
    the k-th/(k+1)-th cut. Under group-limited routing a group near-tie can swap
    whole groups, so every expert counts as contested there."""
    near = np.nonzero(ref.margin <= MARGIN)[0]
    if near.size == 0:
        return {}
    E, k = ref.logits.shape[1], ref.idx.shape[1]
    if max(w.n_group, 1) > 1 and max(w.topk_group, 1) < w.n_group:
        return {int(t): np.ones(E, dtype=bool) for t in near}
    sel = O.selection_scores(ref.logits[near], w.gate_mode, sel_bias)
    out = {}
    for i, t in enumerate(near):
        srt = np.sort(sel[i])[::-1]
        lo = srt[k] if k < E else srt[k - 1]
        out[int(t)] = (sel[i] >= lo - MARGIN) & (sel[i] <= srt[k - 1] + MARGIN)
    return out


def unaffected_tokens(ref: O.OracleResult, contested: dict) -> np.ndarray:
    """Tokens whose routing and kept/dropped status no near-tie can change.

    A near-tie token itself is excluded. For a later assignment (t, e) with
    oracle rank rho in expert e, every earlier near-tie token contesting e
    either holds e in the oracle's choice (it may leave: the layer's rank can be
    one lower) or not (it may join: one higher). With `down` and `up` such
    tokens the layer's rank lies in [rho - down, rho + up], so the status is
    certain when rho + up < C (kept) or rho - down >= C (dropped)."""
    T, k = ref.idx.shape
    ok = ref.margin > MARGIN
    C = ref.capacity
    if C is None or not contested:
        return ok
    E = ref.logits.shape[1]
    up = np.zeros(E, dtype=np.int64)
    down = np.zeros(E, dtype=np.int64)
    rank = np.zeros(E, dtype=np.int64)  # oracle rank of the next assignment, per expert
    for t in range(T):
        for s in range(k):
            e = ref.idx[t, s]
            if (up[e] or down[e]) and not (rank[e] + up[e] < C or rank[e] - down[e] >= C):
                ok[t] = False
            rank[e] += 1
        if t in contested:
            chosen = np.zeros(E, dtype=bool)
            chosen[ref.idx[t]] = True
            down += contested[t] & chosen
            up += contested[t] & ~chosen
    return ok


def compare(w: Workload, gpu, ref: O.OracleResult, check_positions: bool = True) -> dict:
    y, aux, counts, views = gpu
    sel_bias = getattr(ref, "selection_bias", None)
    T, k, E = w.T, w.k, w.E
    near = ref.margin <= MARGIN
    ok = ~near
    idx_g = views["topk_idx"].cpu().numpy()
    gates_g = views["gates"].cpu().numpy()
    assert (idx_g[ok] == ref.idx[ok]).all(), "top-k indices differ on tokens with a clear margin"
    if ok.any():
        gerr = float(np.abs(gates_g[ok] - ref.gates[ok]).max())
        assert gerr <= GATE_TOL, f"gate error {gerr}"
    contested = contested_experts(ref, w, sel_bias)
    # counts: exact for every expert no near-tie token may flip; otherwise off by
    # at most the number of near-tie tokens contesting that expert
    counts_g = counts.cpu().numpy().astype(np.int64)
    slack = np.zeros(E, dtype=np.int64)
    for m in contested.values():
        slack += m
    assert counts_g.sum() == T * k
    assert (np.abs(counts_g - ref.counts) <= slack).all(), "per-expert counts differ"
    # the probability sums do not depend on the choice; the statistic is checked
    # on the layer's own counts (identical to the oracle's without near-ties)
    probsum_g = views["probsum"].cpu().numpy()
    assert np.allclose(probsum_g, ref.probsum, rtol=1e-6, atol=1e-6 * T)
    a = float(aux.cpu()[0])
    a_ref = O.aux_statistic(counts_g, ref.probsum, T, k) if T else 0.0
    assert abs(a - a_ref) <= 1e-6 * max(1.0, abs(a_ref)), (a, a_ref)
    C = ref.capacity
    valid = unaffected_tokens(ref, contested)
    slot_g = views["slot_pos"].cpu().numpy()
    assert ((slot_g[valid] >= 0) == ref.keep[valid]).all(), "capacity cut differs"
    if check_positions and not near.any():
        pos, ts = expected_slot_pos(ref, E)
        assert (slot_g == pos).all(), "permutation rows differ"
        assert (views["tile_start"].cpu().numpy() == ts).all()
    rows = ref.rows
    sel = valid[rows]
    yg = y.float().cpu().numpy()[rows][sel]
    yr = ref.y[sel]
    tol = Y_TOL[w.dtype]
    err = np.abs(yg - yr)
    bound = tol * np.maximum(1.0, np.abs(yr))
    worst = float((err / bound).max()) if err.size else 0.0
    assert worst <= 1.0, f"y error {float(err.max())} exceeds {tol}*max(1,|ref|) (ratio {worst})"
    # dropped tokens (every assignment cut, no shared expert) are exactly zero
    if C is not None and not w.d_s:
        gone = (~ref.keep.any(axis=1)) & valid
        gone_rows = np.nonzero(gone[rows])[0]
        if gone_rows.size:
            assert np.all(y.float().cpu().numpy()[rows][gone_rows] == 0.0)
    return dict(max_err=float(err.max()) if err.size else 0.0, worst_ratio=worst,
                near_ties=int(near.sum()), excluded=int((~valid).sum()),
                rows_compared=int(sel.sum()), rows_sampled=int(len(rows)))


def check_workload(w: Workload, sample: int | None = None, seed: int = 0) -> dict:
    inp = make_inputs(w, device="cuda")
    gpu = run_gpu(w, inp)
    rows = None
    if sample is not None and sample < w.T:
        rng = np.random.default_rng(seed)
        rows = np.sort(rng.choice(w.T, size=sample, replace=False))
    ref = run_oracle(w, inp, rows)
    return compare(w, gpu, ref)


def oracle_quantized_weights(inp: dict, device="cuda") -> dict:
    """E4M3 codes and scales of the drawn dtype weights, computed by the oracle's
    quantiser on the CPU, in the layer's FP8 input layout."""
    out, scales = {}, []
    for name in ("W_g", "W_u", "W_d"):
        wt = inp[name].float().cpu().numpy()
        n, r, c = wt.shape
        codes, sc = O.quantize_rows_fp8(wt.reshape(-1, c))
        out[name] = torch.from_numpy(codes.reshape(n, r, c)).to(device)
        scales.append(torch.from_numpy(sc))
    out["weight_scales"] = torch.cat(scales).to(device)
    return out


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """One 4-bit code per element -> two per byte, the even element in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def oracle_mxfp4_weights(inp: dict, device="cuda") -> dict:
    """MXFP4 codes, block scales and row factors of the drawn dtype weights,
    quantised by the oracle on the CPU, in the layer's input layout; also the
    oracle's own (codes, exponents) per stack for its reference."""
    out, bsc, rfs, mx = {}, [], [], []
    for name in ("W_g", "W_u", "W_d"):
        wt = inp[name].float().cpu().numpy()
        n, r, c = wt.shape
        codes, exps = O.quantize_rows_mxfp4(wt.reshape(-1, c))
        out[name] = torch.from_numpy(pack_e2m1(codes).reshape(n, r, c // 2)).to(device)
        bsc.append(torch.from_numpy((exps + 127).astype(np.uint8).reshape(-1)))
        rfs.append(torch.from_numpy(row_factors_of(codes, exps)))
        mx.append((codes.reshape(n, r, c), exps.reshape(n, r, c // 32)))
    out["block_scales"] = torch.cat(bsc).to(device)
    out["weight_scales"] = torch.cat(rfs).to(device)
    out["oracle_mx"] = mx
    return out


def row_factors_of(codes: np.ndarray, exps: np.ndarray) -> np.ndarray:
    """2^(largest exponent among each row's blocks that hold a non-zero code), 1 if none."""
    rows, K = codes.shape
    nz = (codes.reshape(rows, K // 32, 32) & 0x7).any(axis=2)
    big = np.where(nz, exps, np.iinfo(np.int64).min).max(axis=1)
    return np.where(nz.any(axis=1), np.ldexp(1.0, np.maximum(big, -200)), 1.0).astype(np.float32)

"""Plain fp64 CPU oracle of the top-k routed MoE FFN forward pass.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path. It shares no code with
the CUDA library; the only thing both sides share is the seeded input
generator module, which holds none of the layer's arithmetic.

Every function follows the pages step by step, with numpy fp64 matrix products
as the only library primitive. Sources (page title, then section):

  [ZTF]  Zero to Frontier, ch. 13 section 13.1 "Why MoE": "The MoE layer"
         (router r = x W_r, TopK, gate softmax over the kept logits, SwiGLU
         experts, MoE(x) = sum_{i in K} g_i FFN_i(x)); "Total and active
         parameters"; "Mixtral 8x7B, counted exactly"; "DeepSeek-V3, counted
         exactly"; "In PyTorch" (loop over experts; FLOP table).
  [KL]   kevinluzbetak "Mixture-Of-Experts": routing paragraph (p =
         softmax(h W_r), keep top-k, renormalise), balancing list
         (E * sum_i f_i P_i) and the capacity worked example.
  [AEI]  AI Engineering Illustrated, "Mixture of Experts": "The router is
         small but it decides everything" (router in float32), "The safety
         valve is a capacity limit" (dropped tokens skip the expert),
         "Fine-grained experts and a shared expert".
  [JP]   jacopoparretti "Mixture of experts, token by token": "A hard limit"
         (capacity), "A penalty" (Switch balance statistic).

Readings taken where the pages are silent or disagree (each listed in the
design notes):
  R1 top-k ties go to the lower expert index;
  R2 the router logit is the exact dot product rounded once to float32
     (the pages fix the router precision at float32); every later step is fp64;
  R3 capacity C = floor(cf * T * k / E); within an expert the first C
     assignments in token order are kept; gates are not renormalised over the
     survivors; a dropped assignment contributes 0;
  R4 f_i = routed assignments to i / (T k), counted before the capacity cut;
     P_i = mean over tokens of the full softmax; the statistic is E sum f_i P_i
     with no alpha weight;
  R5 the shared expert is added with weight 1 and is never dropped;
  R6 an optional per-expert router bias is added to the logits before both the
     softmax and the top-k.
The drop ordering of R3 is "parity unpinned" by the pages: it is fixed only by
this definition and a hand-built case.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np

__all__ = [
    "router_logits", "softmax_all", "top_k", "gates_softmax_topk", "gates_renormalised",
    "topk_margin", "capacity_limit", "capacity_keep", "silu", "swiglu_ffn",
    "GATE_RENORM", "GATE_RAW", "GATE_SIGMOID", "sigmoid_affinity", "balance_probs",
    "selection_scores", "group_eligible", "select_experts", "gates_for_mode",
    "E4M3_MAX", "e4m3_round", "e4m3_encode", "e4m3_decode", "quantize_rows_fp8",
    "dequantize_rows_fp8", "fake_quant_rows_fp8", "swiglu_ffn_w8a8",
    "E2M1_MAX", "MX_BLOCK", "e2m1_round", "e2m1_encode", "e2m1_decode", "quantize_rows_mxfp4",
    "dequantize_rows_mxfp4",
    "aux_statistic", "aux_statistic_top1", "dropped_fraction", "moe_forward",
    "moe_param_count", "active_flops", "OracleResult",
]


def _f64(a) -> np.ndarray:
    """Exact upcast of a numpy array or a (CPU) torch tensor to float64."""
    if hasattr(a, "detach"):  # torch tensor: bf16 -> fp32 is exact, then fp64
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# Router  ([ZTF] "The MoE layer"; [AEI] router precision; [KL] routing paragraph)
# ----------------------------------------------------------------------------

def router_logits(x, W_r, bias=None) -> np.ndarray:
    """Router logits r = x W_r for every token, one per expert.

    x: [T, d]; W_r: [E, d] (the router matrix stored expert-major, i.e. W_r^T of
    the page's d x E map); bias: optional [E] added to every token's logits (R6).
    The sum is taken in fp64 on the exact input values, then rounded once to
    float32 (R2); the result is returned as float64 holding float32 values.
    """
    r = _f64(x) @ _f64(W_r).T
    if bias is not None:
        r = r + _f64(bias)[None, :]
    return r.astype(np.float32).astype(np.float64)


def softmax_all(r: np.ndarray) -> np.ndarray:
    """p = softmax(r) over all E experts, per token, max-subtracted ([KL])."""
    z = r - r.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def top_k(r: np.ndarray, k: int) -> np.ndarray:
    """The set K = TopK(r, k) per token, as indices [T, k] in slot order.

    Slot order is descending logit; equal logits go to the lower index (R1).
    A stable sort of -r keeps equal keys in index order, which is that rule.
    """
    order = np.argsort(-r, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def gates_softmax_topk(r: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_i = e^{r_i} / sum_{j in K} e^{r_j} for i in K ([ZTF] "The MoE layer")."""
    rk = np.take_along_axis(r, idx, axis=1)
    z = np.exp(rk - rk.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def gates_renormalised(p: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g = p_K / sum(p_K): softmax over all experts, keep the top-k, renormalise ([KL])."""
    pk = np.take_along_axis(p, idx, axis=1)
    return pk / pk.sum(axis=1, keepdims=True)


def topk_margin(r: np.ndarray, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit per token (+inf when k = E).

    Where this gap is tiny, either top-k set is a correct answer for logits
    carrying float32 rounding, so comparisons of routing decisions use it.
    """
    E = r.shape[1]
    if k >= E:
        return np.full(r.shape[0], np.inf)
    s = -np.sort(-r, axis=1)
    return s[:, k - 1] - s[:, k]


# ----------------------------------------------------------------------------
# Gate variants and DeepSeek-V3 scoring
#   mode 1, raw softmax gates: [JP] "Experts and a router" (Switch takes a
#     softmax over all experts first and keeps only the top one); [KL] routing
#     worked example (some implementations skip the renormalisation).
#   selection-only bias: [AEI] "Fix 2 nudges a bias instead" and [JP] "A bias"
#     (a per-expert bias added to the score only when picking the top k; the
#     mixing weights ignore it).
#   mode 2, sigmoid affinities: [AEI] "The router is small but it decides
#     everything" and [JP] "Experts and a router" (a sigmoid per expert, top k,
#     then the k chosen affinities normalised to sum to one).
#   group-limited selection: [JP] "Smaller experts, more of them" (each token
#     is limited to 4 of its 8 expert groups; the released configuration has
#     n_group 8, topk_group 4).
# Readings where the pages are silent:
#   R7  the raw-probability gates of mode 1 are not renormalised for any k;
#   R8  in mode 2, P_i of the balance statistic is the mean over tokens of the
#       affinity normalised over all experts, s_i / sum_j s_j;
#   R9  groups are contiguous blocks of E / n_group experts; a group's score is
#       its largest selection score; equal group scores go to the lower group;
#   R10 the selection bias is added to the logit (modes 0, 1) or to the
#       affinity (mode 2); the router bias of R6 still enters before everything.
# ----------------------------------------------------------------------------
GATE_RENORM, GATE_RAW, GATE_SIGMOID = 0, 1, 2


def sigmoid_affinity(r: np.ndarray) -> np.ndarray:
    """s = 1 / (1 + e^{-r}), elementwise."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-r))


def balance_probs(r: np.ndarray, gate_mode: int) -> np.ndarray:
    """Per-token, per-expert probabilities whose mean is P_i (R4, R8)."""
    if gate_mode == GATE_SIGMOID:
        s = sigmoid_affinity(r)
        return s / s.sum(axis=1, keepdims=True)
    return softmax_all(r)


def selection_scores(r: np.ndarray, gate_mode: int, selection_bias=None) -> np.ndarray:
    """What the top-k ranks: the logit (modes 0, 1) or the affinity (mode 2),
    plus the selection-only bias (R10)."""
    sel = sigmoid_affinity(r) if gate_mode == GATE_SIGMOID else r.copy()
    if selection_bias is not None:
        sel = sel + _f64(selection_bias)[None, :]
    return sel


def group_eligible(sel: np.ndarray, n_group: int, topk_group: int):
    """Experts a token may pick under group-limited routing (R9), and the gap
    between the topk_group-th and the next group score (+inf if all kept)."""
    T, E = sel.shape
    if n_group <= 1 or topk_group >= n_group:
        return np.ones((T, E), dtype=bool), np.full(T, np.inf)
    gsize = E // n_group
    gscore = sel.reshape(T, n_group, gsize).max(axis=2)
    order = np.argsort(-gscore, axis=1, kind="stable")
    keep_groups = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep_groups, order[:, :topk_group], True, axis=1)
    srt = np.take_along_axis(gscore, order, axis=1)
    return np.repeat(keep_groups, gsize, axis=1), srt[:, topk_group - 1] - srt[:, topk_group]


def select_experts(sel: np.ndarray, k: int, eligible: np.ndarray):
    """Top-k of the selection scores among eligible experts (ties to the lower
    index), in slot order, and the k-th/(k+1)-th gap among the eligible."""
    masked = np.where(eligible, sel, -np.inf)
    order = np.argsort(-masked, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int64)
    srt = np.take_along_axis(masked, order, axis=1)
    if k < sel.shape[1]:
        nxt = srt[:, k]
        gap = np.where(np.isfinite(nxt), srt[:, k - 1] - nxt, np.inf)
    else:
        gap = np.full(sel.shape[0], np.inf)
    return idx, gap


def gates_for_mode(r: np.ndarray, idx: np.ndarray, gate_mode: int) -> np.ndarray:
    """Mixing weights of the chosen experts, from the logits without the
    selection bias: mode 0 softmax over the chosen logits ([ZTF] "The MoE
    layer"); mode 1 the raw softmax probabilities (R7); mode 2 the chosen
    sigmoid affinities normalised to sum to one."""
    if gate_mode == GATE_RAW:
        return np.take_along_axis(softmax_all(r), idx, axis=1)
    if gate_mode == GATE_SIGMOID:
        sk = np.take_along_axis(sigmoid_affinity(r), idx, axis=1)
        return sk / sk.sum(axis=1, keepdims=True)
    return gates_softmax_topk(r, idx)


# ----------------------------------------------------------------------------
# Capacity  ([AEI] "The safety valve is a capacity limit"; [JP] "A hard limit";
#            [KL] capacity worked example)
# ----------------------------------------------------------------------------

def capacity_limit(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """Per-expert slot limit C = floor(cf * T * k / E) (R3); None when cf <= 0."""
    if capacity_factor is None or capacity_factor <= 0:
        return None
    return int(math.floor(float(capacity_factor) * T * k / E))


def capacity_keep(idx: np.ndarray, E: int, C: Optional[int]) -> np.ndarray:
    """Keep mask [T, k]: per expert, the first C assignments in token order (R3)."""
    T, k = idx.shape
    keep = np.ones((T, k), dtype=bool)
    if C is None:
        return keep
    seen = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            e = idx[t, s]
            keep[t, s] = seen[e] < C
            seen[e] += 1
    return keep


def dropped_fraction(counts: np.ndarray, C: Optional[int], T: int, k: int) -> float:
    """Share of the T*k assignments that overflow their expert's capacity."""
    if C is None:
        return 0.0
    return float(np.maximum(0, np.asarray(counts) - C).sum()) / (T * k)


# ----------------------------------------------------------------------------
# Experts  ([ZTF] "The MoE layer": FFN_i(x) = (SiLU(x W_g) (.) x W_u) W_d)
# ----------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + e^{-a})."""
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu_ffn(x, W_g, W_u, W_d) -> np.ndarray:
    """One SwiGLU expert on rows x [n, d].

    W_g, W_u: [d_e, d] and W_d: [d, d_e] in nn.Linear weight layout, so the
    page's x W_g is x @ W_g.T here.
    """
    x = _f64(x)
    a = x @ _f64(W_g).T
    b = x @ _f64(W_u).T
    return (silu(a) * b) @ _f64(W_d).T


# ----------------------------------------------------------------------------
# Balance statistic  ([KL] balancing list; [JP] "A penalty";
#                     [AEI] "Fix 1 adds an auxiliary loss")
# ----------------------------------------------------------------------------

def aux_statistic(counts: np.ndarray, probsum: np.ndarray, T: int, k: int) -> float:
    """E * sum_i f_i P_i with f_i = counts_i / (T k) and P_i = probsum_i / T (R4)."""
    E = len(counts)
    f = np.asarray(counts, dtype=np.float64) / (T * k)
    P = np.asarray(probsum, dtype=np.float64) / T
    return float(E * np.sum(f * P))


def aux_statistic_top1(idx: np.ndarray, p: np.ndarray) -> float:
    """Variant in which f counts only each token's first choice (for reference)."""
    T, E = p.shape
    f = np.bincount(idx[:, 0], minlength=E) / T
    return float(E * np.sum(f * p.mean(axis=0)))


# ----------------------------------------------------------------------------
# The layer
# ----------------------------------------------------------------------------

class OracleResult:
    """Everything the oracle computes for one layer call."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def moe_forward(x, W_r, expert_weights: Callable[[int], Sequence], k: int,
                capacity_factor: float = 0.0, router_bias=None,
                shared_weights: Optional[Sequence] = None,
                rows: Optional[np.ndarray] = None, gate_mode: int = GATE_RENORM,
                selection_bias=None, n_group: int = 1, topk_group: int = 1,
                act_fp8: bool = False) -> OracleResult:
    """Forward pass of the routed MoE FFN layer, looping over experts.

    x: [T, d]; W_r: [E, d]; expert_weights(e) -> (W_g[e], W_u[e], W_d[e]);
    shared_weights: (gate [d_s,d], up [d_s,d], down [d,d_s]) or None.
    rows: the token indices whose output y is evaluated (default: all). Routing,
    counts, capacity and the balance statistic always cover all T tokens.

    Steps ([KL] routing paragraph and layer listing; [ZTF] "The MoE layer" and
    "In PyTorch"): logits for every token; softmax over all experts; top-k;
    gates; counts; capacity cut in token order; then for each expert, its kept
    tokens in one batch through the SwiGLU, scaled by the gate and added into y;
    the shared expert on every token with weight 1; the balance statistic.
    gate_mode, selection_bias, n_group and topk_group select the routing
    variants above (defaults: renormalised softmax top-k, no bias, no groups).
    act_fp8: the routed experts run swiglu_ffn_w8a8 (R13) instead of swiglu_ffn.
    """
    T = x.shape[0]
    r = router_logits(x, W_r, router_bias)
    E = r.shape[1]
    p = balance_probs(r, gate_mode)
    if gate_mode == GATE_RENORM and selection_bias is None and n_group <= 1:
        idx = top_k(r, k)
        margin = topk_margin(r, k)
    else:
        sel = selection_scores(r, gate_mode, selection_bias)
        eligible, gmargin = group_eligible(sel, n_group, topk_group)
        idx, kmargin = select_experts(sel, k, eligible)
        margin = np.minimum(kmargin, gmargin)
    g = gates_for_mode(r, idx, gate_mode)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    C = capacity_limit(capacity_factor, T, k, E)
    keep = capacity_keep(idx, E, C)
    probsum = p.sum(axis=0)
    aux = aux_statistic(counts, probsum, T, k)

    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    want = np.zeros(T, dtype=bool)
    want[rows] = True
    xr = _f64(x) if not hasattr(x, "detach") else None  # lazy: convert rows only
    d = x.shape[1]
    y = np.zeros((T, d), dtype=np.float64)
    for e in range(E):
        tok, slot = np.nonzero((idx == e) & keep & want[:, None])
        if tok.size == 0:
            continue
        Wg, Wu, Wd = expert_weights(e)
        xe = xr[tok] if xr is not None else _f64(x[tok])
        ffn = swiglu_ffn_w8a8 if act_fp8 else swiglu_ffn
        y[tok] += g[tok, slot][:, None] * ffn(xe, Wg, Wu, Wd)
    if shared_weights is not None:
        xs = xr[rows] if xr is not None else _f64(x[rows])
        y[rows] += swiglu_ffn(xs, *shared_weights)

    return OracleResult(logits=r, probs=p, idx=idx, gates=g, counts=counts,
                        capacity=C, keep=keep, probsum=probsum, aux=aux,
                        margin=margin, rows=rows, y=y[rows],
                        dropped_fraction=dropped_fraction(counts, C, T, k))


# ----------------------------------------------------------------------------
# FP8 expert weights (weight-only quantisation)
#   AI Engineering Illustrated "Mixture of Experts", "Trade-offs to weigh" (at
#   small batch MoE inference is limited by reading weights; quantising the
#   expert weights, as gpt-oss does with MXFP4, attacks that directly) and
#   jacopoparretti "Mixture of experts, token by token", "Memory" (DeepSeek-V3
#   ships its weights in FP8, one byte per parameter).
# Readings (the pages fix no format details): R11 the 8-bit format is E4M3
#   (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, largest
#   finite value 448, no infinities), rounded to nearest-even and saturated to
#   +-448; R12 one fp32 scale per output row, scale = fp32(absmax / 448) (1 for
#   an all-zero row), code = E4M3(fp32(w / scale)); the layer uses
#   code_value * scale.
# ----------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_round(v) -> np.ndarray:
    """Nearest E4M3 value (ties to even), saturated to +-448, as float64.
    The spacing is 2^-9 below 2^-6 (subnormals) and 2^(e-3) in [2^e, 2^(e+1))."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    q = np.where(a < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))
    r = np.minimum(np.rint(a / q) * q, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_encode(v) -> np.ndarray:
    """uint8 codes (sign << 7 | exponent << 3 | mantissa) of E4M3 values."""
    r = e4m3_round(v)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << 7
    normal = a >= 2.0 ** -6
    e = np.floor(np.log2(np.where(normal, a, 1.0))).astype(np.int64)
    mant_n = np.rint(a / 2.0 ** e * 8 - 8).astype(np.int64)
    mant_s = np.rint(a / 2.0 ** -9).astype(np.int64)
    code = np.where(normal, ((e + 7) << 3) | mant_n, mant_s)
    return (sign | code.astype(np.uint8)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of E4M3 codes (0x7F / 0xFF, the NaN codes, never occur)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return s * val


def quantize_rows_fp8(w):
    """Per-row E4M3 quantisation (R12) of a [rows, cols] matrix; returns
    (codes uint8 [rows, cols], scales fp32 [rows])."""
    w32 = np.asarray(_f64(w), dtype=np.float32)
    absmax = np.abs(w32).max(axis=1)
    scales = np.where(absmax > 0, absmax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    ratio = (w32 / scales[:, None]).astype(np.float32)
    return e4m3_encode(ratio), scales


def dequantize_rows_fp8(codes, scales) -> np.ndarray:
    """The weights the layer computes with: code value times the row scale (fp64, exact)."""
    return e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]


# R14 (MXFP4, the 4-bit format the pages name for gpt-oss's expert weights;
# AI Engineering Illustrated "Mixture of Experts", "Trade-offs to weigh"): the
# pages give no format details, so the reading follows the Open Compute
# microscaling convention: blocks of 32 consecutive weights along K share one
# power-of-two scale X = 2^(floor(log2(absmax)) - 2) (2 = the largest E2M1
# exponent; X = 1 for an all-zero block), and each weight becomes the E2M1
# value nearest to w / X (1 sign, 2 exponent bits with bias 1, 1 mantissa bit:
# magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even mantissa, saturated
# at +-6. The layer would compute with code_value * X.
E2M1_MAX = 6.0
MX_BLOCK = 32


def e2m1_round(v) -> np.ndarray:
    """Nearest E2M1 value (ties to even), saturated to +-6, as float64. The
    spacing is 0.5 below 2, 1 in [2, 4) and 2 from 4 on."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    q = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    r = np.minimum(np.rint(a / q) * q, E2M1_MAX)
    return np.copysign(r, v)


def e2m1_encode(v) -> np.ndarray:
    """4-bit codes (sign << 3 | exponent << 1 | mantissa), one per uint8."""
    r = e2m1_round(v)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.uint8) << 3
    normal = a >= 1.0
    e = np.floor(np.log2(np.where(normal, a, 1.0))).astype(np.int64)
    mant_n = np.rint(a / 2.0 ** e * 2 - 2).astype(np.int64)
    code = np.where(normal, ((e + 1) << 1) | mant_n, np.rint(a / 0.5).astype(np.int64))
    return (sign | code.astype(np.uint8)).astype(np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    """float64 values of 4-bit E2M1 codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    val = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * 2.0 ** (e - 1))
    return s * val


def quantize_rows_mxfp4(w):
    """Per-block MXFP4 quantisation (R14) of a [rows, K] matrix, K a multiple of
    32; returns (codes uint8 [rows, K], one code per element, and the blocks'
    scale exponents int64 [rows, K / 32], X = 2^exponent)."""
    w32 = np.asarray(_f64(w), dtype=np.float32)
    rows, K = w32.shape
    blocks = w32.reshape(rows, K // MX_BLOCK, MX_BLOCK).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))  # amax = f * 2^ex, f in [0.5, 1)
    exps = np.where(amax > 0, (ex - 1) - 2, 0).astype(np.int64)
    codes = e2m1_encode(blocks / np.ldexp(1.0, exps)[:, :, None])
    return codes.reshape(rows, K), exps


def dequantize_rows_mxfp4(codes, exps) -> np.ndarray:
    """code value * 2^exponent of its block (fp64, exact)."""
    c = np.asarray(codes)
    rows, K = c.shape
    vals = e2m1_decode(c).reshape(rows, K // MX_BLOCK, MX_BLOCK)
    return (vals * np.ldexp(1.0, np.asarray(exps))[:, :, None]).reshape(rows, K)


# R13 (FP8 on both operands): the GEMM inputs of a routed expert, the token
# rows x and the hidden rows H, are quantised like the weights, one scale per
# row (per token for x, per routed (token, expert) row for H); a GEMM then
# computes with code * scale on both sides. Sources as above, plus Zero to
# Frontier 13.1 "Why MoE" (the expert FFN is two GEMMs around SwiGLU).

def fake_quant_rows_fp8(a) -> np.ndarray:
    """Rows of `a` through the per-row E4M3 quantiser and back (fp64, exact)."""
    codes, scales = quantize_rows_fp8(a)
    return dequantize_rows_fp8(codes, scales)


def swiglu_ffn_w8a8(x, W_g, W_u, W_d) -> np.ndarray:
    """One SwiGLU expert with E4M3 activations (R13): x rows quantised per row,
    the gate/up GEMM, SwiGLU in full precision, H rows quantised per row, the
    down GEMM. W_g, W_u, W_d are the weights the layer computes with (for FP8
    weights: code * scale). H is quantised from its fp64 value: the pages fix
    no storage precision for it, and every step after the router is fp64 (R2)."""
    xq = fake_quant_rows_fp8(_f64(x))
    a = xq @ _f64(W_g).T
    b = xq @ _f64(W_u).T
    hq = fake_quant_rows_fp8(silu(a) * b)
    return hq @ _f64(W_d).T


# ----------------------------------------------------------------------------
# Parameter and FLOP accounting ([ZTF] "Total and active parameters",
# "Mixtral 8x7B, counted exactly", "DeepSeek-V3, counted exactly", "FLOPs per
# token, and the 6N rule for MoE" and the dense-versus-MoE table)
# ----------------------------------------------------------------------------

def moe_param_count(cfg: dict) -> tuple:
    """(total, active) parameters of a decoder with MoE FFN layers.

    cfg keys: V, d, L, attn (attention parameters per layer), n_dense (leading
    layers with a dense FFN of width d_ff), d_ff, E (routed experts), E_shared,
    k, d_e, tied. Every FFN/expert is a bias-free SwiGLU (3 d width matrices),
    each layer has two RMSNorm gains of size d, there is one final norm, the
    router is a bias-free d x E matrix, and embeddings count in full in both.
    """
    d = cfg["d"]
    norms = 2 * d
    expert = 3 * d * cfg["d_e"]
    router = d * cfg["E"]
    dense_layer = cfg["attn"] + norms + 3 * d * cfg.get("d_ff", 0)
    moe_total = cfg["attn"] + norms + (cfg["E"] + cfg.get("E_shared", 0)) * expert + router
    moe_active = cfg["attn"] + norms + (cfg["k"] + cfg.get("E_shared", 0)) * expert + router
    n_dense = cfg.get("n_dense", 0)
    n_moe = cfg["L"] - n_dense
    emb = cfg["V"] * d * (1 if cfg.get("tied", False) else 2)
    total = n_dense * dense_layer + n_moe * moe_total + emb + d
    active = n_dense * dense_layer + n_moe * moe_active + emb + d
    return total, active


def active_flops(kept_assignments: int, d: int, d_e: int, T: int = 0, d_s: int = 0) -> int:
    """Forward FLOPs of the expert products: 2 per multiply-add, 3 d d_e per
    assignment, plus the shared expert's 3 d d_s per token (router excluded)."""
    return 2 * 3 * d * d_e * int(kept_assignments) + 2 * 3 * d * d_s * int(T)

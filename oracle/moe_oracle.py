"""CPU oracle for the DeepSeek-V3/R1 Mixture-of-Experts block forward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (``sparse_moe_layer_sum_b200``) never calls it and
shares no code with it; the only thing both sides share is the seeded input
generator, which holds none of the method's arithmetic.

Plain, slow and meant to be checked by eye against the pages:

* "DeepSeek-V3.2-Exp · Router" -- the four equations under "All 4 steps"
  (z = x W_r, s = sigma(z), the group-limited top-8 selection E_sel and the
  gate G_i = 2.5 s_i E_sel_i / sum_j s_j E_sel_j) and the gate-forward code
  excerpt under "Code" (fp32 scoring, sigmoid or softmax, bias added for
  selection only, group score = sum of the top two, top groups, mask, top-k,
  gather of the unbiased scores, renormalise, scale).
* "DeepSeek-V3.2-Exp · Mixture of experts" -- the moe-forward code excerpt
  under "Code" (fp32 accumulator y, bincount of the indices, skip empty
  experts, per-expert ``torch.where`` grouping, ``y[idx] += expert(x[idx]) *
  weight``, ``y += shared_experts(x)``) and the parameter table under
  "Parameters".

Floating point is fp64 everywhere except where the pages fix fp32: the router
scores are fp32 (the excerpt casts x and the weight to float), so the scores
s, the biased scores c = s + b and the group scores used for the *decisions*
are rounded to fp32 exactly as the excerpt's fp32 tensors would be.  Every
decision is reported with its gap so that callers can tell near-ties apart.

Readings of points the pages leave open:

1. The routed/shared expert body is not printed; it is read as SwiGLU with
   three bias-free matrices, w2(silu(w1 x) * w3 x), which matches the printed
   per-expert parameter count 3 * 7168 * 2048 = 44,040,192.
2. top-k order: descending by value, ties to the lower index (groups and
   experts alike).
3. h = silu(a) * u is rounded once to the activation dtype (bf16 for bf16
   activations, fp32 for fp32 ones) because it is the second matmul's operand;
   the rounding is done through fp32 (fp64 -> fp32 -> bf16, each
   round-to-nearest-even), the order a fp32-accumulating kernel uses.
4. Expert outputs are kept unrounded (fp64 here), weighted in fp64 and summed
   into an fp64 y that stands in for the excerpt's fp32 accumulator.
5. FP8 weights: e4m3 codes with one fp32 scale per 128 x 128 block of the
   [out, in] weight matrix; the dequantised weight is fp32(q) * scale.
6. FP8 activations (the optional FP8 x FP8 path of the FP8-weight
   configuration; the pages name FP8 experts but no activation format):
   each row of x, and each row of h after its bf16 rounding, is quantised to
   e4m3 with the weights' rule applied to the row, scale = row amax / 448,
   in fp32 arithmetic (one scale per token and matrix).

Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np

# --------------------------------------------------------------------------
# configuration
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class MoEShape:
    """Block hyper-parameters named as in the gate-init / moe-init excerpts."""

    dim: int                 # model width D
    n_routed_experts: int    # E
    n_expert_groups: int     # G
    n_limited_groups: int    # groups kept per token
    n_activated_experts: int  # k
    moe_inter_dim: int       # I
    n_shared_experts: int = 1
    route_scale: float = 2.5
    score_func: str = "sigmoid"
    has_bias: bool = True


def param_counts(shape: MoEShape) -> dict:
    """Learned parameters of one block.

    Restates the "Exact per-instance accounting" tables of the pages
    "DeepSeek-V3.2-Exp · Mixture of experts" (router, routed expert x 256,
    shared expert) and "DeepSeek-V3.2-Exp · Router" (expert scores
    dim x experts, select-experts bias of one value per expert).  An expert
    is three bias-free matrices (reading 1 in the module docstring).
    """
    d, e, i = shape.dim, shape.n_routed_experts, shape.moe_inter_dim
    expert = 3 * d * i
    shared = 3 * d * (shape.n_shared_experts * i)
    router = d * e + (e if shape.has_bias else 0)
    total = e * expert + shared + router
    per_token = shape.n_activated_experts * expert + shared + router
    return {
        "routed_expert": expert,
        "all_routed": e * expert,
        "shared_expert": shared,
        "router": router,
        "block": total,
        "used_per_token": per_token,
    }


# --------------------------------------------------------------------------
# number formats (definitions written out, used for inputs and roundings)
# --------------------------------------------------------------------------


def round_f32_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even), as fp32.

    bfloat16 keeps the top 16 bits of the fp32 encoding.  Round to nearest
    even: add 0x7FFF plus the lowest kept bit, then clear the low 16 bits.
    Finite inputs only.
    """
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep_lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = (b + np.uint64(0x7FFF) + keep_lsb) & np.uint64(0xFFFF0000)
    return r.astype(np.uint32).view(np.float32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 codes (uint16) as fp32: the code is the top half."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_table() -> np.ndarray:
    """Value of each of the 256 float8 e4m3 ("fn") codes, fp64.

    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    is subnormal (m/8 * 2^-6); there is no infinity and S.1111.111 is NaN.
    Largest finite magnitude is 1.75 * 2^8 = 448.
    """
    out = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        ex = (code >> 3) & 0xF
        man = code & 0x7
        if ex == 0xF and man == 0x7:
            out[code] = math.nan
        elif ex == 0:
            out[code] = sign * (man / 8.0) * 2.0 ** -6
        else:
            out[code] = sign * (1.0 + man / 8.0) * 2.0 ** (ex - 7)
    return out


def round_f32_to_f16(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest IEEE binary16 value (ties to even), as fp64.

    binary16 has 10 fraction bits, exponent bias 15 and subnormals below
    2^-14 with spacing 2^-24.  A finite value v with |v| in [2^e, 2^(e+1))
    (e >= -14) is a multiple of 2^(e-10) once rounded; below 2^-14 the
    spacing stays 2^-24.  Magnitudes that round above 65504 are out of range
    (not used: the callers keep far below it).
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    mag = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, -14.0)
    step = np.exp2(e - 10.0)
    r = np.rint(v / step) * step          # np.rint rounds halves to even
    if np.any(np.abs(r) > 65504.0):
        raise OverflowError("value outside the binary16 range")
    return r


E4M3_MAX = 448.0


def round_to_e4m3(v: np.ndarray) -> np.ndarray:
    """Nearest float8 e4m3 value (ties to even), saturated to +-448, as fp64.

    e4m3 keeps 3 fraction bits with exponent bias 7: a value with |v| in
    [2^e, 2^(e+1)) (e >= -6) rounds to a multiple of 2^(e-3); below 2^-6 the
    subnormal spacing is 2^-9.  Magnitudes beyond the largest finite value
    448 are clamped to it (the "satfinite" conversion).  NaN is not handled.
    """
    v = np.asarray(v, dtype=np.float64)
    mag = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
    e = np.maximum(e, -6.0)
    step = np.exp2(e - 3.0)
    r = np.rint(v / step) * step
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def e4m3_code(values: np.ndarray) -> np.ndarray:
    """The uint8 code of e4m3 values (exact e4m3 values in, e.g. from
    round_to_e4m3); +0 for zero."""
    t = e4m3_table()
    finite = np.nonzero(np.isfinite(t))[0]
    lut = {float(t[c]): c for c in finite if not (t[c] == 0 and c == 0x80)}
    return np.vectorize(lambda x: lut[float(x)], otypes=[np.uint8])(np.asarray(values))


def quantize_e4m3_rows(v: np.ndarray, block: Optional[int] = None):
    """Per-row e4m3 quantisation of activations in 1 x block runs (the whole
    row when block is None), fp32 arithmetic.

    For each row and each run of `block` columns: amax = max |v| (exact),
    scale = fp32(amax / 448) (an IEEE fp32 division), r = fp32(1 / scale)
    (IEEE fp32 reciprocal), code = the e4m3 value nearest fp32(v * r) (ties
    to even, saturated); an all-zero block has scale 0 and codes 0.  This is
    the weights' rule (scale = block amax / 448) applied to 1 x 128 blocks of
    a row, with one reciprocal per block in place of a division per value.
    Returns (values [rows, cols] fp64 of the codes, scales [rows, cols/block] fp32);
    the dequantised activation is values * scale.
    """
    v = np.asarray(v, dtype=np.float32)
    r, c = v.shape
    block = c if block is None else block
    vb = v.reshape(r, c // block, block)
    amax = np.abs(vb).max(axis=-1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    recip = (np.float32(1.0) / safe).astype(np.float32)     # fp32 reciprocal
    q = (vb * recip[:, :, None]).astype(np.float32)         # fp32 product
    vals = round_to_e4m3(q.astype(np.float64))
    vals = np.where(scale[:, :, None] > 0, vals, 0.0)
    return vals.reshape(r, c), scale


def dequant_e4m3_rows(vals: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 activation from the e4m3 values and their per-row scales
    (one or more equal runs of columns per scale)."""
    s = np.asarray(scales, dtype=np.float64)
    s = np.repeat(s, np.asarray(vals).shape[-1] // s.shape[-1], axis=-1)
    return np.asarray(vals, dtype=np.float64) * s


def dequant_e4m3_block(q_codes: np.ndarray, scales: np.ndarray, block: int = 128) -> np.ndarray:
    """fp64 weight from e4m3 codes [out, in] and fp32 scales [ceil(out/128), ceil(in/128)].

    w[r, c] = value(q[r, c]) * scale[r // 128, c // 128]  (reading 5).
    """
    q = np.asarray(q_codes, dtype=np.uint8)
    vals = e4m3_table()[q]
    s = np.asarray(scales, dtype=np.float64)
    r, c = q.shape
    if r % block == 0 and c % block == 0:
        # each block times its scale (the same products as the general form)
        vb = vals.reshape(r // block, block, c // block, block)
        return (vb * s[:, None, :, None]).reshape(r, c)
    rows = np.arange(r) // block
    cols = np.arange(c) // block
    return vals * s[rows][:, cols]


# --------------------------------------------------------------------------
# router  ("DeepSeek-V3.2-Exp · Router")
# --------------------------------------------------------------------------


@dataclass
class RouterResult:
    weights: np.ndarray      # [T, k] fp64 gate weights (unbiased scores, renormalised, scaled)
    indices: np.ndarray      # [T, k] int64, descending by biased score, ties -> lower index
    scores: np.ndarray       # [T, E] fp32 s (sigmoid or softmax)
    biased: np.ndarray       # [T, E] fp32 c = s + b (or s when there is no bias)
    group_scores: Optional[np.ndarray]  # [T, G] fp32, None when G == 1
    kept_groups: Optional[np.ndarray]   # [T, Gk] int64
    gap_set: np.ndarray      # [T] smallest gap of a decision that changes the selected set
    gap_order: np.ndarray    # [T] smallest gap between consecutive selected experts


def _desc_order(v: np.ndarray) -> np.ndarray:
    """Indices that sort each row descending by value, ties to the lower index."""
    # stable sort of the negated values keeps equal values in index order
    return np.argsort(-v, axis=-1, kind="stable")


def router(x: np.ndarray, w_r: np.ndarray, bias: Optional[np.ndarray], shape: MoEShape) -> RouterResult:
    """Route every token (the gate-forward excerpt and "All 4 steps").

    x [T, D] (values exactly representable in fp32), w_r [E, D] fp32,
    bias [E] fp32 or None.
    """
    T = x.shape[0]
    E, G, Gk, k = (shape.n_routed_experts, shape.n_expert_groups,
                   shape.n_limited_groups, shape.n_activated_experts)
    # z = x W_r^T: the excerpt computes linear(x.float(), weight.float()); here
    # the exact fp32 inputs are multiplied and summed in fp64 and the score
    # is rounded to fp32 once.
    z = np.asarray(x, dtype=np.float64) @ np.asarray(w_r, dtype=np.float64).T
    if shape.score_func == "softmax":
        m = z.max(axis=-1, keepdims=True)
        ez = np.exp(z - m)
        s = (ez / ez.sum(axis=-1, keepdims=True)).astype(np.float32)
    else:
        s = (1.0 / (1.0 + np.exp(-z))).astype(np.float32)
    original = s
    if bias is not None:
        c = (s + np.asarray(bias, dtype=np.float32)).astype(np.float32)   # fp32 add
    else:
        c = s
    gap_set = np.full(T, np.inf)
    group_scores = kept = None
    masked = c.astype(np.float64)
    if G > 1:
        cg = c.reshape(T, G, E // G)
        if bias is None:
            group_scores = cg.max(axis=-1)
        else:
            top2 = -np.sort(-cg, axis=-1)[:, :, :2]
            group_scores = (top2[:, :, 0] + top2[:, :, 1]).astype(np.float32)  # fp32 add
        gorder = _desc_order(group_scores)
        kept = np.sort(gorder[:, :Gk], axis=-1)
        if Gk < G:
            gs_sorted = np.take_along_axis(group_scores, gorder, axis=-1).astype(np.float64)
            gap_set = np.minimum(gap_set, gs_sorted[:, Gk - 1] - gs_sorted[:, Gk])
        keep_mask = np.zeros((T, G), dtype=bool)
        np.put_along_axis(keep_mask, kept, True, axis=-1)
        expert_kept = np.repeat(keep_mask, E // G, axis=-1)
        masked = np.where(expert_kept, masked, -np.inf)
    order = _desc_order(masked)
    indices = order[:, :k].astype(np.int64)
    srt = np.take_along_axis(masked, order, axis=-1)
    if k < E:
        boundary = srt[:, k - 1] - srt[:, k]
        gap_set = np.minimum(gap_set, boundary)
    if k > 1:
        gap_order = (srt[:, : k - 1] - srt[:, 1:k]).min(axis=-1)
    else:
        gap_order = np.full(T, np.inf)
    # weights = original_scores.gather(1, indices), renormalised for sigmoid,
    # then scaled by route_scale
    w = np.take_along_axis(original.astype(np.float64), indices, axis=-1)
    if shape.score_func == "sigmoid":
        w = w / w.sum(axis=-1, keepdims=True)
    w = w * shape.route_scale
    return RouterResult(w, indices, original, c, group_scores, kept, gap_set, gap_order)


# --------------------------------------------------------------------------
# token grouping  ("DeepSeek-V3.2-Exp · Mixture of experts", moe-forward)
# --------------------------------------------------------------------------


@dataclass
class Dispatch:
    counts: np.ndarray        # [E] int64, bincount of the indices
    offsets: np.ndarray       # [E+1] int64, exclusive prefix sum of counts
    sorted_token: np.ndarray  # [T*k] int64, token of each expert-contiguous row
    slot_of: np.ndarray       # [T*k] int64, row of pair (t, j) in expert order


def dispatch(indices: np.ndarray, n_experts: int) -> Dispatch:
    """Histogram, exclusive scan and the stable per-expert token lists.

    Within expert e the rows are the pairs (t, j) with indices[t, j] == e in
    ascending token order -- the row-major order ``torch.where(indices == i)``
    returns in the moe-forward excerpt.  A token's k experts are distinct, so
    flat order t*k + j is ascending t within each expert.
    """
    flat = np.asarray(indices, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=n_experts).astype(np.int64)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable")          # rows of the expert-major order
    k = indices.shape[1] if indices.ndim == 2 else 1
    sorted_token = perm // k
    slot_of = np.empty_like(perm)
    slot_of[perm] = np.arange(perm.size)
    return Dispatch(counts, offsets, sorted_token, slot_of)


# --------------------------------------------------------------------------
# experts
# --------------------------------------------------------------------------


def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * sigma(a) = a / (1 + exp(-a)), fp64."""
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def expert_ffn(x_rows: np.ndarray, w1: np.ndarray, w3: np.ndarray, w2: np.ndarray,
               act_dtype: str) -> np.ndarray:
    """One expert on a set of rows: w2(silu(w1 x) * w3 x) (reading 1).

    x_rows [n, D]; w1, w3 [I, D]; w2 [D, I] in the nn.Linear [out, in] layout.
    The hidden activation h is rounded once, through fp32, to the type of
    the second matmul's operand (reading 3): ``act_dtype`` "bf16", "f16" or
    "f32".  "e4m3" (reading 6): each row of x and each row of the
    bf16-rounded h is quantised to e4m3 with one scale per row
    (quantize_e4m3_rows) and the matmuls take the dequantised values.
    Returns fp64 [n, D].
    """
    x64 = np.asarray(x_rows, dtype=np.float64)
    if act_dtype == "e4m3":
        x64 = dequant_e4m3_rows(*quantize_e4m3_rows(x64.astype(np.float32)))
    a = x64 @ np.asarray(w1, dtype=np.float64).T
    u = x64 @ np.asarray(w3, dtype=np.float64).T
    h = (silu(a) * u).astype(np.float32)
    if act_dtype == "bf16":
        h = round_f32_to_bf16(h)
    elif act_dtype == "f16":
        h = round_f32_to_f16(h)
    elif act_dtype == "e4m3":
        h = dequant_e4m3_rows(*quantize_e4m3_rows(round_f32_to_bf16(h)))
    elif act_dtype != "f32":
        raise ValueError(act_dtype)
    return np.asarray(h, dtype=np.float64) @ np.asarray(w2, dtype=np.float64).T


# expert weights are fetched lazily so that callers can keep large weight
# sets off the host: get(e) -> (w1 [I, D], w3 [I, D], w2 [D, I]) as arrays
ExpertGetter = Callable[[int], Sequence[np.ndarray]]


def moe_forward(x: np.ndarray, route: RouterResult, get_expert: ExpertGetter,
                get_shared: Optional[Callable[[], Sequence[np.ndarray]]],
                n_experts: int, act_dtype: str,
                tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """The block output y for the rows ``tokens`` (all rows when None).

    Follows the moe-forward excerpt: an fp64 stand-in for the fp32 zero
    accumulator, then experts in ascending id, skipping experts with no
    tokens, each adding ``expert(x[idx]) * weights[idx, top]`` to its rows,
    then the shared expert on every row with weight 1.  The rows are
    independent, so evaluating a subset gives the same rows as the full call.
    """
    T = x.shape[0]
    rows = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    sub_idx = route.indices[rows]
    sub_w = route.weights[rows]
    y = np.zeros((rows.size, x.shape[1]), dtype=np.float64)
    counts = np.bincount(sub_idx.reshape(-1), minlength=n_experts)
    for e in range(n_experts):
        if counts[e] == 0:
            continue
        r_local, top = np.nonzero(sub_idx == e)     # row-major: ascending token
        w1, w3, w2 = get_expert(e)
        out = expert_ffn(x[rows[r_local]], w1, w3, w2, act_dtype)
        y[r_local] += out * sub_w[r_local, top][:, None]
    if get_shared is not None:
        w1, w3, w2 = get_shared()
        y += expert_ffn(x[rows], w1, w3, w2, act_dtype)
    return y

"""CPU fp64 oracle of the Step-3.5-Flash sparse-MoE FFN layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` do.  It shares no code with the CUDA library and
imports nothing from it; it depends on NumPy alone.

What it computes is the plain definition of the layer as the source pages state
it, written out step by step in float64 (inputs are upcast exactly):

* sglang-jax issue #1367 "[Feature] Support Step 3.5 Flash (StepFun) Model",
  section "Model configuration" (MoE bullet: 288 routed + 1 shared expert,
  intermediate 1280, top-8, sigmoid routing in fp32, router bias, normalised
  top-k weights, routed scaling 3.0; clamped SwiGLU where the limit 0.0 means
  "no clamp"), section "Reuse map" (a SiLU-and-mul with an elementwise clamp
  branch) and section "Key difficulties" item 1 (the routing order: sigmoid
  scores in fp32; the bias is used only to select the top-k; the gating
  weights come from the bias-free scores, are renormalised, then multiplied by
  routed_scaling_factor).
* llm-atlas "Step-3.5-Flash", table "Raw config fields" (moe_num_experts 288,
  moe_top_k 8, moe_intermediate_size 1280, share_expert_dim 1280,
  norm_expert_weight true, moe_router_activation sigmoid,
  moe_router_scaling_factor 3, use_moe_router_bias true, need_fp32_gate true,
  swiglu_limits / swiglu_limits_shared).

Readings taken where the pages are silent (each listed with the design notes):

* the bias is added to the sigmoid scores (not to the logits) to form the
  selection score;
* the selection keeps the k largest selection scores, ordered by descending
  score, equal scores going to the lower expert index;
* the selection decision is taken in fp32, the precision the pages give the
  router ("sigmoid routing computed in fp32", need_fp32_gate): the fp64 logit
  is rounded once to fp32, the sigmoid is the correctly rounded fp32 value of
  the exact sigmoid of that logit, and bias is added in fp32 arithmetic;
* renormalise first, then scale; no epsilon in the renormalisation;
* the shared expert has no gate and weight 1.0 (no config field gives it one);
* clamp: gate = min(gate, L), up = clip(up, -L, L), applied before silu(gate)*up;
  L <= 0 means no clamp; the shared expert has its own limit;
* weight layout: x @ W convention, w_gate/w_up [E, H, I], w_down [E, I, H],
  router_w [H, E].

Parity status: every function here is pinned by tests in
``tests/test_oracle.py`` (brute force, closed forms, invariants, special cases
that reduce to textbook routines).  No page prints a worked numeric example,
so beyond those pins the output values have no page-printed anchor.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Any, Optional, Sequence

import numpy as np

__all__ = [
    "OracleResult",
    "router_logits",
    "sigmoid64",
    "selection_scores_fp32",
    "select_topk",
    "select_topk_by_rounds",
    "gate_weights",
    "swiglu_expert",
    "expert_permutation",
    "moe_routing",
    "moe_forward",
    "moe_forward_rows",
    "moe_forward_dense_masked",
    "near_tie_gaps",
    "dense_mlp",
    "decode_e4m3",
    "dequantize_e4m3",
    "DequantizedExperts",
]


def _f64(a) -> np.ndarray:
    """Exact upcast of any float array (fp32, or bf16 already widened to fp32)."""
    return np.asarray(a, dtype=np.float64)


def router_logits(x, router_w) -> np.ndarray:
    """Router logits l = x . W_r, [T, H] x [H, E] -> [T, E], in float64.

    sglang-jax issue #1367, "Model configuration" (MoE bullet, "computed in
    fp32") and llm-atlas "Step-3.5-Flash", "Raw config fields"
    (need_fp32_gate true).  The exact product in float64 is the target every
    fp32 implementation approximates.
    """
    return _f64(x) @ _f64(router_w)


def sigmoid64(z) -> np.ndarray:
    """The logistic function 1 / (1 + exp(-z)) in float64
    (moe_router_activation = sigmoid, llm-atlas "Raw config fields")."""
    z = _f64(z)
    return 1.0 / (1.0 + np.exp(-z))


def selection_scores_fp32(logits, bias) -> tuple[np.ndarray, np.ndarray]:
    """fp32 sigmoid scores s and fp32 selection scores beta = s + b.

    sglang-jax issue #1367, "Key difficulties" item 1: scores are the sigmoid
    in fp32, the router bias serves the top-k selection only.  The logit is
    rounded once to fp32, s is the fp32 rounding of the exact sigmoid of that
    value, and beta is the fp32 sum s + b (IEEE round-to-nearest).
    Returns (s32, beta32), both float32 [T, E].
    """
    l32 = np.asarray(logits, dtype=np.float64).astype(np.float32)
    s32 = sigmoid64(l32).astype(np.float32)
    if bias is None:
        b32 = np.zeros(s32.shape[-1], dtype=np.float32)
    else:
        b32 = np.asarray(bias, dtype=np.float32)
    beta32 = (s32 + b32[None, :]).astype(np.float32)
    return s32, beta32


def select_topk(beta, k: int) -> np.ndarray:
    """Top-k selection by a full stable sort: indices of the k largest scores,
    ordered by descending score, equal scores to the lower index.  [T, E] ->
    [T, k] int32 (moe_top_k, llm-atlas "Raw config fields")."""
    beta = np.asarray(beta)
    T, E = beta.shape
    out = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        # lexsort sorts by the last key first: primary -beta, secondary index
        order = np.lexsort((idx, -beta[t].astype(np.float64)))
        out[t] = order[:k]
    return out


def select_topk_by_rounds(beta, k: int) -> np.ndarray:
    """The same selection made as k rounds of arg-max (np.argmax returns the
    first, i.e. lowest, index among equal maxima).  Used to cross-check
    :func:`select_topk` by brute force."""
    beta = np.array(beta, dtype=np.float64, copy=True)
    T, E = beta.shape
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        row = beta[t].copy()
        for j in range(k):
            e = int(np.argmax(row))
            out[t, j] = e
            row[e] = -np.inf
    return out


def gate_weights(s_sel, scale: float, norm: bool) -> np.ndarray:
    """Gating weights of the selected experts, from the bias-free scores.

    sglang-jax issue #1367, "Key difficulties" item 1: the weights are gathered
    from the bias-free sigmoid scores, normalised over the top-k
    (norm_expert_weight true), then multiplied by routed_scaling_factor (3).
    s_sel: [T, k] -> g: [T, k] float64.
    """
    g = _f64(s_sel)
    if norm:
        g = g / g.sum(axis=1, keepdims=True)
    return g * float(scale)


def _silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def swiglu_expert(rows, w_gate, w_up, w_down, limit: float) -> np.ndarray:
    """One SwiGLU FFN expert on a block of rows, in float64.

    a = rows . Wg, u = rows . Wu; with a limit L > 0 (sglang-jax issue #1367,
    "Model configuration": swiglu_limits, 0.0 means no clamp; "Reuse map": an
    elementwise clamp branch before SiLU-and-mul) gate = min(a, L) and
    up = clip(u, -L, L); h = silu(gate) * up; y = h . Wd.
    rows [n, H], Wg/Wu [H, I], Wd [I, H] -> y [n, H].
    """
    rows = _f64(rows)
    a = rows @ _f64(w_gate)
    u = rows @ _f64(w_up)
    if limit is not None and limit > 0.0:
        a = np.minimum(a, limit)
        u = np.clip(u, -limit, limit)
    h = _silu(a) * u
    return h @ _f64(w_down)


def expert_permutation(topk_idx, num_experts: int):
    """Token-to-expert grouping of the (token, slot) pairs.

    sglang-jax issue #1367, "Reuse map" / "Implementation strategy" (EPMoE: a
    grouped matmul needs each expert's rows contiguous).  Definition:
    counts[e] = number of pairs (t, j) with topk_idx[t, j] == e;
    offsets = exclusive prefix sum of counts, with offsets[E] = T*k;
    perm lists the pair ids t*k + j of expert 0, then expert 1, ..., each in
    ascending t; pos[t, j] is the slot of pair (t, j) in perm.
    Returns (counts[E], offsets[E+1], perm[T*k], pos[T, k]), all int32/int64.
    """
    idx = np.asarray(topk_idx)
    T, k = idx.shape
    counts = np.zeros(num_experts, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    perm = np.empty(T * k, dtype=np.int64)
    pos = np.empty((T, k), dtype=np.int64)
    for t in range(T):                       # ascending t within each expert
        for j in range(k):
            e = idx[t, j]
            perm[fill[e]] = t * k + j
            pos[t, j] = fill[e]
            fill[e] += 1
    return counts, offsets, perm, pos


def near_tie_gaps(beta32, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest selection scores per token
    (float64 of the fp32 values); +inf when k == E."""
    b = np.sort(np.asarray(beta32, dtype=np.float64), axis=1)[:, ::-1]
    if b.shape[1] <= k:
        return np.full(b.shape[0], np.inf)
    return b[:, k - 1] - b[:, k]


@dataclass
class OracleResult:
    out: np.ndarray            # [T, H] float64
    topk_idx: np.ndarray       # [T, k] int32
    topk_w: np.ndarray         # [T, k] float64
    counts: np.ndarray         # [E]
    offsets: np.ndarray        # [E+1]
    perm: np.ndarray           # [T*k]
    pos: np.ndarray            # [T, k]
    logits: np.ndarray         # [T, E] float64
    beta32: np.ndarray         # [T, E] float32 selection scores
    tie_gap: np.ndarray        # [T] gap between k-th and (k+1)-th beta


def _route(x, router_w, router_bias, top_k, scale, norm, use_bias, forced_idx):
    logits = router_logits(x, router_w)
    bias = router_bias if use_bias else None
    s32, beta32 = selection_scores_fp32(logits, bias)
    if forced_idx is None:
        idx = select_topk(beta32, top_k)
    else:
        idx = np.asarray(forced_idx, dtype=np.int32).reshape(-1, top_k)
    s_sel = np.take_along_axis(s32, idx.astype(np.int64), axis=1)
    w = gate_weights(s_sel, scale, norm)
    return logits, s32, beta32, idx, w


def moe_routing(x, router_w, router_bias, *, top_k: int, scale: float = 3.0,
                norm: bool = True, use_bias: bool = True):
    """Routing of every token without the expert FFNs: a dict of topk_idx,
    topk_w, counts, offsets, perm, pos, logits, s32 (the fp32 bias-free
    scores), beta32 (the fp32 selection scores) and tie_gap.  Same steps as
    :func:`moe_forward` (sglang-jax issue #1367, "Key difficulties" item 1)."""
    x64 = _f64(x)
    E = np.asarray(router_w).shape[1]
    logits, s32, beta32, idx, w = _route(x64, router_w, router_bias, top_k, scale, norm,
                                         use_bias, None)
    counts, offsets, perm, pos = expert_permutation(idx, E)
    return dict(topk_idx=idx, topk_w=w, counts=counts, offsets=offsets, perm=perm, pos=pos,
                s32=s32, beta32=beta32, tie_gap=near_tie_gaps(beta32, top_k), logits=logits)


def moe_forward(x, router_w, router_bias, w_gate, w_up, w_down,
                sh_gate, sh_up, sh_down, *, top_k: int,
                scale: float = 3.0, norm: bool = True, use_bias: bool = True,
                swiglu_limit: float = 0.0, swiglu_limit_shared: float = 0.0,
                forced_idx: Optional[np.ndarray] = None) -> OracleResult:
    """The MoE FFN layer forward for every token, as the pages define it.

    out[t] = sum_j g[t, j] * f_{S[t, j]}(x[t]) + f_shared(x[t])
    (sglang-jax issue #1367, "Model configuration" MoE bullet and "Key
    difficulties" item 1).  The routed experts are evaluated per expert on the
    rows routed to it (the grouped form); ``moe_forward_dense_masked`` is the
    brute-force form of the same sum.

    ``w_gate``/``w_up``/``w_down`` may be arrays [E, H, I] / [E, I, H] or any
    object whose ``[e]`` returns expert e's matrix (for lazy fetching of large
    weight sets).  ``forced_idx`` replaces the selection (used to re-evaluate a
    near-tied token with another valid selection).
    """
    x64 = _f64(x)
    T, H = x64.shape
    E = np.asarray(router_w).shape[1]
    logits, _, beta32, idx, w = _route(x64, router_w, router_bias, top_k, scale,
                                       norm, use_bias, forced_idx)
    counts, offsets, perm, pos = expert_permutation(idx, E)
    out = swiglu_expert(x64, sh_gate, sh_up, sh_down, swiglu_limit_shared)
    for e in range(E):
        if counts[e] == 0:
            continue
        pairs = perm[offsets[e]:offsets[e + 1]]
        toks = pairs // top_k
        slots = pairs % top_k
        y = swiglu_expert(x64[toks], w_gate[e], w_up[e], w_down[e], swiglu_limit)
        out[toks] += w[toks, slots][:, None] * y
    return OracleResult(out=out, topk_idx=idx, topk_w=w, counts=counts,
                        offsets=offsets, perm=perm, pos=pos, logits=logits,
                        beta32=beta32, tie_gap=near_tie_gaps(beta32, top_k))


def moe_forward_rows(rows: Sequence[int], x, router_w, router_bias, w_gate, w_up,
                     w_down, sh_gate, sh_up, sh_down, *, top_k: int,
                     scale: float = 3.0, norm: bool = True, use_bias: bool = True,
                     swiglu_limit: float = 0.0, swiglu_limit_shared: float = 0.0,
                     forced_idx: Optional[np.ndarray] = None) -> OracleResult:
    """The same forward evaluated only for the listed token rows.

    The layer is token-wise independent (each output row depends on its own
    input row only), so this equals the corresponding rows of
    :func:`moe_forward`; it lets large workloads be checked on a sample of
    rows.  The permutation fields describe the sampled sub-batch only.
    """
    rows = np.asarray(rows, dtype=np.int64)
    xs = _f64(np.asarray(x)[rows])
    fi = None if forced_idx is None else np.asarray(forced_idx).reshape(-1, top_k)
    return moe_forward(xs, router_w, router_bias, w_gate, w_up, w_down,
                       sh_gate, sh_up, sh_down, top_k=top_k, scale=scale,
                       norm=norm, use_bias=use_bias, swiglu_limit=swiglu_limit,
                       swiglu_limit_shared=swiglu_limit_shared, forced_idx=fi)


def moe_forward_dense_masked(x, router_w, router_bias, w_gate, w_up, w_down,
                             sh_gate, sh_up, sh_down, *, top_k: int,
                             scale: float = 3.0, norm: bool = True,
                             use_bias: bool = True, swiglu_limit: float = 0.0,
                             swiglu_limit_shared: float = 0.0) -> np.ndarray:
    """Brute-force form: every expert on every token, then a masked sum.

    out = M . Y + f_shared(x) with M[t, e] = g[t, j] if e = S[t, j] else 0
    and Y[e] = f_e(x).  This is the dense side of the "GMM == per-expert-loop"
    check planned in sglang-jax issue #1367, "Implementation strategy".
    Tiny shapes only.
    """
    x64 = _f64(x)
    T, H = x64.shape
    E = np.asarray(router_w).shape[1]
    _, _, _, idx, w = _route(x64, router_w, router_bias, top_k, scale, norm,
                             use_bias, None)
    M = np.zeros((T, E))
    for t in range(T):
        for j in range(top_k):
            M[t, idx[t, j]] = w[t, j]
    Y = np.stack([swiglu_expert(x64, w_gate[e], w_up[e], w_down[e], swiglu_limit)
                  for e in range(E)])                      # [E, T, H]
    out = np.einsum("te,eth->th", M, Y)
    return out + swiglu_expert(x64, sh_gate, sh_up, sh_down, swiglu_limit_shared)


def dense_mlp(x, w_gate, w_up, w_down, swiglu_limit: float = 0.0) -> np.ndarray:
    """The model's dense SwiGLU MLP (the first three decoder layers): the same
    expert function applied to every token, without routing.

    sglang-jax issue #1367, section "Model configuration", MLP bullet (the
    first 3 layers are dense, intermediate 11264; layers 3-44 are MoE);
    llm-atlas "Step-3.5-Flash", table "Raw config fields" (intermediate_size
    11264).  x [T, H]; w_gate, w_up [H, I]; w_down [I, H]; the clamp as in
    the experts (L <= 0: none).
    """
    return swiglu_expert(_f64(x), w_gate, w_up, w_down, swiglu_limit)


def decode_e4m3(codes) -> np.ndarray:
    """Values of FP8 E4M3 codes (the OCP "E4M3FN" encoding), in float64.

    Bit 7 is the sign, bits 6-3 the exponent e (bias 7), bits 2-0 the
    mantissa m: e = 0 gives the subnormals m * 2^-9; e = 1..15 gives
    (1 + m/8) * 2^(e-7), except e = 15, m = 7, which is NaN (there are no
    infinities; the largest finite magnitude is 448).  The pages list FP8
    official weights for the model (sglang-jax issue #1367, section "Model
    configuration", the "Official weights" bullet) without stating a format;
    E4M3FN with one power-of-two scale per output feature is the reading
    taken.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def dequantize_e4m3(codes, scale) -> np.ndarray:
    """Weights from FP8 E4M3 codes [..., K, N] (x @ W layout: N output
    features) and one scale per output feature [..., N]:
    w[..., k, n] = value(codes[..., k, n]) * scale[..., n]."""
    v = decode_e4m3(codes)
    return v * np.asarray(scale, dtype=np.float64)[..., None, :]


class DequantizedExperts:
    """``view[e]`` -> expert e's dequantized matrix (float64) from codes
    [E, K, N] and scales [E, N] (torch tensors or arrays; fetched per expert
    so large weight sets are walked one expert at a time)."""

    def __init__(self, codes, scales):
        self.codes = codes
        self.scales = scales

    def __getitem__(self, e: int) -> np.ndarray:
        return dequantize_e4m3(as_numpy(self.codes[e]), as_numpy(self.scales[e]))

    def __len__(self):
        return len(self.codes)


def as_numpy(t: Any) -> np.ndarray:
    """Exact host copy of a torch tensor (bf16 widened exactly to float32;
    integer codes kept as they are) or array."""
    if hasattr(t, "detach"):
        import torch  # local: the oracle itself needs only NumPy
        t = t.detach()
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.cpu().numpy()
    return np.asarray(t)

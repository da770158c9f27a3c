"""Comparison of the CUDA path with the CPU oracle (used by the GPU tests and
by the smoke check).

Bar (element by element):
* top-k indices bit-exact, except near-tied tokens: those whose oracle k-th
  and (k+1)-th fp32 selection scores differ by less than TIE_BAND, or two of
  whose selected experts do (several selections, or orders, are then
  correct).  Such a token's GPU selection must still be one of the correct
  ones: k distinct experts that differ from the oracle's only in experts whose
  oracle score lies within TIE_BAND of the oracle's k-th score, listed in
  descending oracle score (within TIE_BAND), with the weights the oracle
  gives that selection.  Those tokens are counted, and their outputs are
  re-checked against the oracle evaluated on the GPU's selection;
* ``strict=True`` (inputs built with exact ties, which both sides must break
  to the lower index) allows no exception at all;
* counts, offsets and the permutation bit-exact given the selection;
* gate weights within fp32 rounding (rtol 1e-5);
* router logits of the selected experts within LOGIT_TOL of the fp64 logits
  (fp32 accuracy); every logit within LOGIT_TOL_APPROX (after the tensor-core
  router, experts that cannot be selected keep its approximate logit, whose
  error must stay well inside the top-k guard band);
* outputs: relative Frobenius error <= 1e-2 and max |error| <= 5e-2 * RMS(out).

Layers with fp32 expert weights take the fp32 expert path (tf32 tensor cores
over the two-term split of every operand) and meet a bar a hundred times
tighter, derived from its arithmetic:
* a product w x carries at most ~1.5 * 2^-21 relative error (the lo terms
  are read as tf32, 2^-10 of values below 2^-11 |w|, |x|; w_lo x_lo dropped);
* the tensor cores' fp32 accumulation loses at most one ulp of the partial
  sum per MMA k-step (3K/8 steps: 192 for K = 512), <= 2.3e-5 of the largest
  partial sum, and the SwiGLU, the gate weight and the fp32 combine add
  fp32 roundings;
so relative Frobenius error <= REL_FRO_F32 = 1e-4 and max |error| <=
MAX_ABS_OVER_RMS_F32 = 1e-3 * RMS(out) (the bf16 path measures ~5e-3 and
fails it).  The truncation term is linear in the step count, so the bar
grows with the longest accumulation of the layer (fp32_bar_scale: x8 at
H = 4096, 1536 steps); tests/test_fp32_bar.py checks the bar against an
emulation of this arithmetic with an accumulator that truncates every step
(the tiny fp32 layer: 8e-6 there, 6e-6 measured on the GPU).  A bf16 output (bf16 x) is the fp32 result rounded once more, by at
most 2^-8 of its magnitude: there the error beyond 2^-8 |out| must meet the
same max bar (with its own 2^-8 share), and the relative Frobenius error stays
under 2^-8 + REL_FRO_F32.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

import oracle.moe_oracle as om

TIE_BAND = 1e-6
REL_FRO = 1e-2
MAX_ABS_OVER_RMS = 5e-2
REL_FRO_F32 = 1e-4
MAX_ABS_OVER_RMS_F32 = 1e-3
BF16_U = 2.0 ** -8      # unit roundoff of bf16 (8 significant bits)


def fp32_bar_scale(hidden: int, intermediate: int) -> float:
    """Factor on the fp32 bar for a layer: its longest accumulation
    (3 K / 8 MMA steps, K = H for gate|up, I rounded up to 128 for down)
    over the 192 steps of K = 512 the base bar is derived for."""
    i_pad = -(-intermediate // 128) * 128
    return max(1.0, 3 * max(hidden, i_pad) / 8 / 192)
W_RTOL = 1e-5
LOGIT_TOL = 1e-5
LOGIT_TOL_APPROX = 4e-4


@dataclass
class ParityReport:
    tokens: int
    near_ties: int
    idx_mismatch_rows: int
    rel_fro: float
    max_abs_over_rms: float
    rows_checked: int
    logit_max_err: float = 0.0
    excess_bf16_over_rms: float = 0.0   # max(|error| - 2^-8 |out|) / RMS(out)

    def ok(self) -> bool:
        return self.rel_fro <= REL_FRO and self.max_abs_over_rms <= MAX_ABS_OVER_RMS

    def ok_fp32(self, out_bf16: bool = False, scale: float = 1.0) -> bool:
        """The fp32 expert path's bar (module docstring) times `scale`
        (fp32_bar_scale); out_bf16: the output dtype is bf16, so its own
        rounding is set apart."""
        rel, mx = REL_FRO_F32 * scale, MAX_ABS_OVER_RMS_F32 * scale
        if out_bf16:
            return (self.rel_fro <= BF16_U + rel and
                    self.excess_bf16_over_rms <= mx * (1 + BF16_U))
        return self.rel_fro <= rel and self.max_abs_over_rms <= mx


def order_gaps(beta32: np.ndarray, top_k: int) -> np.ndarray:
    """Per token, the smallest gap between neighbours among the k + 1 largest
    fp32 selection scores.  Below TIE_BAND the token is near-tied: either the
    k-th and (k+1)-th (which expert is selected) or two selected experts
    (their order) are within fp32 rounding of each other, so a GPU whose fp32
    logits differ from the correctly rounded ones in the last bits may
    legitimately decide the other way."""
    b = -np.sort(-np.asarray(beta32, dtype=np.float64), axis=1)
    n = min(top_k + 1, b.shape[1])
    if n < 2:
        return np.full(b.shape[0], np.inf)
    return (b[:, :n - 1] - b[:, 1:n]).min(axis=1)


def check_tied_row(gidx_row, ref: dict, t: int, top_k: int, E: int):
    """A near-tied token whose GPU selection differs from the oracle's: assert
    it is another correct selection (see the module docstring)."""
    beta = ref["beta32"][t].astype(np.float64)
    oidx = ref["topk_idx"][t]
    kth = beta[oidx[top_k - 1]]
    g = [int(e) for e in gidx_row]
    assert all(0 <= e < E for e in g), f"token {t}: expert id out of range {g}"
    assert len(set(g)) == top_k, f"token {t}: repeated expert {g}"
    added = set(g) - set(int(e) for e in oidx)
    dropped = set(int(e) for e in oidx) - set(g)
    for e in added:
        assert beta[e] >= kth - TIE_BAND, \
            f"token {t}: expert {e} (score {beta[e]!r}) is below the k-th score {kth!r}"
    for e in dropped:
        assert beta[e] <= kth + TIE_BAND, \
            f"token {t}: dropped expert {e} (score {beta[e]!r}) is above the k-th {kth!r}"
    for j in range(top_k - 1):
        a, b = beta[g[j]], beta[g[j + 1]]
        assert a >= b - TIE_BAND, f"token {t}: order not descending at slot {j}: {g}"


def check_selection(gidx: np.ndarray, gw: np.ndarray, ref: dict, top_k: int, E: int,
                    scale: float = 3.0, strict: bool = False):
    """Top-k indices and gate weights against the oracle's routing ``ref``.
    Returns (mismatched-row mask, near-tie mask)."""
    tie = order_gaps(ref["beta32"], top_k) < TIE_BAND
    mism = (gidx != ref["topk_idx"]).any(axis=1)
    if strict:
        bad = np.nonzero(mism)[0]
        assert bad.size == 0, f"top-k differs on {bad.size} exactly-tied tokens, first {bad[:8]}"
    bad = np.nonzero(mism & ~tie)[0]
    assert bad.size == 0, f"top-k differs on {bad.size} non-tied tokens, first {bad[:8]}"
    for t in np.nonzero(mism)[0]:
        check_tied_row(gidx[t], ref, int(t), top_k, E)
    # weights: the bias-free scores of the selection, renormalised, scaled --
    # the oracle's own for matching rows, the oracle's for the GPU's selection
    # on the others
    ok = ~mism
    np.testing.assert_allclose(gw[ok], ref["topk_w"][ok], rtol=W_RTOL, atol=1e-7)
    if mism.any():
        s_sel = np.take_along_axis(ref["s32"][mism], gidx[mism].astype(np.int64), axis=1)
        want = om.gate_weights(s_sel, scale, True)
        np.testing.assert_allclose(gw[mism], want, rtol=W_RTOL, atol=1e-7)
    return mism, tie


def check_routing(gpu_rt: dict, ref: dict, top_k: int, E: int, wl=None, strict: bool = False):
    """Selection, weights and grouping.  Returns (mismatched-row mask, near-tie mask)."""
    gidx = gpu_rt["topk_idx"]
    mism, tie = check_selection(gidx, gpu_rt["topk_w"], ref, top_k, E,
                                scale=3.0 if wl is None else wl.scale, strict=strict)
    # grouping: the permutation of the GPU's own selection is unique
    counts, offsets, perm, _ = om.expert_permutation(gidx, E)
    assert np.array_equal(gpu_rt["counts"], counts)
    assert np.array_equal(gpu_rt["offsets"], offsets)
    assert np.array_equal(gpu_rt["perm"], perm)
    if not mism.any():
        assert np.array_equal(gpu_rt["perm"], ref["perm"])
        assert np.array_equal(gpu_rt["counts"], ref["counts"])
    return mism, tie


def output_errors(gpu_out: np.ndarray, ref_out: np.ndarray):
    """(relative Frobenius error, max |error| / RMS, max(|error| - 2^-8
    |ref|) / RMS)."""
    d = gpu_out.astype(np.float64) - ref_out
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref_out), 1e-300))
    rms = float(np.sqrt(np.mean(ref_out ** 2)))
    mx = float(np.max(np.abs(d)) / max(rms, 1e-300))
    ex = float(np.max(np.abs(d) - BF16_U * np.abs(ref_out)) / max(rms, 1e-300))
    return rel, mx, ex


def expert_views(inp: dict) -> dict:
    """Lazy per-expert float views of a workload's expert weights (bf16 / fp32
    tensors widened exactly, FP8 codes dequantized by the oracle), for the
    ``experts`` argument of :func:`compare`."""
    if "s_w_gate" in inp:
        return dict(w_gate=om.DequantizedExperts(inp["w_gate"], inp["s_w_gate"]),
                    w_up=om.DequantizedExperts(inp["w_up"], inp["s_w_up"]),
                    w_down=om.DequantizedExperts(inp["w_down"], inp["s_w_down"]),
                    sh_gate=om.dequantize_e4m3(om.as_numpy(inp["sh_gate"]),
                                               om.as_numpy(inp["s_sh_gate"])),
                    sh_up=om.dequantize_e4m3(om.as_numpy(inp["sh_up"]),
                                             om.as_numpy(inp["s_sh_up"])),
                    sh_down=om.dequantize_e4m3(om.as_numpy(inp["sh_down"]),
                                               om.as_numpy(inp["s_sh_down"])))
    return dict(w_gate=_Widened(inp["w_gate"]), w_up=_Widened(inp["w_up"]),
                w_down=_Widened(inp["w_down"]), sh_gate=om.as_numpy(inp["sh_gate"]),
                sh_up=om.as_numpy(inp["sh_up"]), sh_down=om.as_numpy(inp["sh_down"]))


class _Widened:
    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return om.as_numpy(self.t[e])

    def __len__(self):
        return len(self.t)


def compare(inp_host: dict, wl, gpu_out: np.ndarray, gpu_rt: dict,
            rows: Optional[np.ndarray] = None, experts=None,
            strict: bool = False) -> ParityReport:
    """inp_host: exact fp32 host copies of x, router_w, router_bias (and, when
    ``experts`` is None, of all weights); ``experts`` may supply lazy
    per-expert views (w_gate, w_up, w_down, sh_gate, sh_up, sh_down)."""
    k, E = wl.top_k, wl.num_experts
    x = inp_host["x"]
    ref = om.moe_routing(x, inp_host["router_w"], inp_host["router_bias"], top_k=k,
                         scale=wl.scale)
    mism, tie = check_routing(gpu_rt, ref, k, E, wl=wl, strict=strict)
    logit_err = 0.0
    if "logits" in gpu_rt:
        d = np.abs(gpu_rt["logits"].astype(np.float64) - ref["logits"])
        sel = np.take_along_axis(d, gpu_rt["topk_idx"].astype(np.int64), axis=1)
        logit_err = float(sel.max())
        assert logit_err <= LOGIT_TOL, f"selected router logits off by {logit_err}"
        assert float(d.max()) <= LOGIT_TOL_APPROX, f"router logits off by {float(d.max())}"
    T = x.shape[0]
    if rows is None:
        rows = np.arange(T)
    rows = np.unique(np.concatenate([np.asarray(rows, np.int64), np.nonzero(mism)[0]]))
    w = experts if experts is not None else inp_host
    res = om.moe_forward_rows(rows, x, inp_host["router_w"], inp_host["router_bias"],
                              w["w_gate"], w["w_up"], w["w_down"], w["sh_gate"], w["sh_up"],
                              w["sh_down"], top_k=k, scale=wl.scale,
                              swiglu_limit=wl.swiglu_limit,
                              swiglu_limit_shared=wl.swiglu_limit_shared,
                              forced_idx=gpu_rt["topk_idx"][rows])
    rel, mx, ex = output_errors(gpu_out[rows], res.out)
    return ParityReport(tokens=T, near_ties=int(tie.sum()), idx_mismatch_rows=int(mism.sum()),
                        rel_fro=rel, max_abs_over_rms=mx, rows_checked=int(rows.size),
                        logit_max_err=logit_err, excess_bf16_over_rms=ex)

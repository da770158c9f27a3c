"""The fp32 expert path's parity bar against an emulation of its arithmetic.

tests/parity.py holds fp32-weight layers to relative Frobenius error 1e-4
and max error 1e-3 x RMS times fp32_bar_scale (the longest accumulation over
192 MMA steps), a bar derived from the two-term tf32 split rather than
fitted to GPU results.  This test checks the derivation on the CPU: it
evaluates the layer with every expert GEMM done the way the fp32 path does
it, with the worst-case accumulator, and asserts the result stays inside a
quarter of the bar.  (On the tiny fp32 layer the emulation gives 8.4e-6
relative Frobenius error, the GPU 6.4e-6; an accumulator that rounded to
nearest would give 0.4e-6, so the tensor cores' accumulation behaves like
the truncating model, whose error grows linearly with the step count.)

The emulated arithmetic, written here from its description (not from the
kernels' code):
* every operand value v -> v_hi = v rounded to tf32 (11 significant bits,
  nearest, ties to even) and v_lo = v - v_hi, which the tensor cores read as
  tf32 (modelled as truncation, the worse case);
* a product w . x -> the K-concatenated terms w_hi x_hi, w_lo x_hi, w_hi x_lo,
  in that order, eight K elements per MMA step summed exactly and added to an
  fp32 accumulator that truncates (the worst case the derivation allows);
* h and y stay fp32; the k + 1 rows of a token are summed in fp32 in the
  order j = 0..k-1, then the shared row.
The routing is the oracle's.
"""
from dataclasses import replace

import numpy as np

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, host_f32, make_inputs
from tests.parity import MAX_ABS_OVER_RMS_F32, REL_FRO_F32, fp32_bar_scale, output_errors

MMA_K = 8  # K elements per tf32 MMA step


def _to_tf32(v: np.ndarray, mode: str) -> np.ndarray:
    """v (fp32 values) with an 11-bit significand: 'nearest' (ties to even)
    or 'trunc' (toward zero); exact in fp64."""
    m, e = np.frexp(np.asarray(v, np.float64))  # v = m 2^e, 0.5 <= |m| < 1
    s = m * 2.0 ** 11
    s = np.rint(s) if mode == "nearest" else np.trunc(s)
    return np.ldexp(s, e - 11)


def _split(v: np.ndarray):
    v = np.asarray(v, np.float32).astype(np.float64)
    hi = _to_tf32(v, "nearest")
    lo = (v - hi).astype(np.float32).astype(np.float64)  # exact in fp32
    return hi, _to_tf32(lo, "trunc")


def _f32_trunc(v: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 toward zero."""
    r = v.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(v)
    r[over] = np.nextafter(r[over], np.float32(0))
    return r


def _gemm(rows: np.ndarray, w: np.ndarray) -> np.ndarray:
    """rows [n, K] . w [K, m] the fp32-path way: fp32 result [n, m]."""
    xh, xl = _split(rows)
    wh, wl = _split(w)
    K = rows.shape[1]
    acc = np.zeros((rows.shape[0], w.shape[1]), np.float32)
    for a, b in ((xh, wh), (xh, wl), (xl, wh)):  # terms hi.hi, lo.hi, hi.lo
        for k0 in range(0, K, MMA_K):
            step = a[:, k0:k0 + MMA_K] @ b[k0:k0 + MMA_K, :]
            acc = _f32_trunc(acc.astype(np.float64) + step)
    return acc


def _expert(rows, wg, wu, wd, limit):
    a = _gemm(rows, wg)
    u = _gemm(rows, wu)
    if limit > 0:
        a = np.minimum(a, np.float32(limit))
        u = np.clip(u, np.float32(-limit), np.float32(limit))
    h = (a / (np.float32(1) + np.exp(-a)) * u).astype(np.float32)
    return _gemm(h, wd)


def _emulated_layer(wl, inp):
    x = inp["x"]
    rt = om.moe_routing(x, inp["router_w"], inp["router_bias"], top_k=wl.top_k,
                        scale=wl.scale)
    idx, gw = rt["topk_idx"], rt["topk_w"].astype(np.float32)
    T, k = idx.shape
    y = np.zeros((T, k, wl.hidden), np.float32)
    for e in np.unique(idx):
        t, j = np.nonzero(idx == e)
        y[t, j] = _expert(x[t], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e],
                          wl.swiglu_limit) * gw[t, j][:, None]
    ysh = _expert(x, inp["sh_gate"], inp["sh_up"], inp["sh_down"], wl.swiglu_limit_shared)
    out = np.zeros((T, wl.hidden), np.float32)
    for j in range(k):
        out = out + y[:, j]
    return out + ysh


def _check(wl):
    inp = {kk: host_f32(v) for kk, v in make_inputs(wl, "cpu").items()}
    ref = om.moe_forward(inp["x"], inp["router_w"], inp["router_bias"], inp["w_gate"],
                         inp["w_up"], inp["w_down"], inp["sh_gate"], inp["sh_up"],
                         inp["sh_down"], top_k=wl.top_k, scale=wl.scale,
                         swiglu_limit=wl.swiglu_limit,
                         swiglu_limit_shared=wl.swiglu_limit_shared).out
    rel, mx, _ = output_errors(_emulated_layer(wl, inp), ref)
    sc = fp32_bar_scale(wl.hidden, wl.intermediate) / 4  # a quarter of the bar
    assert rel <= REL_FRO_F32 * sc and mx <= MAX_ABS_OVER_RMS_F32 * sc, (rel, mx)
    return rel, mx


def test_bar_holds_for_the_tiny_fp32_layer():
    _check(WORKLOADS["tiny"])


def test_bar_holds_at_the_full_hidden_size():
    # H = 4096: 1536 MMA steps per gate|up product, the longest accumulation
    # (emulated: 1.2e-4 relative Frobenius error against a bar of 8e-4)
    _check(replace(WORKLOADS["tiny"], name="bk", T=12, hidden=4096, num_experts=4, top_k=2,
                   intermediate=64, shared_intermediate=64, x_dist="rmsnorm_normal",
                   expert_std=0.02))


def test_the_emulation_sees_a_bf16_sized_error(monkeypatch):
    """Guard against an emulation too exact to test anything: rounding the
    operands to bf16 instead of splitting them must break the bar."""
    import sys

    def bf16_only(v):
        v = np.asarray(v, np.float32).astype(np.float64)
        m, e = np.frexp(v)
        return np.ldexp(np.rint(m * 2.0 ** 8), e - 8), np.zeros_like(v)

    monkeypatch.setattr(sys.modules[__name__], "_split", bf16_only)
    wl = WORKLOADS["tiny"]
    inp = {kk: host_f32(v) for kk, v in make_inputs(wl, "cpu").items()}
    ref = om.moe_forward(inp["x"], inp["router_w"], inp["router_bias"], inp["w_gate"],
                         inp["w_up"], inp["w_down"], inp["sh_gate"], inp["sh_up"],
                         inp["sh_down"], top_k=wl.top_k, scale=wl.scale).out
    rel, _, _ = output_errors(_emulated_layer(wl, inp), ref)
    assert rel > REL_FRO_F32, rel

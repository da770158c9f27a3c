"""Pins of the CPU oracle against what the pages and the mathematics fix.

The pages print no worked numeric example, so the oracle is pinned by
brute force on tiny shapes, closed forms, invariants stated by the pages and
special cases that reduce to textbook routines computed here with torch
float64 operations.  The mutation tests at the end plant plausible mistakes in
the oracle (on the CPU) and check that some pin fails.
"""
import os
from dataclasses import replace

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(d):
    return {k: v.float().numpy() if hasattr(v, "numpy") else v for k, v in d.items()}


def _tiny(**kw):
    wl = WORKLOADS["tiny"]
    if kw:
        from dataclasses import replace
        wl = replace(wl, **kw)
    return wl, _np(make_inputs(wl, "cpu"))


def _fwd(inp, wl, **kw):
    args = dict(top_k=wl.top_k, scale=wl.scale, swiglu_limit=wl.swiglu_limit,
                swiglu_limit_shared=wl.swiglu_limit_shared)
    args.update(kw)
    return om.moe_forward(inp["x"], inp["router_w"], inp["router_bias"],
                          inp["w_gate"], inp["w_up"], inp["w_down"],
                          inp["sh_gate"], inp["sh_up"], inp["sh_down"], **args)


def _torch_mlp(x, wg, wu, wd, limit=0.0):
    """Textbook SwiGLU MLP with torch float64 ops (independent of the oracle)."""
    x = torch.as_tensor(np.asarray(x, np.float64))
    a = x @ torch.as_tensor(np.asarray(wg, np.float64))
    u = x @ torch.as_tensor(np.asarray(wu, np.float64))
    if limit > 0:
        a = torch.clamp(a, max=limit)
        u = torch.clamp(u, min=-limit, max=limit)
    return (F.silu(a) * u) @ torch.as_tensor(np.asarray(wd, np.float64))


# --------------------------------------------------------------------------
# pins (plain functions, so the mutation tests can re-run them)
# --------------------------------------------------------------------------

def pin_topk_brute_force():
    rng = np.random.default_rng(1)
    beta = rng.standard_normal((64, 16)).astype(np.float32)
    beta[:, 5] = beta[:, 3]             # exact ties: the lower index must win
    beta[:8, :] = 0.25                  # rows of all-equal scores
    a = om.select_topk(beta, 4)
    b = om.select_topk_by_rounds(beta, 4)
    assert np.array_equal(a, b)
    assert np.array_equal(a[0], [0, 1, 2, 3])
    # hand-worked row: scores 0.5, 0.9, 0.9, 0.1, 0.7 -> 1, 2 (tie, lower first), 4
    hand = np.array([[0.5, 0.9, 0.9, 0.1, 0.7]], np.float32)
    assert np.array_equal(om.select_topk(hand, 3)[0], [1, 2, 4])


def pin_weights_sum_to_scale():
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    assert np.allclose(r.topk_w.sum(axis=1), 3.0, rtol=0, atol=1e-12)
    assert (r.topk_w > 0).all()


def pin_bias_selects_only():
    """The bias changes which experts are selected, never the weights of a
    fixed selection (sglang-jax issue #1367, "Key difficulties" item 1)."""
    wl, inp = _tiny()
    base = _fwd(inp, wl)
    # (i) a uniform shift of the bias keeps the selection -> identical results
    inp2 = dict(inp, router_bias=inp["router_bias"] + np.float32(0.125))
    shifted = _fwd(inp2, wl)
    assert np.array_equal(base.topk_idx, shifted.topk_idx)
    assert np.array_equal(base.topk_w, shifted.topk_w)
    assert np.array_equal(base.out, shifted.out)
    # (ii) force a selection with a large bias, vary the rest: weights unchanged
    E, k = wl.num_experts, wl.top_k
    chosen = np.array([3, 7, 11, 14])
    rng = np.random.default_rng(7)
    ws = []
    for trial in range(3):
        b = rng.standard_normal(E).astype(np.float32) * 0.1
        b[chosen] = 10.0 + np.arange(k, dtype=np.float32)  # fixes order too
        r = _fwd(dict(inp, router_bias=b), wl)
        assert (np.sort(r.topk_idx, axis=1) == np.sort(chosen)).all()
        ws.append(r.topk_w)
    assert np.array_equal(ws[0], ws[1]) and np.array_equal(ws[1], ws[2])
    # and the weights are 3 * s / sum(s) of the chosen experts' bias-free scores
    s = 1.0 / (1.0 + np.exp(-(inp["x"].astype(np.float64) @ inp["router_w"].astype(np.float64))))
    sel = np.take_along_axis(s, r.topk_idx.astype(np.int64), axis=1)
    assert np.allclose(r.topk_w, 3.0 * sel / sel.sum(1, keepdims=True), rtol=1e-6)
    # (iii) a bias that changes the selection changes the output
    b = inp["router_bias"].copy()
    b[base.topk_idx[0, 0]] = -10.0
    other = _fwd(dict(inp, router_bias=b), wl)
    assert not np.array_equal(other.topk_idx[0], base.topk_idx[0])
    assert not np.allclose(other.out[0], base.out[0])


def pin_closed_form_identical_experts():
    """All routed experts equal f: out = 3 f(x) + shared(x) for any routing."""
    wl, inp = _tiny()
    E = wl.num_experts
    wg = np.broadcast_to(inp["w_gate"][2], inp["w_gate"].shape).copy()
    wu = np.broadcast_to(inp["w_up"][2], inp["w_up"].shape).copy()
    wd = np.broadcast_to(inp["w_down"][2], inp["w_down"].shape).copy()
    r = _fwd(dict(inp, w_gate=wg, w_up=wu, w_down=wd), wl)
    f = _torch_mlp(inp["x"], wg[0], wu[0], wd[0]).numpy()
    sh = _torch_mlp(inp["x"], inp["sh_gate"], inp["sh_up"], inp["sh_down"]).numpy()
    assert np.allclose(r.out, 3.0 * f + sh, rtol=1e-10, atol=1e-12)


def pin_single_expert_is_dense_mlp():
    """E = 1, k = 1: the layer is a dense SwiGLU MLP times 3 plus the shared one."""
    rng = np.random.default_rng(3)
    T, H, I = 9, 32, 24
    x = rng.standard_normal((T, H))
    rw = rng.standard_normal((H, 1)) * 0.1
    rb = np.array([0.3], np.float32)
    wg, wu = rng.standard_normal((1, H, I)) * 0.2, rng.standard_normal((1, H, I)) * 0.2
    wd = rng.standard_normal((1, I, H)) * 0.2
    sg, su, sd = (rng.standard_normal((H, I)) * 0.2, rng.standard_normal((H, I)) * 0.2,
                  rng.standard_normal((I, H)) * 0.2)
    r = om.moe_forward(x, rw, rb, wg, wu, wd, sg, su, sd, top_k=1)
    want = 3.0 * _torch_mlp(x, wg[0], wu[0], wd[0]) + _torch_mlp(x, sg, su, sd)
    assert np.allclose(r.out, want.numpy(), rtol=1e-10, atol=1e-12)


def pin_all_experts_mixture():
    """k = E, zero bias: a dense mixture with weights 3 s_e / sum_e s_e."""
    rng = np.random.default_rng(4)
    T, H, I, E = 7, 16, 8, 5
    x = rng.standard_normal((T, H))
    rw = rng.standard_normal((H, E)) * 0.3
    wg, wu = rng.standard_normal((E, H, I)) * 0.3, rng.standard_normal((E, H, I)) * 0.3
    wd = rng.standard_normal((E, I, H)) * 0.3
    sg, su, sd = wg[0] * 0.5, wu[1] * 0.5, wd[2] * 0.5
    r = om.moe_forward(x, rw, np.zeros(E, np.float32), wg, wu, wd, sg, su, sd, top_k=E)
    s = torch.sigmoid(torch.as_tensor(x) @ torch.as_tensor(rw))
    g = 3.0 * s / s.sum(1, keepdim=True)
    want = sum(g[:, e:e + 1] * _torch_mlp(x, wg[e], wu[e], wd[e]) for e in range(E))
    want = want + _torch_mlp(x, sg, su, sd)
    # weights use the fp32-rounded sigmoid scores: relative error ~1e-7
    assert np.allclose(r.out, want.numpy(), rtol=1e-6, atol=1e-7)


def pin_grouped_equals_dense_masked():
    """The grouped (per-expert) evaluation equals the brute-force masked sum
    ("GMM == per-expert-loop", sglang-jax issue #1367, "Implementation strategy")."""
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    dense = om.moe_forward_dense_masked(
        inp["x"], inp["router_w"], inp["router_bias"], inp["w_gate"], inp["w_up"],
        inp["w_down"], inp["sh_gate"], inp["sh_up"], inp["sh_down"], top_k=wl.top_k)
    assert np.allclose(r.out, dense, rtol=1e-12, atol=1e-13)


def pin_row_independence():
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    for t in (0, 5, 31):
        one = _fwd(dict(inp, x=inp["x"][t:t + 1]), wl)
        assert np.array_equal(one.topk_idx[0], r.topk_idx[t])
        assert np.allclose(one.out[0], r.out[t], rtol=1e-13, atol=1e-14)
    p = np.random.default_rng(5).permutation(wl.T)
    rp = _fwd(dict(inp, x=inp["x"][p]), wl)
    assert np.allclose(rp.out, r.out[p], rtol=1e-13, atol=1e-14)
    assert np.array_equal(rp.counts, r.counts)


def pin_permutation():
    """perm is the stable sort of the pair ids by expert; a library stable sort
    gives the same permutation."""
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    T, k, E = wl.T, wl.top_k, wl.num_experts
    flat = r.topk_idx.reshape(-1)
    assert np.array_equal(r.perm, np.argsort(flat, kind="stable"))
    assert np.array_equal(r.counts, np.bincount(flat, minlength=E))
    assert r.offsets[0] == 0 and r.offsets[-1] == T * k
    assert (np.diff(r.offsets) >= 0).all()
    assert np.array_equal(np.sort(r.perm), np.arange(T * k))
    inv = np.empty(T * k, np.int64)
    inv[r.perm] = np.arange(T * k)
    assert np.array_equal(inv.reshape(T, k), r.pos)
    for e in range(E):
        seg = r.perm[r.offsets[e]:r.offsets[e + 1]]
        assert (flat[seg] == e).all()
        assert (np.diff(seg // k) > 0).all()


def pin_clamp_branches():
    """Crafted single-expert layer whose pre-activations are known exactly:
    every branch of the clamp (gate above / below L, up above L, below -L, inside)."""
    H = I = 6
    L, Ls = 2.0, 5.0
    a_vals = np.array([3.0, 1.5, -4.0, 2.0, 10.0, 0.5])   # gate pre-activations
    u_vals = np.array([-7.0, 0.75, 3.0, -1.0, 2.5, 6.0])  # up pre-activations
    x = np.ones((1, H))
    wg = np.diag(a_vals)[None]
    wu = np.diag(u_vals)[None]
    wd = np.eye(I)[None]
    zero = np.zeros((H, I))
    r = om.moe_forward(x, np.zeros((H, 1)), None, wg, wu, wd, zero, zero, np.zeros((I, H)),
                       top_k=1, use_bias=False, swiglu_limit=L)
    gate = np.array([2.0, 1.5, -4.0, 2.0, 2.0, 0.5])
    up = np.array([-2.0, 0.75, 2.0, -1.0, 2.0, 2.0])
    h = gate / (1.0 + np.exp(-gate)) * up
    assert np.allclose(r.out[0], 3.0 * h, rtol=1e-14, atol=0)
    # the shared expert takes its own limit
    r2 = om.moe_forward(x, np.zeros((H, 1)), None, wg * 0, wu * 0, wd * 0,
                        wg[0], wu[0], wd[0], top_k=1, use_bias=False,
                        swiglu_limit=L, swiglu_limit_shared=Ls)
    gate_s = np.minimum(a_vals, Ls)
    up_s = np.clip(u_vals, -Ls, Ls)
    assert np.allclose(r2.out[0], gate_s / (1.0 + np.exp(-gate_s)) * up_s, rtol=1e-14)


def pin_clamp_off():
    wl, inp = _tiny()
    a = _fwd(inp, wl, swiglu_limit=0.0, swiglu_limit_shared=0.0)
    b = _fwd(inp, wl, swiglu_limit=1e30, swiglu_limit_shared=1e30)
    assert np.array_equal(a.out, b.out)
    c = _fwd(inp, wl, swiglu_limit=0.05, swiglu_limit_shared=0.0)
    assert not np.allclose(a.out, c.out)


def pin_routing_fields():
    """moe_routing (the routing half alone, which the GPU checks compare with)
    equals moe_forward's routing fields field by field, and its score arrays
    equal an independent torch recomputation: the fp64 logits rounded once to
    fp32, the fp32 rounding of the float64 sigmoid, plus the bias in fp32;
    tie_gap is the gap between the k-th and (k+1)-th of a full sort."""
    for kw in ({}, dict(swiglu_limit=0.3, swiglu_limit_shared=0.5, T=48, top_k=3)):
        wl, inp = _tiny(**kw)
        f = _fwd(inp, wl)
        r = om.moe_routing(inp["x"], inp["router_w"], inp["router_bias"], top_k=wl.top_k,
                           scale=wl.scale)
        for name in ("topk_idx", "topk_w", "counts", "offsets", "perm", "pos", "beta32",
                     "tie_gap", "logits"):
            assert np.array_equal(np.asarray(r[name]), np.asarray(getattr(f, name))), name
        lt = (torch.as_tensor(inp["x"], dtype=torch.float64)
              @ torch.as_tensor(inp["router_w"], dtype=torch.float64))
        s = torch.sigmoid(lt.float().double()).float()
        beta = s + torch.as_tensor(inp["router_bias"], dtype=torch.float32)
        assert np.array_equal(r["s32"], s.numpy())
        assert np.array_equal(r["beta32"], beta.numpy())
        srt = torch.sort(beta.double(), dim=1, descending=True).values
        gap = (srt[:, wl.top_k - 1] - srt[:, wl.top_k]).numpy()
        assert np.array_equal(r["tie_gap"], gap)
        T, k = wl.T, wl.top_k
        assert np.array_equal(r["perm"][r["pos"].reshape(-1)], np.arange(T * k))
        sel = torch.as_tensor(r["topk_idx"].astype(np.int64))
        ssel = torch.gather(s.double(), 1, sel)
        assert np.allclose(r["topk_w"], (3.0 * ssel / ssel.sum(1, keepdim=True)).numpy(),
                           rtol=1e-15, atol=0)


PINS = [pin_topk_brute_force, pin_weights_sum_to_scale, pin_bias_selects_only,
        pin_closed_form_identical_experts, pin_single_expert_is_dense_mlp,
        pin_all_experts_mixture, pin_grouped_equals_dense_masked,
        pin_row_independence, pin_permutation, pin_clamp_branches, pin_clamp_off,
        pin_routing_fields]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# --------------------------------------------------------------------------
# readings of the pages (documented, not pinned by a printed value)
# --------------------------------------------------------------------------

def test_bias_added_to_scores_not_logits():
    """Reading: the selection score is sigmoid(l) + b.  With logits (0, 4) and
    bias (0.6, 0): scores+bias = (1.1, 0.982) picks expert 0; logits+bias would
    give sigmoid(0.6) < sigmoid(4) and pick expert 1."""
    l = np.array([[0.0, 4.0]])
    s32, beta = om.selection_scores_fp32(l, np.array([0.6, 0.0], np.float32))
    assert om.select_topk(beta, 1)[0, 0] == 0


def test_selection_decided_in_fp32():
    """Two scores that differ in fp64 but round to the same fp32 value tie, and
    the tie goes to the lower index."""
    base = 0.3
    l = np.array([[base + 1e-12, base]])
    _, beta = om.selection_scores_fp32(l, np.zeros(2, np.float32))
    assert beta[0, 0] == beta[0, 1]
    assert om.select_topk(beta, 1)[0, 0] == 0


def test_near_tie_gap():
    beta = np.array([[0.9, 0.5, 0.5 - 1e-7, 0.1]], np.float32)
    gap = om.near_tie_gaps(beta, 2)
    assert 0 < gap[0] < 1e-6


def test_rows_variant_matches_full():
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    rows = [3, 17, 30]
    rr = om.moe_forward_rows(rows, inp["x"], inp["router_w"], inp["router_bias"],
                             inp["w_gate"], inp["w_up"], inp["w_down"], inp["sh_gate"],
                             inp["sh_up"], inp["sh_down"], top_k=wl.top_k)
    assert np.array_equal(rr.topk_idx, r.topk_idx[rows])
    assert np.allclose(rr.out, r.out[rows], rtol=1e-13, atol=1e-14)


def test_forced_selection():
    wl, inp = _tiny()
    r = _fwd(inp, wl)
    forced = r.topk_idx.copy()
    forced[:, [0, 1]] = forced[:, [1, 0]]              # same set, other order
    r2 = _fwd(inp, wl, forced_idx=forced)
    assert np.allclose(r2.out, r.out, rtol=1e-13, atol=1e-14)


# --------------------------------------------------------------------------
# the workloads and the config printed by the pages
# --------------------------------------------------------------------------

def _golden_config():
    vals = {}
    with open(os.path.join(GOLDEN, "step35_flash_moe_config.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split(None, 1)
                vals[k] = v
    return vals


def test_workloads_follow_page_config():
    g = _golden_config()
    for name in ("decode", "prefill", "zipf_prefill", "clamp_ragged"):
        wl = WORKLOADS[name]
        assert wl.hidden == int(g["hidden_size"])
        assert wl.num_experts == int(g["moe_num_experts"])
        assert wl.top_k == int(g["moe_top_k"])
        assert wl.intermediate == int(g["moe_intermediate_size"])
        assert wl.shared_intermediate == int(g["share_expert_dim"])
        assert wl.scale == float(g["moe_router_scaling_factor"])
    assert g["moe_router_activation"] == "sigmoid"
    assert g["norm_expert_weight"] == "true" and g["use_moe_router_bias"] == "true"
    # the clamped workload uses the non-zero routed limit printed by the page
    limits = g["swiglu_limits"].split("+")
    assert float(limits[1].split("x")[0]) == WORKLOADS["clamp_ragged"].swiglu_limit


def test_parameter_count_consistent_with_pages():
    """42 MoE layers x 289 experts x 3 matrices x 4096 x 1280 stays under the
    ~196B total the pages give; one expert is 31,457,280 bf16 bytes."""
    g = _golden_config()
    layers = int(g["moe_layers_last"]) - int(g["moe_layers_first"]) + 1
    assert layers == 42
    per_expert = 3 * 4096 * 1280
    assert per_expert * 2 == 31_457_280 == WORKLOADS["decode"].weight_bytes_per_expert
    moe_params = layers * 289 * per_expert
    assert 190e9 < moe_params <= float(g["total_params_billion"]) * 1e9
    # active: 9 experts per token per layer is below the ~11B active figure
    assert layers * 9 * per_expert < float(g["active_params_billion"]) * 1e9


def test_zipf_bias_values():
    from sparse_moe_layer_gemm_b200.workloads import draw_router
    _, b = draw_router(WORKLOADS["zipf_prefill"], "cpu")
    assert abs(float(b[0])) == 0.0
    assert abs(float(b[9]) - 0.5 * np.log(1.0 / 10 ** 1.1)) < 1e-6


def test_inputs_deterministic():
    a = make_inputs(WORKLOADS["tiny"], "cpu")
    b = make_inputs(WORKLOADS["tiny"], "cpu")
    for k in a:
        assert torch.equal(a[k], b[k])


# --------------------------------------------------------------------------
# planted mistakes: each must make some pin fail
# --------------------------------------------------------------------------

def _fails(pins):
    """True if some pin fails (an assertion, or a shape error for a
    transposed operand)."""
    for p in pins:
        try:
            p()
        except (AssertionError, ValueError):
            return True
    return False


def test_mutant_no_renorm(monkeypatch):
    monkeypatch.setattr(om, "gate_weights", lambda s, scale, norm: np.asarray(s, np.float64) * scale)
    assert _fails([pin_weights_sum_to_scale, pin_all_experts_mixture])


def test_mutant_weights_from_biased_scores(monkeypatch):
    orig = om.selection_scores_fp32

    def biased(logits, bias):
        s, beta = orig(logits, bias)
        return beta, beta
    monkeypatch.setattr(om, "selection_scores_fp32", biased)
    assert _fails([pin_bias_selects_only])


def test_mutant_missing_shared(monkeypatch):
    orig = om.swiglu_expert
    calls = {"n": 0}

    def no_shared(rows, wg, wu, wd, limit):
        calls["n"] += 1
        y = orig(rows, wg, wu, wd, limit)
        return y * 0 if calls["n"] == 1 else y
    monkeypatch.setattr(om, "swiglu_expert", no_shared)
    assert _fails([pin_closed_form_identical_experts])


def test_mutant_silu_sign(monkeypatch):
    monkeypatch.setattr(om, "_silu", lambda z: z / (1.0 + np.exp(z)))
    assert _fails([pin_closed_form_identical_experts, pin_clamp_branches])


def test_mutant_topk_ties_to_higher_index(monkeypatch):
    def bad(beta, k):
        beta = np.asarray(beta)
        E = beta.shape[1]
        return np.stack([np.lexsort((-np.arange(E), -beta[t].astype(np.float64)))[:k]
                         for t in range(beta.shape[0])]).astype(np.int32)
    monkeypatch.setattr(om, "select_topk", bad)
    assert _fails([pin_topk_brute_force])


def test_mutant_clamp_up_one_sided(monkeypatch):
    orig = om.swiglu_expert

    def one_sided(rows, wg, wu, wd, limit):
        rows = np.asarray(rows, np.float64)
        a = rows @ np.asarray(wg, np.float64)
        u = rows @ np.asarray(wu, np.float64)
        if limit and limit > 0:
            a = np.minimum(a, limit)
            u = np.minimum(u, limit)
        return (a / (1 + np.exp(-a)) * u) @ np.asarray(wd, np.float64)
    monkeypatch.setattr(om, "swiglu_expert", one_sided)
    assert _fails([pin_clamp_branches])


def test_mutant_perm_not_stable(monkeypatch):
    orig = om.expert_permutation

    def reversed_within(idx, E):
        counts, offsets, perm, pos = orig(idx, E)
        perm = perm.copy()
        for e in range(E):
            perm[offsets[e]:offsets[e + 1]] = perm[offsets[e]:offsets[e + 1]][::-1]
        return counts, offsets, perm, pos
    monkeypatch.setattr(om, "expert_permutation", reversed_within)
    assert _fails([pin_permutation])


def test_mutant_transposed_down(monkeypatch):
    orig = om.swiglu_expert
    monkeypatch.setattr(om, "swiglu_expert",
                        lambda rows, wg, wu, wd, limit: orig(rows, wg, wu, np.asarray(wd).T, limit))
    assert _fails([pin_closed_form_identical_experts, pin_clamp_branches])


def test_mutant_routing_ignores_bias(monkeypatch):
    orig = om.moe_routing

    def no_bias(x, router_w, router_bias, **kw):
        return orig(x, router_w, None, **kw)
    monkeypatch.setattr(om, "moe_routing", no_bias)
    assert _fails([pin_routing_fields])


def test_mutant_routing_gap_of_wrong_slots(monkeypatch):
    orig = om.near_tie_gaps
    monkeypatch.setattr(om, "near_tie_gaps", lambda beta, k: orig(beta, k + 1))
    assert _fails([pin_routing_fields])


# ---------------------------------------------------------------- FP8 E4M3 weights

def test_e4m3_decode_closed_forms():
    """Values fixed by the encoding's definition (sign, 4-bit exponent with
    bias 7, 3-bit mantissa, subnormals below exponent 1, NaN at S.1111.111)."""
    d = om.decode_e4m3
    assert d([0x00])[0] == 0.0 and np.signbit(d([0x80])[0])
    assert d([0x01])[0] == 2.0 ** -9                 # smallest subnormal
    assert d([0x07])[0] == 7 * 2.0 ** -9             # largest subnormal
    assert d([0x08])[0] == 2.0 ** -6                 # smallest normal
    assert d([0x38])[0] == 1.0
    assert d([0x3C])[0] == 1.5
    assert d([0x40])[0] == 2.0
    assert d([0x7E])[0] == 448.0                     # largest finite
    assert np.isnan(d([0x7F])[0]) and np.isnan(d([0xFF])[0])
    assert d([0xB8])[0] == -1.0


def test_e4m3_decode_structure():
    """Sign symmetry, strict monotonicity over the finite positive codes, and
    every value an integer multiple of the smallest subnormal."""
    v = om.decode_e4m3(np.arange(256))
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(v[0x80:0xFF], -pos)
    k = pos * 2.0 ** 9
    assert np.array_equal(k, np.round(k))


def test_e4m3_decode_matches_torch():
    """Special case that reduces to a library routine: torch's float8_e4m3fn
    (CPU) decodes the same 256 codes to the same values."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = om.decode_e4m3(codes.numpy())
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(np.where(both_nan, 0, ref), np.where(both_nan, 0, got))
    assert np.array_equal(np.isnan(ref), np.isnan(got))


def test_dequantize_scales_columns():
    """Scales apply per output feature (column of the x @ W matrix)."""
    codes = np.array([[0x38, 0x40], [0xB8, 0x3C]], dtype=np.uint8)   # [[1, 2], [-1, 1.5]]
    w = om.dequantize_e4m3(codes, np.array([0.5, 4.0]))
    assert np.array_equal(w, [[0.5, 8.0], [-0.5, 6.0]])


def test_mutant_e4m3_wrong_bias(monkeypatch):
    """A planted mistake (exponent bias 8 instead of 7) fails the pins."""
    real = om.decode_e4m3

    def bad(codes):
        return real(codes) * 0.5
    monkeypatch.setattr(om, "decode_e4m3", bad)
    with pytest.raises(AssertionError):
        test_e4m3_decode_closed_forms()


def test_fp8_workload_quantisation_bound():
    """The FP8 inputs: power-of-two scales, no code out of the finite range,
    and every dequantized weight within half an E4M3 step of the fp32 draw
    (relative 2^-4 for normal values, absolute 2^-10 * scale below them)."""
    wl = replace(WORKLOADS["tiny"], weight_dtype="fp8")
    q = make_inputs(wl, "cpu")
    ref = make_inputs(WORKLOADS["tiny"], "cpu")
    for name in ("w_gate", "w_down", "sh_up"):
        codes, sc = q[name].numpy(), q["s_" + name].numpy().astype(np.float64)
        assert codes.dtype == np.uint8 and not np.any((codes & 0x7F) == 0x7F)
        assert np.array_equal(np.exp2(np.round(np.log2(sc))), sc)
        w = ref[name].double().numpy()
        dq = om.dequantize_e4m3(codes, sc)
        bound = np.maximum(np.abs(w) * 2.0 ** -4, 2.0 ** -10 * sc[..., None, :])
        assert np.all(np.abs(dq - w) <= bound)
    view = om.DequantizedExperts(q["w_up"], q["s_w_up"])
    assert len(view) == wl.num_experts
    assert np.array_equal(view[3], om.dequantize_e4m3(q["w_up"][3].numpy(), q["s_w_up"][3].numpy()))


# ---------------------------------------------------------------- dense MLP

def test_dense_mlp_diagonal_closed_form():
    """Diagonal weights (H = I): out_i = silu(a_i x_i) * (b_i x_i) * c_i per
    element, written with scalar math.exp; with a clamp L the gate is
    min(., L) and up clip(., -L, L) before the product."""
    import math
    rng = np.random.default_rng(11)
    n = 7
    x = rng.normal(size=(3, n))
    a, b, c = rng.normal(size=n) * 2, rng.normal(size=n) * 2, rng.normal(size=n)
    for L in (0.0, 0.7):
        got = om.dense_mlp(x, np.diag(a), np.diag(b), np.diag(c), L)
        for t in range(3):
            for i in range(n):
                g, u = a[i] * x[t, i], b[i] * x[t, i]
                if L > 0:
                    g, u = min(g, L), min(max(u, -L), L)
                want = g / (1.0 + math.exp(-g)) * u * c[i]
                assert abs(got[t, i] - want) <= 1e-12 * max(1.0, abs(want))


def test_dense_mlp_row_independence_and_linearity_in_down():
    """Each row depends only on its own input (to BLAS summation order);
    scaling W_down by a power of two scales the output exactly."""
    rng = np.random.default_rng(12)
    x = rng.normal(size=(5, 16))
    wg, wu, wd = (rng.normal(size=s) * 0.3 for s in ((16, 24), (16, 24), (24, 16)))
    full = om.dense_mlp(x, wg, wu, wd)
    for t in range(5):
        np.testing.assert_allclose(om.dense_mlp(x[t:t + 1], wg, wu, wd)[0], full[t],
                                   rtol=1e-12, atol=1e-12)
    assert np.array_equal(om.dense_mlp(x, wg, wu, 4.0 * wd), 4.0 * full)

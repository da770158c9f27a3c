"""CPU checks of the GPU-parity harness itself (tests/parity.py): on a token
whose oracle k-th and (k+1)-th selection scores are near-tied, the harness
must accept exactly the other correct selections, and reject an unrelated
expert, a wrong order, wrong weights and any mismatch in strict mode.  The
"GPU" results here are planted on the CPU from the oracle's own routing."""
import numpy as np
import pytest

import oracle.moe_oracle as om
from sparse_moe_layer_gemm_b200.workloads import WORKLOADS, make_inputs
from tests.parity import TIE_BAND, check_routing


def _setup():
    wl = WORKLOADS["tiny"]
    inp = {k: v.float().numpy() for k, v in make_inputs(wl, "cpu").items()}
    ref = om.moe_routing(inp["x"], inp["router_w"], inp["router_bias"], top_k=wl.top_k,
                         scale=wl.scale)
    k = wl.top_k
    t = 0
    beta = ref["beta32"][t]
    sel = ref["topk_idx"][t]
    a = int(sel[k - 1])
    rest = [e for e in np.argsort(-beta.astype(np.float64), kind="stable") if e not in sel]
    b = int(rest[0])           # the best expert outside the selection
    worst = int(rest[-1])      # an unrelated expert
    # make token t near-tied: b just below the k-th score
    ref["beta32"] = ref["beta32"].copy()
    ref["beta32"][t, b] = np.float32(beta[a] - np.float32(4e-7))
    ref["tie_gap"] = ref["tie_gap"].copy()
    ref["tie_gap"][t] = float(ref["beta32"][t, a]) - float(ref["beta32"][t, b])
    assert ref["tie_gap"][t] < TIE_BAND
    return wl, ref, t, a, b, worst


def _gpu(ref, idx, wl, weights=None):
    counts, offsets, perm, _ = om.expert_permutation(idx, wl.num_experts)
    if weights is None:
        s_sel = np.take_along_axis(ref["s32"], idx.astype(np.int64), axis=1)
        weights = om.gate_weights(s_sel, wl.scale, True).astype(np.float32)
    return dict(topk_idx=idx.astype(np.int32), topk_w=weights, counts=counts,
                offsets=offsets, perm=perm)


def test_identical_selection_passes():
    wl, ref, *_ = _setup()
    mism, tie = check_routing(_gpu(ref, ref["topk_idx"].copy(), wl), ref, wl.top_k,
                              wl.num_experts, wl=wl)
    assert not mism.any() and tie[0]


def test_other_correct_selection_passes():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, wl.top_k - 1] = b
    mism, _ = check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)
    assert mism[t] and mism.sum() == 1


def test_unrelated_expert_rejected():
    wl, ref, t, a, b, worst = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, wl.top_k - 1] = worst
    with pytest.raises(AssertionError):
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)


def test_dropping_a_top_expert_rejected():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, 0] = b              # drops the best expert, keeps the k-th
    idx[t] = idx[t][np.argsort(-ref["beta32"][t][idx[t]].astype(np.float64), kind="stable")]
    with pytest.raises(AssertionError):
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)


def test_wrong_order_rejected():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, wl.top_k - 1] = b
    idx[t, [0, 1]] = idx[t, [1, 0]]
    with pytest.raises(AssertionError):
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)


def test_wrong_weights_on_tied_row_rejected():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, wl.top_k - 1] = b
    g = _gpu(ref, idx, wl)
    g["topk_w"] = g["topk_w"].copy()
    g["topk_w"][t] = ref["topk_w"][t]          # the oracle's weights of its own set
    with pytest.raises(AssertionError):
        check_routing(g, ref, wl.top_k, wl.num_experts, wl=wl)


def test_strict_mode_rejects_any_mismatch():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    idx[t, wl.top_k - 1] = b
    with pytest.raises(AssertionError):
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl, strict=True)


def test_non_tied_mismatch_rejected():
    wl, ref, t, a, b, _ = _setup()
    idx = ref["topk_idx"].copy()
    u = 1 if t == 0 else 0
    sel = idx[u]
    out = [e for e in np.argsort(-ref["beta32"][u].astype(np.float64), kind="stable")
           if e not in sel]
    idx[u, wl.top_k - 1] = out[0]
    with pytest.raises(AssertionError):
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)


def test_order_swap_of_near_equal_selected_experts():
    """Two selected experts whose scores are within TIE_BAND may come in
    either order; with a larger gap the swap is rejected."""
    wl = WORKLOADS["tiny"]
    inp = {k: v.float().numpy() for k, v in make_inputs(wl, "cpu").items()}
    ref = om.moe_routing(inp["x"], inp["router_w"], inp["router_bias"], top_k=wl.top_k,
                         scale=wl.scale)
    t = 3
    e1, e2 = int(ref["topk_idx"][t, 1]), int(ref["topk_idx"][t, 2])
    idx = ref["topk_idx"].copy()
    idx[t, [1, 2]] = idx[t, [2, 1]]
    with pytest.raises(AssertionError):        # a real gap: the order is fixed
        check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)
    ref["beta32"] = ref["beta32"].copy()
    ref["beta32"][t, e2] = np.nextafter(ref["beta32"][t, e1], np.float32(-1))
    mism, tie = check_routing(_gpu(ref, idx, wl), ref, wl.top_k, wl.num_experts, wl=wl)
    assert mism[t] and tie[t]

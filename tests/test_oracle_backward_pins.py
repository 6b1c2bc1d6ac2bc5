"""Pins of the oracle's layer backward (the next row after the forward: axolotl
ExpertParallelArgs, expert_parallel_save_dispatch) to things other than
itself: central finite differences of the already-pinned forward oracle (run
in fp64 storage, so that nothing is rounded except the fp32 routing weights),
the softmax's shift invariance, and the equality of the save and recompute
strategies for the dispatch outputs.

L = <dout, out>; dx, dW13, dW2 against differences of L in x and the weights;
dlogits and dbias against differences in the logits and the bias (these pass
through the fp32 routing weights, hence a looser bound).
"""
import numpy as np
import pytest

import oracle


def _inputs(seed, T=6, H=8, E=4, k=2, I=4, bias=False, shared=False):
    rng = np.random.default_rng(seed)
    # logits 0.5 apart within a token: the top-k and its weights' order stay put
    # under the perturbations below
    logits = np.stack([rng.permutation(E) * 0.5 + rng.normal(0, 0.01, E) for _ in range(T)])
    logits = logits.astype(np.float32)
    b = rng.normal(0, 0.05, E).astype(np.float32) if bias else None
    x = rng.normal(0, 1, (T, H))
    w13 = rng.normal(0, 1, (E, 2 * I, H)) / np.sqrt(H)
    w2 = rng.normal(0, 1, (E, H, I)) / np.sqrt(I)
    dout = rng.normal(0, 1, (T, H))
    sh = (rng.normal(0, 1, (2 * I, H)) / np.sqrt(H), rng.normal(0, 1, (H, I)) / np.sqrt(I)) if shared else (None, None)
    return dict(logits=logits, bias=b, x=x, w13=w13, w2=w2, dout=dout, w13s=sh[0], w2s=sh[1])


def _loss(d, k, ep, capacity=-1, bias_select_only=False, **over):
    a = {**d, **over}
    r = oracle.moe_layer(a["logits"], a["bias"], a["x"], a["w13"], a["w2"], k, ep, capacity,
                         bias_select_only=bias_select_only, w13_shared=a["w13s"], w2_shared=a["w2s"])
    return float((a["dout"] * r["out"]).sum()), r


def _grad(d, k, ep, capacity=-1, bias_select_only=False, save_dispatch=False):
    return oracle.moe_layer_backward(d["logits"], d["bias"], d["x"], d["w13"], d["w2"], k, ep,
                                     d["dout"], capacity, bias_select_only=bias_select_only,
                                     w13_shared=d["w13s"], w2_shared=d["w2s"],
                                     save_dispatch=save_dispatch)


def _fd(d, name, index, k, ep, eps, capacity=-1, bias_select_only=False):
    """Central difference of L along one entry of d[name]; the routing must not change."""
    base = d[name]
    plus, minus = base.copy(), base.copy()
    plus[index] += eps
    minus[index] -= eps
    lp, rp = _loss(d, k, ep, capacity, bias_select_only, **{name: plus})
    lm, rm = _loss(d, k, ep, capacity, bias_select_only, **{name: minus})
    np.testing.assert_array_equal(rp["topk_idx"], rm["topk_idx"])
    np.testing.assert_array_equal(rp["keep"], rm["keep"])
    step = float(plus[index]) - float(minus[index])       # what the storage really holds
    return (lp - lm) / step


@pytest.mark.parametrize("capacity", [-1, 3])
def test_backward_dx_and_weights_match_finite_differences(capacity):
    d = _inputs(0)
    k, ep = 2, 2
    g = _grad(d, k, ep, capacity)
    if capacity >= 0:
        assert not g["keep"].all(), "the cap must drop something"
    rng = np.random.default_rng(1)
    for _ in range(8):
        t, c = rng.integers(0, 6), rng.integers(0, 8)
        fd = _fd(d, "x", (t, c), k, ep, 1e-5, capacity)
        assert abs(fd - g["dx"][t, c]) <= 1e-7 + 1e-6 * abs(fd), (t, c, fd, g["dx"][t, c])
    kept_experts = sorted(set(g["topk_idx"][g["keep"] != 0].tolist()))
    for e in kept_experts[:2]:
        for name, shape in (("w13", (8, 8)), ("w2", (8, 4))):
            for _ in range(3):
                r, c = rng.integers(0, shape[0]), rng.integers(0, shape[1])
                fd = _fd(d, name, (e, r, c), k, ep, 1e-5, capacity)
                ref = g["dW13" if name == "w13" else "dW2"][e, r, c]
                assert abs(fd - ref) <= 1e-7 + 1e-6 * abs(fd), (name, e, r, c, fd, ref)
    # an expert with no kept row gets no weight gradient
    for e in range(4):
        if e not in kept_experts:
            assert not g["dW13"][e].any() and not g["dW2"][e].any()


@pytest.mark.parametrize("capacity", [-1, 3])
def test_backward_dlogits_match_finite_differences(capacity):
    d = _inputs(2)
    k, ep = 2, 2
    g = _grad(d, k, ep, capacity)
    for t in range(6):
        for e in range(4):
            fd = _fd(d, "logits", (t, e), k, ep, 2.0 ** -10, capacity)
            assert abs(fd - g["dlogits"][t, e]) <= 1e-5 + 2e-3 * abs(fd), (t, e, fd, g["dlogits"][t, e])


def test_backward_dlogits_shift_invariance_and_support():
    d = _inputs(3)
    g = _grad(d, 2, 2)
    # adding a constant to a token's selected logits leaves the softmax unchanged
    assert np.abs(g["dlogits"].sum(axis=1)).max() <= 1e-6 * np.abs(g["dlogits"]).max()
    # only the selected experts get a gradient
    sel = np.zeros((6, 4), bool)
    np.put_along_axis(sel, g["topk_idx"].astype(np.int64), True, axis=1)
    assert not g["dlogits"][~sel].any()


def test_backward_bias_in_weights_and_selection_only():
    d = _inputs(4, bias=True)
    g = _grad(d, 2, 2)
    for e in range(4):
        fd = _fd(d, "bias", (e,), 2, 2, 2.0 ** -10)
        assert abs(fd - g["dbias"][e]) <= 1e-5 + 2e-3 * abs(fd), (e, fd, g["dbias"][e])
    np.testing.assert_allclose(g["dbias"], g["dlogits"].sum(axis=0))
    # the bias steering the selection only: no gradient reaches it
    g2 = _grad(d, 2, 2, bias_select_only=True)
    assert not g2["dbias"].any()
    for e in range(4):
        assert _fd(d, "bias", (e,), 2, 2, 2.0 ** -10, bias_select_only=True) == 0.0


def test_backward_shared_expert_matches_finite_differences():
    d = _inputs(5, shared=True)
    g = _grad(d, 2, 2)
    rng = np.random.default_rng(6)
    for _ in range(6):
        t, c = rng.integers(0, 6), rng.integers(0, 8)
        fd = _fd(d, "x", (t, c), 2, 2, 1e-5)
        assert abs(fd - g["dx"][t, c]) <= 1e-7 + 1e-6 * abs(fd)
    for name, key, shape in (("w13s", "dW13_shared", (8, 8)), ("w2s", "dW2_shared", (8, 4))):
        for _ in range(3):
            r, c = rng.integers(0, shape[0]), rng.integers(0, shape[1])
            fd = _fd(d, name, (r, c), 2, 2, 1e-5)
            assert abs(fd - g[key][r, c]) <= 1e-7 + 1e-6 * abs(fd), (name, r, c, fd, g[key][r, c])


@pytest.mark.parametrize("dtype", ["f64", "bf16"])
def test_backward_save_dispatch_equals_recompute(dtype):
    """Holding the dispatch outputs (the receive rows) or recomputing them gives
    the same gradient, bit for bit: the rows are copies of x."""
    d = _inputs(7, T=16, E=8)
    if dtype == "bf16":
        to_bits = lambda a: (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
        d.update(x=to_bits(d["x"]), w13=to_bits(d["w13"]), w2=to_bits(d["w2"]))
    kw = dict(k=2, ep=2, dout=d["dout"], capacity=5, n_chunks=2)
    a = oracle.moe_layer_backward(d["logits"], None, d["x"], d["w13"], d["w2"], save_dispatch=True, **kw)
    b = oracle.moe_layer_backward(d["logits"], None, d["x"], d["w13"], d["w2"], save_dispatch=False, **kw)
    for key in ("dx", "dlogits", "dW13", "dW2"):
        np.testing.assert_array_equal(a[key], b[key])
    assert not a["keep"].all()


def test_backward_steps_compose_to_the_layer_backward():
    """The combine's and the routing's backward steps, fed the forward's exact
    expert rows (fp64 storage), give the layer backward's dlogits (pinned above by
    finite differences); the rows' backward fed the combine's dy, summed per
    token with unit weights (the permute's backward), gives its dx."""
    d = _inputs(8, T=8, E=4)
    k, ep = 2, 2
    g = _grad(d, k, ep, capacity=3)
    fw = oracle.moe_layer(d["logits"], None, d["x"], d["w13"], d["w2"], k, ep, 3)
    lay = fw["chunks"][0]["layout"]
    y = fw["chunks"][0]["y"]                      # float64 storage: the exact rows
    dy, dw = oracle.combine_backward(d["dout"], y, lay["pos"], fw["topk_w"])
    np.testing.assert_allclose(oracle.route_backward(fw["topk_idx"], fw["topk_w"], dw, 4),
                               g["dlogits"], rtol=1e-12, atol=1e-14)
    # dy[p] = w dout[t] for each kept slot
    for t in range(8):
        for j in range(k):
            p = lay["pos"][t, j]
            if p >= 0:
                np.testing.assert_array_equal(dy[p], np.float64(fw["topk_w"][t, j]) * d["dout"][t])
    # the rows' backward, then the permute's backward (the combine with unit weights)
    n = lay["N"]
    dxr = np.zeros((n, 8))
    eoff = lay["expert_offsets"]
    for e in range(4):
        for p in range(int(eoff[e]), int(eoff[e + 1])):
            dxr[p] = oracle.ffn_row_backward(d["x"][lay["recv_token"][p]], d["w13"][e], d["w2"][e], dy[p])[0]
    dx = oracle.combine(dxr, lay["pos"], np.ones((8, k), np.float32), 8)
    np.testing.assert_allclose(dx, g["dx"], rtol=1e-12, atol=1e-14)


def test_grouped_ffn_backward_step_composes_with_the_row_passes():
    """combine backward -> grouped FFN backward over the receive buffer -> permute
    backward gives the layer backward's dx, dW13 and dW2 (two chunks)."""
    d = _inputs(9, T=8, E=4)
    k, ep = 2, 2
    g = oracle.moe_layer_backward(d["logits"], None, d["x"], d["w13"], d["w2"], k, ep, d["dout"],
                                  capacity=3, n_chunks=2)
    fw = oracle.moe_layer(d["logits"], None, d["x"], d["w13"], d["w2"], k, ep, 3, n_chunks=2)
    dx = np.zeros_like(d["x"])
    dW13 = np.zeros_like(g["dW13"])
    dW2 = np.zeros_like(g["dW2"])
    for c, ch in enumerate(fw["chunks"]):
        lay = ch["layout"]
        dy, _ = oracle.combine_backward(d["dout"], ch["y"], lay["pos"], fw["topk_w"], c * 4)
        dxr, a, b = oracle.ffn_backward(ch["xr"], lay["expert_offsets"], d["w13"], d["w2"], dy)
        dW13 += a
        dW2 += b
        oracle.combine(dxr, lay["pos"], np.ones((8, k), np.float32), 8, c * 4, dx)
    np.testing.assert_allclose(dx, g["dx"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dW13, g["dW13"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dW2, g["dW2"], rtol=1e-12, atol=1e-14)

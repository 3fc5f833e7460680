"""Pins of the backward oracle (CPU): central finite differences of the forward
oracle, and closed forms of the attention backward.

The objective is J = sum(dout * out) + dloss * L_gb.  For a random direction
delta of each input, (J(theta + eps*delta) - J(theta - eps*delta)) / (2 eps)
must equal <grad, delta>; in float64 with eps = 1e-5 the truncation error is
O(eps^2) relative, far below the 1e-7 tolerance, and a dropped term, a wrong
sign or a transposed operand in any gradient moves the inner product by O(1).
The tiny geometry has two shots with one borrowed frame on each side of the
cut, so keys shared by two window groups exercise the accumulation of dK, dV.
"""
import numpy as np
import pytest

from oracle import backward as ob
from oracle import layer as olayer
from oracle import route as oroute

GEOM = dict(T=4, h=4, w=4, win_h=2, win_w=2, shots=[2, 2], tg_max=0, aug=1)
N, H, HD, D, M = 64, 2, 8, 8, 3
ALPHA = 0.1


def _inputs(seed=0, with_bias=True):
    rs = np.random.default_rng(seed)
    w_r = rs.standard_normal((D, M)) / np.sqrt(D)
    bias = rs.standard_normal(M) * 0.1 if with_bias else None
    x = rs.standard_normal((N, D))
    # keep every token's top-2 probability gap >= 1e-3 so that the argmax
    # does not move under the finite-difference steps
    for _ in range(100):
        p = oroute.probabilities(oroute.logits(x, w_r, bias))
        bad = oroute.top2_margin(p) < 1e-3
        if not bad.any():
            break
        x[bad] = rs.standard_normal((int(bad.sum()), D))
    q = rs.standard_normal((N, H, HD))
    k = rs.standard_normal((N, H, HD))
    v = rs.standard_normal((N, H, HD))
    dout = rs.standard_normal((N, H, HD))
    return dict(x=x, w_r=w_r, bias=bias, q=q, k=k, v=v, dout=dout, dloss=0.7)


def _J(inp, **over):
    a = dict(inp)
    a.update(over)
    return ob.objective(a["x"], a["w_r"], a["bias"], a["q"], a["k"], a["v"], M, GEOM, ALPHA, a["dout"],
                        a["dloss"])


@pytest.fixture(scope="module")
def case():
    inp = _inputs()
    grads = ob.layer_backward(inp["x"], inp["w_r"], inp["bias"], inp["q"], inp["k"], inp["v"], M, GEOM, ALPHA,
                              inp["dout"], inp["dloss"])
    return inp, grads


@pytest.mark.parametrize("name,grad", [("q", "dq"), ("k", "dk"), ("v", "dv"), ("x", "dx"), ("w_r", "dw_r"),
                                       ("bias", "dbias")])
def test_directional_derivatives(case, name, grad):
    inp, grads = case
    rs = np.random.default_rng(["q", "k", "v", "x", "w_r", "bias"].index(name) + 10)
    eps = 1e-5
    for _ in range(3):
        delta = rs.standard_normal(np.shape(inp[name]))
        jp = _J(inp, **{name: inp[name] + eps * delta})
        jm = _J(inp, **{name: inp[name] - eps * delta})
        fd = (jp - jm) / (2 * eps)
        an = float(np.sum(grads[grad] * delta))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_argmax_stable_under_steps(case):
    inp, _ = case
    g0 = oroute.route(inp["x"], inp["w_r"], inp["bias"])[0]
    g1 = oroute.route(inp["x"] + 1e-5, inp["w_r"], inp["bias"])[0]
    assert np.array_equal(g0, g1)


def test_single_key_closed_form():
    """One key: P = 1 and O = v, so dv = sum of dO over queries and dq = dk = 0."""
    rs = np.random.default_rng(1)
    q, k, v = rs.standard_normal((5, 4)), rs.standard_normal((1, 4)), rs.standard_normal((1, 3))
    do = rs.standard_normal((5, 3))
    dq, dk, dv = ob.attend_bwd(q, k, v, do, 0.5)
    np.testing.assert_allclose(dv, do.sum(axis=0, keepdims=True), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)


def test_uniform_attention_closed_form():
    """q = 0: P = 1/n everywhere, so dv_j = mean of dO over queries, dk = 0 and
    dq_i = scale/n * sum_j (dO_i . v_j - dO_i . vbar) k_j."""
    rs = np.random.default_rng(2)
    n, scale = 6, 0.3
    q = np.zeros((4, 5))
    k, v, do = rs.standard_normal((n, 5)), rs.standard_normal((n, 3)), rs.standard_normal((4, 3))
    dq, dk, dv = ob.attend_bwd(q, k, v, do, scale)
    np.testing.assert_allclose(dv, np.repeat(do.sum(axis=0, keepdims=True) / n, n, axis=0), atol=1e-14)
    np.testing.assert_allclose(dk, 0.0, atol=1e-14)
    vbar = v.mean(axis=0)
    want = np.stack([scale / n * sum((do[i] @ v[j] - do[i] @ vbar) * k[j] for j in range(n)) for i in range(4)])
    np.testing.assert_allclose(dq, want, atol=1e-13)


def test_loss_only_router_gradient():
    """With dout = 0 the router only sees the balancing loss: the gate gradient is
    zero and, through the softmax Jacobian, each token's dr sums to zero over groups."""
    inp = _inputs(seed=3)
    grads = ob.layer_backward(inp["x"], inp["w_r"], inp["bias"], inp["q"], inp["k"], inp["v"], M, GEOM, ALPHA,
                              np.zeros_like(inp["dout"]), 1.0)
    np.testing.assert_allclose(grads["dr"].sum(axis=1), 0.0, atol=1e-15)
    assert np.all(grads["dgate"] == 0.0)


def test_mean_splits_upstream_gradient():
    """Scaling dout by 3 scales every attention gradient by 3 (linearity of the mean)."""
    inp = _inputs(seed=4)
    a = ob.layer_backward(inp["x"], inp["w_r"], None, inp["q"], inp["k"], inp["v"], M, GEOM, ALPHA, inp["dout"], 0.0)
    b = ob.layer_backward(inp["x"], inp["w_r"], None, inp["q"], inp["k"], inp["v"], M, GEOM, ALPHA,
                          3 * inp["dout"], 0.0)
    for key in ("dq", "dk", "dv", "dgate"):
        np.testing.assert_allclose(b[key], 3 * a[key], rtol=1e-12, atol=1e-12)
    assert olayer.mean3(1.0, 2.0, 3.0) == 2.0

"""Pins for the backward pass of the TTT-linear oracle.

The loss L = sum_t <dout_t, o_t> + <dS_end, S_end> is affine in each single
input coordinate (the layer is multilinear in q, k, v, lr and S0), so a
central difference along one coordinate equals the partial derivative up to
rounding.  Every gradient entry of ``ttt_linear_backward`` is checked that
way against the forward recurrence, which is itself pinned to the pages'
linear-attention theorem.
"""
import numpy as np
import pytest

from oracle import ttt_linear_backward, ttt_linear_recurrent


def _rand(B=1, H=2, N=6, dk=3, dv=4, seed=5):
    r = np.random.default_rng(seed)
    return dict(q=r.standard_normal((B, H, N, dk)), k=r.standard_normal((B, H, N, dk)),
                v=r.standard_normal((B, H, N, dv)), lr=r.uniform(0.05, 0.6, (B, H, N)),
                S0=r.standard_normal((B, H, dk, dv))), \
        r.standard_normal((B, H, N, dv)), r.standard_normal((B, H, dk, dv))


def _loss(x, dout, dS_end, include_diag):
    o, S = ttt_linear_recurrent(x["q"], x["k"], x["v"], x["lr"], x["S0"], include_diag)
    return float((dout * o).sum() + (0.0 if dS_end is None else (dS_end * S).sum()))


def _central_differences(x, dout, dS_end, include_diag, h=0.5):
    # exact for an affine function of the coordinate, whatever h is
    grads = {}
    for name in ("q", "k", "v", "lr", "S0"):
        g = np.empty_like(x[name])
        for idx in np.ndindex(x[name].shape):
            old = x[name][idx]
            x[name][idx] = old + h
            lp = _loss(x, dout, dS_end, include_diag)
            x[name][idx] = old - h
            lm = _loss(x, dout, dS_end, include_diag)
            x[name][idx] = old
            g[idx] = (lp - lm) / (2 * h)
        grads[name] = g
    return grads


@pytest.mark.parametrize("include_diag", [True, False])
@pytest.mark.parametrize("with_dS_end", [False, True])
def test_backward_equals_central_differences(include_diag, with_dS_end):
    x, dout, dS_end = _rand()
    dS_end = dS_end if with_dS_end else None
    fd = _central_differences(x, dout, dS_end, include_diag)
    dq, dk, dv, dlr, dS0 = ttt_linear_backward(x["q"], x["k"], x["v"], x["lr"], dout, x["S0"],
                                               dS_end, include_diag)
    for got, name in ((dq, "q"), (dk, "k"), (dv, "v"), (dlr, "lr"), (dS0, "S0")):
        np.testing.assert_allclose(got, fd[name], rtol=0, atol=1e-10, err_msg=name)


def test_without_initial_state_the_state_gradient_still_appears():
    x, dout, dS_end = _rand(N=5, seed=9)
    x["S0"] = np.zeros_like(x["S0"])
    fd = _central_differences(x, dout, dS_end, True)
    *_, dS0 = ttt_linear_backward(x["q"], x["k"], x["v"], x["lr"], dout, None, dS_end, True)
    np.testing.assert_allclose(dS0, fd["S0"], rtol=0, atol=1e-10)


def test_planted_diagonal_mistake_is_caught():
    """The inclusive layer's gradients taken with the exclusive reverse
    recurrence (an off-by-one in which reads see a token's own update)."""
    x, dout, dS_end = _rand(seed=11)
    fd = _central_differences(x, dout, dS_end, True)
    _, dk, dv, dlr, _ = ttt_linear_backward(x["q"], x["k"], x["v"], x["lr"], dout, x["S0"],
                                            dS_end, include_diag=False)
    assert max(np.abs(dk - fd["k"]).max(), np.abs(dv - fd["v"]).max(),
               np.abs(dlr - fd["lr"]).max()) > 1e-3


def test_planted_missing_end_state_term_is_caught():
    """Dropping the final-state sensitivity dS_end from the reverse pass."""
    x, dout, dS_end = _rand(seed=12)
    fd = _central_differences(x, dout, dS_end, True)
    _, dk, _, _, dS0 = ttt_linear_backward(x["q"], x["k"], x["v"], x["lr"], dout, x["S0"], None,
                                           True)
    assert np.abs(dk - fd["k"]).max() > 1e-3 and np.abs(dS0 - fd["S0"]).max() > 1e-3

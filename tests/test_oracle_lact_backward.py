"""Pins for the LaCT backward oracle: its float64 torch restatement of the
forward equals the numpy oracle, and its gradients equal central differences
of the numpy oracle's loss (the numpy oracle is itself pinned to finite
differences of the binding loss and to linear attention in the W2-only case)."""
import numpy as np
import pytest

from oracle import lact_forward
from oracle.lact import LaCTState
from oracle.lact_backward import lact_backward, lact_forward_torch, _t


def _rand(B=1, H=2, N=7, Nq=None, d=4, dh=3, seed=0):
    r = np.random.default_rng(seed)
    nq = N if Nq is None else Nq
    x = dict(q=r.standard_normal((B, H, nq, d)), k=r.standard_normal((B, H, N, d)) * 0.7,
             v=r.standard_normal((B, H, N, d)), lr=r.uniform(0.05, 0.3, (B, H, N)),
             W1=r.standard_normal((B, H, dh, d)) * 0.5, W3=r.standard_normal((B, H, dh, d)) * 0.5,
             W2=r.standard_normal((B, H, d, dh)) * 0.5)
    dout = r.standard_normal((B, H, nq, d))
    dW = (r.standard_normal((B, H, dh, d)), r.standard_normal((B, H, dh, d)),
          r.standard_normal((B, H, d, dh)))
    return x, dout, dW


def _np_forward(x, **kw):
    opt = kw.get("opt", "gd")
    st = LaCTState(x["W1"].copy(), x["W3"].copy(), x["W2"].copy())
    if opt in ("momentum", "muon"):
        st.M1, st.M3, st.M2 = (np.zeros_like(st.W1), np.zeros_like(st.W3), np.zeros_like(st.W2))
    return lact_forward(x["q"], x["k"], x["v"], x["lr"], st, **kw)


def _np_loss(x, dout, dW, **kw):
    out, st = _np_forward(x, **kw)
    L = float(np.sum(out * dout))
    if dW is not None:
        L += float(sum(np.sum(w * g) for w, g in zip((st.W1, st.W3, st.W2), dW)))
    return L


CASES = [
    dict(chunk=3, order="causal", opt="gd"),
    dict(chunk=3, order="causal", opt="momentum", beta=0.8),
    dict(chunk=4, order="causal", opt="muon", beta=0.9, ns_steps=3),
    dict(chunk=3, order="bidirectional", opt="gd"),
    dict(chunk=2, order="causal", opt="gd", normalize_rows=False, update_mask=4),
    dict(chunk=3, order="causal", opt="gd", update_mask=3),
]


@pytest.mark.parametrize("kw", CASES)
def test_torch_restatement_equals_the_numpy_oracle(kw):
    x, _, _ = _rand(Nq=5 if kw["order"] == "bidirectional" else None, seed=1)
    out_np, st = _np_forward(x, **kw)
    out_t, W_t = lact_forward_torch(*(_t(x[n]) for n in ("q", "k", "v", "lr", "W1", "W3", "W2")),
                                    **kw)
    np.testing.assert_allclose(out_t.numpy(), out_np, rtol=0, atol=1e-12)
    for a, b in zip(W_t, (st.W1, st.W3, st.W2)):
        np.testing.assert_allclose(a.numpy(), b, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kw", CASES)
def test_gradients_equal_central_differences(kw):
    x, dout, dW = _rand(Nq=5 if kw["order"] == "bidirectional" else None, seed=2)
    got = lact_backward(x["q"], x["k"], x["v"], x["lr"], x["W1"], x["W3"], x["W2"], dout, dW, **kw)
    def central(name, idx, h):
        old = x[name][idx]
        x[name][idx] = old + h
        lp = _np_loss(x, dout, dW, **kw)
        x[name][idx] = old - h
        lm = _np_loss(x, dout, dW, **kw)
        x[name][idx] = old
        return (lp - lm) / (2 * h)

    h = 2e-4
    for name, g in zip(("q", "k", "v", "lr", "W1", "W3", "W2"), got):
        fd = np.empty_like(g)
        for idx in np.ndindex(x[name].shape):
            # Richardson extrapolation of the central difference: the h^2
            # truncation term cancels, leaving O(h^4)
            fd[idx] = (4 * central(name, idx, h / 2) - central(name, idx, h)) / 3
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(g, fd, rtol=0, atol=2e-7 * scale, err_msg=name)


def test_planted_missing_second_order_term_is_caught():
    """Treating each chunk gradient as independent of the chunk-start weights
    (a plausible shortcut) gives wrong weight gradients."""
    import torch
    import oracle.lact_backward as lb
    x, dout, dW = _rand(seed=3)
    kw = dict(chunk=3, order="causal", opt="gd")
    good = lact_backward(x["q"], x["k"], x["v"], x["lr"], x["W1"], x["W3"], x["W2"], dout, dW, **kw)
    orig = lb._chunk_gradients

    def detached(W1, W3, W2, k, v, lr):
        return orig(W1.detach(), W3.detach(), W2.detach(), k, v, lr)
    lb._chunk_gradients = detached
    try:
        bad = lact_backward(x["q"], x["k"], x["v"], x["lr"], x["W1"], x["W3"], x["W2"], dout, dW,
                            **kw)
    finally:
        lb._chunk_gradients = orig
    assert max(np.abs(b - g).max() for b, g in zip(bad[4:], good[4:])) > 1e-4
    del torch


EXPLICIT_CASES = CASES + [
    dict(chunk=2, order="causal", opt="momentum", beta=0.7, update_mask=5),
    dict(chunk=7, order="bidirectional", opt="momentum", beta=0.9, normalize_rows=False),
    dict(chunk=3, order="bidirectional", opt="muon", beta=0.8, ns_steps=5),
]


@pytest.mark.parametrize("kw", EXPLICIT_CASES)
def test_written_out_backward_equals_autograd(kw):
    """The step-by-step backward (read VJP, row-norm VJP, momentum carry and
    the chunk gradient's vector-Jacobian product) equals autograd."""
    from oracle.lact_backward import lact_backward_explicit
    x, dout, dW = _rand(B=2, H=2, N=9, Nq=6 if kw["order"] == "bidirectional" else None, seed=7)
    args = (x["q"], x["k"], x["v"], x["lr"], x["W1"], x["W3"], x["W2"], dout, dW)
    ref = lact_backward(*args, **kw)
    got = lact_backward_explicit(*args, **kw)
    for name, g, r in zip(("q", "k", "v", "lr", "W1", "W3", "W2"), got, ref):
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-10 * max(1.0, np.abs(r).max()),
                                   err_msg=name)


def test_muon_chunk_with_zero_learning_rates():
    """A first chunk whose learning rates are all zero leaves the momentum
    buffer at exactly zero, and Newton-Schulz maps it to zero.  X0 = G /
    (||G||_F + eps) is differentiable there (derivative I / eps), so both
    backward oracles must stay finite, agree, and match central differences."""
    from oracle.lact_backward import lact_backward_explicit
    kw = dict(chunk=3, order="causal", opt="muon", beta=0.9, ns_steps=3)
    x, dout, dW = _rand(N=7, seed=4)
    x["lr"][..., :3] = 0.0
    args = (x["q"], x["k"], x["v"], x["lr"], x["W1"], x["W3"], x["W2"], dout, dW)
    ref = lact_backward(*args, **kw)
    got = lact_backward_explicit(*args, **kw)
    for name, g, r in zip(("q", "k", "v", "lr", "W1", "W3", "W2"), got, ref):
        assert np.isfinite(g).all() and np.isfinite(r).all(), name
        np.testing.assert_allclose(g, r, rtol=0, atol=1e-10 * max(1.0, np.abs(r).max()),
                                   err_msg=name)
    # Inside the zero chunk the map is linear only while ||G|| << eps = 1e-7,
    # so the difference step there is 1e-12 (the result is ~1e9, so the
    # rounding of the loss difference stays far below the tolerance); the
    # token of the second chunk (a momentum buffer away from zero) takes the
    # usual step.
    for idx, h in [((0, 0, 0), 1e-12), ((0, 1, 2), 1e-12), ((0, 0, 5), 2e-4)]:
        def loss(val):
            old = x["lr"][idx]
            x["lr"][idx] = val
            L = _np_loss(x, dout, dW, **kw)
            x["lr"][idx] = old
            return L
        c = x["lr"][idx]
        fd1 = (loss(c + h) - loss(c - h)) / (2 * h)
        fd2 = (loss(c + h / 2) - loss(c - h / 2)) / h
        fd = (4 * fd2 - fd1) / 3
        assert abs(got[3][idx] - fd) <= 1e-5 * max(1.0, abs(fd)), (idx, got[3][idx], fd)

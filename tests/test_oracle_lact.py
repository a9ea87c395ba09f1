"""Pins for the LaCT oracle against facts that are not the oracle.

* Finite differences of the lr-weighted binding loss pin the hand-derived
  SwiGLU chunk gradients (sign, transposes, silu').
* Per-token GD whose gradient is taken by finite differences equals the
  oracle at chunk = 1 (chunk semantics, update, normalisation).
* Updating only W2 with GD and no normalisation turns the layer into linear
  attention over the features phi(x) = silu(W1 x) * (W3 x): block-causal for
  the language order, unmasked for the view-synthesis order ("Test-Time
  Training with KV Binding Is Secretly Linear Attention", summary section
  "4. Resultados", variants that update only the last linear layer; podcast
  11:54-12:33).  With momentum the same closed form carries geometric chunk
  weights.
* Newton-Schulz equals U diag(p^5(sigma/||G||_F)) V^T from a library SVD
  (a matrix polynomial in G G^T keeps the singular vectors).
* Invariants: unit row norms after every update, causal outputs unchanged by
  future tokens, bidirectional single-chunk outputs invariant to token order,
  split-call streaming equal to one call.
"""
import numpy as np
import pytest

from oracle import (lact_chunk_gradients, lact_forward, lact_read, newton_schulz,
                    silu)
from oracle.lact import lact_init_state

NS = (3.4445, -4.7750, 2.0315)


def _phi(W1, W3, x):
    return silu(x @ W1.T) * (x @ W3.T)


def _small(B=1, H=2, N=24, d=4, dh=8, seed=0, Nq=None):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, Nq or N, d))
    k = r.standard_normal((B, H, N, d))
    v = r.standard_normal((B, H, N, d))
    lr = r.uniform(0.05, 0.3, (B, H, N))
    W1 = r.standard_normal((H, dh, d)) / np.sqrt(d)
    W3 = r.standard_normal((H, dh, d)) / np.sqrt(d)
    W2 = r.standard_normal((H, d, dh)) / np.sqrt(dh)
    return q, k, v, lr, W1, W3, W2


def _loss(W1, W3, W2, k, v, lr):
    f = (silu(k @ W1.T) * (k @ W3.T)) @ W2.T
    return float(np.sum(lr * -np.sum(f * v, axis=-1)))


def _fd_grad(fn, W, h=1e-6):
    G = np.zeros_like(W)
    for idx in np.ndindex(W.shape):
        Wp, Wm = W.copy(), W.copy()
        Wp[idx] += h
        Wm[idx] -= h
        G[idx] = (fn(Wp) - fn(Wm)) / (2 * h)
    return G


def test_chunk_gradients_match_finite_differences():
    _, k, v, lr, W1, W3, W2 = _small(N=3)
    k, v, lr, W1, W3, W2 = k[0, 0], v[0, 0], lr[0, 0], W1[0], W3[0], W2[0]
    G1, G3, G2 = lact_chunk_gradients(W1, W3, W2, k, v, lr)
    F1 = _fd_grad(lambda W: _loss(W, W3, W2, k, v, lr), W1)
    F3 = _fd_grad(lambda W: _loss(W1, W, W2, k, v, lr), W3)
    F2 = _fd_grad(lambda W: _loss(W1, W3, W, k, v, lr), W2)
    for G, F in ((G1, F1), (G3, F3), (G2, F2)):
        assert np.abs(G - F).max() <= 1e-6 * np.abs(F).max()


def test_chunk1_equals_per_token_gd_with_numerical_gradients():
    q, k, v, lr, W1, W3, W2 = _small(B=1, H=1, N=5, d=3, dh=4, seed=3)
    st = lact_init_state(W1, W3, W2, 1)
    out, st = lact_forward(q, k, v, lr, st, chunk=1, order="causal", opt="gd")
    w1, w3, w2 = W1[0].copy(), W3[0].copy(), W2[0].copy()
    nrm = lambda W: W / np.linalg.norm(W, axis=1, keepdims=True)  # noqa: E731
    for t in range(5):
        x = q[0, 0, t:t + 1]
        ref_o = (silu(x @ w1.T) * (x @ w3.T)) @ w2.T
        np.testing.assert_allclose(out[0, 0, t], ref_o[0], rtol=1e-9, atol=1e-12)
        kt, vt, et = k[0, 0, t:t + 1], v[0, 0, t:t + 1], lr[0, 0, t:t + 1]
        g1 = _fd_grad(lambda W: _loss(W, w3, w2, kt, vt, et), w1)
        g3 = _fd_grad(lambda W: _loss(w1, W, w2, kt, vt, et), w3)
        g2 = _fd_grad(lambda W: _loss(w1, w3, W, kt, vt, et), w2)
        w1, w3, w2 = nrm(w1 - g1), nrm(w3 - g3), nrm(w2 - g2)
    for a, b in ((st.W1[0, 0], w1), (st.W3[0, 0], w3), (st.W2[0, 0], w2)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-7)


def test_w2_only_gd_causal_is_block_causal_feature_attention():
    C = 5
    q, k, v, lr, W1, W3, W2 = _small(B=2, H=2, N=23, seed=1)
    st = lact_init_state(W1, W3, W2, 2)
    out, _ = lact_forward(q, k, v, lr, st, chunk=C, order="causal", opt="gd",
                          normalize_rows=False, update_mask=4)
    for b in range(2):
        for h in range(2):
            pq, pk = _phi(W1[h], W3[h], q[b, h]), _phi(W1[h], W3[h], k[b, h])
            s = pq @ pk.T * lr[b, h][None, :]
            blk = np.arange(23) // C
            s = s * (blk[None, :] < blk[:, None])          # strictly earlier chunks
            ref = pq @ W2[h].T + s @ v[b, h]
            np.testing.assert_allclose(out[b, h], ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_w2_only_gd_bidirectional_is_unmasked_feature_attention():
    q, k, v, lr, W1, W3, W2 = _small(B=1, H=2, N=17, Nq=6, seed=2)
    st = lact_init_state(W1, W3, W2, 1)
    out, _ = lact_forward(q, k, v, lr, st, chunk=6, order="bidirectional", opt="gd",
                          normalize_rows=False, update_mask=4)
    for h in range(2):
        pq, pk = _phi(W1[h], W3[h], q[0, h]), _phi(W1[h], W3[h], k[0, h])
        ref = pq @ W2[h].T + (pq @ pk.T * lr[0, h][None, :]) @ v[0, h]
        np.testing.assert_allclose(out[0, h], ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_w2_only_momentum_has_geometric_chunk_weights():
    C, N, beta = 4, 18, 0.7
    q, k, v, lr, W1, W3, W2 = _small(B=1, H=1, N=N, seed=4)
    st = lact_init_state(W1, W3, W2, 1, opt="momentum")
    out, _ = lact_forward(q, k, v, lr, st, chunk=C, order="causal", opt="momentum", beta=beta,
                          normalize_rows=False, update_mask=4)
    pq, pk = _phi(W1[0], W3[0], q[0, 0]), _phi(W1[0], W3[0], k[0, 0])
    blk = np.arange(N) // C
    # token s in chunk c' contributes to the weights read by chunk c > c' with
    # weight sum_{j=0}^{c-1-c'} beta^j = (1 - beta^(c-c')) / (1 - beta)
    gap = blk[:, None] - blk[None, :]
    w = np.where(gap > 0, (1 - beta ** np.maximum(gap, 0)) / (1 - beta), 0.0)
    ref = pq @ W2[0].T + (pq @ pk.T * lr[0, 0][None, :] * w) @ v[0, 0]
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def _ns_by_svd(G, steps=5, coef=NS, eps=1e-7):
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    x = s / (np.sqrt(np.sum(G * G)) + eps)
    a, b, c = coef
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return (U * x) @ Vt


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (7, 7), (1, 5)])
def test_newton_schulz_equals_svd_polynomial(shape):
    G = np.random.default_rng(5).standard_normal(shape)
    X = newton_schulz(G, 5, NS, 1e-7)
    np.testing.assert_allclose(X, _ns_by_svd(G), rtol=0, atol=1e-12)


def test_newton_schulz_scalar_case():
    g = -3.0
    x = 3.0 / (3.0 + 1e-7)
    for _ in range(5):
        x = NS[0] * x + NS[1] * x ** 3 + NS[2] * x ** 5
    assert np.isclose(newton_schulz(np.array([[g]]))[0, 0], -x, rtol=0, atol=1e-14)


def test_newton_schulz_singular_values_near_one():
    G = np.random.default_rng(6).standard_normal((48, 96))
    s = np.linalg.svd(newton_schulz(G), compute_uv=False)
    assert s.min() > 0.5 and s.max() < 1.3


def test_w2_only_muon_single_chunk_uses_ns_of_gradient():
    q, k, v, lr, W1, W3, W2 = _small(B=1, H=1, N=12, Nq=5, d=4, dh=8, seed=7)
    st = lact_init_state(W1, W3, W2, 1, opt="muon")
    out, st = lact_forward(q, k, v, lr, st, chunk=12, order="bidirectional", opt="muon",
                           beta=0.9, normalize_rows=False, update_mask=4)
    pk = _phi(W1[0], W3[0], k[0, 0])
    G2 = -(lr[0, 0][:, None] * v[0, 0]).T @ pk        # d l / d W2 summed over the chunk
    W2n = W2[0] - _ns_by_svd(G2)
    np.testing.assert_allclose(st.W2[0, 0], W2n, rtol=0, atol=1e-12)
    ref = _phi(W1[0], W3[0], q[0, 0]) @ W2n.T
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("opt", ["gd", "momentum", "muon"])
def test_rows_unit_norm_after_update(opt):
    q, k, v, lr, W1, W3, W2 = _small(B=1, H=2, N=20, seed=8)
    st = lact_init_state(W1, W3, W2, 1, opt=opt)
    _, st = lact_forward(q, k, v, lr, st, chunk=7, order="causal", opt=opt)
    for W in (st.W1, st.W3, st.W2):
        np.testing.assert_allclose(np.linalg.norm(W, axis=-1), 1.0, rtol=0, atol=1e-12)


def test_update_mask_freezes_other_matrices():
    q, k, v, lr, W1, W3, W2 = _small(seed=9)
    st = lact_init_state(W1, W3, W2, 1)
    _, st = lact_forward(q, k, v, lr, st, chunk=8, update_mask=4)
    assert np.array_equal(st.W1[0], W1) and np.array_equal(st.W3[0], W3)
    assert not np.allclose(st.W2[0], W2)


def test_causal_outputs_ignore_future_tokens():
    C = 6
    q, k, v, lr, W1, W3, W2 = _small(N=30, seed=10)
    out, _ = lact_forward(q, k, v, lr, lact_init_state(W1, W3, W2, 1), chunk=C)
    r = np.random.default_rng(11)
    cut = 2 * C
    q2, k2, v2, lr2 = q.copy(), k.copy(), v.copy(), lr.copy()
    for a in (q2, k2, v2):
        a[:, :, cut:] = r.standard_normal(a[:, :, cut:].shape)
    lr2[:, :, cut:] = r.uniform(0.05, 0.3, lr2[:, :, cut:].shape)
    out2, _ = lact_forward(q2, k2, v2, lr2, lact_init_state(W1, W3, W2, 1), chunk=C)
    assert np.array_equal(out[:, :, :cut], out2[:, :, :cut])
    assert not np.allclose(out[:, :, cut:], out2[:, :, cut:])


def test_bidirectional_single_chunk_is_order_invariant():
    q, k, v, lr, W1, W3, W2 = _small(N=16, Nq=5, seed=12)
    out, _ = lact_forward(q, k, v, lr, lact_init_state(W1, W3, W2, 1), chunk=16,
                          order="bidirectional")
    p = np.random.default_rng(13).permutation(16)
    out2, _ = lact_forward(q, k[:, :, p], v[:, :, p], lr[:, :, p],
                           lact_init_state(W1, W3, W2, 1), chunk=16, order="bidirectional")
    np.testing.assert_allclose(out, out2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("opt", ["gd", "momentum", "muon"])
def test_streaming_split_equals_single_call(opt):
    C = 5
    q, k, v, lr, W1, W3, W2 = _small(N=25, seed=14)
    out, st = lact_forward(q, k, v, lr, lact_init_state(W1, W3, W2, 1, opt), chunk=C, opt=opt)
    s2 = lact_init_state(W1, W3, W2, 1, opt)
    oa, s2 = lact_forward(q[:, :, :10], k[:, :, :10], v[:, :, :10], lr[:, :, :10], s2,
                          chunk=C, opt=opt)
    ob, s2 = lact_forward(q[:, :, 10:], k[:, :, 10:], v[:, :, 10:], lr[:, :, 10:], s2,
                          chunk=C, opt=opt)
    np.testing.assert_allclose(np.concatenate([oa, ob], 2), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s2.W2, st.W2, rtol=0, atol=1e-12)


def test_read_is_swiglu_of_the_weights():
    _, _, _, _, W1, W3, W2 = _small(seed=15)
    x = np.random.default_rng(16).standard_normal((3, 4))
    h1, h3 = x @ W1[0].T, x @ W3[0].T
    ref = np.stack([W2[0] @ (h1[i] / (1 + np.exp(-h1[i])) * h3[i]) for i in range(3)])
    np.testing.assert_allclose(lact_read(W1[0], W3[0], W2[0], x), ref, rtol=1e-14, atol=1e-14)


def test_planted_sign_mistake_is_caught():
    """Flipping the loss sign inside the oracle's gradient must break the
    finite-difference pin (shows the pin is sensitive to a dropped minus)."""
    _, k, v, lr, W1, W3, W2 = _small(N=3)
    k, v, lr, W1, W3, W2 = k[0, 0], v[0, 0], lr[0, 0], W1[0], W3[0], W2[0]
    _, _, G2_wrong = lact_chunk_gradients(W1, W3, W2, k, v, -lr)
    F2 = _fd_grad(lambda W: _loss(W1, W3, W, k, v, lr), W2)
    assert np.abs(G2_wrong - F2).max() > 1e-3 * np.abs(F2).max()

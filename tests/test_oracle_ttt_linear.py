"""Pins for the TTT-linear oracle against facts that are not the oracle.

* The pages' theorem: the token-by-token GD recurrence on -<W k, v> equals
  causal linear attention  o_t = sum_{s<=t} eta_s (q_t . k_s) v_s
  ("Test-Time Training with KV Binding Is Secretly Linear Attention",
  summary section "B. Reformulación Teórica"; podcast 7:50-8:26).
* Gradient ascent is the same layer with the sign absorbed (summary,
  "Resolución de Paradojas"; podcast 9:01-9:39): negating eta negates o.
* A hand-worked three-token example (tests/golden/ttt_linear_hand.json).
"""
import json
import os

import numpy as np
import pytest

from oracle import ttt_linear_recurrent, ttt_linear_attention_sum
from ttt_synth import make_linear_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(B=2, H=3, N=37, dk=5, dv=7, seed=0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, N, dk))
    k = r.standard_normal((B, H, N, dk))
    v = r.standard_normal((B, H, N, dv))
    lr = r.uniform(0.01, 0.5, (B, H, N))
    S0 = r.standard_normal((B, H, dk, dv))
    return q, k, v, lr, S0


@pytest.mark.parametrize("include_diag", [True, False])
@pytest.mark.parametrize("with_s0", [False, True])
def test_recurrence_equals_linear_attention(include_diag, with_s0):
    q, k, v, lr, S0 = _rand()
    S0 = S0 if with_s0 else None
    o_rec, _ = ttt_linear_recurrent(q, k, v, lr, S0, include_diag)
    o_sum = ttt_linear_attention_sum(q, k, v, lr, S0, include_diag)
    np.testing.assert_allclose(o_rec, o_sum, rtol=0, atol=1e-12 * np.abs(o_sum).max())


def test_final_state_is_sum_of_outer_products():
    q, k, v, lr, S0 = _rand(N=23)
    _, S = ttt_linear_recurrent(q, k, v, lr, S0)
    expect = S0 + np.einsum("bhn,bhni,bhnj->bhij", lr, k, v)
    np.testing.assert_allclose(S, expect, rtol=0, atol=1e-12 * np.abs(expect).max())


def test_gradient_ascent_sign_is_absorbed():
    q, k, v, lr, _ = _rand(N=19)
    o_pos, _ = ttt_linear_recurrent(q, k, v, lr, None)
    o_neg, _ = ttt_linear_recurrent(q, k, v, -lr, None)
    assert np.array_equal(o_neg, -o_pos)


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "ttt_linear_hand.json")))
    shape = lambda a: np.array(a, dtype=np.float64)[None, None]  # noqa: E731
    q, k, v = shape(g["q"]), shape(g["k"]), shape(g["v"])
    lr = np.array(g["lr"], dtype=np.float64)[None, None]
    o_inc, S = ttt_linear_recurrent(q, k, v, lr, None, True)
    o_exc, _ = ttt_linear_recurrent(q, k, v, lr, None, False)
    assert np.array_equal(o_inc[0, 0], np.array(g["out_inclusive"], dtype=np.float64))
    assert np.array_equal(o_exc[0, 0], np.array(g["out_exclusive"], dtype=np.float64))
    assert np.array_equal(S[0, 0], np.array(g["S_end"], dtype=np.float64))


def test_streaming_split_equals_single_call():
    q, k, v, lr, S0 = _rand(N=40)
    o_all, S_all = ttt_linear_recurrent(q, k, v, lr, S0)
    o_a, S_a = ttt_linear_recurrent(q[:, :, :17], k[:, :, :17], v[:, :, :17], lr[:, :, :17], S0)
    o_b, S_b = ttt_linear_recurrent(q[:, :, 17:], k[:, :, 17:], v[:, :, 17:], lr[:, :, 17:], S_a)
    np.testing.assert_allclose(np.concatenate([o_a, o_b], 2), o_all, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S_b, S_all, rtol=1e-13, atol=1e-13)


def test_sampled_sum_matches_full_on_workload_inputs():
    x = make_linear_inputs(1, 2, 256, 32, 32, chunk=16, dtype="f32", lr_kind="0.1sig", cfg=1)
    o_rec, _ = ttt_linear_recurrent(x.q.values, x.k.values, x.v.values, x.lr)
    idx = [0, 15, 16, 100, 255]
    o_s = ttt_linear_attention_sum(x.q.values, x.k.values, x.v.values, x.lr, t_index=idx)
    np.testing.assert_allclose(o_s, o_rec[:, :, idx], rtol=0, atol=1e-12)


def test_planted_index_mistake_is_caught():
    """A recurrence that reads before its own update (an off-by-one in the
    causal mask) must disagree with the inclusive linear-attention sum."""
    q, k, v, lr, _ = _rand(N=11)
    o_wrong, _ = ttt_linear_recurrent(q, k, v, lr, None, include_diag=False)
    o_sum = ttt_linear_attention_sum(q, k, v, lr, None, include_diag=True)
    assert np.abs(o_wrong - o_sum).max() > 1e-3


# ---------------------------------------------------------------- bidirectional order
# Every token writes, then every query reads the final weight: linear attention
# with no causal mask (the xiaoxiang.io post on the KV-binding paper, section
# "线性注意力视角": TTT-KV(X) = X A X^T X B).

@pytest.mark.parametrize("with_s0", [False, True])
def test_bidirectional_equals_unmasked_attention_sum(with_s0):
    q, k, v, lr, S0 = _rand()
    S0 = S0 if with_s0 else None
    o_rec, _ = ttt_linear_recurrent(q, k, v, lr, S0, order="bidirectional")
    o_sum = ttt_linear_attention_sum(q, k, v, lr, S0, order="bidirectional")
    np.testing.assert_allclose(o_rec, o_sum, rtol=0, atol=1e-12 * np.abs(o_sum).max())


def test_bidirectional_constant_lr_is_the_matrix_product_form():
    """With a constant learning rate c and W0 = 0 the layer is c (Q K^T) V,
    the X A X^T X B form with Q = X A, K = X, V = X B (a matmul identity)."""
    r = np.random.default_rng(3)
    X = r.standard_normal((1, 1, 29, 6))
    A = r.standard_normal((6, 6))
    Bm = r.standard_normal((6, 4))
    c = 0.37
    q, k, v = X @ A, X, X @ Bm
    lr = np.full((1, 1, 29), c)
    o, _ = ttt_linear_recurrent(q, k, v, lr, None, order="bidirectional")
    expect = c * (X[0, 0] @ A @ X[0, 0].T @ X[0, 0] @ Bm)
    np.testing.assert_allclose(o[0, 0], expect, rtol=0, atol=1e-12 * np.abs(expect).max())


def test_bidirectional_read_is_a_causal_read_after_the_sequence():
    """o_t equals what the causal recurrence reads for a query q_t appended
    after the whole sequence with a zero update (k = v = 0, eta = 0)."""
    q, k, v, lr, S0 = _rand(N=17)
    o_bi, S_bi = ttt_linear_recurrent(q, k, v, lr, S0, order="bidirectional")
    for t in (0, 5, 16):
        q2 = np.concatenate([q, q[:, :, t:t + 1]], 2)
        k2 = np.concatenate([k, np.zeros_like(k[:, :, :1])], 2)
        v2 = np.concatenate([v, np.zeros_like(v[:, :, :1])], 2)
        lr2 = np.concatenate([lr, np.zeros_like(lr[:, :, :1])], 2)
        o_c, S_c = ttt_linear_recurrent(q2, k2, v2, lr2, S0)
        np.testing.assert_allclose(o_bi[:, :, t], o_c[:, :, -1], rtol=0,
                                   atol=1e-12 * np.abs(o_c).max())
    np.testing.assert_allclose(S_bi, S_c, rtol=0, atol=1e-12 * np.abs(S_c).max())


def test_bidirectional_is_equivariant_under_token_permutation():
    q, k, v, lr, S0 = _rand(N=21)
    perm = np.random.default_rng(5).permutation(21)
    o, S = ttt_linear_recurrent(q, k, v, lr, S0, order="bidirectional")
    o_p, S_p = ttt_linear_recurrent(q[:, :, perm], k[:, :, perm], v[:, :, perm], lr[:, :, perm],
                                    S0, order="bidirectional")
    np.testing.assert_allclose(o_p, o[:, :, perm], rtol=0, atol=1e-12 * np.abs(o).max())
    np.testing.assert_allclose(S_p, S, rtol=0, atol=1e-12 * np.abs(S).max())


def test_planted_causal_mask_in_bidirectional_is_caught():
    """The causal recurrence (a mask left in place) disagrees with the
    unmasked sum everywhere but the last token."""
    q, k, v, lr, _ = _rand(N=13)
    o_causal, _ = ttt_linear_recurrent(q, k, v, lr, None)
    o_sum = ttt_linear_attention_sum(q, k, v, lr, None, order="bidirectional")
    assert np.abs(o_causal[:, :, :-1] - o_sum[:, :, :-1]).max() > 1e-3
    np.testing.assert_allclose(o_causal[:, :, -1], o_sum[:, :, -1], rtol=0, atol=1e-12)

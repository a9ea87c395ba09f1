"""Oracle: linear fast weight with KV binding (test infrastructure only).

Source: "Test-Time Training with KV Binding Is Secretly Linear Attention"
(gist.science summary, section "B. Reformulación Teórica"; podcast transcript
at 7:50-9:39).  A fast weight W (dv x dk) takes, for every token, one gradient
step on the binding loss  l_t(W) = -<W k_t, v_t>  with the token's learning
rate eta_t.  The gradient is -v_t k_t^T, independent of W, so the step is
    W_t = W_{t-1} + eta_t v_t k_t^T,
and the read is o_t = W q_t.  Unrolled, o_t = W_0 q_t + sum_{s<=t} eta_s
(q_t . k_s) v_s: causal linear attention, which is the pages' central claim.

Conventions (readings of the pages, all stated once here):
  * the state handed across calls is S = W^T with shape [dk, dv];
  * ``include_diag=True`` (default): token t reads W after its own update
    (o_t = W_t q_t, inclusive causal mask); ``False`` reads before it;
  * ``order="bidirectional"``: every token's update is applied first and
    every query then reads the final W, o_t = W_N q_t.  This is the unmasked
    form that the xiaoxiang.io post on the KV-binding paper (section
    "线性注意力视角", the linear-attention view) writes as X A X^T X B: linear
    attention with no causal mask.  It is also the linear counterpart of
    the write-then-read order of posed-image sets in the "Test-Time Training
    Done Right" review ("El orden de lectura evita información futura").
    include_diag plays no role there.
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def ttt_linear_recurrent(q, k, v, lr, S0=None, include_diag=True, order="causal"):
    """Token-by-token TTT recurrence (the definition).

    q, k: [B,H,N,dk]; v: [B,H,N,dv]; lr: [B,H,N]; S0: [B,H,dk,dv] or None.
    order: "causal" (each token reads as it goes) or "bidirectional" (every
    token writes, then every query reads the final weight).
    Returns (out [B,H,N,dv] float64, S_end [B,H,dk,dv] float64).
    """
    if order not in ("causal", "bidirectional"):
        raise ValueError(order)
    q, k, v, lr = _f64(q), _f64(k), _f64(v), _f64(lr)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    # W = S^T  (dv x dk) per (b, h)
    W = np.zeros((B, H, dv, dk)) if S0 is None else np.swapaxes(_f64(S0), -1, -2).copy()
    out = np.empty((B, H, N, dv))
    if order == "bidirectional":
        for t in range(N):
            # the same GD step on -<W k_t, v_t> as the causal order, no reads yet
            W += lr[:, :, t, None, None] * (v[:, :, t, :, None] * k[:, :, t, None, :])
        for t in range(N):
            out[:, :, t] = np.einsum("bhij,bhj->bhi", W, q[:, :, t])
        return out, np.swapaxes(W, -1, -2).copy()
    for t in range(N):
        # gradient of -<W k_t, v_t> w.r.t. W is -v_t k_t^T; one GD step of size eta_t
        step = lr[:, :, t, None, None] * (v[:, :, t, :, None] * k[:, :, t, None, :])
        if include_diag:
            W += step
            out[:, :, t] = np.einsum("bhij,bhj->bhi", W, q[:, :, t])
        else:
            out[:, :, t] = np.einsum("bhij,bhj->bhi", W, q[:, :, t])
            W += step
    return out, np.swapaxes(W, -1, -2).copy()


def ttt_linear_attention_sum(q, k, v, lr, S0=None, include_diag=True, t_index=None,
                             order="causal"):
    """The same outputs written as the causal linear-attention sum
        o_t = S0^T q_t + sum_{s <= t (or s < t)} eta_s (q_t . k_s) v_s
    (bidirectional order: the sum runs over every s), evaluated directly for
    the token positions in ``t_index`` (all if None).
    Cost O(|t_index| * N * d); used for sampled checks at full sizes.
    Returns [B,H,len(t_index),dv] float64.
    """
    q, k, v, lr = _f64(q), _f64(k), _f64(v), _f64(lr)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    idx = np.arange(N) if t_index is None else np.asarray(t_index)
    out = np.zeros((B, H, len(idx), dv))
    for j, t in enumerate(idx):
        last = t + 1 if include_diag else t
        if order == "bidirectional":
            last = N
        if last > 0:
            scores = np.einsum("bhd,bhsd->bhs", q[:, :, t], k[:, :, :last]) * lr[:, :, :last]
            out[:, :, j] = np.einsum("bhs,bhsd->bhd", scores, v[:, :, :last])
        if S0 is not None:
            out[:, :, j] += np.einsum("bhij,bhi->bhj", _f64(S0), q[:, :, t])
    return out


def ttt_linear_backward(q, k, v, lr, dout, S0=None, dS_end=None, include_diag=True):
    """Gradients of the recurrence above for the scalar
        L = sum_t <dout_t, o_t> + <dS_end, S_end>
    with respect to q, k, v, lr and S0 (the backward pass of the layer, which
    the pages' training-speed results rely on: "Test-Time Training with KV
    Binding Is Secretly Linear Attention", section "Resultados Experimentales").

    Written as the reverse-time recurrence of the definition.  With
    R_s = dS_end + sum of q_t dout_t^T over the tokens t whose read sees token
    s's update (t >= s inclusive, t > s exclusive), the token's contributions
    are
        dk_s = eta_s R_s v_s,  dv_s = eta_s R_s^T k_s,  dlr_s = k_s^T R_s v_s,
    and the read gives dq_t = S_t dout_t with S_t the state the token read.
    dS0 = R after the first token.

    q, k: [B,H,N,dk]; v, dout: [B,H,N,dv]; lr: [B,H,N]; S0, dS_end:
    [B,H,dk,dv] or None (zeros).  Returns (dq, dk, dv, dlr, dS0) in float64.
    """
    q, k, v, lr, dout = _f64(q), _f64(k), _f64(v), _f64(lr), _f64(dout)
    B, H, N, dk_ = q.shape
    dv_ = v.shape[-1]
    # forward: the state each token's read sees, S = W^T [dk, dv]
    S = np.zeros((B, H, dk_, dv_)) if S0 is None else _f64(S0).copy()
    dq = np.empty((B, H, N, dk_))
    for t in range(N):
        inc = lr[:, :, t, None, None] * (k[:, :, t, :, None] * v[:, :, t, None, :])
        if include_diag:
            S += inc
        # o_t = S^T q_t  =>  d q_t = S dout_t
        dq[:, :, t] = np.einsum("bhij,bhj->bhi", S, dout[:, :, t])
        if not include_diag:
            S += inc
    # reverse: R accumulates the reads' sensitivities to the state
    R = np.zeros((B, H, dk_, dv_)) if dS_end is None else _f64(dS_end).copy()
    dk = np.empty((B, H, N, dk_))
    dv = np.empty((B, H, N, dv_))
    dlr = np.empty((B, H, N))
    for s in range(N - 1, -1, -1):
        read = q[:, :, s, :, None] * dout[:, :, s, None, :]
        if include_diag:
            R += read
        # token s adds eta_s k_s v_s^T to every later state
        Rv = np.einsum("bhij,bhj->bhi", R, v[:, :, s])
        RTk = np.einsum("bhij,bhi->bhj", R, k[:, :, s])
        dk[:, :, s] = lr[:, :, s, None] * Rv
        dv[:, :, s] = lr[:, :, s, None] * RTk
        dlr[:, :, s] = np.einsum("bhi,bhi->bh", k[:, :, s], Rv)
        if not include_diag:
            R += read
    return dq, dk, dv, dlr, R

"""Oracle: causal sliding-window softmax attention and the full LaCT language
layer (test infrastructure only).

Source: "Test-Time Training Done Right" review, sections "Memoria no lineal y
atención local" and "El orden de lectura evita información futura": the
layer combines local (windowed) attention with the fast-weight memory; the
two branches may share Q, K and V and their outputs are summed; in language
modelling the window is causal and slides (2048 tokens for the 760M model,
4096 for the 3B one, "Lenguaje").

Readings (the pages state none of these):
  * a token attends to itself and the window - 1 tokens before it;
  * scores are scaled by 1 / sqrt(d), the usual dot-product scaling;
  * the memory branch is the LaCT layer of ``oracle.lact`` in causal order,
    and the summed output is  window_attention(q, k, v) + lact(q, k, v).
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np


def sliding_window_attention(q, k, v, window, scale=None, t_index=None):
    """o_t = sum over s in (t - window, t] of softmax_s(scale q_t . k_s) v_s.

    q, k: [B,H,N,d]; v: [B,H,N,dv].  Token by token, float64.  With
    ``t_index`` only those positions are computed (sampled checks at full
    sizes); the result is then [B,H,len(t_index),dv].
    """
    B, H, N, d = np.shape(q)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx = range(N) if t_index is None else list(t_index)
    out = np.empty((B, H, len(idx), np.shape(v)[-1]))
    for j, t in enumerate(idx):
        s0 = max(0, t - window + 1)
        qt = np.asarray(q[:, :, t], dtype=np.float64)
        ks = np.asarray(k[:, :, s0:t + 1], dtype=np.float64)
        vs = np.asarray(v[:, :, s0:t + 1], dtype=np.float64)
        scores = scale * np.einsum("bhd,bhsd->bhs", qt, ks)
        scores -= scores.max(axis=-1, keepdims=True)
        p = np.exp(scores)
        p /= p.sum(axis=-1, keepdims=True)
        out[:, :, j] = np.einsum("bhs,bhsd->bhd", p, vs)
    return out


def lact_layer_forward(q, k, v, lr, state, *, chunk, window, scale=None, **lact_kw):
    """The LaCT language layer: causal LaCT memory plus causal sliding-window
    attention on the same q, k, v, outputs summed.  ``state`` (a LaCTState)
    is updated in place.  Returns (out, state)."""
    from .lact import lact_forward
    mem, state = lact_forward(q, k, v, lr, state, chunk=chunk, order="causal", **lact_kw)
    return mem + sliding_window_attention(q, k, v, window, scale), state

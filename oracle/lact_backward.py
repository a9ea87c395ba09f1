"""Oracle: backward pass of the LaCT layer (test infrastructure only).

The layer is training-time machinery in the pages: the language models are
trained end to end through it ("Test-Time Training Done Right" review,
"Lenguaje: calidad y velocidad no son equivalentes", Table 3 training
throughput).  This module gives the gradients of

    L = sum_t <dout_t, out_t> + sum_m <dW_m, W_m(end)>

with respect to q, k, v, the learning rates and the initial fast weights
W1, W3, W2, through the whole chunk loop: every chunk's gradient G depends
on the chunk-start weights and on k, v and lr, and the update, the optional
momentum or Newton-Schulz step and the row normalisation all sit on the
path.

How it computes them: ``lact_forward_torch`` restates the steps of
``oracle.lact.lact_forward`` (same order, same formulas: chunk gradients
written out, GD / momentum / Muon, row normalisation, causal or
bidirectional order) in float64 torch operations, and torch.autograd
differentiates that restatement.  Autograd is the library primitive here;
the restatement is pinned to the numpy oracle, and the gradients to central
differences of the numpy oracle, in tests/test_oracle_lact_backward.py.
"""
from __future__ import annotations

import torch

MASK_W1, MASK_W3, MASK_W2 = 1, 2, 4


def _t(x):
    return torch.as_tensor(x, dtype=torch.float64)


def _silu(x):
    return x * torch.sigmoid(x)


def _silu_prime(x):
    s = torch.sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


def _read(W1, W3, W2, x):
    """o = W2 (silu(W1 x) * (W3 x)) for every token row; [B,H,T,d]."""
    h1 = torch.einsum("bhtd,bhjd->bhtj", x, W1)
    h3 = torch.einsum("bhtd,bhjd->bhtj", x, W3)
    return torch.einsum("bhtj,bhdj->bhtd", _silu(h1) * h3, W2)


def _chunk_gradients(W1, W3, W2, k, v, lr):
    """Sum over the chunk of lr_t * grad_W(-<f_W(k_t), v_t>) at the
    chunk-start weights, written out as in oracle.lact."""
    h1 = torch.einsum("bhtd,bhjd->bhtj", k, W1)
    h3 = torch.einsum("bhtd,bhjd->bhtj", k, W3)
    a = _silu(h1)
    gm = a * h3
    dy = -lr[..., None] * v
    G2 = torch.einsum("bhtd,bhtj->bhdj", dy, gm)
    dg = torch.einsum("bhtd,bhdj->bhtj", dy, W2)
    G3 = torch.einsum("bhtj,bhtd->bhjd", dg * a, k)
    G1 = torch.einsum("bhtj,bhtd->bhjd", dg * h3 * _silu_prime(h1), k)
    return G1, G3, G2


def _newton_schulz(G, steps, coef, eps):
    a, b, c = coef
    X = G / (torch.sqrt(torch.sum(G * G, dim=(-2, -1), keepdim=True)) + eps)
    tall = X.shape[-2] > X.shape[-1]
    if tall:
        X = X.transpose(-2, -1)
    for _ in range(steps):
        A = X @ X.transpose(-2, -1)
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.transpose(-2, -1) if tall else X


def _normalize_rows(W, eps):
    n = torch.sqrt(torch.sum(W * W, dim=-1, keepdim=True))
    return W / torch.clamp_min(n, eps)


def lact_forward_torch(q, k, v, lr, W1, W3, W2, *, chunk, order="causal", opt="gd", beta=0.9,
                       ns_steps=5, ns_coef=(3.4445, -4.7750, 2.0315), ns_eps=1e-7,
                       normalize_rows=True, norm_eps=1e-12, update_mask=7):
    """The layer's forward in float64 torch ops, differentiable end to end.

    q: causal [B,H,N,d], bidirectional [B,H,Nq,d]; k, v [B,H,N,d]; lr
    [B,H,N]; W1, W3 [B,H,dh,d] and W2 [B,H,d,dh] at the start (momentum
    starts at zero).  Returns (out, (W1, W3, W2) at the end).
    """
    B, H, N, d = k.shape
    W = [W1, W3, W2]
    M = [torch.zeros_like(w) for w in W] if opt in ("momentum", "muon") else None
    outs = []
    for t0 in range(0, N, chunk):
        t1 = min(N, t0 + chunk)
        if order == "causal":
            outs.append(_read(W[0], W[1], W[2], q[:, :, t0:t1]))
        G = _chunk_gradients(W[0], W[1], W[2], k[:, :, t0:t1], v[:, :, t0:t1], lr[:, :, t0:t1])
        for i, bit in enumerate((MASK_W1, MASK_W3, MASK_W2)):
            if not update_mask & bit:
                continue
            if opt == "gd":
                U = G[i]
            elif opt == "momentum":
                M[i] = beta * M[i] + G[i]
                U = M[i]
            elif opt == "muon":
                M[i] = beta * M[i] + G[i]
                U = _newton_schulz(M[i], ns_steps, ns_coef, ns_eps)
            else:
                raise ValueError(opt)
            W[i] = W[i] - U
            if normalize_rows:
                W[i] = _normalize_rows(W[i], norm_eps)
    if order == "causal":
        out = torch.cat(outs, dim=2) if outs else torch.zeros_like(q)
    elif order == "bidirectional":
        out = _read(W[0], W[1], W[2], q)
    else:
        raise ValueError(order)
    return out, tuple(W)


def lact_backward(q, k, v, lr, W1, W3, W2, dout, dW_end=None, **kw):
    """Gradients of sum <dout, out> + sum_m <dW_end[m], W_m(end)> with respect
    to (q, k, v, lr, W1, W3, W2), each a float64 numpy array of its input's
    shape.  W1, W3, W2 are per (b, h): [B,H,...].  dW_end: None or a triple
    of [B,H,...] arrays.  Keyword arguments as for lact_forward_torch."""
    xs = [_t(a).clone().requires_grad_(True) for a in (q, k, v, lr, W1, W3, W2)]
    out, Wend = lact_forward_torch(*xs, **kw)
    L = torch.sum(out * _t(dout))
    if dW_end is not None:
        for w, g in zip(Wend, dW_end):
            L = L + torch.sum(w * _t(g))
    grads = torch.autograd.grad(L, xs, allow_unused=True)
    return tuple(torch.zeros_like(x).numpy() if g is None else g.detach().numpy()
                 for x, g in zip(xs, grads))

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

``lact_backward_explicit`` computes the same gradients step by step (read,
row-norm, Newton-Schulz and chunk-gradient vector-Jacobian products, the
momentum carry), the decomposition a backward kernel follows; it is pinned
to ``lact_backward``.
"""
from __future__ import annotations

import numpy as _np
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
    # X0 = G / (||G||_F + eps) is differentiable at G = 0 (derivative I / eps,
    # since eps > 0); the clamp keeps autograd's sqrt finite there and changes
    # the forward value by less than 1e-150
    n = torch.sqrt(torch.clamp_min(torch.sum(G * G, dim=(-2, -1), keepdim=True), 1e-300))
    X = G / (n + eps)
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


# ---------------------------------------------------------------------------
# The same gradients written out step by step (GD, momentum, Muon), float64
# numpy.  This is the list of products a backward kernel computes; it is
# pinned to lact_backward above.
#
# Per token (key k, value v, lr eta) at the chunk-start weights:
#   h1 = W1 k, h3 = W3 k, a = silu(h1), s = silu'(h1), g = a * h3,
#   dy = -eta v, dg = W2^T dy,
#   G2 += dy g^T,  G3 += (dg * a) k^T,  G1 += (dg * h3 * s) k^T.
# For an upstream R = dL/dG the token contributes
#   phi = <R1, G1_t> + <R3, G3_t> + <R2, G2_t>
#       = r2 . g + dg . (a * r3 + h3 * s * r1),   r1 = R1 k, r3 = R3 k, r2 = R2^T dy,
# whose derivatives give the chunk gradient's vector-Jacobian product (the
# second-order term of training through the update):
#   dphi/dh3 = r2 * a + dg * s * r1
#   dphi/dh1 = (r2 * h3 + dg * r3) * s + (dg * h3 * r1) * silu''(h1)
#   dphi/ddg = a * r3 + h3 * s * r1
#   dW1 += dphi/dh1 k^T,  dW3 += dphi/dh3 k^T,  dW2 += dy (dphi/ddg)^T
#   dk   = W1^T dphi/dh1 + W3^T dphi/dh3 + R1^T (dg * h3 * s) + R3^T (dg * a)
#   dphi/ddy = W2 dphi/ddg + R2 g,  dv = -eta dphi/ddy,  deta = -v . dphi/ddy
# silu''(x) = sigma (1 - sigma) (2 + x (1 - 2 sigma)).
# ---------------------------------------------------------------------------


def _sig(x):
    return 1.0 / (1.0 + _np.exp(-x))


def _np_silu(x):
    return x * _sig(x)


def _np_silu1(x):
    s = _sig(x)
    return s * (1.0 + x * (1.0 - s))


def _np_silu2(x):
    s = _sig(x)
    return s * (1.0 - s) * (2.0 + x * (1.0 - 2.0 * s))


def _read_vjp(W1, W3, W2, x, do):
    """Memory read o = W2 (silu(W1 x) * (W3 x)) for rows x [T,d]: returns
    (dW1, dW3, dW2, dx) for the upstream do [T,d]."""
    h1, h3 = x @ W1.T, x @ W3.T
    a = _np_silu(h1)
    g = a * h3
    dg = do @ W2
    dh3 = dg * a
    dh1 = dg * h3 * _np_silu1(h1)
    return dh1.T @ x, dh3.T @ x, do.T @ g, dh1 @ W1 + dh3 @ W3


def _chunk_gradients_np(W1, W3, W2, k, v, lr):
    h1, h3 = k @ W1.T, k @ W3.T
    a, s = _np_silu(h1), _np_silu1(h1)
    dy = -lr[:, None] * v
    dg = dy @ W2
    return ((dg * h3 * s).T @ k, (dg * a).T @ k, dy.T @ (a * h3))


def _chunk_gradient_vjp(W1, W3, W2, k, v, lr, R1, R3, R2):
    """Vector-Jacobian product of the chunk gradient G(W; k, v, lr) with the
    upstream (R1, R3, R2): returns (dW1, dW3, dW2, dk, dv, dlr)."""
    h1, h3 = k @ W1.T, k @ W3.T
    a, s, s2 = _np_silu(h1), _np_silu1(h1), _np_silu2(h1)
    g = a * h3
    dy = -lr[:, None] * v
    dg = dy @ W2                      # rows: W2^T dy
    r1, r3, r2 = k @ R1.T, k @ R3.T, dy @ R2
    d_h3 = r2 * a + dg * s * r1
    d_h1 = (r2 * h3 + dg * r3) * s + (dg * h3 * r1) * s2
    d_dg = a * r3 + h3 * s * r1
    dW1 = d_h1.T @ k
    dW3 = d_h3.T @ k
    dW2 = dy.T @ d_dg
    dk = d_h1 @ W1 + d_h3 @ W3 + (dg * h3 * s) @ R1 + (dg * a) @ R3
    d_dy = d_dg @ W2.T + g @ R2.T
    return dW1, dW3, dW2, dk, -lr[:, None] * d_dy, -_np.sum(v * d_dy, axis=1)


def _newton_schulz_np(G, steps, coef, eps):
    a, b, c = coef
    X = G / (_np.sqrt(_np.sum(G * G)) + eps)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if tall else X


def _newton_schulz_vjp(G, dY, steps, coef, eps):
    """Y = NS(G) (Frobenius normalisation, wide orientation, quintic steps
    X <- a X + (b A + c A^2) X with A = X X^T): the upstream dY taken back to
    G.  Each step's A and B = b A + c A^2 are symmetric, so
        dX_prev = a dX + B dX + (dA + dA^T) X,  dB = dX X^T,
        dA = b dB + c (dB A + A dB);
    the normalisation X0 = G / (n + eps), n = ||G||_F, gives
        dG = dX0 / (n + eps) - G <dX0, G> / (n (n + eps)^2)."""
    a, b, c = coef
    n = _np.sqrt(_np.sum(G * G))
    X = G / (n + eps)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X, dY = X.T, dY.T
    xs = []
    for _ in range(steps):
        xs.append(X)
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    dX = dY
    for X in reversed(xs):
        A = X @ X.T
        Bm = b * A + c * (A @ A)
        dB = dX @ X.T
        dA = b * dB + c * (dB @ A + A @ dB)
        dX = a * dX + Bm @ dX + (dA + dA.T) @ X
    if tall:
        dX = dX.T
    # at G = 0 the second term's limit is 0 (|G| |G| / n -> 0)
    corr = 0.0 if n == 0 else _np.sum(dX * G) / (n * (n + eps) ** 2)
    return dX / (n + eps) - G * corr


def _norm_rows_vjp(U, dW, eps):
    """W = U / max(||U_row||, eps): the upstream dW taken back to U."""
    n = _np.sqrt(_np.sum(U * U, axis=-1, keepdims=True))
    big = n > eps
    w = U / _np.where(big, n, eps)
    proj = _np.sum(w * dW, axis=-1, keepdims=True)
    return _np.where(big, (dW - w * proj) / _np.where(big, n, 1.0), dW / eps)


def lact_backward_explicit(q, k, v, lr, W1, W3, W2, dout, dW_end=None, *, chunk,
                           order="causal", opt="gd", beta=0.9, ns_steps=5,
                           ns_coef=(3.4445, -4.7750, 2.0315), ns_eps=1e-7, normalize_rows=True,
                           norm_eps=1e-12, update_mask=7):
    """The gradients of lact_backward, computed by the steps above (GD,
    momentum and Muon).  Same arguments and results."""
    if opt not in ("gd", "momentum", "muon"):
        raise ValueError(opt)
    f = lambda a: _np.asarray(a, dtype=_np.float64)  # noqa: E731
    q, k, v, lr, dout = f(q), f(k), f(v), f(lr), f(dout)
    W0 = [f(W1), f(W3), f(W2)]
    B, H, N, d = k.shape
    grads = [_np.zeros_like(q), _np.zeros_like(k), _np.zeros_like(v), _np.zeros_like(lr)] + \
        [_np.zeros_like(w) for w in W0]
    bits = (MASK_W1, MASK_W3, MASK_W2)
    for b in range(B):
        for h in range(H):
            # forward, keeping the chunk-start weights and pre-normalisation updates
            W = [w[b, h].copy() for w in W0]
            M = [_np.zeros_like(w) for w in W]
            saved = []
            for t0 in range(0, N, chunk):
                t1 = min(N, t0 + chunk)
                G = _chunk_gradients_np(*W, k[b, h, t0:t1], v[b, h, t0:t1], lr[b, h, t0:t1])
                start = [w.copy() for w in W]
                Us = [None] * 3
                Ms = [None] * 3
                for i in range(3):
                    if not update_mask & bits[i]:
                        continue
                    if opt == "momentum":
                        M[i] = beta * M[i] + G[i]
                        U = W[i] - M[i]
                    elif opt == "muon":
                        M[i] = beta * M[i] + G[i]
                        Ms[i] = M[i].copy()
                        U = W[i] - _newton_schulz_np(M[i], ns_steps, ns_coef, ns_eps)
                    else:
                        U = W[i] - G[i]
                    Us[i] = U
                    W[i] = _normalize_rows_np(U, norm_eps) if normalize_rows else U
                saved.append((t0, t1, start, Us, Ms))
            # reverse
            dW = [_np.zeros_like(w) for w in W] if dW_end is None else \
                [f(g)[b, h].copy() for g in dW_end]
            if order == "bidirectional":
                r = _read_vjp(*W, q[b, h], dout[b, h])
                for i in range(3):
                    dW[i] += r[i]
                grads[0][b, h] = r[3]
            dM = [_np.zeros_like(w) for w in W]
            for t0, t1, start, Us, Ms in reversed(saved):
                R = [_np.zeros_like(w) for w in W]
                for i in range(3):
                    if Us[i] is None:
                        continue
                    dU = _norm_rows_vjp(Us[i], dW[i], norm_eps) if normalize_rows else dW[i]
                    if opt == "momentum":
                        dM[i] = dM[i] - dU      # U = W - M
                        R[i] = dM[i]            # M = beta M_prev + G
                        dM[i] = beta * dM[i]
                    elif opt == "muon":         # U = W - NS(M)
                        dM[i] = dM[i] + _newton_schulz_vjp(Ms[i], -dU, ns_steps, ns_coef, ns_eps)
                        R[i] = dM[i]
                        dM[i] = beta * dM[i]
                    else:
                        R[i] = -dU              # U = W - G
                    dW[i] = dU                  # U = W_start - ...
                vj = _chunk_gradient_vjp(*start, k[b, h, t0:t1], v[b, h, t0:t1], lr[b, h, t0:t1],
                                         *R)
                for i in range(3):
                    dW[i] = dW[i] + vj[i]
                grads[1][b, h, t0:t1] += vj[3]
                grads[2][b, h, t0:t1] += vj[4]
                grads[3][b, h, t0:t1] += vj[5]
                if order == "causal":
                    r = _read_vjp(*start, q[b, h, t0:t1], dout[b, h, t0:t1])
                    for i in range(3):
                        dW[i] = dW[i] + r[i]
                    grads[0][b, h, t0:t1] = r[3]
            for i in range(3):
                grads[4 + i][b, h] = dW[i]
    return tuple(grads)


def _normalize_rows_np(W, eps):
    n = _np.sqrt(_np.sum(W * W, axis=-1, keepdims=True))
    return W / _np.maximum(n, eps)

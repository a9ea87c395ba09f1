"""Oracle: large-chunk test-time training (LaCT) with a SwiGLU fast-weight
memory (test infrastructure only; float64 numpy).

Sources, "Test-Time Training Done Right" review (iplexlaw page):
  * section "Memoria no lineal y atención local": the memory is a SwiGLU MLP
    with three matrices; a negative inner-product loss binds the memory's
    output for each key to its value; the chunk's gradients are summed with
    per-token learning rates; the optimizer is GD, momentum or Muon (Newton-
    Schulz iterations on the matrix gradient); the weights are L2-normalised
    after the update.
  * section "El orden de lectura evita información futura": for language the
    current chunk reads the memory of earlier chunks and only then updates it;
    for posed images the input set is written first and the target queried
    afterwards.
  * section "Pesos rápidos para recordar el contexto": chunks of 2K up to ~1M
    tokens.

Notation.  Per (b, h): W1, W3 in R^{dh x d}, W2 in R^{d x dh},
    f_W(x) = W2 (silu(W1 x) * (W3 x)),    l_t(W) = -<f_W(k_t), v_t>.
The chunk gradient is  G = sum_{t in chunk} eta_t grad_W l_t(W)  with every
term taken at the chunk-start weights W.  Written out (rows are tokens):
    H1 = K W1^T, H3 = K W3^T, A = silu(H1), Gm = A * H3
    dY = -diag(eta) V                      (d l / d f, lr-weighted)
    G2 = dY^T Gm                           (d x dh)
    dG = dY W2                             (C x dh)
    G3 = (dG * A)^T K                      (dh x d)
    G1 = (dG * H3 * silu'(H1))^T K         (dh x d)
Readings where the pages are silent (each is also listed in the design notes):
  * normalisation rescales every row (first index as stored) of each updated
    matrix to unit L2 norm, W[i,:] /= max(||W[i,:]||, norm_eps); the initial
    weights are not normalised;
  * momentum: M <- beta M + G, U = M (no dampening, no Nesterov, M0 = 0);
  * Muon: U = NS(M) with the quintic Newton-Schulz map below and no extra
    scale, so W <- W - NS(M);
  * a short last chunk is processed as a shorter chunk (no padding);
  * bidirectional order: all input chunks update, then the queries read the
    final weights; only the queries produce output.
"""
from __future__ import annotations

import dataclasses
import numpy as np

MASK_W1, MASK_W3, MASK_W2 = 1, 2, 4

# Token blocks for accumulating the (very long) chunk sums; the sum itself is
# the definition -- the block size only bounds the oracle's memory.
_TOKEN_BLOCK = 16384


def silu(x):
    return x / (1.0 + np.exp(-x))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu_prime(x):
    """d/dx [x * sigmoid(x)] = sigmoid(x) * (1 + x * (1 - sigmoid(x)))."""
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


@dataclasses.dataclass
class LaCTState:
    W1: np.ndarray          # [B,H,dh,d] float64
    W3: np.ndarray          # [B,H,dh,d]
    W2: np.ndarray          # [B,H,d,dh]
    M1: np.ndarray | None = None
    M3: np.ndarray | None = None
    M2: np.ndarray | None = None

    def copy(self):
        c = lambda a: None if a is None else a.copy()  # noqa: E731
        return LaCTState(c(self.W1), c(self.W3), c(self.W2), c(self.M1), c(self.M3), c(self.M2))


def lact_read(W1, W3, W2, x):
    """Memory read o = W2 (silu(W1 x) * (W3 x)) for every row x of ``x``.
    W1, W3: [dh,d]; W2: [d,dh]; x: [T,d] -> [T,d]."""
    h1 = x @ W1.T
    h3 = x @ W3.T
    return (silu(h1) * h3) @ W2.T


def lact_chunk_gradients(W1, W3, W2, k, v, lr):
    """Sum over the chunk's tokens of eta_t * grad_W (-<f_W(k_t), v_t>), each
    gradient at the chunk-start weights.  k, v: [C,d]; lr: [C].
    Returns (G1 [dh,d], G3 [dh,d], G2 [d,dh])."""
    dh, d = W1.shape
    G1 = np.zeros((dh, d))
    G3 = np.zeros((dh, d))
    G2 = np.zeros((d, dh))
    for s in range(0, k.shape[0], _TOKEN_BLOCK):
        kb, vb, eb = k[s:s + _TOKEN_BLOCK], v[s:s + _TOKEN_BLOCK], lr[s:s + _TOKEN_BLOCK]
        h1 = kb @ W1.T
        h3 = kb @ W3.T
        a = silu(h1)
        gm = a * h3
        dy = -eb[:, None] * vb
        G2 += dy.T @ gm
        dg = dy @ W2
        G3 += (dg * a).T @ kb
        G1 += (dg * h3 * silu_prime(h1)).T @ kb
    return G1, G3, G2


def newton_schulz(G, steps=5, coef=(3.4445, -4.7750, 2.0315), eps=1e-7):
    """Quintic Newton-Schulz orthogonalisation used by Muon (K. Jordan, 2024):
        X = G / (||G||_F + eps); work on the wide orientation (rows <= cols);
        repeat: A = X X^T;  X <- a X + (b A + c A A) X.
    Each step applies p(s) = a s + b s^3 + c s^5 to every singular value while
    keeping the singular vectors.  G: [r, c] -> [r, c]."""
    a, b, c = coef
    X = G / (np.sqrt(np.sum(G * G)) + eps)
    tall = X.shape[0] > X.shape[1]
    if tall:
        X = X.T
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if tall else X


def _normalize_rows(W, eps):
    n = np.sqrt(np.sum(W * W, axis=-1, keepdims=True))
    return W / np.maximum(n, eps)


def _broadcast_w(W, B):
    W = np.asarray(W, dtype=np.float64)
    if W.ndim == 3:                       # [H,...] shared across the batch
        W = np.broadcast_to(W[None], (B,) + W.shape)
    return np.array(W, dtype=np.float64)


def lact_init_state(W1, W3, W2, B, opt="gd"):
    st = LaCTState(_broadcast_w(W1, B), _broadcast_w(W3, B), _broadcast_w(W2, B))
    if opt in ("momentum", "muon"):
        st.M1, st.M3, st.M2 = np.zeros_like(st.W1), np.zeros_like(st.W3), np.zeros_like(st.W2)
    return st


def lact_forward(q, k, v, lr, state: LaCTState, *, chunk, order="causal", opt="gd",
                 beta=0.9, ns_steps=5, ns_coef=(3.4445, -4.7750, 2.0315), ns_eps=1e-7,
                 normalize_rows=True, norm_eps=1e-12, update_mask=7):
    """One call of the layer over a sequence.

    q: causal -> [B,H,N,d] (same tokens as k); bidirectional -> [B,H,Nq,d].
    k, v: [B,H,N,d]; lr: [B,H,N].  ``state`` is updated in place and returned.
    Returns (out, state): out is [B,H,N,d] (causal) or [B,H,Nq,d] (bidir).
    """
    if chunk <= 0:
        raise ValueError("chunk must be positive")
    q, k, v, lr = (np.asarray(x, dtype=np.float64) for x in (q, k, v, lr))
    B, H, N, d = k.shape
    out = np.zeros(q.shape)
    for b in range(B):
        for h in range(H):
            W = [state.W1[b, h], state.W3[b, h], state.W2[b, h]]
            Ms = None if state.M1 is None else [state.M1[b, h], state.M3[b, h], state.M2[b, h]]
            for t0 in range(0, N, chunk):
                t1 = min(N, t0 + chunk)
                if order == "causal":
                    # read the memory left by earlier chunks, then update
                    out[b, h, t0:t1] = lact_read(W[0], W[1], W[2], q[b, h, t0:t1])
                G = lact_chunk_gradients(W[0], W[1], W[2], k[b, h, t0:t1], v[b, h, t0:t1],
                                         lr[b, h, t0:t1])
                for i, bit in enumerate((MASK_W1, MASK_W3, MASK_W2)):
                    if not update_mask & bit:
                        continue
                    if opt == "gd":
                        U = G[i]
                    elif opt == "momentum":
                        Ms[i][...] = beta * Ms[i] + G[i]
                        U = Ms[i]
                    elif opt == "muon":
                        Ms[i][...] = beta * Ms[i] + G[i]
                        U = newton_schulz(Ms[i], ns_steps, ns_coef, ns_eps)
                    else:
                        raise ValueError(opt)
                    W[i][...] = W[i] - U
                    if normalize_rows:
                        W[i][...] = _normalize_rows(W[i], norm_eps)
            if order == "bidirectional":
                out[b, h] = lact_read(W[0], W[1], W[2], q[b, h])
            elif order != "causal":
                raise ValueError(order)
    return out, state

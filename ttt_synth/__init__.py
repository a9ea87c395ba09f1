"""Seeded synthetic inputs for the TTT-KV fast-weight layer.

This module only draws random numbers and shapes them into the token tensors
and initial fast weights that the layer consumes.  It contains none of the
layer's arithmetic: no recurrence, no attention, no gradient, no optimizer.
Both the CPU oracle (through the tests and the bench's CPU baseline) and the
GPU path receive the very same bytes from here.

Recipe (one PCG64 stream per tensor): ``numpy.random.default_rng([cfg, tid])``
with ``tid`` 0:q 1:k 2:v 3:lr 4:W1 5:W3 6:W2 7:dout 8:dS_end (or dW1_end)
9:dW3_end 10:dW2_end (the output and end-state gradients a backward pass
receives); float32 draws; per-token L2
normalisation where the workload says so; a single round-to-nearest-even cast
to bfloat16 for bf16 workloads.  The workloads mirror the pages' settings:
the linear fast weight of "Test-Time Training with KV Binding Is Secretly
Linear Attention" (section "Reformulación Teórica") and the LaCT language
(32K tokens), 48-view and 128-view novel-view-synthesis settings of "Test-Time
Training Done Right" (sections "Síntesis de vistas" and "Lenguaje").
"""
from __future__ import annotations

import dataclasses
import numpy as np

TID_Q, TID_K, TID_V, TID_LR, TID_W1, TID_W3, TID_W2, TID_DOUT, TID_DSEND, TID_DW3, TID_DW2 = range(11)


# ---------------------------------------------------------------- bf16 bits
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- draws
def _rng(cfg: int, tid: int, seed: int = 0) -> np.random.Generator:
    key = [cfg, tid] if seed == 0 else [cfg, tid, seed]
    return np.random.default_rng(key)


def _normal(cfg, tid, shape, seed=0, mean=0.0):
    x = _rng(cfg, tid, seed).standard_normal(size=shape, dtype=np.float32)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def _l2_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _sigmoid(x):
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _softplus(x):
    x = x.astype(np.float64)
    return (np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x)))).astype(np.float32)


# ---------------------------------------------------------------- containers
@dataclasses.dataclass
class TokenTensor:
    """A token tensor as delivered to both sides: float32 values that are
    exactly representable in ``dtype`` plus, for bf16, the raw bits."""
    values: np.ndarray            # float32, exact values the layer consumes
    bits: np.ndarray | None       # uint16 bf16 bits (None for fp32 tensors)
    dtype: str                    # "f32" | "bf16"


def _token(x: np.ndarray, dtype: str) -> TokenTensor:
    if dtype == "bf16":
        bits = f32_to_bf16_bits(x)
        return TokenTensor(bf16_bits_to_f32(bits), bits, "bf16")
    return TokenTensor(np.ascontiguousarray(x, dtype=np.float32), None, "f32")


@dataclasses.dataclass
class LinearInputs:
    q: TokenTensor
    k: TokenTensor
    v: TokenTensor
    lr: np.ndarray                # float32 [B,H,N]
    S0: np.ndarray | None         # float32 [B,H,dk,dv] or None (zeros)
    chunk: int


@dataclasses.dataclass
class LaCTInputs:
    q: TokenTensor                # causal: [B,H,N,d]; bidirectional: [B,H,Nq,d]
    k: TokenTensor
    v: TokenTensor
    lr: np.ndarray                # float32 [B,H,N]
    W1: np.ndarray                # float32 [H,dh,d]  (identical across B)
    W3: np.ndarray                # float32 [H,dh,d]
    W2: np.ndarray                # float32 [H,d,dh]
    chunk: int
    order: str                    # "causal" | "bidirectional"


# ---------------------------------------------------------------- generic makers
def make_linear_inputs(B, H, N, dk, dv, *, chunk, dtype, lr_kind, cfg=100, seed=0,
                       with_S0=False) -> LinearInputs:
    """q, k ~ N(0,1) L2-normalised per token, v ~ N(0,1); lr_kind picks the
    per-token learning-rate distribution ("0.1sig" or "sig-2")."""
    q = _l2_rows(_normal(cfg, TID_Q, (B, H, N, dk), seed))
    k = _l2_rows(_normal(cfg, TID_K, (B, H, N, dk), seed))
    v = _normal(cfg, TID_V, (B, H, N, dv), seed)
    z = _normal(cfg, TID_LR, (B, H, N), seed)
    if lr_kind == "0.1sig":
        lr = np.float32(0.1) * _sigmoid(z)
    elif lr_kind == "sig-2":
        lr = _sigmoid(z - np.float32(2.0))
    else:
        raise ValueError(lr_kind)
    S0 = None
    if with_S0:
        S0 = 0.1 * _normal(cfg, TID_W1, (B, H, dk, dv), seed)
    return LinearInputs(_token(q, dtype), _token(k, dtype), _token(v, dtype),
                        np.ascontiguousarray(lr, np.float32), S0, chunk)


@dataclasses.dataclass
class LinearGrads:
    dout: TokenTensor             # [B,H,N,dv], the dtype of the layer's inputs
    dS_end: np.ndarray            # float32 [B,H,dk,dv]


def make_linear_grads(x: LinearInputs, *, cfg=100, seed=0) -> LinearGrads:
    """Upstream gradients for a backward pass over ``x``: dout ~ N(0,1) in
    the inputs' dtype and dS_end ~ 0.1 N(0,1)."""
    B, H, N, dk = x.q.values.shape
    dv = x.v.values.shape[-1]
    dout = _normal(cfg, TID_DOUT, (B, H, N, dv), seed)
    dS_end = np.float32(0.1) * _normal(cfg, TID_DSEND, (B, H, dk, dv), seed)
    return LinearGrads(_token(dout, x.q.dtype), dS_end)


@dataclasses.dataclass
class LaCTGrads:
    dout: TokenTensor             # [B,H,R,d] bf16 (R: the output rows of the layer)
    dW_end: tuple                 # float32 ([B,H,dh,d], [B,H,dh,d], [B,H,d,dh])


def make_lact_grads(x: LaCTInputs, *, cfg=200, seed=0) -> LaCTGrads:
    """Upstream gradients for a backward pass over ``x``: dout ~ N(0,1) (bf16)
    and dW_end ~ 0.1 N(0,1) per weight (ids 8, 9, 10)."""
    B, H, R, d = x.q.values.shape
    dh = x.W1.shape[-2]
    dout = _normal(cfg, TID_DOUT, (B, H, R, d), seed)
    dW = tuple(np.float32(0.1) * _normal(cfg, tid, shp, seed) for tid, shp in
               ((TID_DSEND, (B, H, dh, d)), (TID_DW3, (B, H, dh, d)), (TID_DW2, (B, H, d, dh))))
    return LaCTGrads(_token(dout, "bf16"), dW)


def make_lact_inputs(B, H, N, d, dh, *, chunk, order, Nq=None, qk_norm=True,
                     v_norm=False, lr_kind="0.01softplus", cfg=200, seed=0,
                     dtype="bf16") -> LaCTInputs:
    """Token tensors and SwiGLU fast weights W ~ N(0, std = 1/sqrt(fan_in))."""
    nq = N if order == "causal" else (Nq if Nq is not None else N)
    q = _normal(cfg, TID_Q, (B, H, nq, d), seed)
    k = _normal(cfg, TID_K, (B, H, N, d), seed)
    v = _normal(cfg, TID_V, (B, H, N, d), seed)
    if qk_norm:
        q, k = _l2_rows(q), _l2_rows(k)
    if v_norm:
        v = _l2_rows(v)
    z = _normal(cfg, TID_LR, (B, H, N), seed)
    if lr_kind == "0.01softplus":
        lr = np.float32(0.01) * _softplus(z)
    elif lr_kind == "0.01sig":
        lr = np.float32(0.01) * _sigmoid(z)
    else:
        raise ValueError(lr_kind)
    W1 = _normal(cfg, TID_W1, (H, dh, d), seed) * np.float32(1.0 / np.sqrt(d))
    W3 = _normal(cfg, TID_W3, (H, dh, d), seed) * np.float32(1.0 / np.sqrt(d))
    W2 = _normal(cfg, TID_W2, (H, d, dh), seed) * np.float32(1.0 / np.sqrt(dh))
    return LaCTInputs(_token(q, dtype), _token(k, dtype), _token(v, dtype),
                      np.ascontiguousarray(lr, np.float32),
                      W1.astype(np.float32), W3.astype(np.float32), W2.astype(np.float32),
                      chunk, order)


# ---------------------------------------------------------------- named workloads
# The five workloads, with their sizes.  ``small`` variants keep every
# property (dtype, distributions, chunk structure incl. a ragged last chunk)
# at sizes the CPU oracle finishes in seconds.
WORKLOADS = {
    "ttt_linear_f32_n256": dict(kind="linear", B=1, H=2, N=256, dk=32, dv=32, chunk=16,
                                dtype="f32", lr_kind="0.1sig", cfg=1),
    "ttt_linear_bf16_n32k": dict(kind="linear", B=4, H=16, N=32768, dk=64, dv=64, chunk=64,
                                 dtype="bf16", lr_kind="sig-2", cfg=2),
    # backward pass of the 32K linear layer (upstream gradients from make_linear_grads)
    "ttt_linear_bwd_bf16_n32k": dict(kind="linear", B=4, H=16, N=32768, dk=64, dv=64, chunk=64,
                                     dtype="bf16", lr_kind="sig-2", cfg=2, backward=True),
    "lact_causal_n32k": dict(kind="lact", B=2, H=4, N=32768, d=128, dh=256, chunk=2048,
                             order="causal", qk_norm=True, v_norm=False,
                             lr_kind="0.01softplus", opt="gd", cfg=3),
    # the 32K causal shape with only W2 updated (plain GD, no row norm): the
    # layer is block-causal linear attention on silu(W1 x) * (W3 x)
    "lact_w2only_causal_n32k": dict(kind="lact", B=2, H=4, N=32768, d=128, dh=256, chunk=2048,
                                    order="causal", qk_norm=True, v_norm=False,
                                    lr_kind="0.01softplus", opt="gd", update_mask=4,
                                    normalize_rows=False, cfg=3),
    # the backward pass of that layer (upstream gradients from make_lact_grads)
    "lact_bwd_causal_n32k": dict(kind="lact", B=2, H=4, N=32768, d=128, dh=256, chunk=2048,
                                 order="causal", qk_norm=True, v_norm=False,
                                 lr_kind="0.01softplus", opt="gd", backward=True, cfg=3),
    # the full language layer at that shape: memory + causal sliding-window
    # attention with the 760M model's 2048-token window ("Lenguaje")
    "lact_layer_causal_n32k": dict(kind="lact", B=2, H=4, N=32768, d=128, dh=256, chunk=2048,
                                   order="causal", qk_norm=True, v_norm=False,
                                   lr_kind="0.01softplus", opt="gd", window=2048, cfg=3),
    "lact_bidir_196k": dict(kind="lact", B=1, H=2, N=196608, Nq=4096, d=384, dh=768,
                            chunk=196608, order="bidirectional", qk_norm=True, v_norm=True,
                            lr_kind="0.01sig", opt="gd", cfg=4),
    "lact_bidir_muon_1m": dict(kind="lact", B=1, H=2, N=1029120, Nq=8040, d=384, dh=768,
                               chunk=65536, order="bidirectional", qk_norm=True, v_norm=True,
                               lr_kind="0.01sig", opt="muon", beta=0.9, ns_steps=5,
                               cfg=5),
    # the first two 64K chunks of that scene: the same kernels on a case small
    # enough to profile (a few hundred MB on the device)
    "lact_bidir_muon_128k": dict(kind="lact", B=1, H=2, N=131072, Nq=8040, d=384, dh=768,
                                 chunk=65536, order="bidirectional", qk_norm=True, v_norm=True,
                                 lr_kind="0.01sig", opt="muon", beta=0.9, ns_steps=5,
                                 cfg=5),
}


def make_workload(name: str, **overrides):
    w = dict(WORKLOADS[name])
    w.update(overrides)
    kind = w.pop("kind")
    if kind == "linear":
        return make_linear_inputs(w["B"], w["H"], w["N"], w["dk"], w["dv"], chunk=w["chunk"],
                                  dtype=w["dtype"], lr_kind=w["lr_kind"], cfg=w["cfg"],
                                  seed=w.get("seed", 0))
    return make_lact_inputs(w["B"], w["H"], w["N"], w["d"], w["dh"], chunk=w["chunk"],
                            order=w["order"], Nq=w.get("Nq"), qk_norm=w["qk_norm"],
                            v_norm=w["v_norm"], lr_kind=w["lr_kind"], cfg=w["cfg"],
                            seed=w.get("seed", 0))

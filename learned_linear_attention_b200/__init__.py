"""B200 (sm_100a) TTT-KV fast-weight layer.

The compute lives in ``libttt_b200.so`` (hand-written CUDA for sm_100a behind
the C ABI of ``include/ttt.h``).  This package is its Python binding: the
functions below have the same names as the C entry points and only marshal
arguments; ``make_*_desc`` and ``alloc_*`` are conveniences that fill the
descriptor structs and allocate caller-owned device buffers with PyTorch.
"""
from __future__ import annotations

from ._lib import (  # noqa: F401
    LIB_PATH, TTT_BF16, TTT_BIDIRECTIONAL, TTT_CAUSAL, TTT_ERR_ALIGN, TTT_ERR_ARG, TTT_ERR_CUDA,
    TTT_ERR_DTYPE, TTT_ERR_SHAPE, TTT_ERR_TIMEOUT, TTT_ERR_UNSUPPORTED, TTT_ERR_WORKSPACE,
    TTT_F32, TTT_OK, TTT_OPT_GD, TTT_OPT_MOMENTUM, TTT_OPT_MUON, TTT_STATUS_BYTES, TTTError,
    lact_apply_grad, lact_bwd_workspace_bytes, lact_chunk_bwd, lact_chunk_fwd, lact_chunk_fwd_noalloc, lact_chunk_grad, lact_grad_bytes,
    lact_noalloc_check_status, lact_desc, lact_read,
    lact_layer_fwd, ttt_window_attn_fwd,
    ttt_window_desc, lact_state_bytes, lact_state_init, lact_state_readout,
    lact_workspace_bytes, lact_workspace_bytes_min, load, status_string, ttt_build_info, ttt_check_device_status,
    ttt_linear_bwd, ttt_linear_bwd_workspace_bytes, ttt_linear_desc, ttt_linear_fwd,
    ttt_linear_state_init, ttt_linear_state_readout,
    ttt_linear_workspace_bytes, ttt_profile_begin, ttt_profile_end, ttt_selftest_wait_timeout)

_DT = {"f32": TTT_F32, "fp32": TTT_F32, "bf16": TTT_BF16}
_ORDER = {"causal": TTT_CAUSAL, "bidirectional": TTT_BIDIRECTIONAL}
_OPT = {"gd": TTT_OPT_GD, "momentum": TTT_OPT_MOMENTUM, "muon": TTT_OPT_MUON}


def make_linear_desc(B, H, N, dk, dv, chunk, include_diag=True, in_dtype="bf16",
                     out_dtype="f32", order="causal") -> ttt_linear_desc:
    return ttt_linear_desc(B, H, N, dk, dv, chunk, _ORDER[order], int(bool(include_diag)),
                           _DT[in_dtype], _DT[out_dtype])


def make_lact_desc(B, H, N_in, d, dh, chunk, *, N_q=None, order="causal", opt="gd", beta=0.9,
                   ns_steps=5, ns_coef=(3.4445, -4.7750, 2.0315), ns_eps=1e-7,
                   normalize_rows=True, norm_eps=1e-12, update_mask=7,
                   out_dtype="f32", split_operands=None) -> lact_desc:
    """Fill a lact_desc.  split_operands defaults to on for Muon (its update
    amplifies bf16 operand rounding) and off otherwise."""
    nq = N_in if order == "causal" else (N_q if N_q is not None else 0)
    desc = lact_desc()
    desc.B, desc.H, desc.N_in, desc.N_q, desc.d, desc.dh, desc.chunk = B, H, N_in, nq, d, dh, chunk
    desc.order, desc.opt, desc.beta, desc.ns_steps = _ORDER[order], _OPT[opt], beta, ns_steps
    for i in range(3):
        desc.ns_coef[i] = ns_coef[i]
    desc.ns_eps, desc.normalize_rows, desc.norm_eps = ns_eps, int(bool(normalize_rows)), norm_eps
    desc.update_mask, desc.in_dtype, desc.out_dtype = update_mask, TTT_BF16, _DT[out_dtype]
    desc.split_operands = int(opt == "muon") if split_operands is None else int(bool(split_operands))
    return desc


def make_window_desc(B, H, N, d, window, *, scale=0.0, out_dtype="f32",
                     accumulate=False) -> ttt_window_desc:
    """Fill a ttt_window_desc (bf16 q, k, v; scale <= 0 selects 1/sqrt(d))."""
    return ttt_window_desc(B, H, N, d, window, scale, TTT_BF16, _DT[out_dtype],
                           int(bool(accumulate)))


def alloc_workspace(nbytes: int, device="cuda"):
    """Zero-filled byte workspace (the status block must start zeroed)."""
    import torch
    return torch.zeros(max(int(nbytes), TTT_STATUS_BYTES), dtype=torch.uint8, device=device)


def alloc_lact_state(desc: lact_desc, device="cuda"):
    import torch
    return torch.empty(lact_state_bytes(desc) // 4, dtype=torch.float32, device=device)

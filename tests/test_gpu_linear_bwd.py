"""GPU parity for the backward pass of the linear fast weight against the
fp64 oracle (the reverse-time recurrence, pinned to central differences),
through the C ABI.

The CUDA path computes every gradient as a forward-time scan with the roles
of q, k, v and dout exchanged, on the forward kernels.  Tolerances as for the
forward pass (normwise max relative error): 1e-4 for fp32 inputs (CUDA-core
kernel), 2e-2 for bf16 inputs with fp32 accumulation (tensor-core kernel)."""
import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from oracle import ttt_linear_backward
from ttt_synth import make_linear_grads, make_linear_inputs, make_workload
from gpu_util import rel_err, to_dev

pytestmark = pytest.mark.gpu
TOL_F32, TOL_BF16 = 1e-4, 2e-2
NAMES = ("dq", "dk", "dv", "dlr", "dS0")


def run_bwd(x, g, include_diag=True, S0=None, with_dS_end=True):
    B, H, N, dk = x.q.values.shape
    dv = x.v.values.shape[-1]
    desc = T.make_linear_desc(B, H, N, dk, dv, x.chunk, include_diag, in_dtype=x.q.dtype,
                              out_dtype="f32")
    q, k, v, dout = to_dev(x.q), to_dev(x.k), to_dev(x.v), to_dev(g.dout)
    lr = torch.from_numpy(x.lr).cuda()
    S0d = None if S0 is None else torch.from_numpy(np.asarray(S0, np.float32)).cuda()
    dSe = torch.from_numpy(g.dS_end).cuda() if with_dS_end else None
    nan = float("nan")
    outs = [torch.full(s, nan, device="cuda") for s in
            ((B, H, N, dk), (B, H, N, dk), (B, H, N, dv), (B, H, N), (B, H, dk, dv))]
    ws = T.alloc_workspace(T.ttt_linear_bwd_workspace_bytes(desc))
    T.ttt_linear_bwd(desc, q, k, v, lr, S0d, dout, dSe, *outs, ws)
    assert T.ttt_check_device_status(ws) == T.TTT_OK
    return [o.cpu().numpy() for o in outs]


def oracle_bwd(x, g, include_diag=True, S0=None, with_dS_end=True, heads=None):
    sel = (lambda a: a) if heads is None else (lambda a: np.stack([a[b, h] for b, h in heads])[None])
    return ttt_linear_backward(sel(x.q.values), sel(x.k.values), sel(x.v.values), sel(x.lr),
                               sel(g.dout.values), None if S0 is None else sel(S0),
                               sel(g.dS_end) if with_dS_end else None, include_diag)


def _compare(got, ref, tol):
    for name, a, r in zip(NAMES, got, ref):
        assert not np.isnan(a).any(), name
        assert rel_err(a, r) <= tol, (name, rel_err(a, r))


def test_f32_n256_workload(cuda_device):
    x = make_workload("ttt_linear_f32_n256")
    g = make_linear_grads(x, cfg=1)
    _compare(run_bwd(x, g), oracle_bwd(x, g), TOL_F32)


@pytest.mark.parametrize("include_diag", [True, False])
def test_f32_ragged_unequal_dims_with_states(cuda_device, include_diag):
    x = make_linear_inputs(2, 3, 77, 24, 40, chunk=9, dtype="f32", lr_kind="0.1sig", cfg=61,
                           with_S0=True)
    g = make_linear_grads(x, cfg=61)
    _compare(run_bwd(x, g, include_diag, S0=x.S0), oracle_bwd(x, g, include_diag, S0=x.S0),
             TOL_F32)


def test_f32_without_end_state_gradient(cuda_device):
    x = make_linear_inputs(1, 2, 50, 16, 16, chunk=16, dtype="f32", lr_kind="0.1sig", cfg=62)
    g = make_linear_grads(x, cfg=62)
    _compare(run_bwd(x, g, with_dS_end=False), oracle_bwd(x, g, with_dS_end=False), TOL_F32)


@pytest.mark.parametrize("include_diag", [True, False])
@pytest.mark.parametrize("N", [1, 300, 1000])
def test_bf16_tensor_core_path(cuda_device, include_diag, N):
    x = make_linear_inputs(2, 3, N, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=63,
                           with_S0=True)
    g = make_linear_grads(x, cfg=63)
    _compare(run_bwd(x, g, include_diag, S0=x.S0), oracle_bwd(x, g, include_diag, S0=x.S0),
             TOL_BF16)


@pytest.mark.parametrize("include_diag", [True, False])
def test_bf16_sequence_split(cuda_device, include_diag):
    """5000 tokens: every scan runs as segments on separate SMs."""
    x = make_linear_inputs(1, 3, 5000, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=64,
                           with_S0=True)
    g = make_linear_grads(x, cfg=64)
    _compare(run_bwd(x, g, include_diag, S0=x.S0), oracle_bwd(x, g, include_diag, S0=x.S0),
             TOL_BF16)


def test_bf16_unsplit_dims_on_cuda_cores(cuda_device):
    x = make_linear_inputs(1, 2, 200, 32, 48, chunk=32, dtype="bf16", lr_kind="sig-2", cfg=65)
    g = make_linear_grads(x, cfg=65)
    _compare(run_bwd(x, g), oracle_bwd(x, g), TOL_BF16)


def test_empty_sequence_passes_the_end_state_gradient(cuda_device):
    x = make_linear_inputs(1, 2, 0, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=66)
    g = make_linear_grads(x, cfg=66)
    *_, dS0 = run_bwd(x, g)
    assert np.array_equal(dS0, g.dS_end)


@pytest.mark.slow
def test_bf16_n32k_workload_sampled_heads(cuda_device):
    """The 32K-token, 64-head shape; the oracle recomputes eight whole heads,
    two per batch row, spread over the head index."""
    x = make_workload("ttt_linear_bf16_n32k")
    g = make_linear_grads(x, cfg=2)
    got = run_bwd(x, g)
    heads = [(0, 0), (0, 9), (1, 4), (1, 13), (2, 2), (2, 11), (3, 7), (3, 15)]
    ref = oracle_bwd(x, g, heads=heads)
    _compare([np.stack([a[b, h] for b, h in heads])[None] for a in got], ref, TOL_BF16)

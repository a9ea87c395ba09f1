"""lact_chunk_fwd_noalloc: the LaCT layer for callers that cannot allocate
device memory (code hosted by a program that owns every device allocation,
or paths where cudaMalloc/cudaFree are not allowed).  It must give the same
result as lact_chunk_fwd with a caller-allocated workspace, and as the
oracle, call after call, although every call reuses the library's one fixed
scratch array; lact_noalloc_check_status reads that array's status block.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from oracle import lact_forward
from oracle.lact import lact_init_state
from ttt_synth import make_lact_inputs, make_workload
from gpu_util import rel_err, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _problem():
    x = make_lact_inputs(1, 2, 1000, 128, 256, chunk=256, order="causal", cfg=77)
    desc = T.make_lact_desc(1, 2, 1000, 128, 256, 256, opt="momentum")
    W = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
    q, k, v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
    lr = torch.from_numpy(x.lr).cuda()
    return x, desc, W, q, k, v, lr


def _run(desc, W, q, k, v, lr, noalloc, shape, ws_bytes=None):
    state = T.alloc_lact_state(desc)
    T.lact_state_init(desc, *W, 0, state)
    out = torch.full(shape, float("nan"), device="cuda")
    if noalloc:
        T.lact_chunk_fwd_noalloc(desc, q, k, v, lr, state, out)
        assert T.lact_noalloc_check_status() == T.TTT_OK
    else:
        ws = T.alloc_workspace(ws_bytes or T.lact_workspace_bytes(desc))
        T.lact_chunk_fwd(desc, q, k, v, lr, state, out, ws)
        assert T.ttt_check_device_status(ws) == T.TTT_OK
    torch.cuda.synchronize()
    return out.cpu().numpy(), state.cpu().numpy()


def test_noalloc_matches_allocating_entry_point_and_oracle_twice(cuda_device):
    x, desc, W, q, k, v, lr = _problem()
    shape = (1, 2, 1000, 128)
    ref_out, ref_state = _run(desc, W, q, k, v, lr, False, shape)
    o_ref, st_ref = lact_forward(x.q.values, x.k.values, x.v.values, x.lr,
                                 lact_init_state(x.W1, x.W3, x.W2, 1, "momentum"), chunk=256,
                                 opt="momentum")
    n = 1 * 2 * 256 * 128
    for _ in range(2):
        out, state = _run(desc, W, q, k, v, lr, True, shape)
        assert not np.isnan(out).any()
        assert rel_err(out, ref_out) <= TOL
        assert rel_err(state, ref_state) <= TOL
        assert rel_err(out, o_ref) <= TOL
        assert rel_err(state[:n].reshape(st_ref.W1.shape), st_ref.W1) <= TOL
        assert rel_err(state[2 * n:3 * n].reshape(st_ref.W2.shape), st_ref.W2) <= TOL


def test_noalloc_runs_the_chunk_loop_when_the_fast_form_does_not_fit(cuda_device):
    """The 32K-token W2-only layer (GD, no row norm): its parallel form needs
    more than the 64 MiB scratch, its chunk loop fits, so the entry point runs
    the loop; it must agree with the parallel form that lact_chunk_fwd runs in
    a full-size workspace.  The array still holds the previous test's
    contents when this runs."""
    x = make_workload("lact_w2only_causal_n32k")
    B, H, N, d = x.k.values.shape
    dh = x.W1.shape[-2]
    desc = T.make_lact_desc(B, H, N, d, dh, x.chunk, update_mask=4, normalize_rows=False)
    assert T.lact_workspace_bytes(desc) > 64 << 20 >= T.lact_workspace_bytes_min(desc)
    W = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
    q, k, v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
    lr = torch.from_numpy(x.lr).cuda()
    ref_out, ref_state = _run(desc, W, q, k, v, lr, False, (B, H, N, d))
    for _ in range(2):
        out, state = _run(desc, W, q, k, v, lr, True, (B, H, N, d))
        assert not np.isnan(out).any()
        assert rel_err(out, ref_out) <= TOL
        assert rel_err(state, ref_state) <= TOL


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_device):
    big = T.make_lact_desc(1, 2, 196608, 384, 768, 196608, N_q=4096, order="bidirectional")
    st = T.load().lact_chunk_fwd_noalloc(ctypes.byref(big), 16, 16, 16, 16, 16, 16, None)
    assert st == T.TTT_ERR_WORKSPACE
    assert T.lact_noalloc_check_status() == T.TTT_OK

"""lact_chunk_fwd_noalloc: the LaCT layer for callers that cannot allocate
device memory (code hosted by a program that owns every device allocation,
or paths where cudaMalloc/cudaFree are not allowed).  It must give the same
result as lact_chunk_fwd with a caller-allocated workspace, call after call,
although both calls reuse the library's one fixed scratch array.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from ttt_synth import make_lact_inputs
from gpu_util import rel_err, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _problem():
    x = make_lact_inputs(1, 2, 1000, 128, 256, chunk=256, order="causal", cfg=77)
    desc = T.make_lact_desc(1, 2, 1000, 128, 256, 256, opt="momentum")
    W = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
    q, k, v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
    lr = torch.from_numpy(x.lr).cuda()
    return desc, W, q, k, v, lr


def _run(desc, W, q, k, v, lr, noalloc):
    state = T.alloc_lact_state(desc)
    T.lact_state_init(desc, *W, 0, state)
    out = torch.full((1, 2, 1000, 128), float("nan"), device="cuda")
    if noalloc:
        T.lact_chunk_fwd_noalloc(desc, q, k, v, lr, state, out)
    else:
        ws = T.alloc_workspace(T.lact_workspace_bytes(desc))
        T.lact_chunk_fwd(desc, q, k, v, lr, state, out, ws)
        assert T.ttt_check_device_status(ws) == T.TTT_OK
    torch.cuda.synchronize()
    return out.cpu().numpy(), state.cpu().numpy()


def test_noalloc_matches_allocating_entry_point_twice(cuda_device):
    desc, W, q, k, v, lr = _problem()
    ref_out, ref_state = _run(desc, W, q, k, v, lr, noalloc=False)
    for _ in range(2):
        out, state = _run(desc, W, q, k, v, lr, noalloc=True)
        assert not np.isnan(out).any()
        assert rel_err(out, ref_out) <= TOL
        assert rel_err(state, ref_state) <= TOL


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_device):
    big = T.make_lact_desc(1, 2, 196608, 384, 768, 196608, N_q=4096, order="bidirectional")
    st = T.load().lact_chunk_fwd_noalloc(ctypes.byref(big), 16, 16, 16, 16, 16, 16, None)
    assert st == T.TTT_ERR_WORKSPACE

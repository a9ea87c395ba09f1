"""Context parallelism through the C ABI on one GPU: the ranks of a
world-size-2 run execute one after another, each with its own share of every
chunk, its own copy of the state and its own gradient buffer; between the
gradient and the update of each chunk the test sums the ranks' gradients
(standing in for the all-reduce, which needs several GPUs).  The result must
match the unsharded oracle ("Test-Time Training Done Right" review, "Vídeo y
cálculo distribuido") within the bf16 tolerance, on every rank."""
import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from learned_linear_attention_b200.context_parallel import (DeviceOps, chunk_plan, local_tokens,
                                                            max_share, run_rank, shares)
from oracle import lact_forward
from oracle.lact import lact_init_state
from ttt_synth import make_lact_inputs
from gpu_util import LaCTRun, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


class _Rank:
    def __init__(self, x, rank, world, opt, kw):
        B, H, N, d = x.k.values.shape
        dh = x.W1.shape[-2]
        self.idx = np.array(local_tokens(N, x.chunk, world, rank), dtype=np.int64)
        take = lambda a: np.ascontiguousarray(a[:, :, self.idx])  # noqa: E731
        bits = lambda tt: torch.from_numpy(take(tt.bits).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731,E501
        self.k, self.v = bits(x.k), bits(x.v)
        self.lr = torch.from_numpy(take(x.lr)).cuda()
        n_local = len(self.idx)
        if x.order == "causal":
            self.q, nq, self.rows = bits(x.q), n_local, self.idx
        else:
            s, m = shares(x.q.values.shape[2], world)[rank]
            self.rows = np.arange(s, s + m)
            qb = np.ascontiguousarray(x.q.bits[:, :, s:s + m]).view(np.int16)
            self.q, nq = torch.from_numpy(qb).view(torch.bfloat16).cuda(), m
        self.desc = T.make_lact_desc(B, H, n_local, d, dh, max(1, max_share(N, x.chunk, world)),
                                     N_q=nq, order=x.order, opt=opt, **kw)
        self.state = T.alloc_lact_state(self.desc)
        W = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
        T.lact_state_init(self.desc, *W, 0, self.state)
        self.ws = T.alloc_workspace(T.lact_workspace_bytes(self.desc))
        self.G = torch.empty(T.lact_grad_bytes(self.desc) // 4, device="cuda")
        self.out = torch.full((B, H, nq, d), float("nan"), device="cuda")
        self.ops = DeviceOps(self.desc, self.q, self.k, self.v, self.lr, self.state, self.out,
                             self.ws, self.G)


def _run_sharded(x, world, opt, **kw):
    """The loop of run_rank, rank by rank within each chunk (one GPU)."""
    N = x.k.values.shape[2]
    ranks = [_Rank(x, r, world, opt, kw) for r in range(world)]
    offs = [0] * world
    for _, _, sh in chunk_plan(N, x.chunk, world):
        for r, rk in enumerate(ranks):
            n = sh[r][1]
            if x.order == "causal":
                rk.ops.read(offs[r], n)
            rk.ops.grad(offs[r], n)
        total = sum(rk.G for rk in ranks)      # the all-reduce
        for r, rk in enumerate(ranks):
            rk.G.copy_(total)
            rk.ops.apply()
            offs[r] += sh[r][1]
    if x.order != "causal":
        for rk in ranks:
            rk.ops.read_queries()
    torch.cuda.synchronize()
    for rk in ranks:
        assert T.ttt_check_device_status(rk.ws) == T.TTT_OK
    return ranks


def _oracle(x, opt, **kw):
    st = lact_init_state(x.W1, x.W3, x.W2, x.k.values.shape[0], opt)
    return lact_forward(x.q.values, x.k.values, x.v.values, x.lr, st, chunk=x.chunk,
                        order=x.order, opt=opt, **kw)


def _check(x, world, opt, **kw):
    ranks = _run_sharded(x, world, opt, **kw)
    okw = {k: v for k, v in kw.items() if k in ("beta", "ns_steps")}
    ref, st = _oracle(x, opt, **okw)
    out = np.full(ref.shape, np.nan)
    n = st.W1.size
    for rk in ranks:
        out[:, :, rk.rows] = rk.out.cpu().numpy()
        s = rk.state.cpu().numpy()
        assert rel_err(s[:n].reshape(st.W1.shape), st.W1) <= TOL
        assert rel_err(s[2 * n:3 * n].reshape(st.W2.shape), st.W2) <= TOL
    assert not np.isnan(out).any()
    assert rel_err(out, ref) <= TOL, rel_err(out, ref)


@pytest.mark.parametrize("opt", ["gd", "momentum"])
def test_causal_two_ranks_fused_key_gradient_path(cuda_device, opt):
    """d = 128: each share's gradient runs on the fused key/gradient kernel;
    chunks of 256 split 128/128, the last (168 tokens) 84/84."""
    x = make_lact_inputs(1, 2, 680, 128, 256, chunk=256, order="causal", cfg=71)
    _check(x, 2, opt)


def test_bidirectional_three_ranks_muon(cuda_device):
    """Muon (split operands, fused Newton-Schulz) on the summed gradient;
    shares 86/86/84 of each 256-token chunk and 63/63/62 of the last one."""
    x = make_lact_inputs(1, 2, 700, 128, 256, chunk=256, order="bidirectional", Nq=130,
                         v_norm=True, lr_kind="0.01sig", cfg=72)
    _check(x, 3, "muon", beta=0.9, ns_steps=5)


def test_bidirectional_two_ranks_view_synthesis_dims(cuda_device):
    """d = 384, dh = 768: the key pass and split-K gradient GEMMs on a share."""
    x = make_lact_inputs(1, 2, 600, 384, 768, chunk=600, order="bidirectional", Nq=100,
                         v_norm=True, lr_kind="0.01sig", cfg=73)
    _check(x, 2, "gd")


def test_one_rank_loop_equals_the_layer_call(cuda_device):
    """run_rank with one rank (no collective) is the layer itself."""
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=256, order="causal", cfg=74)
    rk = _Rank(x, 0, 1, "momentum", {})
    run_rank(512, 256, 1, 0, True, rk.ops)
    run = LaCTRun(x, opt="momentum")
    ref = run.run()
    assert rel_err(rk.out.cpu().numpy(), ref) <= 1e-2
    assert rel_err(rk.state.cpu().numpy(), run.state.cpu().numpy()) <= 1e-3


def test_empty_share_and_argument_checks(cuda_device):
    x = make_lact_inputs(1, 1, 128, 128, 256, chunk=128, order="causal", cfg=75)
    rk = _Rank(x, 0, 1, "gd", {})
    rk.ops.grad(0, 0)                       # no tokens: a zero gradient
    assert float(rk.G.abs().max()) == 0.0
    bad = T.load().lact_chunk_grad
    import ctypes
    st = bad(ctypes.byref(rk.desc), 100, 100, rk.k.data_ptr(), rk.v.data_ptr(), rk.lr.data_ptr(),
             rk.state.data_ptr(), rk.G.data_ptr(), rk.ws.data_ptr(), rk.ws.numel(), None)
    assert st == T.TTT_ERR_SHAPE

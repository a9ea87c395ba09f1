"""Context parallelism on CPU ranks: the chunk loop of
learned_linear_attention_b200.context_parallel run by world-size-2 (and 3)
gloo process groups, with the oracle's per-chunk pieces standing in for the
device kernels and a real all-reduce of the chunk gradient between them.
The sharded result must equal the unsharded oracle ("Test-Time Training Done
Right" review, "Vídeo y cálculo distribuido": summing the shares' gradients
is the chunk gradient, so every rank applies the same update)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from learned_linear_attention_b200.context_parallel import (chunk_plan, local_tokens, run_rank,
                                                            shares)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shares_cover_every_token_once():
    for n in (0, 1, 5, 64, 65, 1000):
        for world in (1, 2, 3, 8):
            sh = shares(n, world)
            assert len(sh) == world
            got = [i for s, m in sh for i in range(s, s + m)]
            assert got == list(range(n))
    idx = sorted(i for r in range(3) for i in local_tokens(700, 256, 3, r))
    assert idx == list(range(700))
    assert [C for _, C, _ in chunk_plan(700, 256, 2)] == [256, 256, 188]


class _OracleOps:
    """The oracle's chunk pieces for one rank: reads, the chunk gradient of
    the local share at the current weights, the update.  Per (b, h)."""

    def __init__(self, x, rank, world, opt, kw, dist):
        from oracle.lact import lact_init_state
        self.x, self.opt, self.kw, self.dist = x, opt, kw, dist
        B, H, N, d = x.k.values.shape
        self.idx = np.array(local_tokens(N, x.chunk, world, rank), dtype=np.int64)
        self.k = x.k.values[:, :, self.idx].astype(np.float64)
        self.v = x.v.values[:, :, self.idx].astype(np.float64)
        self.lr = x.lr[:, :, self.idx].astype(np.float64)
        if x.order == "causal":
            self.q = x.q.values[:, :, self.idx].astype(np.float64)
        else:   # each rank reads its share of the queries
            nq = x.q.values.shape[2]
            s, m = shares(nq, world)[rank]
            self.qrows = np.arange(s, s + m)
            self.q = x.q.values[:, :, self.qrows].astype(np.float64)
        self.st = lact_init_state(x.W1, x.W3, x.W2, B, opt)
        self.out = np.full(self.q.shape, np.nan)
        self.G = None

    def read(self, t0, n):
        from oracle.lact import lact_read
        B, H = self.q.shape[:2]
        for b in range(B):
            for h in range(H):
                self.out[b, h, t0:t0 + n] = lact_read(self.st.W1[b, h], self.st.W3[b, h],
                                                      self.st.W2[b, h], self.q[b, h, t0:t0 + n])

    def read_queries(self):
        self.read(0, self.q.shape[2])

    def grad(self, t0, n):
        from oracle.lact import lact_chunk_gradients
        B, H = self.k.shape[:2]
        G = [np.zeros_like(self.st.W1), np.zeros_like(self.st.W3), np.zeros_like(self.st.W2)]
        for b in range(B):
            for h in range(H):
                g = lact_chunk_gradients(self.st.W1[b, h], self.st.W3[b, h], self.st.W2[b, h],
                                         self.k[b, h, t0:t0 + n], self.v[b, h, t0:t0 + n],
                                         self.lr[b, h, t0:t0 + n])
                for i in range(3):
                    G[i][b, h] = g[i]
        self.G = G

    def allreduce(self):
        import torch
        for i in range(3):
            t = torch.from_numpy(self.G[i])
            self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM)
            self.G[i] = t.numpy()

    def apply(self):
        from oracle.lact import newton_schulz
        W = [self.st.W1, self.st.W3, self.st.W2]
        M = [self.st.M1, self.st.M3, self.st.M2]
        kw = self.kw
        B, H = W[0].shape[:2]
        for i in range(3):
            for b in range(B):
                for h in range(H):
                    g = self.G[i][b, h]
                    if self.opt == "gd":
                        U = g
                    else:
                        M[i][b, h] = kw["beta"] * M[i][b, h] + g
                        U = M[i][b, h] if self.opt == "momentum" else newton_schulz(
                            M[i][b, h], kw["ns_steps"])
                    w = W[i][b, h] - U
                    W[i][b, h] = w / np.maximum(np.sqrt(np.sum(w * w, -1, keepdims=True)), 1e-12)


def _rank_main(rank, world, port, case, outq):
    import datetime
    import torch.distributed as dist
    from ttt_synth import make_lact_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        order, opt, N, chunk = case
        x = make_lact_inputs(1, 2, N, 8, 16, chunk=chunk, order=order, Nq=11, cfg=61)
        kw = dict(beta=0.9, ns_steps=3)
        ops = _OracleOps(x, rank, world, opt, kw, dist)
        run_rank(N, chunk, world, rank, order == "causal", ops)
        rows = ops.idx if order == "causal" else ops.qrows
        outq.put((rank, rows, ops.out, ops.st.W1, ops.st.W2))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [("causal", "gd", 70, 32), ("causal", "momentum", 70, 32),
                                  ("bidirectional", "muon", 70, 32),
                                  ("bidirectional", "gd", 45, 45)])
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_chunks_equal_the_unsharded_oracle(case, world):
    """70 tokens in chunks of 32 (32, 32, 6): shares of 16/16 (world 2) and
    11/11/10 (world 3), and 3/3/0 in the last chunk of world 3; one 45-token
    chunk bidirectionally.  Every rank ends with the unsharded weights, and
    the ranks' outputs together are the unsharded outputs."""
    from oracle import lact_forward
    from oracle.lact import lact_init_state
    from ttt_synth import make_lact_inputs
    order, opt, N, chunk = case
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = make_lact_inputs(1, 2, N, 8, 16, chunk=chunk, order=order, Nq=11, cfg=61)
    ref, st = lact_forward(x.q.values, x.k.values, x.v.values, x.lr,
                           lact_init_state(x.W1, x.W3, x.W2, 1, opt), chunk=chunk, order=order,
                           opt=opt, beta=0.9, ns_steps=3)
    out = np.full(ref.shape, np.nan)
    for _, rows, o, W1, W2 in res:
        out[:, :, rows] = o
        np.testing.assert_allclose(W1, st.W1, rtol=0, atol=1e-12)
        np.testing.assert_allclose(W2, st.W2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_a_planted_missing_allreduce_is_caught():
    """Without the sum over ranks, a rank's weights follow only its own share
    and leave the unsharded oracle's."""
    from oracle import lact_forward
    from oracle.lact import lact_init_state
    from ttt_synth import make_lact_inputs

    class _NoSum(_OracleOps):
        def allreduce(self):
            pass

    x = make_lact_inputs(1, 2, 70, 8, 16, chunk=32, order="causal", cfg=61)
    ops = _NoSum(x, 0, 2, "gd", {}, None)
    run_rank(70, 32, 2, 0, True, ops)
    _, st = lact_forward(x.q.values, x.k.values, x.v.values, x.lr,
                         lact_init_state(x.W1, x.W3, x.W2, 1, "gd"), chunk=32)
    assert np.abs(ops.st.W1 - st.W1).max() > 1e-4

"""Context-parallel LaCT layer: the tokens of every chunk split across ranks.

"Test-Time Training Done Right" review, "Vídeo y cálculo distribuido": a
chunk's tokens are spread over devices; every device computes the gradient
of its share at the chunk-start weights, the shares' gradients are summed
(one all-reduce per chunk, float32, into each rank's own buffer), and every
device applies the same optimizer step and row normalisation to its own copy
of the weights.  The weights therefore stay identical on every rank.

Layout: chunk c of the global sequence covers tokens [c C, c C + C_c).  Rank
r holds the contiguous share ``shares(C_c, world)[r]`` of every chunk; its
local token tensors ([B, H, n_local, d]) concatenate its shares in chunk
order.  In causal order every rank reads its own share's queries before the
chunk's update; in bidirectional order every rank reads its own queries
after the last chunk.

The device work is the C ABI's lact_read, lact_chunk_grad and
lact_apply_grad (hand-written kernels); the only other step is the
all-reduce (NCCL through torch.distributed).  ``run_rank`` is the chunk loop
of one rank over any object with those four operations, so the same loop
runs on the GPU (``DeviceOps``) and, in the tests, on CPU ranks.
"""
from __future__ import annotations

from typing import List, Tuple


def shares(n: int, world: int) -> List[Tuple[int, int]]:
    """(start, length) of each rank's contiguous share of n tokens: the first
    ranks take ceil(n / world) tokens, the last ones what is left (possibly
    nothing)."""
    per = -(-n // world) if n > 0 else 0
    out = []
    for r in range(world):
        s = min(n, r * per)
        out.append((s, min(n, s + per) - s))
    return out


def chunk_plan(N_in: int, chunk: int, world: int):
    """Per chunk: (global start, length, [(start within chunk, length)] per rank)."""
    plan = []
    for t0 in range(0, N_in, chunk):
        C = min(chunk, N_in - t0)
        plan.append((t0, C, shares(C, world)))
    return plan


def local_tokens(N_in: int, chunk: int, world: int, rank: int) -> List[int]:
    """Global token indices held by `rank`, in local order."""
    idx = []
    for t0, _, sh in chunk_plan(N_in, chunk, world):
        s, n = sh[rank]
        idx.extend(range(t0 + s, t0 + s + n))
    return idx


def max_share(N_in: int, chunk: int, world: int) -> int:
    return max([n for _, _, sh in chunk_plan(N_in, chunk, world) for _, n in sh] + [0])


def run_rank(N_in: int, chunk: int, world: int, rank: int, causal: bool, ops) -> None:
    """The chunk loop of one rank.  ops.read(t0, n) reads local query rows
    [t0, t0 + n) with the current weights; ops.grad(t0, n) forms the gradient
    of local tokens [t0, t0 + n); ops.allreduce() sums it over the ranks;
    ops.apply() updates the weights with the sum; ops.read_queries() reads
    the bidirectional queries.  Every rank takes the same collective steps
    in the same order, whatever its share."""
    off = 0
    for _, _, sh in chunk_plan(N_in, chunk, world):
        n = sh[rank][1]
        if causal:
            ops.read(off, n)
        ops.grad(off, n)
        ops.allreduce()
        ops.apply()
        off += n
    if not causal:
        ops.read_queries()


class DeviceOps:
    """The four operations on this rank's GPU through the C ABI.

    desc: the lact_desc of the local problem (N_in = this rank's token count,
    chunk >= its largest share, N_q = its query count when bidirectional);
    q, k, v, lr: its local tensors; state: its copy of the state; out: its
    output rows; ws: a workspace of lact_workspace_bytes(desc); G: a float32
    buffer of lact_grad_bytes(desc); group: the process group of the
    all-reduce (None: a single rank, no collective)."""

    def __init__(self, desc, q, k, v, lr, state, out, ws, G, group=None, stream=None):
        self.desc, self.q, self.k, self.v, self.lr = desc, q, k, v, lr
        self.state, self.out, self.ws, self.G = state, out, ws, G
        self.group, self.stream = group, stream

    def read(self, t0, n):
        from . import _lib
        _lib.lact_read(self.desc, t0, n, self.q, self.state, self.out, self.ws, stream=self.stream)

    def grad(self, t0, n):
        from . import _lib
        _lib.lact_chunk_grad(self.desc, t0, n, self.k, self.v, self.lr, self.state, self.G,
                             self.ws, stream=self.stream)

    def allreduce(self):
        if self.group is None:
            return
        import torch.distributed as dist
        dist.all_reduce(self.G, op=dist.ReduceOp.SUM, group=self.group)

    def apply(self):
        from . import _lib
        _lib.lact_apply_grad(self.desc, self.G, self.state, self.ws, stream=self.stream)

    def read_queries(self):
        from . import _lib
        _lib.lact_read(self.desc, 0, self.desc.N_q, self.q, self.state, self.out, self.ws,
                       stream=self.stream)

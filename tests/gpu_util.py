"""Shared helpers for the GPU parity tests: move seeded inputs to the device
and call the C ABI through the package binding."""
from __future__ import annotations

import os

import numpy as np
import torch

import learned_linear_attention_b200 as T


def to_dev(tt, device="cuda"):
    """TokenTensor -> device tensor with the exact values (bf16 bits or f32)."""
    if tt.dtype == "bf16":
        bits = np.ascontiguousarray(tt.bits).view(np.int16)
        return torch.from_numpy(bits).view(torch.bfloat16).to(device).contiguous()
    return torch.from_numpy(np.ascontiguousarray(tt.values)).to(device).contiguous()


# Every comparison made through rel_err is also recorded with the
# elementwise measure, and the session's terminal summary lists both per test
# (the elementwise ratio is reported, not asserted: it is unbounded where the
# reference crosses zero).
ERROR_LOG: list = []


def elem_err(a, ref):
    """Elementwise relative error, max_i |a_i - ref_i| / (|ref_i| + 1e-3 max|ref|)."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if a.size == 0:
        return 0.0
    return float((np.abs(a - ref) / (np.abs(ref) + 1e-3 * np.abs(ref).max())).max())


def rel_err(a, ref):
    """Normwise max relative error: max|a - ref| / max|ref|."""
    a = np.asarray(a, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if a.size == 0:
        return 0.0
    norm = float(np.abs(a - ref).max() / max(np.abs(ref).max(), 1e-300))
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    ERROR_LOG.append((test, a.size, norm, elem_err(a, ref)))
    return norm


def run_linear(x, include_diag=True, out_dtype="f32", S0=None, chunk=None, stream=None,
               ws_bytes=None, order="causal"):
    B, H, N, dk = x.q.values.shape
    dv = x.v.values.shape[-1]
    desc = T.make_linear_desc(B, H, N, dk, dv, chunk or x.chunk, include_diag,
                              in_dtype=x.q.dtype, out_dtype=out_dtype, order=order)
    q, k, v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
    lr = torch.from_numpy(np.ascontiguousarray(x.lr)).cuda()
    S = torch.zeros(B, H, dk, dv, dtype=torch.float32, device="cuda")
    if S0 is not None:
        S.copy_(torch.from_numpy(np.asarray(S0, dtype=np.float32)))
    odt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = torch.full((B, H, N, dv), float("nan"), dtype=odt, device="cuda")
    ws = T.alloc_workspace(ws_bytes or T.ttt_linear_workspace_bytes(desc))
    T.ttt_linear_fwd(desc, q, k, v, lr, S, out, ws, stream=stream)
    assert T.ttt_check_device_status(ws, stream) == T.TTT_OK
    return out.float().cpu().numpy(), S.cpu().numpy()


class LaCTRun:
    """One LaCT problem on the device: descriptor, state, workspace."""

    def __init__(self, x, opt="gd", out_dtype="f32", min_workspace=False, **kw):
        B, H, N, d = x.k.values.shape
        dh = x.W1.shape[-2]
        nq = x.q.values.shape[2]
        self.x, self.opt = x, opt
        self.desc = T.make_lact_desc(B, H, N, d, dh, x.chunk, N_q=nq, order=x.order, opt=opt,
                                     out_dtype=out_dtype, **kw)
        self.q, self.k, self.v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
        self.lr = torch.from_numpy(x.lr).cuda()
        self.state = T.alloc_lact_state(self.desc)
        size = T.lact_workspace_bytes_min if min_workspace else T.lact_workspace_bytes
        self.ws = T.alloc_workspace(size(self.desc))
        odt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        self.out = torch.full((B, H, nq, d), float("nan"), dtype=odt, device="cuda")
        self.init_state()

    def init_state(self, W1=None, W3=None, W2=None, per_batch=False):
        W1 = self.x.W1 if W1 is None else W1
        W3 = self.x.W3 if W3 is None else W3
        W2 = self.x.W2 if W2 is None else W2
        dev = [torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).cuda()
               for w in (W1, W3, W2)]
        T.lact_state_init(self.desc, *dev, int(per_batch), self.state)

    def set_momentum(self, M1, M3, M2):
        n = M1.size
        flat = np.concatenate([np.asarray(m, np.float32).ravel() for m in (M1, M3, M2)])
        self.state[3 * n:6 * n].copy_(torch.from_numpy(flat))

    def run(self):
        T.lact_chunk_fwd(self.desc, self.q, self.k, self.v, self.lr, self.state, self.out,
                         self.ws)
        assert T.ttt_check_device_status(self.ws) == T.TTT_OK
        return self.out.float().cpu().numpy()

    def weights(self):
        B, H = self.desc.B, self.desc.H
        d, dh = self.desc.d, self.desc.dh
        W1 = torch.empty(B, H, dh, d, device="cuda")
        W3 = torch.empty(B, H, dh, d, device="cuda")
        W2 = torch.empty(B, H, d, dh, device="cuda")
        M = torch.empty(3 * B * H * d * dh, device="cuda") if self.opt != "gd" else None
        T.lact_state_readout(self.desc, self.state, W1, W3, W2, M)
        torch.cuda.synchronize()
        res = [W1.cpu().numpy(), W3.cpu().numpy(), W2.cpu().numpy()]
        if M is not None:
            n = B * H * d * dh
            m = M.cpu().numpy()
            res += [m[:n].reshape(W1.shape), m[n:2 * n].reshape(W3.shape),
                    m[2 * n:].reshape(W2.shape)]
        return res

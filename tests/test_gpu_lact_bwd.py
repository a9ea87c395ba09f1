"""GPU parity for the backward pass of the LaCT layer (lact_chunk_bwd)
against the written-out backward oracle (oracle.lact_backward, itself pinned
to autograd and to central differences of the forward oracle).  Tolerance:
normwise 2e-2 per gradient (bf16 operands, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from oracle.lact_backward import lact_backward_explicit
from ttt_synth import make_lact_grads, make_lact_inputs
from gpu_util import rel_err, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2
NAMES = ("q", "k", "v", "lr", "W1", "W3", "W2")


def _nan_at16(shape):
    """A NaN-filled float32 tensor whose data starts 16 bytes past a 32-byte
    boundary (the API asks for 16-byte alignment only)."""
    n = int(np.prod(shape))
    base = torch.full((n + 8,), float("nan"), device="cuda")
    off = (4 - (base.data_ptr() % 32) // 4) % 8
    t = base[off:off + n]
    assert t.data_ptr() % 32 == 16
    return t.view(shape)


def _run(x, g, opt="gd", with_dw=True, offset16=False, **kw):
    B, H, N, d = x.k.values.shape
    dh = x.W1.shape[-2]
    R = x.q.values.shape[2]
    desc = T.make_lact_desc(B, H, N, d, dh, x.chunk, N_q=R, order=x.order, opt=opt,
                            split_operands=False, **kw)
    state0 = T.alloc_lact_state(desc)
    T.lact_state_init(desc, *[torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)], 0, state0)
    mat = B * H * d * dh
    dW_end = None
    if with_dw:
        dW_end = torch.from_numpy(np.concatenate([w.ravel() for w in g.dW_end])).cuda()
    shapes = [(B, H, R, d), (B, H, N, d), (B, H, N, d), (B, H, N), (3 * mat,)]
    if offset16:
        grads = [_nan_at16(sh) for sh in shapes]
        nb = T.lact_bwd_workspace_bytes(desc)
        raw = T.alloc_workspace(nb + 64)
        skip = (16 - raw.data_ptr() % 32) % 32
        ws = raw[skip:skip + nb]
        assert ws.data_ptr() % 32 == 16
    else:
        grads = [torch.full(sh, float("nan"), device="cuda") for sh in shapes]
        ws = T.alloc_workspace(T.lact_bwd_workspace_bytes(desc))
    T.lact_chunk_bwd(desc, to_dev(x.q), to_dev(x.k), to_dev(x.v), torch.from_numpy(x.lr).cuda(),
                     state0, to_dev(g.dout), dW_end, *grads, ws)
    assert T.ttt_check_device_status(ws) == T.TTT_OK
    out = [t.cpu().numpy() for t in grads[:4]]
    dW = grads[4].cpu().numpy()
    out += [dW[:mat].reshape(B, H, dh, d), dW[mat:2 * mat].reshape(B, H, dh, d),
            dW[2 * mat:].reshape(B, H, d, dh)]
    return out


def _oracle(x, g, opt="gd", with_dw=True, **kw):
    B = x.k.values.shape[0]
    W = [np.broadcast_to(w[None], (B,) + w.shape).astype(np.float64) for w in (x.W1, x.W3, x.W2)]
    okw = {k: v for k, v in kw.items() if k in ("beta", "normalize_rows", "update_mask")}
    return lact_backward_explicit(x.q.values, x.k.values, x.v.values, x.lr, *W, g.dout.values,
                                  g.dW_end if with_dw else None, chunk=x.chunk, order=x.order,
                                  opt=opt, **okw)


def _check(x, g, opt="gd", with_dw=True, offset16=False, **kw):
    got = _run(x, g, opt, with_dw, offset16, **kw)
    ref = _oracle(x, g, opt, with_dw, **kw)
    for name, a, r in zip(NAMES, got, ref):
        assert not np.isnan(a).any(), name
        assert rel_err(a, r) <= TOL, (name, rel_err(a, r))


@pytest.mark.parametrize("opt", ["gd", "momentum"])
def test_causal_chunks(cuda_device, opt):
    """Three chunks (128, 128, 72 tokens: the last ragged), d = 128, dh = 256."""
    x = make_lact_inputs(1, 2, 328, 128, 256, chunk=128, order="causal", cfg=81)
    _check(x, make_lact_grads(x, cfg=81), opt, beta=0.9)


def test_buffers_only_16_byte_aligned(cuda_device):
    """Gradient outputs and workspace 16 bytes past a 32-byte boundary: the
    kernels' 256-bit stores give way to 128-bit ones."""
    x = make_lact_inputs(1, 2, 300, 128, 256, chunk=128, order="causal", cfg=86)
    _check(x, make_lact_grads(x, cfg=86), "momentum", beta=0.9, offset16=True)


@pytest.mark.parametrize("dh", [128, 384])
def test_hidden_widths_on_the_fused_route(cuda_device, dh):
    """d = 128 with dh = 128 (a hidden width below one 256-wide product tile)
    and dh = 384 (one and a half tiles), causal, a ragged last chunk."""
    x = make_lact_inputs(1, 2, 200, 128, dh, chunk=128, order="causal", cfg=87)
    _check(x, make_lact_grads(x, cfg=87), "momentum", beta=0.9)


def test_causal_without_end_gradient(cuda_device):
    x = make_lact_inputs(2, 1, 256, 128, 256, chunk=128, order="causal", cfg=82)
    _check(x, make_lact_grads(x, cfg=82), with_dw=False)


def test_bidirectional(cuda_device):
    x = make_lact_inputs(1, 2, 300, 128, 256, chunk=128, order="bidirectional", Nq=90,
                         v_norm=True, lr_kind="0.01sig", cfg=83)
    _check(x, make_lact_grads(x, cfg=83), "momentum", beta=0.8)


def test_w2_only_without_normalisation(cuda_device):
    x = make_lact_inputs(1, 2, 256, 128, 256, chunk=128, order="causal", cfg=84)
    _check(x, make_lact_grads(x, cfg=84), update_mask=4, normalize_rows=False)


def test_view_synthesis_dims(cuda_device):
    x = make_lact_inputs(1, 1, 256, 384, 768, chunk=128, order="bidirectional", Nq=64,
                         v_norm=True, lr_kind="0.01sig", cfg=85)
    _check(x, make_lact_grads(x, cfg=85))


def test_muon_is_rejected(cuda_device):
    d = T.make_lact_desc(1, 1, 128, 128, 256, 128, opt="muon")
    with pytest.raises(T.TTTError):
        T.lact_bwd_workspace_bytes(d)

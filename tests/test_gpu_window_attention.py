"""GPU parity for the causal sliding-window attention kernel and the LaCT
language layer (memory + window attention, outputs summed) against the fp64
oracle, through the C ABI.  Tolerance: normwise max relative error 2e-2
(bf16 q, k, v and P operands, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from oracle import lact_layer_forward, sliding_window_attention
from oracle.lact import lact_init_state
from ttt_synth import make_lact_inputs, make_workload
from gpu_util import LaCTRun, rel_err, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-2


def run_window(x, window, out_dtype="f32", scale=0.0, init=None):
    B, H, N, d = x.q.values.shape
    q, k, v = to_dev(x.q), to_dev(x.k), to_dev(x.v)
    desc = T.make_window_desc(B, H, N, d, window, scale=scale, out_dtype=out_dtype,
                              accumulate=init is not None)
    odt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    if init is None:
        out = torch.full((B, H, N, d), float("nan"), dtype=odt, device="cuda")
    else:
        out = torch.from_numpy(np.asarray(init, np.float32)).to("cuda", odt)
    ws = T.alloc_workspace(T.TTT_STATUS_BYTES)
    T.ttt_window_attn_fwd(desc, q, k, v, out, ws)
    assert T.ttt_check_device_status(ws) == T.TTT_OK
    return out.float().cpu().numpy()


def _x(N, cfg, B=1, H=2, qk_norm=False):
    return make_lact_inputs(B, H, N, 128, 256, chunk=128, order="causal", qk_norm=qk_norm, cfg=cfg)


@pytest.mark.parametrize("window", [1, 100, 128, 300, 5000])
def test_matches_oracle_ragged(cuda_device, window):
    # 700 tokens: 6 query tiles, the last ragged; windows inside one tile,
    # exactly one tile, across tiles, and covering the whole sequence
    x = _x(700, 71)
    got = run_window(x, window)
    ref = sliding_window_attention(x.q.values, x.k.values, x.v.values, window)
    assert not np.isnan(got).any()
    assert rel_err(got, ref) <= TOL, rel_err(got, ref)


def test_sharper_scores_and_bf16_output(cuda_device):
    x = _x(520, 72, B=2, H=1)
    got = run_window(x, 200, out_dtype="bf16", scale=0.3)
    ref = sliding_window_attention(x.q.values, x.k.values, x.v.values, 200, scale=0.3)
    assert rel_err(got, ref) <= TOL, rel_err(got, ref)


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_accumulate_adds_to_out(cuda_device, out_dtype):
    x = _x(300, 73)
    base = np.random.default_rng(73).standard_normal(x.q.values.shape).astype(np.float32)
    if out_dtype == "bf16":
        base = torch.from_numpy(base).bfloat16().float().numpy()
    got = run_window(x, 150, out_dtype=out_dtype, init=base)
    ref = base + sliding_window_attention(x.q.values, x.k.values, x.v.values, 150)
    assert rel_err(got, ref) <= TOL, rel_err(got, ref)


def test_single_token(cuda_device):
    x = _x(1, 74)
    got = run_window(x, 16)
    np.testing.assert_allclose(got, x.v.values, rtol=0, atol=1e-6)


def test_lact_layer_memory_plus_window(cuda_device):
    """The LaCT language layer: causal memory and window branch summed."""
    x = make_lact_inputs(1, 2, 640, 128, 256, chunk=256, order="causal", cfg=75)
    run = LaCTRun(x)
    T.lact_layer_fwd(run.desc, 200, 0.0, run.q, run.k, run.v, run.lr, run.state, run.out, run.ws)
    assert T.ttt_check_device_status(run.ws) == T.TTT_OK
    got = run.out.float().cpu().numpy()
    st = lact_init_state(x.W1, x.W3, x.W2, 1, "gd")
    ref, st = lact_layer_forward(x.q.values, x.k.values, x.v.values, x.lr, st, chunk=x.chunk,
                                 window=200)
    assert rel_err(got, ref) <= TOL, rel_err(got, ref)
    W = run.weights()
    for g, r in zip(W[:3], (st.W1, st.W3, st.W2)):
        assert rel_err(g, r) <= TOL


@pytest.mark.slow
def test_n32k_window_2048_sampled_positions(cuda_device):
    """The 32K-token, 8-head shape with the pages' 2048-token window; the
    oracle recomputes tile edges, window edges and the end, every 61st token
    (a stride that walks through all rows of the 128-token query tiles), and
    two whole query tiles, one inside the first window and one far past it."""
    x = make_workload("lact_causal_n32k")
    got = run_window(x, 2048)
    edges = [0, 127, 128, 2046, 2047, 2048, 2049, 4095, 17000, 32767]
    idx = sorted(set(edges) | set(range(0, 32768, 61)) | set(range(1024, 1152)) |
                 set(range(20480, 20608)))
    ref = sliding_window_attention(x.q.values, x.k.values, x.v.values, 2048, t_index=idx)
    assert rel_err(got[:, :, idx], ref) <= TOL, rel_err(got[:, :, idx], ref)

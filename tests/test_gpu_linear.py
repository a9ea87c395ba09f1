"""GPU parity for the linear fast weight (TTT-linear == causal linear
attention) against the fp64 oracle, through the C ABI.

Tolerances (normwise max relative error, max|gpu-ref| / max|ref|): 1e-4 for
fp32 inputs on the CUDA-core kernel, 2e-2 for bf16 inputs with fp32
accumulation on the tensor-core kernel."""
import numpy as np
import pytest
import torch

import learned_linear_attention_b200 as T
from oracle import ttt_linear_attention_sum, ttt_linear_recurrent
from ttt_synth import make_linear_inputs, make_workload
from gpu_util import rel_err, run_linear

pytestmark = pytest.mark.gpu
TOL_F32, TOL_BF16 = 1e-4, 2e-2


def _oracle(x, include_diag=True, S0=None):
    return ttt_linear_recurrent(x.q.values, x.k.values, x.v.values, x.lr, S0, include_diag)


def test_f32_n256_workload(cuda_device):
    x = make_workload("ttt_linear_f32_n256")
    out, S = run_linear(x)
    ref, Sref = _oracle(x)
    assert rel_err(out, ref) <= TOL_F32
    assert rel_err(S, Sref) <= TOL_F32


@pytest.mark.parametrize("include_diag", [True, False])
def test_f32_ragged_with_initial_state(cuda_device, include_diag):
    x = make_linear_inputs(2, 3, 77, 24, 40, chunk=9, dtype="f32", lr_kind="0.1sig", cfg=11,
                           with_S0=True)
    out, S = run_linear(x, include_diag, S0=x.S0)
    ref, Sref = _oracle(x, include_diag, x.S0)
    assert rel_err(out, ref) <= TOL_F32
    assert rel_err(S, Sref) <= TOL_F32


@pytest.mark.parametrize("include_diag", [True, False])
@pytest.mark.parametrize("N", [1, 128, 300, 1000])
def test_bf16_tensor_core_kernel(cuda_device, include_diag, N):
    x = make_linear_inputs(2, 3, N, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=12,
                           with_S0=True)
    out, S = run_linear(x, include_diag, S0=x.S0)
    ref, Sref = _oracle(x, include_diag, x.S0)
    assert not np.isnan(out).any()
    assert rel_err(out, ref) <= TOL_BF16
    assert rel_err(S, Sref) <= TOL_BF16


@pytest.mark.parametrize("include_diag", [True, False])
def test_bf16_sequence_split_matches_oracle(cuda_device, include_diag):
    """5000 tokens over 3 heads: each head's 40 tiles run as 5 segments on
    separate SMs, their start states summed by the segment pre-pass from S0
    and the earlier segments' increments; the last tile is ragged."""
    x = make_linear_inputs(1, 3, 5000, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=19,
                           with_S0=True)
    out, S = run_linear(x, include_diag, S0=x.S0)
    ref, Sref = _oracle(x, include_diag, x.S0)
    assert not np.isnan(out).any()
    assert rel_err(out, ref) <= TOL_BF16
    assert rel_err(S, Sref) <= TOL_BF16


def test_bf16_split_and_unsplit_agree(cuda_device):
    """A workspace of only the status block runs every head unsplit; the
    split run differs from it by fp32 summation order and the bf16 rounding
    of the segments' start states only."""
    x = make_linear_inputs(2, 2, 4096, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=20,
                           with_S0=True)
    o_split, S_split = run_linear(x, S0=x.S0)
    o_one, S_one = run_linear(x, S0=x.S0, ws_bytes=T.TTT_STATUS_BYTES)
    assert rel_err(o_split, o_one) <= 1e-2
    assert rel_err(S_split, S_one) <= 1e-5


def test_bf16_output_dtype(cuda_device):
    x = make_linear_inputs(1, 2, 400, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=13)
    out, _ = run_linear(x, out_dtype="bf16")
    ref, _ = _oracle(x)
    assert rel_err(out, ref) <= TOL_BF16


def test_bf16_cuda_core_dims(cuda_device):
    x = make_linear_inputs(1, 2, 150, 32, 48, chunk=16, dtype="bf16", lr_kind="sig-2", cfg=14)
    out, S = run_linear(x)
    ref, Sref = _oracle(x)
    assert rel_err(out, ref) <= TOL_BF16 and rel_err(S, Sref) <= TOL_BF16


def test_chunk_size_invariance(cuda_device):
    x = make_linear_inputs(1, 2, 96, 32, 32, chunk=16, dtype="f32", lr_kind="0.1sig", cfg=15)
    outs = [run_linear(x, chunk=c)[0] for c in (1, 5, 16, 32, 96)]
    for o in outs[1:]:
        assert rel_err(o, outs[0]) <= 1e-5


def test_gradient_ascent_negates_output(cuda_device):
    x = make_linear_inputs(1, 2, 260, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=16)
    o1, _ = run_linear(x)
    x.lr = -x.lr
    o2, _ = run_linear(x)
    assert np.abs(o1 + o2).max() <= 1e-6 * np.abs(o1).max()


def test_streaming_two_calls_equal_one(cuda_device):
    x = make_linear_inputs(1, 2, 512, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=17)
    full, Sfull = run_linear(x)
    import copy
    a, b = copy.deepcopy(x), copy.deepcopy(x)
    for tt, src in ((a.q, x.q), (a.k, x.k), (a.v, x.v)):
        tt.values, tt.bits = src.values[:, :, :256], src.bits[:, :, :256]
    a.lr = x.lr[:, :, :256]
    for tt, src in ((b.q, x.q), (b.k, x.k), (b.v, x.v)):
        tt.values, tt.bits = src.values[:, :, 256:], src.bits[:, :, 256:]
    b.lr = x.lr[:, :, 256:]
    oa, Sa = run_linear(a)
    ob, Sb = run_linear(b, S0=Sa)
    assert rel_err(np.concatenate([oa, ob], 2), full) <= 1e-2
    assert rel_err(Sb, Sfull) <= 1e-3


def test_empty_sequence_is_a_no_op(cuda_device):
    desc = T.make_linear_desc(1, 2, 0, 64, 64, 64)
    S = torch.ones(1, 2, 64, 64, device="cuda")
    ws = T.alloc_workspace(256)
    e = torch.empty(0, device="cuda")
    T.ttt_linear_fwd(desc, e, e, e, e, S, e, ws)
    assert T.ttt_check_device_status(ws) == T.TTT_OK
    assert bool((S == 1).all())


@pytest.mark.slow
@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_bf16_n32k_workload_sampled(cuda_device, out_dtype):
    """Full 4x16x32768 (d = 64) workload: sampled outputs against the
    linear-attention sum, and the final state against sum eta k v^T."""
    x = make_workload("ttt_linear_bf16_n32k")
    out, S = run_linear(x, out_dtype=out_dtype)
    idx = np.array([0, 1, 127, 128, 4095, 16384, 32766, 32767])
    ref = ttt_linear_attention_sum(x.q.values, x.k.values, x.v.values, x.lr, t_index=idx)
    assert rel_err(out[:, :, idx], ref) <= TOL_BF16
    k64 = x.k.values.astype(np.float64)
    ev = x.lr[..., None].astype(np.float64) * x.v.values.astype(np.float64)
    Sref = np.matmul(np.swapaxes(k64, -1, -2), ev)
    assert rel_err(S, Sref) <= TOL_BF16
    assert not np.isnan(out).any()


@pytest.mark.slow
def test_bf16_n32k_workload_two_heads_in_full(cuda_device):
    """Full 4x16x32768 (d = 64) workload in the launch configuration the
    benchmark times (bf16 output, 64-token chunks): two whole (b, h) heads,
    every token, against the token-by-token recurrence, and their end states."""
    x = make_workload("ttt_linear_bf16_n32k")
    out, S = run_linear(x, out_dtype="bf16")
    for b, h in ((0, 0), (3, 15)):
        def sl(t):
            return t[b:b + 1, h:h + 1]
        ref, Sref = ttt_linear_recurrent(sl(x.q.values), sl(x.k.values), sl(x.v.values), sl(x.lr))
        assert rel_err(sl(out), ref) <= TOL_BF16
        assert rel_err(sl(S), Sref) <= TOL_BF16
        assert not np.isnan(sl(out)).any()


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    ws = T.alloc_workspace(256)
    assert T.ttt_selftest_wait_timeout(ws, 2000) == T.TTT_OK
    assert T.ttt_check_device_status(ws) == T.TTT_ERR_TIMEOUT
    assert T.ttt_check_device_status(ws) == T.TTT_OK      # cleared
    x = make_linear_inputs(1, 1, 64, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=18)
    out, _ = run_linear(x)
    assert rel_err(out, _oracle(x)[0]) <= TOL_BF16


# ---------------------------------------------------------------- bidirectional order
# Every token writes, then every query reads the final state: linear attention
# with no causal mask.

def _oracle_bi(x, S0=None):
    return ttt_linear_recurrent(x.q.values, x.k.values, x.v.values, x.lr, S0,
                                order="bidirectional")


def test_bidirectional_f32_n256_workload_shape(cuda_device):
    """The fp32 configuration's shapes (B1 H2 N256 d32, chunk 16) in
    bidirectional order, on the CUDA-core kernel."""
    x = make_workload("ttt_linear_f32_n256")
    out, S = run_linear(x, order="bidirectional")
    ref, Sref = _oracle_bi(x)
    assert rel_err(out, ref) <= TOL_F32
    assert rel_err(S, Sref) <= TOL_F32


def test_bidirectional_f32_ragged_with_initial_state(cuda_device):
    x = make_linear_inputs(2, 3, 77, 24, 40, chunk=9, dtype="f32", lr_kind="0.1sig", cfg=21,
                           with_S0=True)
    out, S = run_linear(x, S0=x.S0, order="bidirectional")
    ref, Sref = _oracle_bi(x, x.S0)
    assert rel_err(out, ref) <= TOL_F32
    assert rel_err(S, Sref) <= TOL_F32


@pytest.mark.parametrize("N", [1, 128, 300, 5000])
def test_bidirectional_bf16_tensor_core(cuda_device, N):
    """State pass over the whole sequence, then reads only, in segments that
    all start from the final state; ragged last tile for N = 300, 5000."""
    x = make_linear_inputs(2, 3, N, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=22,
                           with_S0=True)
    out, S = run_linear(x, S0=x.S0, order="bidirectional")
    ref, Sref = _oracle_bi(x, x.S0)
    assert not np.isnan(out).any()
    assert rel_err(out, ref) <= TOL_BF16
    assert rel_err(S, Sref) <= TOL_BF16


def test_bidirectional_bf16_small_workspace_runs_on_cuda_cores(cuda_device):
    x = make_linear_inputs(1, 2, 700, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=23,
                           with_S0=True)
    out, S = run_linear(x, S0=x.S0, order="bidirectional", ws_bytes=T.TTT_STATUS_BYTES)
    ref, Sref = _oracle_bi(x, x.S0)
    assert rel_err(out, ref) <= TOL_BF16
    assert rel_err(S, Sref) <= TOL_BF16
    o_tc, S_tc = run_linear(x, S0=x.S0, order="bidirectional")
    assert rel_err(o_tc, out) <= 1e-2


def test_bidirectional_bf16_other_dims_and_bf16_out(cuda_device):
    x = make_linear_inputs(1, 2, 150, 32, 48, chunk=16, dtype="bf16", lr_kind="sig-2", cfg=24)
    out, S = run_linear(x, order="bidirectional", out_dtype="bf16")
    ref, Sref = _oracle_bi(x)
    assert rel_err(out, ref) <= TOL_BF16 and rel_err(S, Sref) <= TOL_BF16
    y = make_linear_inputs(1, 2, 400, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=25)
    out, _ = run_linear(y, order="bidirectional", out_dtype="bf16")
    assert rel_err(out, _oracle_bi(y)[0]) <= TOL_BF16


def test_bidirectional_output_is_permutation_equivariant(cuda_device):
    """Permuting the tokens permutes the outputs and leaves the state (up to
    fp32 summation order), as the unmasked form requires."""
    x = make_linear_inputs(1, 2, 384, 64, 64, chunk=64, dtype="bf16", lr_kind="sig-2", cfg=26)
    o, S = run_linear(x, order="bidirectional")
    import copy
    perm = np.random.default_rng(0).permutation(384)
    y = copy.deepcopy(x)
    for tt in (y.q, y.k, y.v):
        tt.values = np.ascontiguousarray(tt.values[:, :, perm])
        tt.bits = np.ascontiguousarray(tt.bits[:, :, perm])
    y.lr = np.ascontiguousarray(x.lr[:, :, perm])
    o_p, S_p = run_linear(y, order="bidirectional")
    assert rel_err(o_p, o[:, :, perm]) <= 1e-2
    assert rel_err(S_p, S) <= 1e-5

"""GPU parity for the LaCT SwiGLU fast-weight layer against the fp64 oracle,
through the C ABI.  Tolerance: normwise max relative error 2e-2 (bf16
operands, fp32 accumulation and fp32 state)."""
import numpy as np
import pytest

from oracle import lact_forward
from oracle.lact import lact_init_state
from ttt_synth import make_lact_inputs, make_workload
from gpu_util import LaCTRun, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _oracle(x, opt="gd", **kw):
    B = x.k.values.shape[0]
    st = lact_init_state(x.W1, x.W3, x.W2, B, opt)
    return lact_forward(x.q.values, x.k.values, x.v.values, x.lr, st, chunk=x.chunk,
                        order=x.order, opt=opt, **kw)


def _check(x, opt="gd", out_dtype="f32", tol=TOL, **kw):
    run = LaCTRun(x, opt=opt, out_dtype=out_dtype, **kw)
    out = run.run()
    ref, st = _oracle(x, opt, **kw)
    assert not np.isnan(out).any()
    assert rel_err(out, ref) <= tol, rel_err(out, ref)
    W = run.weights()
    for g, r in zip(W[:3], (st.W1, st.W3, st.W2)):
        assert rel_err(g, r) <= tol, rel_err(g, r)
    return run, out, ref, st


@pytest.mark.parametrize("opt", ["gd", "momentum"])
def test_causal_ragged_chunks(cuda_device, opt):
    # chunks 256, 256, 128+40: several token tiles and a ragged last chunk
    x = make_lact_inputs(1, 2, 680, 128, 256, chunk=256, order="causal", cfg=31)
    _check(x, opt)


def test_causal_bf16_output(cuda_device):
    x = make_lact_inputs(2, 1, 384, 128, 256, chunk=128, order="causal", cfg=32)
    _check(x, out_dtype="bf16")


@pytest.mark.parametrize("opt", ["gd", "momentum", "muon"])
def test_bidirectional_ragged_queries(cuda_device, opt):
    x = make_lact_inputs(1, 2, 700, 128, 256, chunk=256, order="bidirectional", Nq=200,
                         v_norm=True, lr_kind="0.01sig", cfg=33)
    _check(x, opt)


def test_wide_hidden_and_head_dims(cuda_device):
    x = make_lact_inputs(1, 1, 300, 384, 768, chunk=300, order="bidirectional", Nq=130,
                         v_norm=True, lr_kind="0.01sig", cfg=34)
    _check(x)


def test_update_mask_without_normalisation(cuda_device):
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=128, order="causal", cfg=35)
    run, *_ = _check(x, update_mask=4, normalize_rows=False)
    W = run.weights()
    assert np.array_equal(W[0][0], x.W1) and np.array_equal(W[1][0], x.W3)


def test_rows_are_unit_norm_after_update(cuda_device):
    x = make_lact_inputs(1, 2, 256, 128, 256, chunk=128, order="causal", cfg=36)
    run = LaCTRun(x)
    run.run()
    for W in run.weights():
        assert np.abs(np.linalg.norm(W.astype(np.float64), axis=-1) - 1).max() < 1e-5


def test_causal_outputs_ignore_future_tokens(cuda_device):
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=128, order="causal", cfg=37)
    o1 = LaCTRun(x).run()
    x2 = make_lact_inputs(1, 2, 512, 128, 256, chunk=128, order="causal", cfg=38)
    for a, b in ((x2.q, x.q), (x2.k, x.k), (x2.v, x.v)):
        a.values[:, :, :256], a.bits[:, :, :256] = b.values[:, :, :256], b.bits[:, :, :256]
    x2.lr[:, :, :256] = x.lr[:, :, :256]
    x2.W1, x2.W3, x2.W2 = x.W1, x.W3, x.W2
    o2 = LaCTRun(x2).run()
    assert np.array_equal(o1[:, :, :256], o2[:, :, :256])


def test_streaming_split_equals_single_call(cuda_device):
    import copy
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=128, order="causal", cfg=39)
    full = LaCTRun(x, opt="momentum")
    of = full.run()
    a = copy.deepcopy(x)
    for tt in (a.q, a.k, a.v):
        tt.values, tt.bits = tt.values[:, :, :256], tt.bits[:, :, :256]
    a.lr = a.lr[:, :, :256]
    b = copy.deepcopy(x)
    for tt in (b.q, b.k, b.v):
        tt.values, tt.bits = tt.values[:, :, 256:], tt.bits[:, :, 256:]
    b.lr = b.lr[:, :, 256:]
    ra = LaCTRun(a, opt="momentum")
    oa = ra.run()
    Wa = ra.weights()
    rb = LaCTRun(b, opt="momentum")
    rb.init_state(Wa[0], Wa[1], Wa[2], per_batch=True)
    rb.set_momentum(*Wa[3:])
    ob = rb.run()
    assert rel_err(np.concatenate([oa, ob], 2), of) <= 1e-5


@pytest.mark.slow
def test_causal_n32k_workload(cuda_device):
    x = make_workload("lact_causal_n32k")
    _check(x)


@pytest.mark.slow
def test_bidirectional_196k_workload(cuda_device):
    x = make_workload("lact_bidir_196k")
    _check(x)


def test_split_operands_tighten_gd(cuda_device):
    """hi+lo bf16 operands (about 16 significant bits) must track the fp64
    oracle at least 4x closer than plain bf16 operands."""
    x = make_lact_inputs(1, 2, 640, 128, 256, chunk=256, order="causal", cfg=40)
    ref, _ = _oracle(x)
    e_plain = rel_err(LaCTRun(x, split_operands=False).run(), ref)
    e_split = rel_err(LaCTRun(x, split_operands=True).run(), ref)
    assert e_split <= TOL and e_split * 4 <= e_plain, (e_split, e_plain)


@pytest.mark.slow
def test_bidirectional_muon_1m_workload(cuda_device):
    """~1M input tokens in 64K chunks (15 full + one 46080-token chunk) with
    momentum 0.9 and five Newton-Schulz steps, then 8040 queries."""
    x = make_workload("lact_bidir_muon_1m")
    _check(x, "muon", beta=0.9, ns_steps=5)


def test_cuda_graph_replay_matches_eager(cuda_device):
    """The whole call (fork/join helper streams, memsets, programmatic
    dependent launches) is capturable; replaying the graph reproduces the
    eagerly launched result bit for bit."""
    import torch
    import learned_linear_attention_b200 as T
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=128, order="causal", cfg=41)
    run = LaCTRun(x, opt="momentum")
    eager = run.run()
    W0 = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        T.lact_state_init(run.desc, *W0, 0, run.state)
        T.lact_chunk_fwd(run.desc, run.q, run.k, run.v, run.lr, run.state, run.out, run.ws)
    run.out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(run.out.cpu().numpy(), eager)


def test_causal_many_chunks_multi_tile_groups(cuda_device):
    """Chunks of 1024 tokens over 8 heads: every fused key/gradient work item
    covers several token tiles, and the read of each chunk runs beside the
    gradient of the same chunk."""
    x = make_lact_inputs(2, 4, 4096, 128, 256, chunk=1024, order="causal", cfg=42)
    _check(x)


def test_causal_update_mask_w1_w3_with_norm_keeps_w2(cuda_device):
    """W2 excluded from the update on the fused path: every bf16 buffer must
    hold the initial W2, which stays exactly unchanged, and the rows of W1
    and W3 are normalised."""
    x = make_lact_inputs(1, 2, 640, 128, 256, chunk=128, order="causal", cfg=43)
    run, *_ = _check(x, update_mask=3)
    W = run.weights()
    assert np.array_equal(W[2][0], x.W2)
    for w in W[:2]:
        assert np.abs(np.linalg.norm(w.astype(np.float64), axis=-1) - 1).max() < 1e-5


def test_causal_chunk_not_a_multiple_of_the_tile(cuda_device):
    """Chunks of 200 tokens: the last tile of each chunk holds rows of the
    next chunk, which must not enter this chunk's gradient."""
    x = make_lact_inputs(1, 2, 600, 128, 256, chunk=200, order="causal", cfg=44)
    _check(x)
    _check(x, "momentum")


def test_causal_head_dim_256_fused_gemm_update(cuda_device):
    """d = dh = 256 runs the key pass and the gradient GEMMs with the update
    fused into their epilogues (momentum)."""
    x = make_lact_inputs(1, 2, 512, 256, 256, chunk=256, order="causal", cfg=45)
    _check(x, "momentum")


def test_causal_hidden_128_and_many_items_per_cta(cuda_device):
    """dh = 128 (two hidden blocks per head) over 64 heads: more work items
    than SMs, so CTAs of the fused kernel run several items."""
    x = make_lact_inputs(4, 16, 512, 128, 128, chunk=256, order="causal", cfg=46)
    _check(x)


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_w2_only_parallel_form(cuda_device, out_dtype):
    """Only W2 updated, plain GD, no row norm: the layer is block-causal linear
    attention on silu(W1 x) * (W3 x) and runs in its parallel form (one key
    pass, per-chunk increments as the splits of one GEMM, a prefix over
    chunks, one batched read).  W1 and W3 stay exactly as given."""
    x = make_lact_inputs(2, 2, 2048, 128, 256, chunk=256, order="causal", cfg=47)
    run, *_ = _check(x, out_dtype=out_dtype, update_mask=4, normalize_rows=False)
    W = run.weights()
    assert np.array_equal(W[0][0], x.W1) and np.array_equal(W[1][0], x.W3)


def test_w2_only_chunk_loop_in_the_minimum_workspace(cuda_device):
    """Given only lact_workspace_bytes_min, the same W2-only layer runs the
    chunk loop instead of the parallel form; both match the oracle."""
    x = make_lact_inputs(2, 2, 2048, 128, 256, chunk=256, order="causal", cfg=47)
    kw = dict(update_mask=4, normalize_rows=False)
    fast, loop = LaCTRun(x, **kw), LaCTRun(x, min_workspace=True, **kw)
    assert loop.ws.numel() < fast.ws.numel()
    a, b = fast.run(), loop.run()
    ref, st = _oracle(x, "gd", **kw)
    assert rel_err(b, ref) <= TOL, rel_err(b, ref)
    assert rel_err(a, ref) <= TOL, rel_err(a, ref)
    assert rel_err(loop.weights()[2], st.W2) <= TOL


# ---------------------------------------------------------------- fused Newton-Schulz
# The Muon step runs every Newton-Schulz step of a chunk in one cooperative
# launch with grid-wide barriers between its phases.

@pytest.mark.parametrize("ns_steps", [1, 2, 5])
def test_muon_fused_newton_schulz_view_synthesis_dims(cuda_device, ns_steps):
    """d = 384, dh = 768 (the view-synthesis shapes): six 384 x 768 matrices
    per chunk, three chunks, the last ragged."""
    x = make_lact_inputs(1, 2, 600, 384, 768, chunk=256, order="bidirectional", Nq=150,
                         v_norm=True, lr_kind="0.01sig", cfg=43)
    _check(x, "muon", beta=0.9, ns_steps=ns_steps)


def test_muon_fused_newton_schulz_plain_bf16_operands(cuda_device):
    """The fused kernel with plain bf16 operands (one product per step).
    Muon amplifies operand rounding, so plain bf16 lands near the 2e-2 bar
    (about 2.2e-2 here); the default split operands (hi + lo) must meet it and
    be at least twice as close."""
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=256, order="bidirectional", Nq=128,
                         v_norm=True, lr_kind="0.01sig", cfg=44)
    ref, st = _oracle(x, "muon", beta=0.9, ns_steps=5)
    plain = LaCTRun(x, opt="muon", beta=0.9, ns_steps=5, split_operands=False)
    e_plain = rel_err(plain.run(), ref)
    split = LaCTRun(x, opt="muon", beta=0.9, ns_steps=5, split_operands=True)
    e_split = rel_err(split.run(), ref)
    assert e_plain <= 5e-2 and e_split <= TOL and 2 * e_split <= e_plain, (e_plain, e_split)
    for g, r in zip(split.weights()[:3], (st.W1, st.W3, st.W2)):
        assert rel_err(g, r) <= TOL, rel_err(g, r)


def test_muon_cuda_graph_replay_matches_eager(cuda_device):
    """The cooperative Newton-Schulz launch is capturable; replay is bit-exact."""
    import torch
    import learned_linear_attention_b200 as T
    x = make_lact_inputs(1, 2, 512, 128, 256, chunk=256, order="bidirectional", Nq=128,
                         v_norm=True, lr_kind="0.01sig", cfg=45)
    run = LaCTRun(x, opt="muon")
    eager = run.run()
    W0 = [torch.from_numpy(w).cuda() for w in (x.W1, x.W3, x.W2)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        T.lact_state_init(run.desc, *W0, 0, run.state)
        T.lact_chunk_fwd(run.desc, run.q, run.k, run.v, run.lr, run.state, run.out, run.ws)
    run.out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(run.out.cpu().numpy(), eager)


# ---------------------------------------------------------------- chunk loop
# A causal head-dim-128 GD / momentum call whose items leave spare SMs runs as
# one cooperative launch over all chunks; TTT_LACT_CHUNK_LOOP=0 keeps one
# launch per chunk.  Both must agree.

_LOOP_SCRIPT = r"""
import sys, numpy as np
sys.path.insert(0, sys.argv[1])
from ttt_synth import make_lact_inputs
from gpu_util import LaCTRun
x = make_lact_inputs(2, 4, int(sys.argv[3]), 128, 256, chunk=1024, order="causal", cfg=47)
run = LaCTRun(x, opt="momentum")
out = run.run()
W = run.weights()
np.savez(sys.argv[2], out=out, W1=W[0], W3=W[1], W2=W[2])
"""


@pytest.mark.parametrize("n", [4096, 4096 + 1000])
def test_chunk_loop_matches_per_chunk_launches(cuda_device, tmp_path, n):
    """The same call with the chunk loop and with per-chunk launches, each
    in a fresh process: identical arithmetic, so the outputs and weights
    agree to rounding (bit for bit when every chunk is full), and both match
    the oracle."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = {}
    for mode in ("1", "0"):
        path = tmp_path / f"loop{mode}.npz"
        env = dict(os.environ, TTT_LACT_CHUNK_LOOP=mode)
        r = subprocess.run([sys.executable, "-c", _LOOP_SCRIPT, os.path.join(root, "tests"), str(path), str(n)],
                           env=env, cwd=root, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        res[mode] = np.load(path)
    for key in ("out", "W1", "W3", "W2"):
        a, b = res["1"][key], res["0"][key]
        if n % 1024 == 0:
            assert np.array_equal(a, b), (key, rel_err(a, b))
        else:
            assert rel_err(a, b) <= 1e-5, (key, rel_err(a, b))
    x = make_lact_inputs(2, 4, n, 128, 256, chunk=1024, order="causal", cfg=47)
    ref, st = _oracle(x, "momentum")
    assert rel_err(res["1"]["out"], ref) <= TOL
    for key, r in (("W1", st.W1), ("W3", st.W3), ("W2", st.W2)):
        assert rel_err(res["1"][key], r) <= TOL


def test_chunk_loop_is_one_launch(cuda_device):
    """An eligible causal call runs as one chunk-loop launch (plus the bf16
    weight copy), not as per-chunk kernels."""
    import learned_linear_attention_b200 as T
    x = make_lact_inputs(1, 2, 4096, 128, 256, chunk=1024, order="causal", cfg=48)
    run = LaCTRun(x)
    run.run()
    T.ttt_profile_begin()
    run.run()
    prof = T.ttt_profile_end()
    assert prof.get("lact_loop", {}).get("launches") == 1, prof
    assert "lact_keygrad" not in prof and "lact_update" not in prof, prof

"""The C ABI without a GPU: the library loads, exports every entry point that
include/ttt.h declares, the ctypes structs match the C layout, and host-side
validation rejects bad arguments before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import learned_linear_attention_b200 as T
from learned_linear_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^(?:int|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from learned_linear_attention_b200 import build
        build.build()
    return T.load()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("ttt_linear_fwd", "lact_chunk_fwd", "lact_state_init", "lact_state_readout",
              "ttt_linear_state_init", "ttt_linear_state_readout", "ttt_check_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared_functions()) <= set(_lib._SIGS)


def test_ctypes_structs_match_c_layout(lib):
    fields = {"ttt_linear_desc": [f[0] for f in T.ttt_linear_desc._fields_],
              "lact_desc": [f[0] for f in T.lact_desc._fields_],
              "ttt_window_desc": [f[0] for f in T.ttt_window_desc._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', 'int main(void){']
    for s, fl in fields.items():
        lines.append(f'printf("{s} %zu\\n", sizeof({s}));')
        for f in fl:
            lines.append(f'printf("{s}.{f} %zu\\n", offsetof({s}, {f}));')
    lines.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "l.c")
        open(c, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-o", os.path.join(d, "l"), c], check=True)
        out = subprocess.run([os.path.join(d, "l")], capture_output=True, text=True,
                             check=True).stdout.split("\n")
    got = dict(line.split() for line in out if line)
    for s, fl in fields.items():
        cls = getattr(T, s)
        assert int(got[s]) == ctypes.sizeof(cls), s
        for f in fl:
            assert int(got[f"{s}.{f}"]) == getattr(cls, f).offset, f"{s}.{f}"


def test_status_strings(lib):
    assert T.status_string(0) == "TTT_OK"
    assert T.status_string(-8) == "TTT_ERR_TIMEOUT"
    assert T.status_string(-99) == "TTT_ERR_UNKNOWN"
    assert "sm_100a" in T.ttt_build_info()


def _call_linear_fwd(desc, q=16, k=16, v=16, lr=16, S=16, out=16, ws=16, ws_bytes=256):
    return T.load().ttt_linear_fwd(ctypes.byref(desc), q, k, v, lr, S, out, ws, ws_bytes, None)


def test_linear_validation_before_launch(lib):
    good = T.make_linear_desc(1, 2, 8, 64, 64, 16)
    bad_shape = T.make_linear_desc(0, 2, 8, 64, 64, 16)
    assert _call_linear_fwd(bad_shape) == T.TTT_ERR_SHAPE
    assert _call_linear_fwd(T.make_linear_desc(1, 2, 8, 64, 64, 0)) == T.TTT_ERR_ARG
    assert _call_linear_fwd(T.make_linear_desc(1, 2, 8, 256, 64, 16)) == T.TTT_ERR_UNSUPPORTED
    d = T.make_linear_desc(1, 2, 8, 64, 64, 16)
    d.in_dtype = 7
    assert _call_linear_fwd(d) == T.TTT_ERR_DTYPE
    assert _call_linear_fwd(good, ws_bytes=8) == T.TTT_ERR_WORKSPACE
    assert _call_linear_fwd(good, q=0) == T.TTT_ERR_ARG
    assert _call_linear_fwd(good, k=24) == T.TTT_ERR_ALIGN
    # N = 0 is a valid empty call and launches nothing
    assert _call_linear_fwd(T.make_linear_desc(1, 2, 0, 64, 64, 16)) == T.TTT_OK
    assert T.ttt_linear_workspace_bytes(good) == T.TTT_STATUS_BYTES
    d = T.make_linear_desc(1, 2, 8, 64, 64, 16)
    d.order = 5
    assert _call_linear_fwd(d) == T.TTT_ERR_ARG


def test_linear_bidirectional_desc(lib):
    """order sits between chunk and include_diag, as the boundary table has it;
    the bidirectional tensor-core path sizes room for the state pass's
    partial sums (a CUDA-core fallback runs with less), and the backward pass
    is causal only."""
    d = T.make_linear_desc(1, 2, 8, 64, 64, 16, order="bidirectional")
    assert d.order == T.TTT_BIDIRECTIONAL
    assert [f[0] for f in T.ttt_linear_desc._fields_][6] == "order"
    assert _call_linear_fwd(T.make_linear_desc(1, 2, 0, 64, 64, 16, order="bidirectional")) == \
        T.TTT_OK
    assert T.ttt_linear_workspace_bytes(d) > T.TTT_STATUS_BYTES
    f32 = T.make_linear_desc(1, 2, 8, 32, 32, 16, in_dtype="f32", order="bidirectional")
    assert T.ttt_linear_workspace_bytes(f32) == T.TTT_STATUS_BYTES
    assert _call_linear_bwd(d) == T.TTT_ERR_UNSUPPORTED
    n = ctypes.c_size_t(0)
    assert T.load().ttt_linear_bwd_workspace_bytes(ctypes.byref(d), ctypes.byref(n)) == \
        T.TTT_ERR_UNSUPPORTED


def _call_linear_bwd(desc, ws_bytes=1 << 40, **ptrs):
    p = dict(q=16, k=16, v=16, lr=16, S0=0, dout=16, dS_end=0, dq=16, dk=16, dv=16, dlr=16,
             dS0=16, ws=16)
    p.update(ptrs)
    return T.load().ttt_linear_bwd(ctypes.byref(desc), p["q"], p["k"], p["v"], p["lr"], p["S0"],
                                   p["dout"], p["dS_end"], p["dq"], p["dk"], p["dv"], p["dlr"],
                                   p["dS0"], p["ws"], ws_bytes, None)


def test_linear_backward_validation_before_launch(lib):
    good = T.make_linear_desc(1, 2, 8, 64, 64, 16)
    assert _call_linear_bwd(T.make_linear_desc(0, 2, 8, 64, 64, 16)) == T.TTT_ERR_SHAPE
    assert _call_linear_bwd(T.make_linear_desc(1, 2, 8, 256, 64, 16)) == T.TTT_ERR_UNSUPPORTED
    assert _call_linear_bwd(good, ws_bytes=T.TTT_STATUS_BYTES) == T.TTT_ERR_WORKSPACE
    assert _call_linear_bwd(good, dS0=0) == T.TTT_ERR_ARG
    assert _call_linear_bwd(good, dq=0) == T.TTT_ERR_ARG
    assert _call_linear_bwd(good, dout=0) == T.TTT_ERR_ARG
    assert _call_linear_bwd(good, dv=40) == T.TTT_ERR_ALIGN
    assert _call_linear_bwd(good, S0=8) == T.TTT_ERR_ALIGN


def test_linear_backward_workspace(lib):
    # 32K tokens x 64 heads of dims 64: a float32 lr = 1 array per token, four
    # [64][64] float32 states per head and the segment states of one scan
    d = T.make_linear_desc(4, 16, 32768, 64, 64, 64)
    need = T.ttt_linear_bwd_workspace_bytes(d)
    floor = T.TTT_STATUS_BYTES + 64 * 32768 * 4 + 4 * 64 * 64 * 64 * 4
    assert floor <= need <= floor + T.ttt_linear_workspace_bytes(d) + 4096
    small = T.make_linear_desc(1, 2, 100, 24, 40, 9, in_dtype="f32")
    assert T.ttt_linear_bwd_workspace_bytes(small) >= T.TTT_STATUS_BYTES + 2 * 100 * 4 + \
        4 * 2 * 24 * 40 * 4


def _call_lact(desc, ws_bytes=1 << 40, **ptrs):
    p = dict(q=16, k=16, v=16, lr=16, state=16, out=16, ws=16)
    p.update(ptrs)
    return T.load().lact_chunk_fwd(ctypes.byref(desc), p["q"], p["k"], p["v"], p["lr"],
                                   p["state"], p["out"], p["ws"], ws_bytes, None)


def test_lact_validation_before_launch(lib):
    assert _call_lact(T.make_lact_desc(1, 2, 64, 96, 256, 32)) == T.TTT_ERR_UNSUPPORTED
    assert _call_lact(T.make_lact_desc(1, 2, 64, 128, 200, 32)) == T.TTT_ERR_UNSUPPORTED
    assert _call_lact(T.make_lact_desc(1, 2, 64, 128, 256, 0)) == T.TTT_ERR_ARG
    d = T.make_lact_desc(1, 2, 64, 128, 256, 32)
    d.N_q = 10                                    # causal needs N_q == N_in
    assert _call_lact(d) == T.TTT_ERR_SHAPE
    d = T.make_lact_desc(1, 2, 64, 128, 256, 32, update_mask=0)
    assert _call_lact(d) == T.TTT_ERR_ARG
    d = T.make_lact_desc(1, 2, 64, 128, 256, 32)
    d.in_dtype = T.TTT_F32
    assert _call_lact(d) == T.TTT_ERR_DTYPE
    good = T.make_lact_desc(1, 2, 64, 128, 256, 32)
    assert _call_lact(good, ws_bytes=100) == T.TTT_ERR_WORKSPACE
    assert _call_lact(good, k=0) == T.TTT_ERR_ARG
    assert _call_lact(good, v=40) == T.TTT_ERR_ALIGN


@pytest.mark.parametrize("opt,mult", [("gd", 3), ("momentum", 6), ("muon", 6)])
def test_lact_state_bytes(lib, opt, mult):
    d = T.make_lact_desc(2, 4, 32768, 128, 256, 2048, opt=opt)
    assert T.lact_state_bytes(d) == mult * 2 * 4 * 128 * 256 * 4


def test_lact_workspace_sizes_for_the_workloads(lib):
    # 32K-token causal layer: bf16 weights + four [BH, 2048, dh] intermediates + partials
    d3 = T.make_lact_desc(2, 4, 32768, 128, 256, 2048)
    ws3 = T.lact_workspace_bytes(d3)
    assert 4 * 8 * 2048 * 256 * 2 < ws3 < 64 << 20
    # a short W2-only layer: the workspace of its fastest form is never
    # smaller than the chunk loop's, which every call accepts
    dw = T.make_lact_desc(1, 2, 256, 128, 256, 128, update_mask=4, normalize_rows=False)
    assert T.lact_workspace_bytes(dw) >= T.lact_workspace_bytes_min(dw)
    # 196K-token view-synthesis set in one chunk: intermediates dominate
    d4 = T.make_lact_desc(1, 2, 196608, 384, 768, 196608, N_q=4096, order="bidirectional")
    assert T.lact_workspace_bytes(d4) > 3 * 2 * 196608 * 768 * 2
    # ~1M tokens in 64K chunks with Muon: Newton-Schulz buffers present
    d5 = T.make_lact_desc(1, 2, 1029120, 384, 768, 65536, N_q=8040, order="bidirectional",
                          opt="muon")
    assert T.lact_workspace_bytes(d5) < 2 << 30
    for d in (d3, d4, d5):
        assert T.lact_workspace_bytes_min(d) == T.lact_workspace_bytes(d)


def test_w2_only_parallel_form_workspace(lib):
    # the W2-only GD layer without normalisation holds every chunk's features
    # ([BH, N, dh] bf16 twice) and W2 increment ([chunks, BH, d, dh] fp32 and
    # bf16); the chunk loop it falls back to needs the 32K layer's size
    full = T.make_lact_desc(2, 4, 32768, 128, 256, 2048)
    w2 = T.make_lact_desc(2, 4, 32768, 128, 256, 2048, update_mask=4, normalize_rows=False)
    need = T.lact_workspace_bytes(w2)
    assert need >= 2 * 8 * 32768 * 256 * 2 + 16 * 8 * 128 * 256 * 6
    assert T.lact_workspace_bytes_min(w2) <= T.lact_workspace_bytes(full) < 64 << 20
    # not eligible: row norm on, a chunk that does not divide N, momentum
    for kw in (dict(normalize_rows=True), dict(chunk=3000), dict(opt="momentum")):
        args = dict(update_mask=4, normalize_rows=False, chunk=2048)
        args.update(kw)
        chunk = args.pop("chunk")
        d = T.make_lact_desc(2, 4, 32768, 128, 256, chunk, **args)
        assert T.lact_workspace_bytes(d) == T.lact_workspace_bytes_min(d)
    # a workspace below the minimum is rejected before any launch
    assert _call_lact(w2, ws_bytes=T.lact_workspace_bytes_min(w2) - 256) == T.TTT_ERR_WORKSPACE


def test_window_attention_validation_before_launch(lib):
    def call(desc, **p):
        a = dict(q=16, k=16, v=16, out=16, ws=16, ws_bytes=256)
        a.update(p)
        return T.load().ttt_window_attn_fwd(ctypes.byref(desc), a["q"], a["k"], a["v"], a["out"],
                                            a["ws"], a["ws_bytes"], None)
    assert call(T.make_window_desc(1, 2, 64, 64, 16)) == T.TTT_ERR_UNSUPPORTED
    assert call(T.make_window_desc(1, 2, 64, 128, 0)) == T.TTT_ERR_ARG
    assert call(T.make_window_desc(0, 2, 64, 128, 16)) == T.TTT_ERR_SHAPE
    d = T.make_window_desc(1, 2, 64, 128, 16)
    d.in_dtype = T.TTT_F32
    assert call(d) == T.TTT_ERR_DTYPE
    good = T.make_window_desc(1, 2, 64, 128, 16)
    assert call(good, ws_bytes=8) == T.TTT_ERR_WORKSPACE
    assert call(good, k=0) == T.TTT_ERR_ARG
    assert call(good, out=24) == T.TTT_ERR_ALIGN
    assert call(T.make_window_desc(1, 2, 0, 128, 16)) == T.TTT_OK    # empty: nothing launched
    # the layer: causal order only, and the window's own checks
    lact = T.make_lact_desc(1, 2, 64, 128, 256, 32, order="bidirectional", N_q=8)
    assert T.load().lact_layer_fwd(ctypes.byref(lact), 16, ctypes.c_float(0), 16, 16, 16, 16, 16,
                                   16, 16, 1 << 40, None) == T.TTT_ERR_ARG
    lact = T.make_lact_desc(1, 2, 64, 128, 256, 32)
    assert T.load().lact_layer_fwd(ctypes.byref(lact), 0, ctypes.c_float(0), 16, 16, 16, 16, 16,
                                   16, 16, 1 << 40, None) == T.TTT_ERR_ARG


def test_context_parallel_pieces_validate_before_launch(lib):
    """lact_chunk_grad / lact_apply_grad / lact_read reject bad ranges, null
    buffers and short workspaces on the host, before anything is enqueued."""
    L = T.load()
    d = T.make_lact_desc(1, 2, 512, 128, 256, 256)
    assert T.lact_grad_bytes(d) == 3 * 2 * 128 * 256 * 4
    ws = T.lact_workspace_bytes(d)
    g = lambda t0, n, G=16, w=ws: L.lact_chunk_grad(ctypes.byref(d), t0, n, 16, 16, 16, 16, G, 16,  # noqa: E731,E501
                                                    w, None)
    assert g(500, 20) == T.TTT_ERR_SHAPE           # past N_in
    assert g(0, 300) == T.TTT_ERR_SHAPE            # more than one chunk
    assert g(-1, 10) == T.TTT_ERR_SHAPE
    assert g(0, 10, G=0) == T.TTT_ERR_ARG
    assert g(0, 10, w=64) == T.TTT_ERR_WORKSPACE
    assert g(0, 10, G=24) == T.TTT_ERR_ALIGN
    assert L.lact_apply_grad(ctypes.byref(d), 0, 16, 16, ws, None) == T.TTT_ERR_ARG
    assert L.lact_apply_grad(ctypes.byref(d), 16, 16, 16, 64, None) == T.TTT_ERR_WORKSPACE
    r = lambda t0, n: L.lact_read(ctypes.byref(d), t0, n, 16, 16, 16, 16, ws, None)  # noqa: E731
    assert r(400, 200) == T.TTT_ERR_SHAPE
    assert r(0, 0) == T.TTT_OK                     # nothing to read
    bi = T.make_lact_desc(1, 2, 512, 128, 256, 256, N_q=100, order="bidirectional")
    assert L.lact_read(ctypes.byref(bi), 50, 60, 16, 16, 16, 16, T.lact_workspace_bytes(bi),
                       None) == T.TTT_ERR_SHAPE

"""The bounds-checked build (libmoba_debug.so) on the GPU.

Every entry point runs clean under it (no index check fails, no guard is
overwritten) and gives the release library's results bit for bit, and the
forward still matches the oracle.  Each check is then made to fire by a slip
planted through moba_debug_poison -- a bucket entry read as a slot outside
the query chunk (caught before the access; the row is dropped), one guard
word overwritten between the fill and the check -- and the same workspace
runs clean right after.
"""
import ctypes

import pytest
import torch

import block_sparse_long_11_b200 as mb
import synth
from tests import parity as P
from tests.debug_lib import load_both, using

pytestmark = pytest.mark.gpu

DEV = "cuda"
SITE_ATTN_ENTRY = 2  # the block-attention kernel's bucket-entry check


@pytest.fixture(scope="module")
def libs():
    assert torch.cuda.is_available()
    return load_both()


def _forward(x, w, ws, chunk=None):
    out, lse, idx = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], w.block_size, w.topk,
                                    chunk_tokens=chunk, workspace=ws, return_idx=True)
    return out, lse, idx


def _error_info(lib, ws):
    info = ctypes.c_int(-1)
    rc = lib.moba_debug_error_info(ws.buf.data_ptr(), torch.cuda.current_stream().cuda_stream,
                                   ctypes.byref(info))
    assert rc == 0
    return info.value


@pytest.mark.parametrize("shape,chunk", [
    (([1500, 700], 4, 2, 128, 128, 4), 512),    # varlen, GQA, several query chunks
    (([2048], 2, 1, 64, 256, 8), None),         # d64, one chunk
])
def test_forward_clean_same_as_release_and_oracle(libs, shape, chunk):
    rel, dbg = libs
    seqlens, Hq, Hkv, d, B, topk = shape
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=4242, device=DEV)
    with using(rel):
        ws_r = mb.Workspace()
        ref = _forward(x, w, ws_r, chunk)
        mb.moba_check(ws_r)
    with using(dbg):
        ws_d = mb.Workspace()
        got = _forward(x, w, ws_d, chunk)
        mb.moba_check(ws_d)
        assert _error_info(dbg, ws_d) == 0
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    P.check_rows(x, w, got[0], got[1], got[2], P.all_rows(w))


def test_other_entry_points_clean_same_as_release(libs):
    rel, dbg = libs
    w, x = synth.make_custom([1300, 700], 4, 2, 128, 128, 4, seed=4343, device=DEV)
    dout = synth.normal_bf16(tuple(x["q"].shape), 4343, 50, DEV)
    dec = synth.make_decode(2, 320, 4, 2, 128, seed=4344, device=DEV)
    sl = torch.tensor([200, 257], dtype=torch.int32, device=DEV)

    def run():
        ws = mb.Workspace()
        res = {}
        res["gate"] = mb.moba_gate(x["q"], x["k"], x["cu_seqlens"], w.block_size, w.topk,
                                   workspace=ws)
        mb.moba_check(ws)
        res["noalloc"] = mb.moba_gate_noalloc(x["q"], x["k"], x["cu_seqlens"], w.block_size,
                                              w.topk)
        res["full"] = mb.moba_forward_full(x["q"], x["k"], x["v"], x["cu_seqlens"], workspace=ws)
        mb.moba_check(ws)
        out, lse, idx = _forward(x, w, ws)
        mb.moba_check(ws)
        res["bwd"] = mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"],
                                      idx, w.block_size, w.topk, chunk_tokens=600, workspace=ws)
        mb.moba_check(ws)
        kbar = mb.moba_decode_init(dec["k_cache"], sl, 64)
        res["dec"] = mb.moba_decode(dec["q"], dec["k_cache"], dec["v_cache"], sl, kbar, 64, 3,
                                    workspace=ws, return_idx=True)
        mb.moba_check(ws)
        torch.cuda.synchronize()
        return res

    with using(rel):
        ref = run()
    with using(dbg):
        got = run()
    for key in ref:
        a, b = got[key], ref[key]
        a = a if isinstance(a, (tuple, list)) else (a,)
        b = b if isinstance(b, (tuple, list)) else (b,)
        for u, v in zip(a, b):
            assert torch.equal(u, v), key


def test_index_check_catches_a_planted_entry_then_runs_clean(libs):
    _, dbg = libs
    w, x = synth.make_custom([1500, 700], 4, 2, 128, 128, 4, seed=4545, device=DEV)
    with using(dbg):
        ws = mb.Workspace()
        assert dbg.moba_debug_poison(1) == 0
        try:
            _forward(x, w, ws)
            with pytest.raises(mb.MobaError) as ei:
                mb.moba_check(ws)
            assert ei.value.code == 8                     # MOBA_ERR_BOUNDS
            assert _error_info(dbg, ws) == SITE_ATTN_ENTRY
        finally:
            dbg.moba_debug_poison(0)
        out, lse, idx = _forward(x, w, ws)
        mb.moba_check(ws)
        torch.cuda.synchronize()
    P.check_rows(x, w, out, lse, idx, P.all_rows(w))


def test_guard_check_catches_an_overwrite_then_runs_clean(libs):
    _, dbg = libs
    w, x = synth.make_custom([1500, 700], 4, 2, 128, 128, 4, seed=4646, device=DEV)
    with using(dbg):
        ws = mb.Workspace()
        assert dbg.moba_debug_poison(2) == 0
        try:
            _forward(x, w, ws)
            with pytest.raises(mb.MobaError) as ei:
                mb.moba_check(ws)
            assert ei.value.code == 9                     # MOBA_ERR_CANARY
            assert _error_info(dbg, ws) == 0              # the first guard
        finally:
            dbg.moba_debug_poison(0)
        out, lse, idx = _forward(x, w, ws)
        mb.moba_check(ws)
        torch.cuda.synchronize()
    P.check_rows(x, w, out, lse, idx, P.all_rows(w))

"""moba_gate_noalloc: the gate run on the library's static scratch.

Some callers cannot allocate device memory when they run the gate (their
device memory belongs to another allocator they must not call into, or their
setup forbids allocations after start-up).  This checks, through the C ABI,
that the allocation-free entry point selects exactly the blocks that
moba_gate selects with a caller-provided workspace, on two calls in a row
(the second one on scratch that still holds the first call's contents), and
that shapes whose scratch would not fit are refused on the host.
"""
import ctypes

import pytest
import torch

import block_sparse_long_11_b200 as mb
import synth

pytestmark = pytest.mark.gpu


def _call(L, x, w, out):
    q, k, cu = x["q"], x["k"], x["cu_seqlens"]
    T, Hq, d = q.shape
    return L.moba_gate_noalloc(q.data_ptr(), k.data_ptr(), cu.data_ptr(), cu.numel() - 1, T, Hq,
                               k.shape[1], d, w.block_size, w.topk, out.data_ptr(),
                               torch.cuda.current_stream().cuda_stream)


def test_gate_noalloc_matches_gate_on_two_calls():
    from block_sparse_long_11_b200 import build
    build.build()
    L = mb.lib()
    shapes = [([5000, 3000, 777], 8, 2, 128, 256, 5, 71),
              ([4096 * 3 + 100], 4, 4, 64, 128, 3, 72)]
    for seqlens, Hq, Hkv, d, B, topk, seed in shapes:
        w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=seed, device="cuda")
        ref = mb.moba_gate(x["q"], x["k"], x["cu_seqlens"], B, topk)
        mb.moba_check()
        for _ in range(2):
            out = torch.full_like(ref, -7)
            assert _call(L, x, w, out) == 0
            assert L.moba_gate_noalloc_check(torch.cuda.current_stream().cuda_stream) == 0
            torch.cuda.synchronize()
            assert torch.equal(out, ref)


def test_gate_noalloc_refuses_scratch_beyond_the_static_array():
    L = mb.lib()
    P = 1 << 20   # aligned fake pointers: the call must return before touching them
    # 2^24 tokens in blocks of 64 need far more than 32 MiB of pooled-key scratch
    rc = L.moba_gate_noalloc(P, P, P, 1, 1 << 24, 8, 8, 128, 64, 4, P, None)
    assert rc == 3


def test_gate_noalloc_error_word_is_per_call():
    """A malformed call's error is reported by the check that follows it; the
    next call, even an empty one, starts from a clean error word."""
    from block_sparse_long_11_b200 import build
    build.build()
    L = mb.lib()
    w, x = synth.make_custom([512], 2, 2, 64, 64, 3, seed=73, device="cuda")
    out = torch.empty((512, 2, 3), dtype=torch.int32, device="cuda")
    bad = torch.tensor([0, 600], dtype=torch.int32, device="cuda")   # beyond the tokens
    st = torch.cuda.current_stream().cuda_stream
    q, k = x["q"], x["k"]
    assert L.moba_gate_noalloc(q.data_ptr(), k.data_ptr(), bad.data_ptr(), 1, 512, 2, 2, 64, 64,
                               3, out.data_ptr(), st) == 0
    assert L.moba_gate_noalloc_check(st) == 6
    assert L.moba_gate_noalloc(q.data_ptr(), k.data_ptr(), bad.data_ptr(), 1, 0, 2, 2, 64, 64,
                               3, out.data_ptr(), st) == 0
    assert L.moba_gate_noalloc_check(st) == 0

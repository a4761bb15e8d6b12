"""The C-ABI library loads, exports every symbol moba.h declares, and rejects
bad arguments on the host (no compute call, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

import block_sparse_long_11_b200 as mb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moba.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(moba_\w+)\s*\(", src, re.M)))


@pytest.fixture(scope="module")
def L():
    from block_sparse_long_11_b200 import build
    build.build()
    return mb.lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert set(names) == set(mb.EXPORTS), names
    for n in names:
        assert hasattr(L, n), n
        ctypes.cast(getattr(L, n), ctypes.c_void_p)


def test_status_strings(L):
    for code, name in mb._lib.STATUS.items():
        assert mb.moba_status_string(code) == name
    assert mb.moba_status_string(99) == "MOBA_ERR_UNKNOWN"


def test_workspace_size_host_only(L):
    n1 = mb.moba_workspace_size(2048, 1, 1, 1, 64, 256, 3, 0)
    n2 = mb.moba_workspace_size(2048, 1, 1, 1, 64, 256, 3, 512)
    assert n1 > n2 > 0
    # partial buffer grows by chunk * Hq * topk * (2d + 4) bytes
    a = mb.moba_workspace_size(1 << 20, 1, 32, 8, 128, 4096, 12, 65536)
    b = mb.moba_workspace_size(1 << 20, 1, 32, 8, 128, 4096, 12, 131072)
    assert abs((b - a) - 65536 * 32 * 12 * (2 * 128 + 4)) < 65536 * 32 * 12 * 4 + 4096


@pytest.mark.parametrize("args", [
    (2048, 1, 1, 1, 96, 256, 3, 0),     # head_dim not in {64, 128}
    (2048, 1, 3, 2, 64, 256, 3, 0),     # Hq % Hkv != 0
    (2048, 1, 1, 1, 64, 100, 3, 0),     # block not a multiple of 64
    (2048, 1, 1, 1, 64, 256, 65, 0),    # topk > 64
    (2048, 1, 1, 1, 64, 256, 0, 0),     # topk < 1
    (2048, 0, 1, 1, 64, 256, 3, 0),     # no sequences
    (1 << 30, 1, 4, 1, 64, 256, 3, 0),  # T * Hq >= 2^31
])
def test_workspace_size_rejects(L, args):
    assert L.moba_workspace_size(*args) == 0


def test_forward_rejects_before_touching_the_device(L):
    # invalid arguments are answered on the host; pointers are never dereferenced
    P = 1 << 20   # an aligned fake device address
    rc = L.moba_forward(P, P, P, P, 1, 2048, 1, 1, 96, 256, 3, 0.0, P, P, None, 0, P, 1 << 30, None)
    assert rc == 2   # head_dim unsupported
    rc = L.moba_forward(P, P, P, None, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, None, 0, P, 1 << 30, None)
    assert rc == 1   # cu_seqlens NULL
    rc = L.moba_forward(P + 8, P, P, P, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, None, 0, P, 1 << 30, None)
    assert rc == 1   # q not 16-byte aligned
    rc = L.moba_forward(P, P, P, P, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, None, 0, None, 0, None)
    assert rc == 3   # no workspace
    rc = L.moba_forward(P, P, P, P, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, None, 0, P, 16, None)
    assert rc == 3   # workspace too small
    rc = L.moba_forward(P, P, P, P, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, None, 0, P + 64, 1 << 30, None)
    assert rc == 3   # workspace misaligned
    rc = L.moba_gate(P, P, P, 1, 2048, 1, 1, 64, 256, 3, None, P, 1 << 30, None)
    assert rc == 1   # idx NULL


def test_full_workspace_and_rejects(L):
    # the dense causal path needs only the block plan: a few bytes per 256 tokens
    n = mb.moba_full_workspace_size(1 << 20, 1, 32, 8, 128)
    assert 0 < n < (1 << 20)
    assert L.moba_full_workspace_size(2048, 1, 1, 1, 96) == 0     # head_dim unsupported
    assert L.moba_full_workspace_size(2048, 1, 3, 2, 64) == 0     # Hq % Hkv != 0
    assert L.moba_full_workspace_size(1 << 30, 1, 4, 1, 64) == 0  # T * Hq >= 2^31
    P = 1 << 20
    rc = L.moba_forward_full(P, P, P, P, 1, 2048, 1, 1, 96, 0.0, P, P, P, 1 << 30, None)
    assert rc == 2   # head_dim unsupported
    rc = L.moba_forward_full(P, P, P, None, 1, 2048, 1, 1, 64, 0.0, P, P, P, 1 << 30, None)
    assert rc == 1   # cu_seqlens NULL
    rc = L.moba_forward_full(P, P, P + 8, P, 1, 2048, 1, 1, 64, 0.0, P, P, P, 1 << 30, None)
    assert rc == 1   # v not 16-byte aligned
    rc = L.moba_forward_full(P, P, P, P, 1, 2048, 1, 1, 64, 0.0, P, P, P, 8, None)
    assert rc == 3   # workspace too small


def test_decode_workspace_and_rejects(L):
    n = mb._lib.lib().moba_decode_workspace_size(8, 1 << 20, 32, 8, 128, 4096, 12)
    assert n >= 8 * 32 * 12 * (128 * 4 + 8)
    assert L.moba_decode_workspace_size(8, 1 << 20, 32, 8, 96, 4096, 12) == 0   # head_dim
    assert L.moba_decode_workspace_size(8, 1 << 20, 32, 8, 128, 100, 12) == 0   # block
    assert L.moba_decode_workspace_size(8, 1 << 20, 32, 8, 128, 4096, 65) == 0  # topk


def test_decode_rejects_before_touching_the_device(L):
    P = 1 << 20
    rc = L.moba_decode(P, P, P, P, 2, 1024, 4, 2, 96, 64, 3, 0.0, P, P, P, None, P, 1 << 30, None)
    assert rc == 2   # head_dim unsupported
    rc = L.moba_decode(P, P, P, None, 2, 1024, 4, 2, 128, 64, 3, 0.0, P, P, P, None, P, 1 << 30, None)
    assert rc == 1   # seqlens NULL
    rc = L.moba_decode(P, P + 8, P, P, 2, 1024, 4, 2, 128, 64, 3, 0.0, P, P, P, None, P, 1 << 30, None)
    assert rc == 1   # k_cache misaligned
    rc = L.moba_decode(P, P, P, P, 2, 1024, 4, 2, 128, 64, 3, 0.0, P, P, P, None, P, 64, None)
    assert rc == 3   # workspace too small
    rc = L.moba_decode_init(P, P, 2, 1024, 2, 128, 64, None, P, 1 << 20, None)
    assert rc == 1   # kbar NULL with full blocks possible


def test_backward_rejects_before_touching_the_device(L):
    P = 1 << 20
    n = L.moba_backward_workspace_size(2048, 1, 1, 1, 64, 256, 3, 0)
    assert n > 0
    # a smaller dQ chunk needs fewer partial-slot bytes
    assert L.moba_backward_workspace_size(2048, 1, 1, 1, 64, 256, 3, 512) < n
    assert L.moba_backward_workspace_size(2048, 1, 1, 1, 96, 256, 3, 0) == 0
    args = [P, P, P, P, P, P, P, P, 1, 2048, 1, 1, 64, 256, 3, 0.0, P, P, P, 0, P, n, None]
    bad = list(args); bad[12] = 96
    assert L.moba_backward(*bad) == 2        # head_dim unsupported
    bad = list(args); bad[7] = None
    assert L.moba_backward(*bad) == 1        # cu_seqlens NULL
    bad = list(args); bad[16] = P + 4
    assert L.moba_backward(*bad) == 1        # dq misaligned
    bad = list(args); bad[14] = 65
    assert L.moba_backward(*bad) == 2        # topk > 64
    bad = list(args); bad[21] = n - 1
    assert L.moba_backward(*bad) == 3        # workspace too small
    bad = list(args); bad[20] = P + 64
    assert L.moba_backward(*bad) == 3        # workspace misaligned

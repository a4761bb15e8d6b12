"""The bounds-checked build on the host: it links, exports what moba.h
declares, reports itself, takes the planted-slip modes only where it should,
and guards every carved workspace region (no GPU needed)."""
import pytest

import block_sparse_long_11_b200 as mb
from tests.debug_lib import load_both, using
from tests.test_abi import _declared


@pytest.fixture(scope="module")
def libs():
    return load_both()


def test_both_libraries_export_every_declared_symbol(libs):
    for L in libs:
        for n in _declared():
            assert hasattr(L, n), n


def test_build_flag(libs):
    rel, dbg = libs
    assert rel.moba_debug_build() == 0
    assert dbg.moba_debug_build() == 1


def test_poison_modes(libs):
    rel, dbg = libs
    assert rel.moba_debug_poison(0) == 0
    assert rel.moba_debug_poison(1) == 2      # MOBA_ERR_UNSUPPORTED in a release build
    assert dbg.moba_debug_poison(3) == 1      # MOBA_ERR_INVALID_ARG
    assert dbg.moba_debug_poison(-1) == 1
    assert dbg.moba_debug_poison(2) == 0
    assert dbg.moba_debug_poison(0) == 0


SIZES = [
    ("moba_workspace_size", (1 << 20, 1, 32, 8, 128, 4096, 12, 65536)),
    ("moba_workspace_size", (2200, 2, 4, 2, 64, 128, 4, 0)),
    ("moba_full_workspace_size", (2200, 2, 4, 2, 128)),
    ("moba_decode_workspace_size", (4, 1 << 20, 32, 8, 128, 4096, 12)),
    ("moba_backward_workspace_size", (32768, 1, 32, 8, 128, 4096, 12, 0)),
]


@pytest.mark.parametrize("fn,args", SIZES, ids=[f"{f}-{i}" for i, (f, _) in enumerate(SIZES)])
def test_one_guard_per_region(libs, fn, args):
    """The debug layout is the release layout with a 256-byte guard after
    each region, and a call records at most 32 guards: so every region of
    every workspace kind is guarded."""
    rel, dbg = libs
    a, b = getattr(rel, fn)(*args), getattr(dbg, fn)(*args)
    assert a > 0 and b > a
    assert (b - a) % 256 == 0
    assert 1 <= (b - a) // 256 <= 32


def test_status_strings_of_the_debug_codes(libs):
    with using(libs[1]):
        assert mb.moba_status_string(8) == "MOBA_ERR_BOUNDS"
        assert mb.moba_status_string(9) == "MOBA_ERR_CANARY"

"""Loading the bounds-checked library (libmoba_debug.so) beside the release
one in the same process, and running binding calls against either."""
import contextlib

from block_sparse_long_11_b200 import _lib as L_
from block_sparse_long_11_b200 import build


def load_both():
    """(release CDLL, debug CDLL), both built and configured by the binding."""
    build.build()
    build.build(debug=True)
    saved_path, saved = L_.LIB_PATH, L_._lib
    try:
        L_.LIB_PATH, L_._lib = build.LIB, None
        rel = L_.lib()
        L_.LIB_PATH, L_._lib = build.LIB_DEBUG, None
        dbg = L_.lib()
    finally:
        L_.LIB_PATH, L_._lib = saved_path, saved
    return rel, dbg


@contextlib.contextmanager
def using(lib):
    """Route the binding's calls to `lib` inside the block."""
    saved = L_._lib
    L_._lib = lib
    try:
        yield lib
    finally:
        L_._lib = saved

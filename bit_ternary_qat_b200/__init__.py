"""B200-native BitNet b1.58 BitLinear hot path.

The compute lives in ``libbitlinear.so`` (hand-written sm_100a CUDA kernels behind a
C ABI declared in ``include/bitlinear.h``).  This package only marshals arguments
into that library: it loads it lazily on first use and raises if it is missing --
there is no CPU fallback.
"""
from . import synth  # noqa: F401  (seeded inputs; no layer arithmetic)


def load():
    """Load the CUDA library (raises if it is not built)."""
    from . import _lib
    return _lib.lib()


def __getattr__(name):
    from . import ops
    try:
        return getattr(ops, name)
    except AttributeError:
        raise AttributeError(name) from None

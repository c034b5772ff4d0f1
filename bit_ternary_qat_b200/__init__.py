"""B200-native BitNet b1.58 BitLinear hot path.

The compute lives in ``libbitlinear.so`` (hand-written sm_100a CUDA kernels behind the
C ABI declared in ``include/bitlinear.h``).  This package only marshals arguments into
that library (``ops``): the library is loaded on the first call and every call raises
if it is missing -- there is no CPU fallback.
"""
from . import synth  # noqa: F401  (seeded inputs; none of the layer's arithmetic)
from . import ops  # noqa: F401
from .ops import (  # noqa: F401
    bitlinear_act_quant, bitlinear_backward, bitlinear_backward_input, bitlinear_backward_weight,
    bitlinear_grad_input, bitlinear_rmsnorm_backward,
    bitlinear_forward, bitlinear_forward_qat, bitlinear_linear, bitlinear_quant_weight,
    bitlinear_quant_weight_noalloc, check_device_status, launch_count,
    selftest_bounded_wait, set_wait_limit_ns, ternary_gemv, ternary_pack, workspace, workspace_bytes,
    bitlinear_act_quant_tensor, bitlinear_linear_rows, bitlinear_quant_weight_rows, bitlinear_quant_weight_tau,
    ternary_gemv_rows, bitlinear_optimizer_step, bitlinear_linear_packed, mma_peak_probe, read_peak_probe,
)


def load():
    """Load the CUDA library now (raises if it is not built)."""
    from . import _lib
    return _lib.lib()

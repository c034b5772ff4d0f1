"""The workspace-free weight quantiser against the workspace one.

bitlinear_quant_weight_noalloc exists for callers that cannot allocate device memory
(their pool belongs to another allocator), so cannot hand the library a workspace for
the partial sums of |W|; it keeps them in a scratch array built into the library
instead.  Its outputs must be identical to bitlinear_quant_weight's.  Two calls in a row
with different sizes check that nothing left in the shared scratch by one call leaks
into the next.  This file is collected last so that a failure here, in a run that stops
at the first failure, comes after every other test has run.
"""
import pytest
import torch

from bit_ternary_qat_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _outputs(N, K):
    return dict(gamma=torch.empty(1, dtype=torch.float32, device=DEV),
                wq_i8=torch.empty(N, K, dtype=torch.int8, device=DEV),
                wq_bf16=torch.empty(N, K, dtype=torch.bfloat16, device=DEV),
                packed=torch.empty(N, K // 4, dtype=torch.uint8, device=DEV))


def test_noalloc_matches_workspace_entry_point(bl):
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(2048, 2048, 21), (48, 160, 22)]       # two calls in a row, different sizes
    for N, K, seed in cases:
        W = synth.normal((N, K), synth.W_STD, synth.generator(seed)).to(DEV)
        ref = _outputs(N, K)
        ws = bl.workspace(1, N, K, DEV)
        _lib.call("bitlinear_quant_weight", W.data_ptr(), N, K, ref["wq_i8"].data_ptr(), ref["wq_bf16"].data_ptr(),
                  ref["packed"].data_ptr(), ref["gamma"].data_ptr(), ws.data_ptr(), ws.numel(), stream)
        out = _outputs(N, K)
        _lib.call("bitlinear_quant_weight_noalloc", W.data_ptr(), N, K, out["wq_i8"].data_ptr(),
                  out["wq_bf16"].data_ptr(), out["packed"].data_ptr(), out["gamma"].data_ptr(), stream)
        torch.cuda.synchronize()
        assert bl.check_device_status() == 0
        for k in ("gamma", "wq_i8", "wq_bf16", "packed"):
            assert torch.equal(out[k], ref[k]), (N, K, k)


def test_noalloc_allocates_nothing(bl):
    """Once the first call has looked up the scratch address, a call changes neither torch's
    allocator count nor the device's free memory: no allocation happens on its path."""
    stream = torch.cuda.current_stream().cuda_stream
    N, K = 1024, 512
    W = synth.normal((N, K), synth.W_STD, synth.generator(23)).to(DEV)
    out = _outputs(N, K)
    args = (W.data_ptr(), N, K, out["wq_i8"].data_ptr(), out["wq_bf16"].data_ptr(), out["packed"].data_ptr(),
            out["gamma"].data_ptr(), stream)
    _lib.call("bitlinear_quant_weight_noalloc", *args)          # set-up call
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        _lib.call("bitlinear_quant_weight_noalloc", *args)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == torch_before
    assert free_after == free_before
    assert bl.check_device_status() == 0

// fused_quant.cuh -- activation quantisation (K1) and the |W| partial sums of the weight
// quantiser (K2 pass 1) in one launch, for the quantisation-aware forward.
//
// P3 ("BitNet 1.5技术解析…") §3.1's BitLinear.forward quantises the activations and the
// weights of the same layer before the linear; the two are independent, so one grid does
// both: blocks [0, nparts) compute the fp64 partial sums of |W| exactly as
// absmean_partial_kernel does (same slices, hence the same gamma), blocks [nparts, ..) run
// the warp-per-row activation quantiser on 8 rows each.  The partial-sum blocks come first:
// they only stream W and finish early, and the quantiser blocks fill the SMs behind them.
#pragma once
#include "common.cuh"
#include "act_quant.cuh"
#include "weight_quant.cuh"

namespace bl {

template <bool kBf16, int VPL>
__global__ void __launch_bounds__(256, 2) act_quant_absmean_kernel(
    const void* __restrict__ X, int T, int K, int apply_norm, const float* __restrict__ g, float eps,
    int8_t* __restrict__ Xq, float* __restrict__ sx, float* __restrict__ rinv, void* __restrict__ Xdq,
    const float* __restrict__ W, int64_t n, int nparts, double* __restrict__ partials) {
    static_assert(kWqThreads == 256, "one block size for both parts");
    __shared__ typename DqLut<kBf16>::T lut_all[8][256];
    __shared__ double red[kWqThreads / 32];
    pdl_trigger_and_wait();
    if (static_cast<int>(blockIdx.x) < nparts)
        absmean_partial_block(W, n, blockIdx.x, nparts, partials, red);
    else
        act_quant_warp_rows<kBf16, VPL>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, blockIdx.x - nparts,
                                        lut_all);
}

}  // namespace bl

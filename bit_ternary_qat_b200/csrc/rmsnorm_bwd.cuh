// rmsnorm_bwd.cuh -- K6: RMSNorm backward behind the straight-through activation quantiser.
//
// P3 ("BitNet 1.5技术解析…") §3.1 puts RMSNorm in front of activation_quant and §2.2's
// detach() passes the gradient of the quantised activation straight to the RMSNorm
// output, so the input gradient is the textbook derivative of x_hat = x * r * g with the
// saved fp32 r:
//   u = x r,  h = g dX_hat,  c_t = (1/K) sum_k h u,  dX = r (h - u c_t),
//   dg_k = sum_t dX_hat[t,k] u[t,k].
//
// Memory-bound row kernel.  dX_hat arrives in the dX buffer (written there by the grad-
// input GEMM) and is overwritten in place: each thread reads its elements in pass A,
// the block reduces c_t, then the same thread rewrites the same elements in pass B (the
// second read of the row hits L1/L2).  Blocks stride over rows; with dg requested each
// block accumulates its rows' dg in shared memory and writes one partial row, and a
// second small kernel sums the partials in a fixed order.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kBwdThreads = 512;
constexpr int kBwdBlocks = 296;   // partial rows of dg; fixed so workspace size is device-independent

template <bool kBf16X>
__global__ void __launch_bounds__(kBwdThreads) rmsnorm_bwd_kernel(const void* __restrict__ X,
                                                                  const float* __restrict__ rinv,
                                                                  const float* __restrict__ g, float* dX, int T,
                                                                  int K, float* __restrict__ dg_partial) {
    extern __shared__ float dg_s[];     // [K] when dg_partial != nullptr
    __shared__ float red[kBwdThreads / 32];
    const bool want_dg = dg_partial != nullptr;
    if (want_dg)
        for (int k = threadIdx.x; k < K; k += kBwdThreads) dg_s[k] = 0.0f;
    __syncthreads();
    const int nvec = K / 4;
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const float r = __ldg(rinv + t);
        float4* drow = reinterpret_cast<float4*>(dX + static_cast<int64_t>(t) * K);
        float part = 0.0f;
        for (int i = threadIdx.x; i < nvec; i += kBwdThreads) {
            const float4 d = drow[i];
            float x[4];
            if constexpr (kBf16X) {
                const uint2 raw = __ldg(reinterpret_cast<const uint2*>(X) + static_cast<int64_t>(t) * nvec + i);
                x[0] = __uint_as_float(raw.x << 16); x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
                x[2] = __uint_as_float(raw.y << 16); x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
            } else {
                const float4 raw = __ldg(reinterpret_cast<const float4*>(X) + static_cast<int64_t>(t) * nvec + i);
                x[0] = raw.x; x[1] = raw.y; x[2] = raw.z; x[3] = raw.w;
            }
            const float dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float gk = g != nullptr ? __ldg(g + 4 * i + e) : 1.0f;
                const float u = x[e] * r;
                part += gk * dv[e] * u;
                if (want_dg) dg_s[4 * i + e] += dv[e] * u;
            }
        }
        part = warp_sum(part);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
        __syncthreads();
        float tot = 0.0f;
#pragma unroll
        for (int w = 0; w < kBwdThreads / 32; ++w) tot += red[w];
        const float c = tot / static_cast<float>(K);
        __syncthreads();
        for (int i = threadIdx.x; i < nvec; i += kBwdThreads) {
            const float4 d = drow[i];
            float x[4];
            if constexpr (kBf16X) {
                const uint2 raw = __ldg(reinterpret_cast<const uint2*>(X) + static_cast<int64_t>(t) * nvec + i);
                x[0] = __uint_as_float(raw.x << 16); x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
                x[2] = __uint_as_float(raw.y << 16); x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
            } else {
                const float4 raw = __ldg(reinterpret_cast<const float4*>(X) + static_cast<int64_t>(t) * nvec + i);
                x[0] = raw.x; x[1] = raw.y; x[2] = raw.z; x[3] = raw.w;
            }
            const float dv[4] = {d.x, d.y, d.z, d.w};
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float gk = g != nullptr ? __ldg(g + 4 * i + e) : 1.0f;
                const float u = x[e] * r;
                o[e] = r * (gk * dv[e] - u * c);
            }
            drow[i] = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
    if (want_dg) {
        __syncthreads();
        for (int k = threadIdx.x; k < K; k += kBwdThreads) dg_partial[static_cast<int64_t>(blockIdx.x) * K + k] = dg_s[k];
    }
}

__global__ void __launch_bounds__(256) dg_reduce_kernel(const float* __restrict__ partial, int nparts, int K,
                                                        float* __restrict__ dg) {
    const int k = blockIdx.x * 256 + threadIdx.x;
    if (k >= K) return;
    float s = 0.0f;
    for (int p = 0; p < nparts; ++p) s += partial[static_cast<int64_t>(p) * K + k];
    dg[k] = s;
}

}  // namespace bl

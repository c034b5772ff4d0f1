// rmsnorm_bwd.cuh -- K6: RMSNorm backward behind the straight-through activation quantiser.
//
// P3 ("BitNet 1.5技术解析…") §3.1 puts RMSNorm in front of activation_quant and §2.2's
// detach() passes the gradient of the quantised activation straight to the RMSNorm
// output, so the input gradient is the textbook derivative of x_hat = x * r * g with the
// saved fp32 r:
//   u = x r,  h = g dX_hat,  c_t = (1/K) sum_k h u,  dX = r (h - u c_t),
//   dg_k = sum_t dX_hat[t,k] u[t,k].
//
// Memory-bound.  dX_hat arrives in the dX buffer (written there by the grad-input GEMM)
// and is overwritten in place.  Thread i of a block always owns the same column vectors
// (i + j*NT, 4 columns each), so:
//   * a row's data stays in registers between the reduction and the update (dX_hat and X
//     are read from HBM exactly once, dX written once, in place, by the same thread);
//   * dg accumulates in registers across all rows the block visits, and each block writes
//     one partial dg row; dg_reduce_kernel sums the partials in a fixed order.
// A block processes R rows per iteration (rows b, b + G, ...) with a single block
// reduction for the R row sums, so R rows of loads are in flight per thread.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kBwdThreads = 256;
constexpr int kBwdMaxBlocks = 592;   // partial dg rows; fixed so the workspace size is device-independent
constexpr int kBwdMaxVpt = 16;       // K <= 16 * 4 * 256 = 16384

template <bool kBf16X>
__device__ __forceinline__ void load_x4(const void* X, int64_t idx_vec4, float (&x)[4]) {
    if constexpr (kBf16X) {
        const uint2 raw = __ldcs(reinterpret_cast<const uint2*>(X) + idx_vec4);
        x[0] = __uint_as_float(raw.x << 16); x[1] = __uint_as_float(raw.x & 0xFFFF0000u);
        x[2] = __uint_as_float(raw.y << 16); x[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    } else {
        const float4 raw = __ldcs(reinterpret_cast<const float4*>(X) + idx_vec4);
        x[0] = raw.x; x[1] = raw.y; x[2] = raw.z; x[3] = raw.w;
    }
}

// grid = G blocks (<= kBwdMaxBlocks), block = kBwdThreads; thread i owns vectors i + j*NT.
template <bool kBf16X, int VPT, int R>
__global__ void __launch_bounds__(kBwdThreads) rmsnorm_bwd_kernel(const void* __restrict__ X,
                                                                  const float* __restrict__ rinv,
                                                                  const float* __restrict__ g, float* dX, int T,
                                                                  int K, float* __restrict__ dg_partial) {
    constexpr int NT = kBwdThreads;
    __shared__ float red[R][NT / 32];
    pdl_trigger_and_wait();
    const int nvec = K / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float gk[VPT][4];
    float dga[VPT][4];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + j * NT;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            gk[j][e] = (g != nullptr && v < nvec) ? __ldg(g + 4 * v + e) : 1.0f;
            dga[j][e] = 0.0f;
        }
    }

    const int G = gridDim.x;
    for (int t0 = blockIdx.x; t0 < T; t0 += G * R) {
        float d[R][VPT][4], u[R][VPT][4], rr[R];
        float part[R];
#pragma unroll
        for (int q = 0; q < R; ++q) {
            const int t = t0 + q * G;
            part[q] = 0.0f;
            rr[q] = t < T ? __ldg(rinv + t) : 0.0f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int v = threadIdx.x + j * NT;
                if (t < T && v < nvec) {
                    const float4 dv = reinterpret_cast<const float4*>(dX + static_cast<int64_t>(t) * K)[v];
                    d[q][j][0] = dv.x; d[q][j][1] = dv.y; d[q][j][2] = dv.z; d[q][j][3] = dv.w;
                    float x[4];
                    load_x4<kBf16X>(X, static_cast<int64_t>(t) * nvec + v, x);
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[q][j][e] = x[e] * rr[q];
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) { d[q][j][e] = 0.0f; u[q][j][e] = 0.0f; }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
            for (int j = 0; j < VPT; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    part[q] = fmaf(gk[j][e] * d[q][j][e], u[q][j][e], part[q]);
                    dga[j][e] = fmaf(d[q][j][e], u[q][j][e], dga[j][e]);
                }
#pragma unroll
        for (int q = 0; q < R; ++q) {
            const float w = warp_sum(part[q]);
            if (lane == 0) red[q][warp] = w;
        }
        __syncthreads();
        float c[R];
#pragma unroll
        for (int q = 0; q < R; ++q) {
            float tot = 0.0f;
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) tot += red[q][w];
            c[q] = tot / static_cast<float>(K);
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < R; ++q) {
            const int t = t0 + q * G;
            if (t >= T) continue;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                const int v = threadIdx.x + j * NT;
                if (v >= nvec) continue;
                float o[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) o[e] = rr[q] * (gk[j][e] * d[q][j][e] - u[q][j][e] * c[q]);
                reinterpret_cast<float4*>(dX + static_cast<int64_t>(t) * K)[v] = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
    }
    if (dg_partial != nullptr) {
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            if (v < nvec)
                reinterpret_cast<float4*>(dg_partial + static_cast<int64_t>(blockIdx.x) * K)[v] =
                    make_float4(dga[j][0], dga[j][1], dga[j][2], dga[j][3]);
        }
    }
}

// dg[k] = sum_p partial[p][k] in a fixed order.  A block handles 32 columns with 32 warps:
// lane = column, warp w loads partial rows w, w + 32, ... all at once (at most
// kBwdMaxBlocks / 32 loads, all in flight), adds them in order, then warp 0 adds the 32
// warp sums in order.
__global__ void __launch_bounds__(1024) dg_reduce_kernel(const float* __restrict__ partial, int nparts, int K,
                                                         float* __restrict__ dg) {
    constexpr int kPerWarp = (kBwdMaxBlocks + 31) / 32;
    __shared__ float red[32][33];
    pdl_trigger_and_wait();
    const int c = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int k = blockIdx.x * 32 + c;
    float v[kPerWarp];
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) {
        const int p = w + 32 * i;
        v[i] = (k < K && p < nparts) ? __ldcs(partial + static_cast<int64_t>(p) * K + k) : 0.0f;
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kPerWarp; ++i) s += v[i];
    red[w][c] = s;
    __syncthreads();
    if (w == 0 && k < K) {
        float tot = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) tot += red[i][c];
        dg[k] = tot;
    }
}

}  // namespace bl

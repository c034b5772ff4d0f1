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
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kBwdMaxBlocks = 592;   // partial dg rows; fixed so the workspace size is device-independent

// Persistent row kernel: grid = G blocks (<= kBwdMaxBlocks, all resident), block = NT
// threads; thread i owns column vectors i + j*NT (4 columns each), j < VPT, of every row.
// Block b visits rows b, b + G, b + 2G, ...; while it reduces and stores one row, the loads of
// its next row are already in flight (two register buffers, the loop unrolled by two so the
// buffers alternate without copies), so every SM keeps about two rows per block in flight.
// One block barrier per row: the warp sums go to one of two shared arrays, alternating by row.
// The arithmetic of a row is fixed (per thread over j and the 4 columns, then the warp
// butterfly, then the warps in order), so results do not depend on the grid.
template <bool kBf16X>
struct BwdXRaw;
template <>
struct BwdXRaw<true> {
    using T = uint2;   // 4 bf16
    __device__ __forceinline__ static void widen(const uint2& r, float (&x)[4]) {
        x[0] = __uint_as_float(r.x << 16); x[1] = __uint_as_float(r.x & 0xFFFF0000u);
        x[2] = __uint_as_float(r.y << 16); x[3] = __uint_as_float(r.y & 0xFFFF0000u);
    }
};
template <>
struct BwdXRaw<false> {
    using T = float4;
    __device__ __forceinline__ static void widen(const float4& r, float (&x)[4]) {
        x[0] = r.x; x[1] = r.y; x[2] = r.z; x[3] = r.w;
    }
};

template <bool kBf16X, int NT, int VPT, bool kGain, bool kPf = (NT < 1024 || (kBf16X && VPT <= 3 && !kGain))>
__global__ void __launch_bounds__(NT) rmsnorm_bwd_kernel(const void* __restrict__ X,
                                                         const float* __restrict__ rinv,
                                                         const float* __restrict__ g, float* dX, int T,
                                                         int K, float* __restrict__ dg_partial) {
    using XR = typename BwdXRaw<kBf16X>::T;
    __shared__ float red[2][NT / 32];
    pdl_trigger_and_wait();
    const int nvec = K / 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;

    float dga[VPT][4];
#pragma unroll
    for (int j = 0; j < VPT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) dga[j][e] = 0.0f;

    float4 dA[VPT], dB[kPf ? VPT : 1];
    XR xA[VPT], xB[kPf ? VPT : 1];
    auto load_row = [&](int t, float4 (&d)[VPT], XR (&x)[VPT]) {
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            if (v < nvec) {
                d[j] = __ldcs(reinterpret_cast<const float4*>(dX + static_cast<int64_t>(t) * K) + v);
                x[j] = __ldcs(reinterpret_cast<const XR*>(X) + static_cast<int64_t>(t) * nvec + v);
            } else {
                d[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                x[j] = XR{};
            }
        }
    };
    // one row: c_t = (1/K) sum_k g d u, dX = r (g d - u c_t), dg += d u
    auto row = [&](int t, int par, const float4 (&d4)[VPT], const XR (&xr)[VPT]) {
        const float rr = __ldg(rinv + t);
        float d[VPT][4], u[VPT][4], gk[VPT][4];
        float part = 0.0f;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            float x[4];
            BwdXRaw<kBf16X>::widen(xr[j], x);
            d[j][0] = d4[j].x; d[j][1] = d4[j].y; d[j][2] = d4[j].z; d[j][3] = d4[j].w;
            float4 gv = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            if constexpr (kGain) {
                if (v < nvec) gv = __ldg(reinterpret_cast<const float4*>(g) + v);
            }
            gk[j][0] = gv.x; gk[j][1] = gv.y; gk[j][2] = gv.z; gk[j][3] = gv.w;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                u[j][e] = x[e] * rr;
                part = fmaf(gk[j][e] * d[j][e], u[j][e], part);
                dga[j][e] = fmaf(d[j][e], u[j][e], dga[j][e]);
            }
        }
        const float w = warp_sum(part);
        if (lane == 0) red[par][warp] = w;
        __syncthreads();
        float tot = 0.0f;
#pragma unroll
        for (int i = 0; i < NT / 32; ++i) tot += red[par][i];
        const float c = tot / static_cast<float>(K);
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            if (v >= nvec) continue;
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = rr * (gk[j][e] * d[j][e] - u[j][e] * c);
            reinterpret_cast<float4*>(dX + static_cast<int64_t>(t) * K)[v] = make_float4(o[0], o[1], o[2], o[3]);
        }
    };

    int t = blockIdx.x;
    if constexpr (kPf) {
        if (t < T) load_row(t, dA, xA);
        while (t < T) {
            if (t + G < T) load_row(t + G, dB, xB);
            row(t, 0, dA, xA);
            t += G;
            if (t >= T) break;
            if (t + G < T) load_row(t + G, dA, xA);
            row(t, 1, dB, xB);
            t += G;
        }
    } else {
        // 1024-thread blocks hold at most 64 registers per thread: one row buffer
        for (int par = 0; t < T; t += G, par ^= 1) {
            load_row(t, dA, xA);
            row(t, par, dA, xA);
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

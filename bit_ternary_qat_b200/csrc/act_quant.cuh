// act_quant.cuh -- K1: fused RMSNorm + per-token absmax int8 activation quantiser.
//
// Restates P3 ("BitNet 1.5技术解析…") §3.1 (RMSNorm applied before the activation
// quantiser) and §2.2 activation_quant (scale = 127 / row absmax clamped at 1e-5,
// round, clamp to [-128, 127], dequantised value forwarded through the STE), and
// P2 ("BitNet 三元权重量化训练工程…") per-token 8-bit absmax.
//
// One block per token row.  Memory-bound: X is read once from HBM (the two further
// passes over the row hit L1), X_q / X_dq / s / r are written once.  Every quantiser
// operation is an explicitly rounded fp32 intrinsic (no FMA contraction), and the
// sum of squares is an fp64 sum in a fixed order, so the codes are reproducible.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kActThreads = 128;

// 16-byte vector of the input row: 8 bf16 or 4 fp32 values.
template <bool kBf16>
struct ActVec {
    static constexpr int kElems = kBf16 ? 8 : 4;
    float v[kElems];
    __device__ __forceinline__ void load(const void* base, int64_t idx_vec) {
        uint4 raw = __ldg(reinterpret_cast<const uint4*>(base) + idx_vec);
        if constexpr (kBf16) {
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            }
        } else {
            v[0] = __uint_as_float(raw.x);
            v[1] = __uint_as_float(raw.y);
            v[2] = __uint_as_float(raw.z);
            v[3] = __uint_as_float(raw.w);
        }
    }
};

__device__ __forceinline__ double block_sum_f64(double v, double* red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0) {
        for (int w = 0; w < kActThreads / 32; ++w) s += red[w];
        red[0] = s;
    }
    __syncthreads();
    s = red[0];
    __syncthreads();
    return s;
}

__device__ __forceinline__ float block_max_f32(float v, float* red) {
    v = warp_max(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int w = 1; w < kActThreads / 32; ++w) m = fmaxf(m, red[w]);
        red[0] = m;
    }
    __syncthreads();
    float m = red[0];
    __syncthreads();
    return m;
}

// grid = T blocks, block = kActThreads.  K % 32 == 0 so a row is a whole number of
// 16-byte vectors for both input types.
template <bool kBf16>
__global__ void __launch_bounds__(kActThreads) act_quant_kernel(const void* __restrict__ X, int K,
                                                                int apply_norm, const float* __restrict__ g,
                                                                float eps, int8_t* __restrict__ Xq,
                                                                float* __restrict__ sx, float* __restrict__ rinv,
                                                                void* __restrict__ Xdq) {
    using V = ActVec<kBf16>;
    constexpr int E = V::kElems;
    __shared__ double red_d[kActThreads / 32];
    __shared__ float red_f[kActThreads / 32];

    const int64_t t = blockIdx.x;
    const int nvec = K / E;
    const int64_t row_vec0 = t * static_cast<int64_t>(nvec);

    // pass 1: r_t = 1 / sqrt(mean x^2 + eps), fp64 sum in a fixed order
    float r = 1.0f;
    if (apply_norm) {
        double ss = 0.0;
        for (int i = threadIdx.x; i < nvec; i += kActThreads) {
            V x;
            x.load(X, row_vec0 + i);
#pragma unroll
            for (int e = 0; e < E; ++e) ss += static_cast<double>(x.v[e]) * static_cast<double>(x.v[e]);
        }
        ss = block_sum_f64(ss, red_d);
        r = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(eps)));
        if (threadIdx.x == 0) rinv[t] = r;
    }

    // pass 2: absmax of x_hat = fl(fl(x * r) * g)
    float m = 0.0f;
    for (int i = threadIdx.x; i < nvec; i += kActThreads) {
        V x;
        x.load(X, row_vec0 + i);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float h = x.v[e];
            if (apply_norm) {
                h = __fmul_rn(h, r);
                if (g != nullptr) h = __fmul_rn(h, __ldg(g + i * E + e));
            }
            m = fmaxf(m, fabsf(h));
        }
    }
    m = block_max_f32(m, red_f);
    const float s = __fdiv_rn(127.0f, fmaxf(m, 1e-5f));
    if (threadIdx.x == 0) sx[t] = s;

    // pass 3: codes and dequantised values
    for (int i = threadIdx.x; i < nvec; i += kActThreads) {
        V x;
        x.load(X, row_vec0 + i);
        int8_t q[E];
        float dq[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float h = x.v[e];
            if (apply_norm) {
                h = __fmul_rn(h, r);
                if (g != nullptr) h = __fmul_rn(h, __ldg(g + i * E + e));
            }
            int qi = __float2int_rn(__fmul_rn(h, s));
            qi = max(-128, min(127, qi));
            q[e] = static_cast<int8_t>(qi);
            dq[e] = __fdiv_rn(static_cast<float>(qi), s);
        }
        if constexpr (kBf16) {
            uint2 packed;
            packed.x = (uint32_t)(uint8_t)q[0] | ((uint32_t)(uint8_t)q[1] << 8) | ((uint32_t)(uint8_t)q[2] << 16) |
                       ((uint32_t)(uint8_t)q[3] << 24);
            packed.y = (uint32_t)(uint8_t)q[4] | ((uint32_t)(uint8_t)q[5] << 8) | ((uint32_t)(uint8_t)q[6] << 16) |
                       ((uint32_t)(uint8_t)q[7] << 24);
            reinterpret_cast<uint2*>(Xq)[row_vec0 + i] = packed;
            if (Xdq != nullptr) {
                uint4 o;
                o.x = (uint32_t)float_to_bf16_bits(dq[0]) | ((uint32_t)float_to_bf16_bits(dq[1]) << 16);
                o.y = (uint32_t)float_to_bf16_bits(dq[2]) | ((uint32_t)float_to_bf16_bits(dq[3]) << 16);
                o.z = (uint32_t)float_to_bf16_bits(dq[4]) | ((uint32_t)float_to_bf16_bits(dq[5]) << 16);
                o.w = (uint32_t)float_to_bf16_bits(dq[6]) | ((uint32_t)float_to_bf16_bits(dq[7]) << 16);
                reinterpret_cast<uint4*>(Xdq)[row_vec0 + i] = o;
            }
        } else {
            uint32_t packed = (uint32_t)(uint8_t)q[0] | ((uint32_t)(uint8_t)q[1] << 8) |
                              ((uint32_t)(uint8_t)q[2] << 16) | ((uint32_t)(uint8_t)q[3] << 24);
            reinterpret_cast<uint32_t*>(Xq)[row_vec0 + i] = packed;
            if (Xdq != nullptr) {
                reinterpret_cast<float4*>(Xdq)[row_vec0 + i] = make_float4(dq[0], dq[1], dq[2], dq[3]);
            }
        }
    }
}

}  // namespace bl

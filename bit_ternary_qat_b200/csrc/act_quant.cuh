// act_quant.cuh -- K1: fused RMSNorm + per-token absmax int8 activation quantiser.
//
// Restates P3 ("BitNet 1.5技术解析…") §3.1 (RMSNorm applied before the activation
// quantiser) and §2.2 activation_quant (scale = 127 / row absmax clamped at 1e-5,
// round, clamp to [-128, 127], dequantised value forwarded through the STE), and
// P2 ("BitNet 三元权重量化训练工程…") per-token 8-bit absmax.
//
// One block per token row; each thread loads its 16-byte vectors of the row once into
// registers (the row is read from HBM exactly once) and the three steps -- sum of
// squares, absmax, quantise -- run from registers with two block reductions in between.
// Memory-bound: X is read once, X_q / X_dq / s / r are written once.
//
// Exactness (the codes must equal the fp32 oracle's bit for bit):
//   * sum of squares in fp64 in a fixed order (per thread, then a fixed butterfly);
//   * x_hat = (x * r) * g and x_hat * s_t with explicitly rounded fp32 multiplies;
//   * round half to even without a float->int conversion: for |v| < 2^22,
//     fl(v + 1.5*2^23) = 1.5*2^23 + rint(v) exactly, so the integer and its float value
//     are read off that sum;
//   * X_dq = fl(q / s_t) from one correctly rounded reciprocal c = fl(1/s_t) per row and
//     two FMA corrections (Markstein): y0 = fl(q c); y1 = fl(y0 + fl(q - s_t y0) c) is a
//     faithful quotient, so e1 = q - s_t y1 is exact and fl(y1 + e1 c) is the correctly
//     rounded quotient.  tests/test_kernel_arith.py checks this in exact rational
//     arithmetic for every q in [-128, 127] over a wide range of s_t, and the GPU parity
//     tests compare X_dq with the oracle's division.
#pragma once
#include "common.cuh"

namespace bl {

// 16-byte vector of the input row: 8 bf16 or 4 fp32 values.
template <bool kBf16>
struct ActVec {
    static constexpr int kElems = kBf16 ? 8 : 4;
    __device__ __forceinline__ static float elem(const uint4& raw, int e) {
        if constexpr (kBf16) {
            const uint32_t word = e < 2 ? raw.x : (e < 4 ? raw.y : (e < 6 ? raw.z : raw.w));
            return (e & 1) ? __uint_as_float(word & 0xFFFF0000u) : __uint_as_float(word << 16);
        } else {
            const uint32_t word = e == 0 ? raw.x : (e == 1 ? raw.y : (e == 2 ? raw.z : raw.w));
            return __uint_as_float(word);
        }
    }
};

constexpr float kRoundMagic = 12582912.0f;        // 1.5 * 2^23
constexpr int32_t kRoundMagicBits = 0x4B400000;   // bit pattern of 1.5 * 2^23

// fl(q / s) for integer-valued q in [-128, 127] and s > 0, given c = fl(1/s): two FMA
// corrections; after the first, y1 is a faithful quotient, so the second residual is
// exact and the second correction rounds correctly.
__device__ __forceinline__ float div_by_scale(float q, float s, float c) {
    const float y0 = __fmul_rn(q, c);
    const float e0 = __fmaf_rn(-y0, s, q);
    const float y1 = __fmaf_rn(e0, c, y0);
    const float e1 = __fmaf_rn(-y1, s, q);
    return __fmaf_rn(e1, c, y1);
}

template <int NT>
__device__ __forceinline__ double block_sum_f64(double v, double* red) {
    v = warp_sum(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) s += red[w];
    return s;
}

template <int NT>
__device__ __forceinline__ float block_max_f32(float v, float* red) {
    v = warp_max(v);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, red[w]);
    return m;
}

// grid = T blocks, block = NT threads; thread i owns vectors i + j*NT, j < VPT.
template <bool kBf16, int NT, int VPT>
__global__ void __launch_bounds__(NT) act_quant_kernel(const void* __restrict__ X, int K, int apply_norm,
                                                       const float* __restrict__ g, float eps,
                                                       int8_t* __restrict__ Xq, float* __restrict__ sx,
                                                       float* __restrict__ rinv, void* __restrict__ Xdq) {
    using V = ActVec<kBf16>;
    constexpr int E = V::kElems;
    __shared__ double red_d[NT / 32];
    __shared__ float red_f[NT / 32];

    const int64_t t = blockIdx.x;
    const int nvec = K / E;
    const int64_t row_vec0 = t * static_cast<int64_t>(nvec);
    const uint4* xrow = reinterpret_cast<const uint4*>(X) + row_vec0;

    // the row, widened to fp32, in registers (read from HBM once)
    float x[VPT][E];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + j * NT;
        const uint4 raw = v < nvec ? __ldcs(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int e = 0; e < E; ++e) x[j][e] = V::elem(raw, e);
    }

    // r_t = 1 / sqrt(mean x^2 + eps): fp64 sum, fixed order
    float r = 1.0f;
    if (apply_norm) {
        double ss = 0.0;
#pragma unroll
        for (int j = 0; j < VPT; ++j)
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const double xd = static_cast<double>(x[j][e]);
                ss = fma(xd, xd, ss);
            }
        ss = block_sum_f64<NT>(ss, red_d);
        r = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(eps)));
    }

    // x_hat = fl(fl(x * r) * g) (kept in place of x) and its absmax
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + j * NT;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float h = x[j][e];
            if (apply_norm) {
                h = __fmul_rn(h, r);
                if (g != nullptr && v < nvec) h = __fmul_rn(h, __ldg(g + v * E + e));
            }
            x[j][e] = h;
            m = fmaxf(m, fabsf(h));
        }
    }
    m = block_max_f32<NT>(m, red_f);
    const float s = __fdiv_rn(127.0f, fmaxf(m, 1e-5f));
    const float c = __frcp_rn(s);
    if (threadIdx.x == 0) {
        sx[t] = s;
        if (apply_norm) rinv[t] = r;
    }

    // codes and dequantised values.  |x_hat * s| <= 127 * (1 + 2^-23) for finite inputs,
    // so rint(x_hat * s) is in [-127, 127]; the integer clamp is kept for robustness.
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
        const int v = threadIdx.x + j * NT;
        if (v >= nvec) continue;
        uint32_t qb[E];
        float dq[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const float tq = __fadd_rn(__fmul_rn(x[j][e], s), kRoundMagic);   // 1.5*2^23 + rint(x_hat*s)
            const int qi = max(-128, min(127, __float_as_int(tq) - kRoundMagicBits));
            qb[e] = static_cast<uint32_t>(qi) & 0xFFu;
            dq[e] = div_by_scale(__fsub_rn(tq, kRoundMagic), s, c);
        }
        if constexpr (kBf16) {
            uint2 packed;
            packed.x = qb[0] | (qb[1] << 8) | (qb[2] << 16) | (qb[3] << 24);
            packed.y = qb[4] | (qb[5] << 8) | (qb[6] << 16) | (qb[7] << 24);
            reinterpret_cast<uint2*>(Xq)[row_vec0 + v] = packed;
            if (Xdq != nullptr) {
                uint32_t o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(dq[2 * i], dq[2 * i + 1]);
                    o[i] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                reinterpret_cast<uint4*>(Xdq)[row_vec0 + v] = make_uint4(o[0], o[1], o[2], o[3]);
            }
        } else {
            reinterpret_cast<uint32_t*>(Xq)[row_vec0 + v] = qb[0] | (qb[1] << 8) | (qb[2] << 16) | (qb[3] << 24);
            if (Xdq != nullptr) reinterpret_cast<float4*>(Xdq)[row_vec0 + v] = make_float4(dq[0], dq[1], dq[2], dq[3]);
        }
    }
}

// Largest row (elements) the register-resident kernel handles: 16 vectors per thread.
constexpr int kActMaxVpt = 16;
template <bool kBf16>
constexpr int act_threads() { return kBf16 ? 128 : 256; }

}  // namespace bl

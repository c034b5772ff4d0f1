// optim.cuh -- fused optimizer step of the latent weight.
//
// Restates, in the order the pages give them: per-matrix gradient clipping to a maximum L2
// norm (P5 §6.2 clip_grad_norm_(p, 1.0) for weight matrices), AdamW with decoupled weight
// decay and bias-corrected moments (P1 "BitNet量化感知训练中的梯度传播优化", optimizer
// configuration: lr 1e-3, betas (0.9, 0.95), weight decay 0.01, eps 1e-6), then the clamp of
// the latent weight to [-1, 1] (P1 "梯度裁剪与权重约束").
//
// Two launches, both HBM-bound:
//   pass 1  fp64 partial sums of dW^2, one per block, over the slices the weight
//           quantiser's |W| pass uses; block 0 also publishes the step index t = *step + 1;
//   pass 2  every block re-derives the clip coefficient from the partials in a fixed order,
//           then streams dW, W, m, v once (dW is an L2 hit when it fits there), updates them
//           in fp32 and writes W, m, v back -- and, in the same slices and order as the
//           quantiser's pass 1, the fp64 partial sums of |W_new|, so the next step's ternary
//           codes need only the quantiser's pass 2.
// Per element (fp32, one rounding per operation):
//   g = c dW;  m' = fma(b1, m, (1 - b1) g);  v' = fma(b2, v, ((1 - b2) g) g)
//   W' = clamp( W (1 - lr wd) - (lr / bc1) m' / (sqrt(v') / sqrt(bc2) + eps), -1, 1 )
#pragma once
#include "common.cuh"
#include "weight_quant.cuh"

namespace bl {

struct AdamwArgs {
    float lr;             // learning rate
    float beta1, beta2;   // moment decay rates
    float eps;            // added to the bias-corrected root of the second moment
    float decay;          // fl32(1 - lr * weight_decay)
    float omb1, omb2;     // fl32(1 - beta1), fl32(1 - beta2)
    float max_norm;       // clip threshold; <= 0 disables clipping
};

__global__ void __launch_bounds__(kWqThreads) grad_sumsq_partial_kernel(const float* __restrict__ dW, int64_t n,
                                                                        double* __restrict__ partials,
                                                                        const int32_t* __restrict__ step,
                                                                        int32_t* __restrict__ step_next) {
    __shared__ double red[kWqThreads / 32];
    pdl_trigger_and_wait();
    const int64_t nvec = n / 4;
    const float4* g4 = reinterpret_cast<const float4*>(dW);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWqThreads;
    double acc = 0.0;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kWqThreads + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(g4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc = fma((double)v[u].x, (double)v[u].x, acc);
            acc = fma((double)v[u].y, (double)v[u].y, acc);
            acc = fma((double)v[u].z, (double)v[u].z, acc);
            acc = fma((double)v[u].w, (double)v[u].w, acc);
        }
    }
    for (; i < nvec; i += stride) {
        const float4 v = __ldg(g4 + i);
        acc = fma((double)v.x, (double)v.x, acc);
        acc = fma((double)v.y, (double)v.y, acc);
        acc = fma((double)v.z, (double)v.z, acc);
        acc = fma((double)v.w, (double)v.w, acc);
    }
    acc = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < kWqThreads / 32; ++w) s += red[w];
        partials[blockIdx.x] = s;
        if (blockIdx.x == 0) *step_next = *step + 1;
    }
}

struct AdamwScalars {
    float c;           // clip coefficient
    float step_size;   // lr / (1 - beta1^t)
    float bc2_sqrt;    // sqrt(1 - beta2^t)
};

__device__ __forceinline__ float adamw_elem(float w, float dw, float& m, float& v, const AdamwArgs& a,
                                            const AdamwScalars& s) {
    const float g = __fmul_rn(s.c, dw);
    m = __fmaf_rn(a.beta1, m, __fmul_rn(a.omb1, g));
    v = __fmaf_rn(a.beta2, v, __fmul_rn(__fmul_rn(a.omb2, g), g));
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(v), s.bc2_sqrt), a.eps);
    float wn = __fsub_rn(__fmul_rn(w, a.decay), __fdiv_rn(__fmul_rn(s.step_size, m), denom));
    return fminf(fmaxf(wn, -1.0f), 1.0f);
}

// Grid = the partial count of the weight quantiser's pass 1 for n (wq_num_partials), so
// block b visits exactly the vectors that pass 1's block b would, in the same order.
__global__ void __launch_bounds__(kWqThreads) adamw_clamp_kernel(
    float* __restrict__ W, const float* __restrict__ dW, float* __restrict__ m, float* __restrict__ v, int64_t n,
    const double* __restrict__ gpart, int nparts, AdamwArgs a, const int32_t* __restrict__ step_next,
    int32_t* __restrict__ step, double* __restrict__ wpart) {
    __shared__ double red[kWqThreads / 32];
    __shared__ AdamwScalars s_sc;
    pdl_trigger_and_wait();
    {
        // fixed-order sum of the dW^2 partials (as the quantiser's pass 2 sums its partials)
        constexpr int kPerThread = (kWqMaxPartials + kWqThreads - 1) / kWqThreads;
        double acc = 0.0;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
            const int i = threadIdx.x + kWqThreads * k;
            acc += i < nparts ? gpart[i] : 0.0;
        }
        acc = warp_sum(acc);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            double S = 0.0;
#pragma unroll
            for (int w = 0; w < kWqThreads / 32; ++w) S += red[w];
            double c = 1.0;
            if (a.max_norm > 0.0f) {
                c = static_cast<double>(a.max_norm) / (sqrt(S) + 1e-6);
                if (c > 1.0) c = 1.0;
            }
            const double t = static_cast<double>(*step_next);
            const double bc1 = 1.0 - pow(static_cast<double>(a.beta1), t);
            const double bc2 = 1.0 - pow(static_cast<double>(a.beta2), t);
            AdamwScalars sc;
            sc.c = static_cast<float>(c);
            sc.step_size = static_cast<float>(static_cast<double>(a.lr) / bc1);
            sc.bc2_sqrt = static_cast<float>(sqrt(bc2));
            s_sc = sc;
            if (blockIdx.x == 0) *step = *step_next;
        }
        __syncthreads();
    }
    const AdamwScalars sc = s_sc;
    const int64_t nvec = n / 4;
    float4* w4 = reinterpret_cast<float4*>(W);
    const float4* g4 = reinterpret_cast<const float4*>(dW);
    float4* m4 = reinterpret_cast<float4*>(m);
    float4* v4 = reinterpret_cast<float4*>(v);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kWqThreads;
    auto update = [&](float4 w, const float4 g, float4& mm, float4& vv) -> float4 {
        w.x = adamw_elem(w.x, g.x, mm.x, vv.x, a, sc);
        w.y = adamw_elem(w.y, g.y, mm.y, vv.y, a, sc);
        w.z = adamw_elem(w.z, g.z, mm.z, vv.z, a, sc);
        w.w = adamw_elem(w.w, g.w, mm.w, vv.w, a, sc);
        return w;
    };
    double acc = 0.0;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kWqThreads + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        float4 wv[4], gv[4], mv[4], vv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            wv[u] = w4[i + u * stride];            // W stays in L2 for the next quantiser pass
            gv[u] = __ldcs(g4 + i + u * stride);
            mv[u] = __ldcs(m4 + i + u * stride);
            vv[u] = __ldcs(v4 + i + u * stride);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 wn = update(wv[u], gv[u], mv[u], vv[u]);
            w4[i + u * stride] = wn;
            __stcs(m4 + i + u * stride, mv[u]);
            __stcs(v4 + i + u * stride, vv[u]);
            acc += (double)fabsf(wn.x);
            acc += (double)fabsf(wn.y);
            acc += (double)fabsf(wn.z);
            acc += (double)fabsf(wn.w);
        }
    }
    for (; i < nvec; i += stride) {
        float4 mm = __ldcs(m4 + i), vv = __ldcs(v4 + i);
        const float4 wn = update(w4[i], __ldcs(g4 + i), mm, vv);
        w4[i] = wn;
        __stcs(m4 + i, mm);
        __stcs(v4 + i, vv);
        acc += (double)fabsf(wn.x);
        acc += (double)fabsf(wn.y);
        acc += (double)fabsf(wn.z);
        acc += (double)fabsf(wn.w);
    }
    acc = warp_sum(acc);
    __syncthreads();   // red[] is reused
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0 && wpart != nullptr) {
        double s = 0.0;
        for (int w = 0; w < kWqThreads / 32; ++w) s += red[w];
        wpart[blockIdx.x] = s;
    }
}

}  // namespace bl

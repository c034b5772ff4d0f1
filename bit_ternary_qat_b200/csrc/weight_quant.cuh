// weight_quant.cuh -- K2: per-tensor absmean ternary weight quantiser + 2-bit packing.
//
// Restates P3 ("BitNet 1.5技术解析…") §2.1 weight_quant and P5 ("1.58-bit量化技术…")
// §2.2 ternary_quantize:  gamma = max(mean|W|, 1e-5),  W_q = clamp(round(W/gamma), -1, 1),
// and P5 §4.1 (2-bit codes 00 -> 0, 01 -> +1, 10 -> -1) / §5.1 (64-bit aligned packing).
//
// Two launches, both memory-bound:
//   pass 1  each block sums |W| over a fixed slice in fp64 -> one partial per block;
//   pass 2  every block re-derives gamma from the partials in a fixed order (so no third
//           launch and no atomics: the result is bit-identical run to run), then streams W
//           again (an L2 hit when W fits in L2) and writes int8 codes, bf16 codes and the
//           packed 2-bit codes in one go.
//
// The ternary decision needs no per-element division.  fl32(w / gamma) is monotone in w,
// so {w > 0 : fl32(w/gamma) > 0.5} = {w >= w*} for one fp32 threshold w*, found by a
// bisection over fp32 bit patterns (near gamma/2) that evaluates the IEEE division itself.
// Because the division is sign-symmetric, W_q = sign(w) * [|w| >= w*] reproduces
// clamp(round_half_even(fl32(w/gamma)), -1, 1) exactly for every finite w.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kWqThreads = 256;
constexpr int kWqMaxPartials = 1184;   // 8 blocks per SM on 148 SMs

// Number of pass-1 blocks for n elements (4 float4 loads per thread): depends on n only, so
// gamma is the same on every device.
__host__ __device__ inline int wq_num_partials(int64_t n) {
    int64_t vecs = n / 4;
    int64_t p = (vecs + kWqThreads * 4 - 1) / (kWqThreads * 4);
    if (p < 1) p = 1;
    if (p > kWqMaxPartials) p = kWqMaxPartials;
    return static_cast<int>(p);
}

// Partial sum number `part` of `nparts` (256 threads, 4 float4 loads in flight per thread,
// stride nparts * 256 vectors): the same slices whichever launch runs it.
__device__ __forceinline__ void absmean_partial_block(const float* __restrict__ W, int64_t n, int part, int nparts,
                                                      double* __restrict__ partials, double* red) {
    const int64_t nvec = n / 4;
    const float4* w4 = reinterpret_cast<const float4*>(W);
    const int64_t stride = (int64_t)nparts * kWqThreads;
    double acc = 0.0;
    int64_t i = part * (int64_t)kWqThreads + threadIdx.x;
    // four independent loads in flight per thread
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(w4 + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc += (double)fabsf(v[u].x);
            acc += (double)fabsf(v[u].y);
            acc += (double)fabsf(v[u].z);
            acc += (double)fabsf(v[u].w);
        }
    }
    for (; i < nvec; i += stride) {
        float4 v = __ldg(w4 + i);
        acc += (double)fabsf(v.x);
        acc += (double)fabsf(v.y);
        acc += (double)fabsf(v.z);
        acc += (double)fabsf(v.w);
    }
    acc = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
        for (int w = 0; w < kWqThreads / 32; ++w) s += red[w];
        partials[part] = s;
    }
}

__global__ void __launch_bounds__(kWqThreads) absmean_partial_kernel(const float* __restrict__ W, int64_t n,
                                                                     double* __restrict__ partials) {
    __shared__ double red[kWqThreads / 32];
    pdl_trigger_and_wait();
    absmean_partial_block(W, n, blockIdx.x, gridDim.x, partials, red);
}

__device__ __forceinline__ bool above_half(uint32_t bits, float gamma) {
    return __fdiv_rn(__uint_as_float(bits), gamma) > 0.5f;
}

// Smallest positive fp32 w with fl32(w / gamma) > 0.5 (gamma >= 1e-5 > 0), computed by the
// 32 lanes of one warp.  The answer is within a few ulps of gamma/2: lane i tests the bit
// pattern of gamma/2 - 16 + i (monotone predicate, so the ballot is 0..01..1) and the first
// set bit is the answer; if the window does not bracket it, lane 0 bisects the whole
// positive range.
__device__ __forceinline__ float ternary_threshold_warp(float gamma) {
    const int lane = threadIdx.x & 31;
    const uint32_t c = __float_as_uint(__fmul_rn(0.5f, gamma));
    const uint32_t base = c - 16u;
    const unsigned mask = __ballot_sync(0xffffffffu, above_half(base + lane, gamma));
    uint32_t thr = base + (uint32_t)(__ffs((int)mask) - 1);
    if (mask == 0u || (mask & 1u)) {
        uint32_t lo = 0u, hi = 0x7f7fffffu;      // 0/gamma = 0 is not above; FLT_MAX/gamma is
        while (hi - lo > 1u) {
            const uint32_t mid = lo + ((hi - lo) >> 1);
            if (above_half(mid, gamma)) hi = mid; else lo = mid;
        }
        thr = hi;
    }
    return __uint_as_float(thr);
}

constexpr uint32_t kBf16One = 0x3F80u;   // bf16 bits of +1.0

// Codes of 16 consecutive weights (group gi).  thr > 0: W_q = sign(w) [|w| >= thr].  With
// kNonzero the rule also holds for thr = 0 (a zero weight keeps code 0).  The bf16 output
// holds W_q times the magnitude whose bf16 bits are mag_bits (the codes themselves for +1).
template <bool kNonzero = false>
__device__ __forceinline__ void quantise16(const float (&w)[16], float thr, int64_t gi, int8_t* __restrict__ wq_i8,
                                           uint16_t* __restrict__ wq_bf16, uint8_t* __restrict__ packed,
                                           uint32_t mag_bits = kBf16One) {
    int q[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        if constexpr (kNonzero)
            q[e] = (w[e] >= thr && w[e] > 0.0f) ? 1 : ((w[e] <= -thr && w[e] < 0.0f) ? -1 : 0);
        else
            q[e] = (w[e] >= thr) ? 1 : ((w[e] <= -thr) ? -1 : 0);
    }
    if (wq_i8 != nullptr) {
        uint32_t b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            b[j] = (uint32_t)(q[4 * j] & 0xFF) | ((uint32_t)(q[4 * j + 1] & 0xFF) << 8) |
                   ((uint32_t)(q[4 * j + 2] & 0xFF) << 16) | ((uint32_t)(q[4 * j + 3] & 0xFF) << 24);
        reinterpret_cast<uint4*>(wq_i8)[gi] = make_uint4(b[0], b[1], b[2], b[3]);
    }
    if (wq_bf16 != nullptr) {
        // bf16 bits of -m, 0, +m
        const uint32_t neg = mag_bits | 0x8000u;
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t lo = q[2 * j] == 0 ? 0u : (q[2 * j] > 0 ? mag_bits : neg);
            const uint32_t hi = q[2 * j + 1] == 0 ? 0u : (q[2 * j + 1] > 0 ? mag_bits : neg);
            h[j] = lo | (hi << 16);
        }
        uint4* dst = reinterpret_cast<uint4*>(wq_bf16) + gi * 2;
        dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
        dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    }
    if (packed != nullptr) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) word |= (q[e] > 0 ? 1u : (q[e] < 0 ? 2u : 0u)) << (2 * e);
        reinterpret_cast<uint32_t*>(packed)[gi] = word;
    }
}

// n % 32 == 0.  Each thread loads kTqGroups groups of 16 weights (all loads in flight)
// before the block waits for gamma and the threshold, then quantises them; weights beyond
// grid * kWqThreads * kTqGroups groups are handled in further rounds of the same kind.
// kTau: the zero threshold is tau = fl32(tau_factor * gamma) (P2, "直通估计器在三元权重量化
// 中的作用": tau = 0.7 scale, |W| < tau -> 0) instead of the round/clamp threshold.
constexpr int kTqGroups = 2;

template <bool kTau>
__global__ void __launch_bounds__(kWqThreads, 4) ternary_quant_kernel(
    const float* __restrict__ W, int64_t n, const double* __restrict__ partials, int nparts,
    int8_t* __restrict__ wq_i8, uint16_t* __restrict__ wq_bf16, uint8_t* __restrict__ packed,
    float* __restrict__ gamma_out, float tau_factor) {
    __shared__ float s_thr;
    __shared__ double s_red[kWqThreads / 32];
    pdl_trigger_and_wait();
    const int64_t ngroups = n / 16;
    const float4* w4 = reinterpret_cast<const float4*>(W);
    const int64_t round_groups = static_cast<int64_t>(gridDim.x) * kWqThreads * kTqGroups;
    auto load1 = [&](int64_t r0, int q, float (&wq)[16], int64_t& g) {
        g = r0 + (static_cast<int64_t>(blockIdx.x) * kTqGroups + q) * kWqThreads + threadIdx.x;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 v = g < ngroups ? __ldg(w4 + g * 4 + j) : make_float4(0.f, 0.f, 0.f, 0.f);
            wq[4 * j] = v.x; wq[4 * j + 1] = v.y; wq[4 * j + 2] = v.z; wq[4 * j + 3] = v.w;
        }
    };
    auto load = [&](int64_t r0, float (&w)[kTqGroups][16], int64_t (&gi)[kTqGroups]) {
#pragma unroll
        for (int q = 0; q < kTqGroups; ++q) load1(r0, q, w[q], gi[q]);
    };
    float w[kTqGroups][16];
    int64_t gi[kTqGroups];
    load(0, w, gi);
    {
        // fixed-order sum of the partials by the whole block: thread i adds partials
        // i, i + 256, ... (all loaded at once), then a fixed butterfly per warp and the warp
        // sums in order
        constexpr int kPerThread = (kWqMaxPartials + kWqThreads - 1) / kWqThreads;
        double pv[kPerThread];
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
            const int i = threadIdx.x + kWqThreads * k;
            pv[k] = i < nparts ? partials[i] : 0.0;
        }
        double a = 0.0;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) a += pv[k];
        a = warp_sum(a);
        if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = a;
        __syncthreads();
    }
    if (threadIdx.x < 32) {
        double sum = 0.0;
#pragma unroll
        for (int wi = 0; wi < kWqThreads / 32; ++wi) sum += s_red[wi];
        const float gamma = fmaxf(static_cast<float>(sum / static_cast<double>(n)), 1e-5f);
        float thr;
        if constexpr (kTau)
            thr = __fmul_rn(tau_factor, gamma);
        else
            thr = ternary_threshold_warp(gamma);
        if (threadIdx.x == 0) {
            s_thr = thr;
            if (blockIdx.x == 0) *gamma_out = gamma;
        }
    }
    __syncthreads();
    const float thr = s_thr;
    // each group's registers are refilled with the next round's group as soon as it is
    // quantised, so the next round's loads overlap the current round's other group
    for (int64_t r0 = 0; r0 < ngroups; r0 += round_groups) {
        const bool more = r0 + round_groups < ngroups;
#pragma unroll
        for (int q = 0; q < kTqGroups; ++q) {
            if (gi[q] < ngroups) quantise16<kTau>(w[q], thr, gi[q], wq_i8, wq_bf16, packed);
            if (more) load1(r0 + round_groups, q, w[q], gi[q]);
        }
    }
}

// Per-row scale (P4 §9 "Quantizer": scale = mean |W| over each output row), with the b1.58
// round/clamp: gamma_n = max(mean_k |W[n, k]|, 1e-5), W_q = clamp(round(fl32(W / gamma_n)), -1, 1).
// One warp per row, 8 rows per block: fp64 sum of |W| over the row, the row's threshold
// (as above), then the row again (an L1/L2 hit) in groups of 16.  The bf16 output holds
// W_q * bf16(gamma_n), the dequantised weight that the backward contraction uses.  K % 16 == 0.
__global__ void __launch_bounds__(256) ternary_quant_rows_kernel(const float* __restrict__ W, int N, int K,
                                                                 int8_t* __restrict__ wq_i8,
                                                                 uint16_t* __restrict__ wq_bf16,
                                                                 uint8_t* __restrict__ packed,
                                                                 float* __restrict__ gamma_rows) {
    pdl_trigger_and_wait();
    const int lane = threadIdx.x & 31;
    const int64_t n = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (n >= N) return;
    const float4* row = reinterpret_cast<const float4*>(W + n * K);
    const int nvec = K / 4;
    double acc = 0.0;
    for (int v = lane; v < nvec; v += 32) {
        const float4 x = __ldg(row + v);
        acc += (double)fabsf(x.x);
        acc += (double)fabsf(x.y);
        acc += (double)fabsf(x.z);
        acc += (double)fabsf(x.w);
    }
    acc = warp_sum(acc);
    const float gamma = fmaxf(static_cast<float>(acc / static_cast<double>(K)), 1e-5f);
    const float thr = ternary_threshold_warp(gamma);
    if (lane == 0) gamma_rows[n] = gamma;
    const uint32_t mag = float_to_bf16_bits(gamma);
    const int groups = K / 16;
    const int64_t g0 = n * groups;
    for (int q = lane; q < groups; q += 32) {
        float w[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 v = __ldg(row + 4 * q + j);
            w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
        }
        quantise16(w, thr, g0 + q, wq_i8, wq_bf16, packed, mag);
    }
}

// Standalone packing of int8 codes (ternary_pack): one thread per 16 codes.
__global__ void __launch_bounds__(256) ternary_pack_kernel(const int8_t* __restrict__ wq, int64_t n,
                                                           uint8_t* __restrict__ packed) {
    pdl_trigger_and_wait();
    const int64_t ngroups = n / 16;
    for (int64_t gi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; gi < ngroups;
         gi += (int64_t)gridDim.x * blockDim.x) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(wq) + gi);
        const uint32_t b[4] = {v.x, v.y, v.z, v.w};
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            int8_t q = static_cast<int8_t>((b[e >> 2] >> (8 * (e & 3))) & 0xFFu);
            uint32_t code = q == 1 ? 1u : (q == -1 ? 2u : 0u);
            word |= code << (2 * e);
        }
        reinterpret_cast<uint32_t*>(packed)[gi] = word;
    }
}

}  // namespace bl

// act_quant.cuh -- K1: fused RMSNorm + per-token absmax int8 activation quantiser.
//
// Restates P3 ("BitNet 1.5技术解析…") §3.1 (RMSNorm applied before the activation
// quantiser) and §2.2 activation_quant (scale = 127 / row absmax clamped at 1e-5,
// round, clamp to [-128, 127], dequantised value forwarded through the STE), and
// P2 ("BitNet 三元权重量化训练工程…") per-token 8-bit absmax.
//
// One block per R adjacent token rows; each thread loads its 16-byte vectors of the rows
// once into registers (every row is read from HBM exactly once) and the three steps -- sum
// of squares, absmax, quantise -- run from registers with two block reductions in between
// (each reduction covers the R rows at once).
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
//     tests compare X_dq with the oracle's division.  The 256 quotients of a row are
//     computed once into a shared-memory table (already in the output type) and every
//     element looks its value up by code.
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


// R independent block sums / maxima with one barrier each (fixed order: per thread, then a
// fixed butterfly, then the warps in order).
// X_dq through a per-row table: entry q + 128 holds fl32(q / s_t) (computed with
// div_by_scale), stored as the output element type (bf16 bits after one RNE rounding, or
// fp32), so each element costs one shared-memory load instead of the five-op division.
template <bool kBf16>
struct DqLut;
template <>
struct DqLut<true> {
    using T = uint16_t;
    __device__ __forceinline__ static uint16_t make(float d) { return float_to_bf16_bits(d); }
};
template <>
struct DqLut<false> {
    using T = float;
    __device__ __forceinline__ static float make(float d) { return d; }
};

// Quantise one vector of E values of x_hat with scale s and store its codes (E int8) and,
// when wanted, its dequantised values from the row's table.  With tq = fl(fl(x_hat s) +
// 1.5*2^23) = 1.5*2^23 + q (q = rint(x_hat s), |q| <= 127 for finite inputs), the low byte
// of tq's bits is q mod 256 -- the int8 code itself -- because 1.5*2^23's low byte is zero;
// the table index is that byte with its top bit flipped (q + 128).  So codes need no
// integer conversion, no clamp and no shift: three byte permutes gather four codes.
__device__ __forceinline__ uint32_t quant_bits(float h, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(h, s), kRoundMagic));   // 1.5*2^23 + rint(x_hat*s)
}
__device__ __forceinline__ uint32_t lut_index(uint32_t tq_bits) { return (tq_bits & 0xFFu) ^ 0x80u; }
__device__ __forceinline__ uint32_t gather_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

template <bool kBf16, int E>
__device__ __forceinline__ void quant_store_vec(const float (&h)[E], float s, int8_t* Xq, void* Xdq, int64_t vec,
                                                const typename DqLut<kBf16>::T* lut) {
    uint32_t tb[E];
#pragma unroll
    for (int e = 0; e < E; ++e) tb[e] = quant_bits(h[e], s);
    if constexpr (kBf16) {
        reinterpret_cast<uint2*>(Xq)[vec] =
            make_uint2(gather_low_bytes(tb[0], tb[1], tb[2], tb[3]), gather_low_bytes(tb[4], tb[5], tb[6], tb[7]));
        if (Xdq != nullptr) {
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o[i] = static_cast<uint32_t>(lut[lut_index(tb[2 * i])]) |
                       (static_cast<uint32_t>(lut[lut_index(tb[2 * i + 1])]) << 16);
            reinterpret_cast<uint4*>(Xdq)[vec] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    } else {
        reinterpret_cast<uint32_t*>(Xq)[vec] = gather_low_bytes(tb[0], tb[1], tb[2], tb[3]);
        if (Xdq != nullptr)
            reinterpret_cast<float4*>(Xdq)[vec] = make_float4(lut[lut_index(tb[0])], lut[lut_index(tb[1])],
                                                              lut[lut_index(tb[2])], lut[lut_index(tb[3])]);
    }
}

template <int NT, int R>
__device__ __forceinline__ void block_sum_f64(double (&v)[R], double (*red)[NT / 32]) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
        const double w = warp_sum(v[q]);
        if ((threadIdx.x & 31) == 0) red[q][threadIdx.x >> 5] = w;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < R; ++q) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) s += red[q][w];
        v[q] = s;
    }
}

template <int NT, int R>
__device__ __forceinline__ void block_max_f32(float (&v)[R], float (*red)[NT / 32]) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
        const float w = warp_max(v[q]);
        if ((threadIdx.x & 31) == 0) red[q][threadIdx.x >> 5] = w;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < R; ++q) {
        float m = red[q][0];
#pragma unroll
        for (int w = 1; w < NT / 32; ++w) m = fmaxf(m, red[q][w]);
        v[q] = m;
    }
}

// grid = ceil(T / R) blocks, block = NT threads; block b quantises rows R*b .. R*b + R - 1
// (adjacent rows: one contiguous span), thread i owns vectors i + j*NT of each row, j < VPT.
// All R rows are loaded before the first reduction, so R rows of loads are in flight per block.
template <bool kBf16, int NT, int VPT, int R>
__global__ void __launch_bounds__(NT) act_quant_kernel(const void* __restrict__ X, int T, int K, int apply_norm,
                                                       const float* __restrict__ g, float eps,
                                                       int8_t* __restrict__ Xq, float* __restrict__ sx,
                                                       float* __restrict__ rinv, void* __restrict__ Xdq) {
    using V = ActVec<kBf16>;
    using LutT = typename DqLut<kBf16>::T;
    constexpr int E = V::kElems;
    __shared__ double red_d[R][NT / 32];
    __shared__ float red_f[R][NT / 32];
    __shared__ LutT lut[R][256];
    pdl_trigger_and_wait();

    const int nvec = K / E;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * R;

    // the rows' raw 16-byte vectors in registers (read from HBM once, widened on use)
    uint4 raw[R][VPT];
#pragma unroll
    for (int q = 0; q < R; ++q) {
        const bool live = t0 + q < T;
        const uint4* xrow = reinterpret_cast<const uint4*>(X) + (t0 + q) * static_cast<int64_t>(nvec);
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            raw[q][j] = (live && v < nvec) ? __ldcs(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
        }
    }

    // r_t = 1 / sqrt(mean x^2 + eps): fp64 sum, fixed order; max |x| on the way
    float r[R], mx[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
        r[q] = 1.0f;
        mx[q] = 0.0f;
    }
    {
        double ss[R];
#pragma unroll
        for (int q = 0; q < R; ++q) {
            ss[q] = 0.0;
#pragma unroll
            for (int j = 0; j < VPT; ++j)
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float xf = V::elem(raw[q][j], e);
                    mx[q] = fmaxf(mx[q], fabsf(xf));
                    const double xd = static_cast<double>(xf);
                    ss[q] = fma(xd, xd, ss[q]);
                }
        }
        if (apply_norm) {
            block_sum_f64<NT, R>(ss, red_d);
#pragma unroll
            for (int q = 0; q < R; ++q)
                r[q] = static_cast<float>(1.0 / sqrt(ss[q] / static_cast<double>(K) + static_cast<double>(eps)));
        }
    }

    // x_hat = fl(fl(x * r) * g), recomputed where needed from the raw vector
    auto xhat = [&](int q, int j, float (&h)[E]) {
        const int v = threadIdx.x + j * NT;
        float gk[E];
#pragma unroll
        for (int e = 0; e < E; e += 4) {
            const float4 gv = (apply_norm && g != nullptr && v < nvec)
                                  ? __ldg(reinterpret_cast<const float4*>(g + static_cast<int64_t>(v) * E + e))
                                  : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            gk[e] = gv.x; gk[e + 1] = gv.y; gk[e + 2] = gv.z; gk[e + 3] = gv.w;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float x = V::elem(raw[q][j], e);
            if (apply_norm) {
                x = __fmul_rn(x, r[q]);
                if (g != nullptr) x = __fmul_rn(x, gk[e]);
            }
            h[e] = x;
        }
    };
    // max |x_hat|: without a gain, rounding is monotone, so max |fl(x r)| = fl(max |x| * r)
    float m[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
        if (apply_norm && g != nullptr) {
            m[q] = 0.0f;
#pragma unroll
            for (int j = 0; j < VPT; ++j) {
                float h[E];
                xhat(q, j, h);
#pragma unroll
                for (int e = 0; e < E; ++e) m[q] = fmaxf(m[q], fabsf(h[e]));
            }
        } else {
            m[q] = apply_norm ? __fmul_rn(mx[q], r[q]) : mx[q];
        }
    }
    block_max_f32<NT, R>(m, red_f);

    float s[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
        s[q] = __fdiv_rn(127.0f, fmaxf(m[q], 1e-5f));
        if (Xdq != nullptr) {
            // row q's table of fl(q / s) for q = -128..127
            const float c = __frcp_rn(s[q]);
            for (int i = threadIdx.x; i < 256; i += NT)
                lut[q][i] = DqLut<kBf16>::make(div_by_scale(static_cast<float>(i - 128), s[q], c));
        }
    }
    if (Xdq != nullptr) __syncthreads();
#pragma unroll
    for (int q = 0; q < R; ++q) {
        const int64_t t = t0 + q;
        if (t >= T) break;
        if (threadIdx.x == 0) {
            sx[t] = s[q];
            if (apply_norm) rinv[t] = r[q];
        }
        const int64_t row_vec0 = t * static_cast<int64_t>(nvec);
        // codes and dequantised values.  |x_hat * s| <= 127 * (1 + 2^-23) for finite inputs,
        // so rint(x_hat * s) is in [-127, 127] (no clamp needed; a non-finite input still
        // gives an in-range table index).
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
            const int v = threadIdx.x + j * NT;
            if (v >= nvec) continue;
            float h[E];
            xhat(q, j, h);
            quant_store_vec<kBf16, E>(h, s[q], Xq, Xdq, row_vec0 + v, lut[q]);
        }
    }
}

// Short rows (at most 32 * VPL 16-byte vectors): one warp per row, 8 rows per block, no
// shared memory and no block barrier -- both reductions are warp butterflies (fixed order).
// Each lane keeps its VPL raw vectors of the row in registers and widens them on use, so a
// warp has the whole row in flight at once.  The kernel is persistent (two blocks per SM,
// rows strided over the grid) and loads a warp's next row before it quantises the current
// one, so loads stay in flight through the reductions and there is no partial last wave.
template <int VPL>
__device__ __forceinline__ void act_quant_warp_load(const void* __restrict__ X, int64_t t, int nvec,
                                                    uint4 (&raw)[VPL]) {
    const int lane = threadIdx.x & 31;
    const uint4* xrow = reinterpret_cast<const uint4*>(X) + t * static_cast<int64_t>(nvec);
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int v = lane + 32 * j;
        raw[j] = v < nvec ? __ldcs(xrow + v) : make_uint4(0u, 0u, 0u, 0u);
    }
}

template <bool kBf16, int VPL>
__device__ __forceinline__ void act_quant_warp_row(const uint4 (&raw)[VPL], int64_t t, int K, int apply_norm,
                                                   const float* __restrict__ g, float eps, int8_t* __restrict__ Xq,
                                                   float* __restrict__ sx, float* __restrict__ rinv,
                                                   void* __restrict__ Xdq, typename DqLut<kBf16>::T* lut) {
    using V = ActVec<kBf16>;
    constexpr int E = V::kElems;
    const int lane = threadIdx.x & 31;
    const int nvec = K / E;
    const int64_t row_vec0 = t * static_cast<int64_t>(nvec);
    __syncwarp();   // every lane is done with the previous row's table

    // r_t = 1 / sqrt(mean x^2 + eps): fp64 sum, fixed order; max |x| on the way
    float r = 1.0f;
    float mx = 0.0f;
    {
        double ss = 0.0;
#pragma unroll
        for (int j = 0; j < VPL; ++j)
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float xf = V::elem(raw[j], e);
                mx = fmaxf(mx, fabsf(xf));
                if (apply_norm) {
                    const double xd = static_cast<double>(xf);
                    ss = fma(xd, xd, ss);
                }
            }
        if (apply_norm) {
            ss = warp_sum(ss);
            r = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(eps)));
        }
    }
    // x_hat = fl(fl(x * r) * g) of the E elements of vector j (recomputed where needed)
    auto xhat = [&](int j, float (&h)[E]) {
        const int v = lane + 32 * j;
        float gk[E];
#pragma unroll
        for (int e = 0; e < E; e += 4) {
            const float4 gv = (apply_norm && g != nullptr && v < nvec)
                                  ? __ldg(reinterpret_cast<const float4*>(g + static_cast<int64_t>(v) * E + e))
                                  : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
            gk[e] = gv.x; gk[e + 1] = gv.y; gk[e + 2] = gv.z; gk[e + 3] = gv.w;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            float x = V::elem(raw[j], e);
            if (apply_norm) {
                x = __fmul_rn(x, r);
                if (g != nullptr) x = __fmul_rn(x, gk[e]);
            }
            h[e] = x;
        }
    };
    // max |x_hat|: without a gain, rounding is monotone, so max |fl(x r)| = fl(max |x| * r)
    float m = 0.0f;
    if (apply_norm && g != nullptr) {
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            float h[E];
            xhat(j, h);
#pragma unroll
            for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(h[e]));
        }
    } else {
        m = apply_norm ? __fmul_rn(mx, r) : mx;
    }
    m = warp_max(m);
    const float s = __fdiv_rn(127.0f, fmaxf(m, 1e-5f));
    const float c = __frcp_rn(s);
    if (lane == 0) {
        sx[t] = s;
        if (apply_norm) rinv[t] = r;
    }
    if (Xdq != nullptr) {
        // this row's table of fl(q / s) for q = -128..127 (8 entries per lane)
#pragma unroll
        for (int i = lane; i < 256; i += 32) lut[i] = DqLut<kBf16>::make(div_by_scale(static_cast<float>(i - 128), s, c));
        __syncwarp();
    }
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const int v = lane + 32 * j;
        if (v >= nvec) continue;
        float h[E];
        xhat(j, h);
        quant_store_vec<kBf16, E>(h, s, Xq, Xdq, row_vec0 + v, lut);
    }
}

template <bool kBf16, int VPL>
__global__ void __launch_bounds__(256, 2) act_quant_warp_kernel(const void* __restrict__ X, int T, int K, int apply_norm,
                                                                const float* __restrict__ g, float eps,
                                                                int8_t* __restrict__ Xq, float* __restrict__ sx,
                                                                float* __restrict__ rinv, void* __restrict__ Xdq) {
    __shared__ typename DqLut<kBf16>::T lut_all[8][256];
    pdl_trigger_and_wait();
    const int warp = threadIdx.x >> 5;
    const int nvec = K / ActVec<kBf16>::kElems;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * 8;
    int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    if (t >= T) return;
    uint4 cur[VPL];
    act_quant_warp_load<VPL>(X, t, nvec, cur);
    for (;;) {
        const int64_t tn = t + stride;
        uint4 nxt[VPL];
        if (tn < T) act_quant_warp_load<VPL>(X, tn, nvec, nxt);
        act_quant_warp_row<kBf16, VPL>(cur, t, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, lut_all[warp]);
        if (tn >= T) break;
#pragma unroll
        for (int j = 0; j < VPL; ++j) cur[j] = nxt[j];
        t = tn;
    }
}

// ------------------------------------------------------------------------------------
// Per-tensor activation scale (P5 §5.1 quantize_activation: one scale 127 / max|x| over the
// whole tensor), applied to x_hat with the same 1e-5 floor, rounding and clamp as above.
// Two launches over one warp per row, 8 rows per block, a grid of at most kActMaxPartials
// blocks looping over row groups:
//   pass 1  r_t and max |x_hat| of every row; block maxima -> partials[blockIdx];
//   pass 2  every block takes the max of the partials (max is exact in any order), builds
//           one table of fl(q / s) and quantises its rows again with the shared s.
// X is read twice (the second read hits L2 when X fits there).
// ------------------------------------------------------------------------------------
constexpr int kActMaxPartials = 1184;

template <bool kBf16>
__device__ __forceinline__ float act_xhat(const uint4& raw, int e, int v, float r, int apply_norm,
                                          const float* __restrict__ g) {
    float h = ActVec<kBf16>::elem(raw, e);
    if (apply_norm) {
        h = __fmul_rn(h, r);
        if (g != nullptr) h = __fmul_rn(h, __ldg(g + v * ActVec<kBf16>::kElems + e));
    }
    return h;
}

template <bool kBf16>
__global__ void __launch_bounds__(256) act_tensor_max_kernel(const void* __restrict__ X, int T, int K, int apply_norm,
                                                             const float* __restrict__ g, float eps,
                                                             float* __restrict__ rinv, float* __restrict__ partials) {
    constexpr int E = ActVec<kBf16>::kElems;
    __shared__ float red[8];
    pdl_trigger_and_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = K / E;
    float m = 0.0f;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp; t < T; t += static_cast<int64_t>(gridDim.x) * 8) {
        const uint4* xrow = reinterpret_cast<const uint4*>(X) + t * nvec;
        float r = 1.0f;
        if (apply_norm) {
            double ss = 0.0;
            for (int v = lane; v < nvec; v += 32) {
                const uint4 raw = __ldg(xrow + v);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const double xd = static_cast<double>(ActVec<kBf16>::elem(raw, e));
                    ss = fma(xd, xd, ss);
                }
            }
            ss = warp_sum(ss);
            r = static_cast<float>(1.0 / sqrt(ss / static_cast<double>(K) + static_cast<double>(eps)));
            if (lane == 0) rinv[t] = r;
        }
        for (int v = lane; v < nvec; v += 32) {
            const uint4 raw = __ldg(xrow + v);
#pragma unroll
            for (int e = 0; e < E; ++e) m = fmaxf(m, fabsf(act_xhat<kBf16>(raw, e, v, r, apply_norm, g)));
        }
    }
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) b = fmaxf(b, red[w]);
        partials[blockIdx.x] = b;
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(256) act_tensor_quant_kernel(const void* __restrict__ X, int T, int K,
                                                               int apply_norm, const float* __restrict__ g,
                                                               const float* __restrict__ partials, int nparts,
                                                               int8_t* __restrict__ Xq, float* __restrict__ sx,
                                                               const float* __restrict__ rinv,
                                                               void* __restrict__ Xdq) {
    constexpr int E = ActVec<kBf16>::kElems;
    using LutT = typename DqLut<kBf16>::T;
    __shared__ float red[8];
    __shared__ LutT lut[256];
    pdl_trigger_and_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float m = 0.0f;
    for (int i = threadIdx.x; i < nparts; i += 256) m = fmaxf(m, partials[i]);
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    const float s = __fdiv_rn(127.0f, fmaxf(m, 1e-5f));
    if (Xdq != nullptr) {
        const float c = __frcp_rn(s);
        lut[threadIdx.x] = DqLut<kBf16>::make(div_by_scale(static_cast<float>(static_cast<int>(threadIdx.x) - 128), s, c));
        __syncthreads();
    }
    const int nvec = K / E;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + warp; t < T; t += static_cast<int64_t>(gridDim.x) * 8) {
        const uint4* xrow = reinterpret_cast<const uint4*>(X) + t * nvec;
        const float r = apply_norm ? __ldg(rinv + t) : 1.0f;
        if (lane == 0) sx[t] = s;
        for (int v = lane; v < nvec; v += 32) {
            const uint4 raw = __ldg(xrow + v);
            float h[E];
#pragma unroll
            for (int e = 0; e < E; ++e) h[e] = act_xhat<kBf16>(raw, e, v, r, apply_norm, g);
            quant_store_vec<kBf16, E>(h, s, Xq, Xdq, t * nvec + v, lut);
        }
    }
}

// Largest row (elements) the register-resident kernel handles: 16 vectors per thread.
constexpr int kActMaxVpt = 16;
template <bool kBf16>
constexpr int act_threads() { return kBf16 ? 128 : 256; }

}  // namespace bl

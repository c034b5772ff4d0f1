// gemm_simt.cuh -- fp32 CUDA-core GEMM for the fp32 (single-precision) layer path.
//
// The backward contractions of a layer run in fp32 (X, dY fp32) need fp32 products;
// tcgen05 has no fp32-input kind, so this path runs on the FMA pipes:
//   C[m, n] = alpha * sum_k A(m, k) * B(n, k)
// with arbitrary element strides for A and B (so dY, dY^T, X_dq and W_q bf16 are read in
// place, no transposes), fp32 accumulation, 64 x 64 output tiles, 16-deep k slices
// staged in shared memory, 4 x 4 outputs per thread.
#pragma once
#include "common.cuh"

namespace bl {

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_as_float<uint16_t>(const uint16_t* p) {
    return bf16_bits_to_float(__ldg(p));
}

template <typename TA, typename TB>
__global__ void __launch_bounds__(256) simt_gemm_kernel(int M, int N, int K, const TA* __restrict__ A,
                                                        int64_t sam, int64_t sak, const TB* __restrict__ B,
                                                        int64_t sbn, int64_t sbk, const float* __restrict__ alpha,
                                                        float* __restrict__ C, int64_t ldc) {
    constexpr int BM = 64, BN = 64, BK = 16;
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    pdl_trigger_and_wait();
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += BK) {
        for (int i = threadIdx.x; i < BM * BK; i += 256) {
            const int mm = i % BM, kk = i / BM;
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < M && k < K) ? load_as_float(A + m * sam + k * sak) : 0.0f;
            const int n = n0 + mm;
            Bs[kk][mm] = (n < N && k < K) ? load_as_float(B + n * sbn + k * sbk) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    const float al = alpha != nullptr ? __ldg(alpha) : 1.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) C[m * ldc + n] = al * acc[i][j];
        }
    }
}

}  // namespace bl

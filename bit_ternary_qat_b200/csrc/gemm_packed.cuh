// gemm_packed.cuh -- pieces of the int8 x packed-ternary linear (P3 §3.1's linear on the
// 2-bit codes of P5 §4.1 / §5.1) shared by its kernels: the launch arguments, the decode of a
// packed word, the ring constants, and the split-K finaliser.  The tensor-core kernel itself is
// in gemm_packed2.cuh (CTA pairs); up to 16 tokens the call runs the decode GEMV (gemv.cuh).
//
// Decode of one 32-bit word (16 codes, code i at bits 2i..2i+1): with a byte table
// TAB = {0, +1, -1, 0}, a byte permute whose selector nibbles are the codes looks four of them
// up at once:
//   even = prmt(TAB, sel = w & 0x33333333), odd = prmt(TAB, sel = (w >> 2) & 0x33333333)
// (and their upper halves), then two permutes interleave even and odd codes -- 13 integer
// operations per 16 codes.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kPkDecGroups = 4;              // decoder groups of 4 warps
constexpr int kPkThreads = 192 + kPkDecGroups * 128;
constexpr int kPkMaxBT = 256;                 // tokens per tile (UMMA N)
constexpr int kPkMaxPStages = 12;             // packed ring depth
constexpr int kPkKbPerP = 4;                  // 128-code k-blocks per packed stage
constexpr int kPkPBytes = 128 * 128;          // packed tile per stage per CTA: 128 rows x 512 codes
constexpr uint32_t kPkTab = 0x00FF0100u;      // byte c = int8 value of code c

struct PkArgs {
    int T, N, K;
    int bt;                        // tokens per tile: multiple of 32, <= 256
    int t_tiles, n_tiles, splits;  // work units = n_tiles * t_tiles * splits
    int k_blocks;                  // blocks of 128 codes along K
    int pstages;                   // packed ring depth
    const float* sx;               // s_t [T]
    const float* gamma;            // [1]
    void* y;                       // [T x N], written when splits == 1
    int32_t* acc;                  // splits == 1: optional int32 copy [T x N]; splits > 1: partial
                                   // sums [splits x T x N], slice sp written by the units of split sp
    uint64_t wait_ns;
};

// 16 codes of one packed word -> 16 int8 values (byte i = code i).
__device__ __forceinline__ uint4 pk_decode_word(uint32_t w) {
    const uint32_t se = w & 0x33333333u;
    const uint32_t so = (w >> 2) & 0x33333333u;
    const uint32_t e_lo = __byte_perm(kPkTab, 0u, se);          // codes 0, 2, 4, 6
    const uint32_t e_hi = __byte_perm(kPkTab, 0u, se >> 16);    // codes 8, 10, 12, 14
    const uint32_t o_lo = __byte_perm(kPkTab, 0u, so);          // codes 1, 3, 5, 7
    const uint32_t o_hi = __byte_perm(kPkTab, 0u, so >> 16);    // codes 9, 11, 13, 15
    return make_uint4(__byte_perm(e_lo, o_lo, 0x5140), __byte_perm(e_lo, o_lo, 0x7362),
                      __byte_perm(e_hi, o_hi, 0x5140), __byte_perm(e_hi, o_hi, 0x7362));
}

// y = fl(acc * fl(gamma / s_t)) with acc = the split-K partial sums added in split order
// (exact int32); acc_out optional (N % 4 == 0).
template <bool kBf16Out>
__global__ void __launch_bounds__(256) pk_finalize_kernel(const int32_t* __restrict__ part, int splits,
                                                          const float* __restrict__ sx,
                                                          const float* __restrict__ gamma, int T, int N,
                                                          void* __restrict__ y, int32_t* __restrict__ acc_out) {
    pdl_trigger_and_wait();
    const float gm = __ldg(gamma);
    const int64_t nv = static_cast<int64_t>(T) * N / 4;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>((i * 4) / N);
        const float c = __fdiv_rn(gm, __ldg(sx + t));
        int4 a = __ldcs(reinterpret_cast<const int4*>(part) + i);
        for (int sp = 1; sp < splits; ++sp) {
            const int4 b = __ldcs(reinterpret_cast<const int4*>(part) + sp * nv + i);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        if (acc_out != nullptr) reinterpret_cast<int4*>(acc_out)[i] = a;
        const float v0 = __fmul_rn(static_cast<float>(a.x), c), v1 = __fmul_rn(static_cast<float>(a.y), c);
        const float v2 = __fmul_rn(static_cast<float>(a.z), c), v3 = __fmul_rn(static_cast<float>(a.w), c);
        if constexpr (kBf16Out) {
            reinterpret_cast<uint2*>(y)[i] =
                make_uint2((uint32_t)float_to_bf16_bits(v0) | ((uint32_t)float_to_bf16_bits(v1) << 16),
                           (uint32_t)float_to_bf16_bits(v2) | ((uint32_t)float_to_bf16_bits(v3) << 16));
        } else {
            reinterpret_cast<float4*>(y)[i] = make_float4(v0, v1, v2, v3);
        }
    }
}

}  // namespace bl

// mma_peak.cuh -- tensor-pipe peak probe (sm_100a).
//
// The roofline of the BitLinear GEMMs needs a measured denominator for each operand kind.
// This kernel issues tcgen05.mma back to back from shared-memory operands that never
// change, accumulating into one TMEM accumulator: no global-memory traffic, no epilogue, so
// its rate is the tensor pipe's own ceiling for that instruction shape at the clocks the
// GPU holds while running it.  Shapes are those of the GEMMs: M = 128 x N = 256 per CTA
// (cta_group::1) or M = 256 x N = 256 per CTA pair (cta_group::2), 32 bytes of K per
// instruction (32 int8 or 16 bf16 values), four instructions per 128-byte swizzle atom.
//
// The operands hold pseudo-random values (any int8; bf16 of magnitude 2^-7..1 with random
// signs), so the datapath toggles as it does on real data.  The final wait is bounded.
#pragma once
#include "common.cuh"
#include "gemv.cuh"

namespace bl {

constexpr int kPeakThreads = 128;
// dynamic shared memory per CTA: more than half of an SM's, so exactly one CTA per SM
constexpr int kPeakSmemBytes = 120 * 1024;

__device__ __forceinline__ uint32_t peak_hash(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

// Fill `bytes` of shared memory with the probe's operand values.
template <bool kInt8>
__device__ __forceinline__ void peak_fill(uint8_t* dst, int bytes, uint32_t seed) {
    for (int i = threadIdx.x; i < bytes / 4; i += blockDim.x) {
        const uint32_t h = peak_hash(seed + static_cast<uint32_t>(i));
        uint32_t w;
        if constexpr (kInt8) {
            w = h;
        } else {
            // two bf16: sign random, exponent 120..127, mantissa random
            const uint32_t lo = (h & 0x807Fu) | ((120u + ((h >> 7) & 7u)) << 7);
            const uint32_t h2 = h >> 16;
            const uint32_t hi = ((h2 & 0x7Fu) | ((h2 << 8) & 0x8000u)) | ((120u + ((h2 >> 8) & 7u)) << 7);
            w = lo | (hi << 16);
        }
        reinterpret_cast<uint32_t*>(dst)[i] = w;
    }
}

// One CTA per SM: A 128 x 128 bytes, B 256 x 128 bytes, `iters` x 4 MMAs (M = 128, N = 256).
template <bool kInt8>
__global__ void __launch_bounds__(kPeakThreads, 1) mma_peak_kernel(int iters, uint64_t wait_ns) {
    constexpr uint32_t kIdesc = umma_idesc(kInt8, false, false, 128, 256);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    uint8_t* sA = smem;                  // 16 KB
    uint8_t* sB = smem + 16384;          // 32 KB
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + 49152);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    const int warp = threadIdx.x >> 5;

    peak_fill<kInt8>(sA, 16384, blockIdx.x * 0x10001u);
    peak_fill<kInt8>(sB, 32768, blockIdx.x * 0x10001u + 0x8000u);
    fence_proxy_async_shared();          // generic writes -> visible to the tensor core's reads
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger_and_wait();

    if (warp == 0) {
        if (elect_one()) {
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
            for (int it = 0; it < iters; ++it) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma<kInt8>(tmem, umma_desc_sw128(a0 + kk * 32, 16, 1024), umma_desc_sw128(b0 + kk * 32, 16, 1024),
                                  kIdesc, (it | kk) != 0 ? 1u : 0u);
            }
            tc_commit(done);
            // the MMAs must finish before TMEM is released: after a timeout, wait once more
            if (!mbar_wait(done, 0, wait_ns, nullptr)) mbar_wait(done, 0, 100000000ull, nullptr);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// One CTA pair per two SMs: each CTA holds its half of A (128 x 128 bytes) and of B
// (128 x 128 bytes); the leader issues `iters` x 4 MMAs with M = 256, N = 256 and its commit
// arrives on both CTAs' barriers.
template <bool kInt8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPeakThreads, 1) mma_peak2_kernel(int iters,
                                                                                           uint64_t wait_ns) {
    constexpr uint32_t kIdesc = umma_idesc(kInt8, false, false, 256, 256);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    uint8_t* sA = smem;                  // 16 KB
    uint8_t* sB = smem + 16384;          // 16 KB
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + 32768);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    const int warp = threadIdx.x >> 5;
    const bool leader = cluster_ctarank() == 0;

    peak_fill<kInt8>(sA, 16384, blockIdx.x * 0x10001u);
    peak_fill<kInt8>(sB, 16384, blockIdx.x * 0x10001u + 0x8000u);
    fence_proxy_async_shared();
    if (threadIdx.x == 0) {
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(tmem_slot, 256);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' operands written, barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_trigger_and_wait();

    if (warp == 0) {
        if (leader && elect_one()) {
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
            for (int it = 0; it < iters; ++it) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_pair<kInt8>(tmem, umma_desc_sw128(a0 + kk * 32, 16, 1024),
                                       umma_desc_sw128(b0 + kk * 32, 16, 1024), kIdesc, (it | kk) != 0 ? 1u : 0u);
            }
            tc_commit_pair(done, 0x3);
        }
        __syncwarp();
        if (threadIdx.x == 0) {
            if (!mbar_wait(done, 0, wait_ns, nullptr)) mbar_wait(done, 0, 100000000ull, nullptr);
        }
        __syncwarp();
    }
    tc_fence_before();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 256);
    }
}

// The warp-level integer MMA the decode GEMV uses (mma.sync m16n8k32, u8 x s8 -> s32) from
// register operands: 16 warps per SM, each with 8 independent accumulator chains, so the
// rate is the IMMA pipe's throughput rather than one chain's latency.
constexpr int kImmaWarps = 16;
constexpr int kImmaChains = 8;
__global__ void __launch_bounds__(kImmaWarps * 32, 1) imma_sync_peak_kernel(int iters) {
    pdl_trigger_and_wait();
    const uint32_t h = peak_hash(blockIdx.x * 1024u + threadIdx.x);
    const uint32_t a[4] = {h & 0x3F3F3F3Fu, (h >> 3) & 0x3F3F3F3Fu, (h >> 5) & 0x3F3F3F3Fu, (h >> 7) & 0x3F3F3F3Fu};
    const uint32_t b0 = peak_hash(h), b1 = peak_hash(h + 1u);
    int d[kImmaChains][4] = {};
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int c = 0; c < kImmaChains; ++c) mma_u8s8_16832(d[c], a, b0, b1);
    }
    int acc = 0;
#pragma unroll
    for (int c = 0; c < kImmaChains; ++c) acc += d[c][0] + d[c][1] + d[c][2] + d[c][3];
    if (acc == 0x7fffffff) record_status(0);   // keeps the chains live; never true in practice
}

}  // namespace bl

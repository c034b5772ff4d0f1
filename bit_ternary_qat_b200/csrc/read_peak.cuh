// read_peak.cuh -- read-bandwidth probe (sm_100a).
//
// The decode GEMV is bounded by HBM reads of the packed weight.  Its roofline denominator is
// a copy bandwidth; this kernel gives the read-only ceiling of the same bytes read the same
// way, with no arithmetic: the loads of a launch are XOR-folded into one register per thread,
// which is stored only if it equals a value that no input here produces (so no load can be
// dropped).  Like the GEMV, every launch triggers its dependants and then waits for the
// kernel before it (programmatic dependent launch), so chained launches measure the same
// per-launch fixed costs.
//   pattern 0: the GEMV's partition -- block b owns a balanced range of 16-row groups, each
//              warp an equally long run of (row group, 64-byte column block) steps, and lane
//              (g = lane / 4, t = lane % 4) loads 16 bytes of rows g and g + 8 at byte 16 t of
//              the step (8 rows x 64 contiguous bytes per warp instruction);
//   pattern 1: coalesced -- block b owns a contiguous, equally long span of the buffer and
//              each warp instruction loads 512 contiguous bytes.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kReadWarps = 16;
constexpr uint32_t kReadMagic = 0x9e3779b9u;

__global__ void __launch_bounds__(kReadWarps * 32, 1) read_peak_gemv_kernel(const uint8_t* __restrict__ buf,
                                                                           int rows, int row_bytes,
                                                                           uint32_t* __restrict__ sink) {
    pdl_trigger_and_wait();
    const int n_rg = rows / 16, spr = row_bytes / 64;
    const int rg0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * n_rg / gridDim.x);
    const int rg1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * n_rg / gridDim.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int nsteps = (rg1 - rg0) * spr;
    const int i0 = static_cast<int>(static_cast<int64_t>(warp) * nsteps / kReadWarps);
    const int i1 = static_cast<int>(static_cast<int64_t>(warp + 1) * nsteps / kReadWarps);
    const int64_t r8 = 8 * static_cast<int64_t>(row_bytes);
    uint32_t acc = 0;
#pragma unroll 8
    for (int i = i0; i < i1; ++i) {
        const int rg = rg0 + i / spr, s = i - (i / spr) * spr;
        const uint8_t* p = buf + (static_cast<int64_t>(rg) * 16 + g) * row_bytes + s * 64 + 16 * t;
        const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p));
        const uint4 b = __ldcs(reinterpret_cast<const uint4*>(p + r8));
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w;
    }
    if (acc == kReadMagic) sink[0] = acc;
}

__global__ void __launch_bounds__(kReadWarps * 32, 1) read_peak_coalesced_kernel(const uint4* __restrict__ buf,
                                                                                int64_t n16,
                                                                                uint32_t* __restrict__ sink) {
    pdl_trigger_and_wait();
    const int64_t lo = static_cast<int64_t>(blockIdx.x) * n16 / gridDim.x;
    const int64_t hi = static_cast<int64_t>(blockIdx.x + 1) * n16 / gridDim.x;
    uint32_t acc = 0;
#pragma unroll 8
    for (int64_t i = lo + threadIdx.x; i < hi; i += blockDim.x) {
        const uint4 a = __ldcs(buf + i);
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
    if (acc == kReadMagic) sink[0] = acc;
}

}  // namespace bl

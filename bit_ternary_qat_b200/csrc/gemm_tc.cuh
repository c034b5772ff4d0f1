// gemm_tc.cuh -- tcgen05 / TMEM / TMA GEMMs of the BitLinear path (sm_100a).
//
//   D[m, n] = sum_k A[m, k] * B[n, k]
//
// Three uses, one kernel template:
//   forward      kind::i8   A = X_q  [T x K] (K-major), B = W_q int8 [N x K] (K-major)
//                           epilogue y = (acc * gamma) / s_t  (P3 §3.1 output * scale)
//   grad input   kind::f16  A = dY   [T x N] (K-major), B = W_q bf16 [N x K] read MN-major
//                           epilogue dX_hat = gamma * acc     (STE: dY . W_dq)
//   grad weight  kind::f16  A = dY read MN-major (contraction over tokens),
//                           B = X_dq [T x K] read MN-major; epilogue dW = acc
//
// Structure (one CTA per SM, persistent over output tiles of 128 x kBN):
//   warp 0      TMA producer: one elected thread streams A/B k-blocks (128 bytes of K per
//               operand row, 128-byte swizzle) into a kStages-deep shared-memory ring.
//   warp 1      allocates 2*kBN TMEM columns (two fp32/int32 accumulators), then one elected
//               thread issues tcgen05.mma (M=128, N=kBN, K=32 bytes per instruction) and
//               tcgen05.commit to release ring slots and to publish finished accumulators.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time, rescale, store.
//               Accumulators are double-buffered, so the epilogue of tile i overlaps the
//               main loop of tile i+1.
// Out-of-range rows/columns/k are zero-filled by TMA; the epilogue masks stores.
// Every mbarrier wait is bounded (see common.cuh): on a timeout all roles unwind, the
// producer drains the loads it issued, the MMA thread drains its MMAs, TMEM is freed.
#pragma once
#include <cuda.h>
#include "common.cuh"

namespace bl {

enum TcEpilogue : int { kEpiLinear = 0, kEpiScaleF32 = 1, kEpiF32 = 2 };

constexpr int kTcStages = 4;
constexpr int kTcThreads = 192;
constexpr int kTcBM = 128;
constexpr int kTcABytes = kTcBM * 128;   // one stage of A: 128 rows x 128 bytes

struct TcGemmArgs {
    int M, N, K;                 // D is M x N, contraction length K (elements)
    int m_tiles, n_tiles, k_blocks;
    void* out;                   // D, row stride ldo elements
    int64_t ldo;
    int out_bf16;                // kEpiLinear: 1 = bf16 output, 0 = fp32
    int32_t* acc_out;            // kEpiLinear: optional int32 accumulators (row stride ldo)
    const float* row_scale;      // kEpiLinear: s_t of each output row
    const float* gamma;          // kEpiLinear / kEpiScaleF32
    uint64_t wait_ns;            // bound of every mbarrier wait
};

template <int kBN>
__host__ __device__ constexpr int tc_b_bytes() { return kBN * 128; }

template <int kBN>
__host__ __device__ constexpr size_t tc_smem_bytes() {
    return 1024 /* alignment slack */ + (size_t)kTcStages * (kTcABytes + tc_b_bytes<kBN>()) +
           (2 * kTcStages + 4) * sizeof(uint64_t) + 16;
}

template <bool kInt8, bool kAMN, bool kBMN, int kBN, int kEpi>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TcGemmArgs args) {
    static_assert(kBN % 64 == 0 && kBN <= 256, "kBN");
    static_assert(!kInt8 || (!kAMN && !kBMN), "int8 operands are K-major here");
    constexpr int kBBytes = tc_b_bytes<kBN>();
    constexpr uint32_t kStageTx = kTcABytes + kBBytes;
    constexpr int kKbElems = kInt8 ? 128 : 64;           // elements of K per stage
    constexpr int kInstrK = 4;                            // MMAs per stage (32 bytes of K each)
    constexpr uint32_t kIdesc = umma_idesc(kInt8, kAMN, kBMN, kTcBM, kBN);
    constexpr uint32_t kTmemCols = 2 * kBN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kTcStages * kTcABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + kTcStages * kBBytes);
    uint64_t* empty = full + kTcStages;
    uint64_t* tfull = empty + kTcStages;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = args.m_tiles * args.n_tiles;
    const uint64_t lim = args.wait_ns;

    if (warp == 0) {
        // ----------------------------------------------------------------- producer
        if (elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile % args.m_tiles;
                const int nb = tile / args.m_tiles;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, lim, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], kStageTx);
                    uint8_t* a_dst = sA + s * kTcABytes;
                    uint8_t* b_dst = sB + s * kBBytes;
                    if constexpr (!kAMN) {
                        tma_load_2d(a_dst, &tmA, &full[s], kb * kKbElems, mb * kTcBM);
                    } else {
#pragma unroll
                        for (int c = 0; c < kTcBM / 64; ++c)
                            tma_load_2d(a_dst + c * 8192, &tmA, &full[s], mb * kTcBM + c * 64, kb * 64);
                    }
                    if constexpr (!kBMN) {
                        tma_load_2d(b_dst, &tmB, &full[s], kb * kKbElems, nb * kBN);
                    } else {
#pragma unroll
                        for (int c = 0; c < kBN / 64; ++c)
                            tma_load_2d(b_dst + c * 8192, &tmB, &full[s], nb * kBN + c * 64, kb * 64);
                    }
                    if (++s == kTcStages) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok) {
                // Drain: wait (briefly) for the loads of the last kTcStages slots to land
                // before the block can exit.
                for (int i = 0; i < kTcStages; ++i) {
                    int ss = (s - 1 - i + 2 * kTcStages) % kTcStages;
                    uint32_t pp = (s - 1 - i < 0) ? (ph ^ 1u) : ph;
                    mbar_wait(&full[ss], pp, 100000000ull, nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA issuer
        if (elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            int tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
                const int b = tcount & 1;
                const uint32_t tph = (tcount >> 1) & 1;
                if (!mbar_wait(&tempty[b], tph ^ 1u, lim, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kBN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(&full[s], ph, lim, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * kTcABytes);
                    const uint32_t b_base = smem_u32(sB + s * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kInstrK; ++kk) {
                        uint64_t adesc, bdesc;
                        if constexpr (!kAMN) adesc = umma_desc_sw128(a_base + kk * 32, 16, 1024);
                        else adesc = umma_desc_sw128(a_base + kk * 2048, 8192, 1024);
                        if constexpr (!kBMN) bdesc = umma_desc_sw128(b_base + kk * 32, 16, 1024);
                        else bdesc = umma_desc_sw128(b_base + kk * 2048, 8192, 1024);
                        tc_mma<kInt8>(d_tmem, adesc, bdesc, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                    if (++s == kTcStages) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tfull[b]);
            }
            if (!ok) {
                // Drain outstanding MMAs: a final commit on a free accumulator barrier.
                tc_commit(&tfull[tcount & 1]);
                mbar_wait(&tfull[tcount & 1], ((tcount >> 1) & 1), 100000000ull, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------------- epilogue
        const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad + 32) belong to this warp
        int tcount = 0;
        float gm = 1.0f;
        if constexpr (kEpi != kEpiF32) gm = __ldg(args.gamma);
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
            const int b = tcount & 1;
            const uint32_t tph = (tcount >> 1) & 1;
            if (!mbar_wait(&tfull[b], tph, lim, abort_flag)) break;
            tc_fence_after();
            const int mb = tile % args.m_tiles;
            const int nb = tile / args.m_tiles;
            const int row = mb * kTcBM + quad * 32 + lane;
            const bool row_ok = row < args.M;
            float rs = 1.0f;
            if constexpr (kEpi == kEpiLinear) rs = row_ok ? __ldg(args.row_scale + row) : 1.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(b * kBN);
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t r[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + c0, r);
                tmem_ld_wait();
                const int col0 = nb * kBN + c0;
#pragma unroll
                for (int g8 = 0; g8 < 4; ++g8) {
                    const int col = col0 + g8 * 8;
                    // N % 16 == 0: a group of 8 columns is entirely in or entirely out
                    if (!row_ok || col >= args.N) continue;
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const uint32_t raw = r[g8 * 8 + e];
                        if constexpr (kEpi == kEpiLinear) {
                            v[e] = __fdiv_rn(__fmul_rn(static_cast<float>(static_cast<int32_t>(raw)), gm), rs);
                        } else if constexpr (kEpi == kEpiScaleF32) {
                            v[e] = __fmul_rn(gm, __uint_as_float(raw));
                        } else {
                            v[e] = __uint_as_float(raw);
                        }
                    }
                    const int64_t off = static_cast<int64_t>(row) * args.ldo + col;
                    if (kEpi == kEpiLinear && args.out_bf16) {
                        uint4 o;
                        o.x = (uint32_t)float_to_bf16_bits(v[0]) | ((uint32_t)float_to_bf16_bits(v[1]) << 16);
                        o.y = (uint32_t)float_to_bf16_bits(v[2]) | ((uint32_t)float_to_bf16_bits(v[3]) << 16);
                        o.z = (uint32_t)float_to_bf16_bits(v[4]) | ((uint32_t)float_to_bf16_bits(v[5]) << 16);
                        o.w = (uint32_t)float_to_bf16_bits(v[6]) | ((uint32_t)float_to_bf16_bits(v[7]) << 16);
                        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(args.out) + off) = o;
                    } else {
                        float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(args.out) + off);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    }
                    if constexpr (kEpi == kEpiLinear) {
                        if (args.acc_out != nullptr) {
                            int4* dst = reinterpret_cast<int4*>(args.acc_out + off);
                            dst[0] = make_int4((int)r[g8 * 8 + 0], (int)r[g8 * 8 + 1], (int)r[g8 * 8 + 2], (int)r[g8 * 8 + 3]);
                            dst[1] = make_int4((int)r[g8 * 8 + 4], (int)r[g8 * 8 + 5], (int)r[g8 * 8 + 6], (int)r[g8 * 8 + 7]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace bl

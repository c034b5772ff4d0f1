// gemm_tc.cuh -- tcgen05 / TMEM / TMA GEMMs of the BitLinear path (sm_100a).
//
//   D[m, n] = sum_k A[m, k] * B[n, k]
//
// Three uses, one kernel template:
//   forward      kind::i8   A = X_q  [T x K] (K-major), B = W_q int8 [N x K] (K-major)
//                           epilogue y = acc * (gamma / s_t)   (P3 §3.1: the linear of the
//                           dequantised operands times the scales, one factor per token)
//   grad input   kind::f16  A = dY   [T x N] (K-major), B = W_q bf16 [N x K] read MN-major
//                           epilogue dX_hat = gamma * acc       (STE: dY . W_dq)
//   grad weight  kind::f16  A = dY read MN-major (contraction over tokens),
//                           B = X_dq [T x K] read MN-major; epilogue dW = acc
//
// Structure (one CTA per SM, persistent over output tiles of 128 x kBN):
//   warp 0      TMA producer: one elected thread streams A/B k-blocks (128 bytes of K per
//               operand row, 128-byte swizzle) into a kTcStages-deep shared-memory ring.
//   warp 1      allocates 2*kBN TMEM columns (two fp32/int32 accumulators), then one elected
//               thread issues tcgen05.mma (M=128, N=kBN, K=32 bytes per instruction) and
//               tcgen05.commit to release ring slots and to publish finished accumulators.
//   warps 2..5  epilogue: each warp owns 32 accumulator rows (its TMEM lane quadrant).  Per
//               128-byte column chunk it loads the accumulators with tcgen05.ld, rescales,
//               writes its 32 rows into a 128-byte-swizzled shared-memory buffer (conflict
//               free, one 16-byte chunk per store) and one lane issues a TMA tensor store of
//               the 32-row box.  Two buffers per warp overlap the store of one chunk with
//               the math of the next; the TMA store clips rows/columns past the matrix edge.
//               Accumulators are double-buffered in TMEM, so the epilogue of tile i
//               overlaps the main loop of tile i+1.
// Out-of-range rows/columns/k of the operands are zero-filled by TMA.
// Every mbarrier wait is bounded (see common.cuh): on a timeout all roles unwind, the
// producer drains the loads it issued, the MMA thread drains its MMAs, TMEM is freed.
#pragma once
#include <cuda.h>
#include "common.cuh"

namespace bl {

enum TcEpilogue : int {
    kEpiLinearBf16 = 0,   // y = acc * (gamma / s_t) -> bf16
    kEpiScaleF32 = 1,     // gamma * acc -> fp32
    kEpiF32 = 2,          // acc -> fp32
    kEpiLinearF32 = 3,    // y = acc * (gamma / s_t) -> fp32
    kEpiLinearColBf16 = 4,  // y = acc * (gamma_n / s_t) -> bf16 (one scale per output column; 2-SM kernel only)
    kEpiLinearColF32 = 5,   // y = acc * (gamma_n / s_t) -> fp32 (2-SM kernel only)
};

constexpr int kTcStages = 4;
constexpr int kTcThreads = 192;
constexpr int kTcBM = 128;
constexpr int kTcABytes = kTcBM * 128;   // one stage of A: 128 rows x 128 bytes
constexpr int kEpiBufBytes = 32 * 128;   // one staging buffer: 32 rows x 128 bytes
constexpr int kEpiBytes = 4 * 2 * kEpiBufBytes;

struct TcGemmArgs {
    int M, N, K;                 // D is M x N, contraction length K (elements)
    int m_tiles, n_tiles, k_blocks;
    int32_t* acc_out;            // linear epilogues: optional int32 accumulators [M x N] (plain stores)
    const float* row_scale;      // linear epilogues: s_t of each output row
    const float* gamma;          // linear / scale epilogues
    uint64_t wait_ns;            // bound of every mbarrier wait
};

template <int kBN>
__host__ __device__ constexpr int tc_b_bytes() { return kBN * 128; }

template <int kBN>
__host__ __device__ constexpr size_t tc_smem_bytes() {
    return 1024 /* alignment slack */ + (size_t)kTcStages * (kTcABytes + tc_b_bytes<kBN>()) + kEpiBytes +
           (2 * kTcStages + 4) * sizeof(uint64_t) + 16;
}

__host__ __device__ constexpr bool epi_is_col(int e) { return e == kEpiLinearColBf16 || e == kEpiLinearColF32; }
__host__ __device__ constexpr bool epi_is_linear(int e) {
    return e == kEpiLinearBf16 || e == kEpiLinearF32 || epi_is_col(e);
}
__host__ __device__ constexpr bool epi_is_bf16(int e) { return e == kEpiLinearBf16 || e == kEpiLinearColBf16; }
// Output columns per 128-byte chunk.
__host__ __device__ constexpr int epi_chunk_cols(int e) { return epi_is_bf16(e) ? 64 : 32; }

template <bool kInt8, bool kAMN, bool kBMN, int kBN, int kEpi>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmD, const TcGemmArgs args) {
    static_assert(kBN % 64 == 0 && kBN <= 256, "kBN");
    static_assert(!kInt8 || (!kAMN && !kBMN), "int8 operands are K-major here");
    static_assert(!epi_is_col(kEpi), "per-column scales are in the 2-SM kernel only");
    constexpr int kBBytes = tc_b_bytes<kBN>();
    constexpr uint32_t kStageTx = kTcABytes + kBBytes;
    constexpr int kKbElems = kInt8 ? 128 : 64;           // elements of K per stage
    constexpr int kInstrK = 4;                            // MMAs per stage (32 bytes of K each)
    constexpr uint32_t kIdesc = umma_idesc(kInt8, kAMN, kBMN, kTcBM, kBN);
    constexpr uint32_t kTmemCols = 2 * kBN;
    constexpr int kChunkCols = epi_chunk_cols(kEpi);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kTcStages * kTcABytes;
    uint8_t* sE = sB + kTcStages * kBBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + kEpiBytes);
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
        tma_prefetch_desc(&tmD);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger_and_wait();

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
        const int quad = warp & 3;          // TMEM lanes [32*quad, 32*quad + 32) belong to this warp
        uint8_t* ebuf = sE + (warp - 2) * 2 * kEpiBufBytes;
        int buf = 0;
        int tcount = 0;
        float gm = 1.0f;
        if constexpr (kEpi != kEpiF32) gm = __ldg(args.gamma);
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
            const int b = tcount & 1;
            const uint32_t tph = (tcount >> 1) & 1;
            if (!mbar_wait_warp(&tfull[b], tph, lim, abort_flag)) break;
            tc_fence_after();
            const int mb = tile % args.m_tiles;
            const int nb = tile / args.m_tiles;
            const int row0 = mb * kTcBM + quad * 32;
            const int row = row0 + lane;
            const bool row_ok = row < args.M;
            float cs = 1.0f;   // per-token factor gamma / s_t
            if constexpr (epi_is_linear(kEpi)) cs = row_ok ? __fdiv_rn(gm, __ldg(args.row_scale + row)) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(b * kBN);
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += kChunkCols) {
                const int col0 = nb * kBN + c0;
                if (col0 >= args.N) break;                     // warp-uniform
                uint32_t ra[32], rb[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + c0, ra);
                if constexpr (kChunkCols == 64) {
                    tmem_ld_32x32b_x32(t_row + c0 + 32, rb);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rb[i] = 0u;
                }
                tmem_ld_wait();
                auto r = [&](int i) -> uint32_t { return i < 32 ? ra[i] : rb[i - 32]; };
                // this lane's 128-byte row segment as 8 x 16-byte chunks
                uint4 v[8];
                if constexpr (kEpi == kEpiLinearBf16) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = __fmul_rn(static_cast<float>(static_cast<int32_t>(r(8 * j + 2 * e))), cs);
                            const float hi = __fmul_rn(static_cast<float>(static_cast<int32_t>(r(8 * j + 2 * e + 1))), cs);
                            w[e] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
                        }
                        v[j] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float f[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t raw = r(4 * j + e);
                            if constexpr (kEpi == kEpiLinearF32)
                                f[e] = __fmul_rn(static_cast<float>(static_cast<int32_t>(raw)), cs);
                            else if constexpr (kEpi == kEpiScaleF32)
                                f[e] = __fmul_rn(gm, __uint_as_float(raw));
                            else
                                f[e] = __uint_as_float(raw);
                        }
                        v[j] = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                          __float_as_uint(f[3]));
                    }
                }
                // the staging buffer's previous store (two chunks ago) must have been read
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                uint8_t* sb = ebuf + buf * kEpiBufBytes;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4*>(sb + lane * 128 + ((j ^ (lane & 7)) << 4)) = v[j];
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmD, sb, col0, row0);
                    bulk_commit_group();
                }
                buf ^= 1;
                if constexpr (epi_is_linear(kEpi)) {
                    if (args.acc_out != nullptr && row_ok) {
                        // debug copy of the exact int32 accumulators (plain stores)
                        int32_t* dst = args.acc_out + static_cast<int64_t>(row) * args.N + col0;
#pragma unroll
                        for (int j = 0; j < kChunkCols / 4; ++j)
                            if (col0 + 4 * j < args.N)
                                reinterpret_cast<int4*>(dst)[j] = make_int4((int)r(4 * j), (int)r(4 * j + 1),
                                                                            (int)r(4 * j + 2), (int)r(4 * j + 3));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ====================================================================================
// 2-SM variant: a cluster of two CTAs computes a 256 x 256 tile with tcgen05.mma
// .cta_group::2 (M = 256, N = 256).  CTA r of the pair loads rows [128 r, 128 r + 128) of
// the tile's A and of the tile's B (its half of the N columns) into its own shared memory;
// the leader (r = 0) issues the MMAs, which read both CTAs' shared memory and write the
// accumulators of rows [128 r, 128 r + 128) into CTA r's TMEM.  Per SM a pipeline stage is
// 16 KB of A + 16 KB of B for the same MMA work that costs 16 + 32 KB in the 1-SM kernel,
// so six stages fit and 1.5x more MMA work is in flight per byte of shared memory.
// Barrier protocol:
//   full[s]   leader only: the leader's producer posts the pair's bytes (expect_tx); both
//             CTAs' TMA loads complete bytes on it (2-SM TMA form, no multicast);
//   empty[s]  each CTA: arrived by the leader's tcgen05.commit multicast to both CTAs;
//   tfull[b]  each CTA: arrived by the leader's commit multicast after a tile's last MMA;
//   tempty[b] leader only: 4 epilogue warps of each CTA arrive when they drained TMEM.
// Cross-CTA barrier addresses come from mapa.  Cluster barriers only at set-up and
// teardown; every other wait is bounded.
// ====================================================================================
constexpr int kTc2Stages = 6;
constexpr int kTc2HalfBytes = 128 * 128;   // one operand half per stage per CTA: 128 rows x 128 bytes

__host__ __device__ constexpr size_t tc2_smem_bytes() {
    return 1024 + (size_t)kTc2Stages * 2 * kTc2HalfBytes + kEpiBytes + (2 * kTc2Stages + 4) * sizeof(uint64_t) + 16;
}

// Tile order of the 2-SM kernel (grouped raster): tiles are taken in groups of kTileGroupM
// consecutive m-tiles; inside a group the m-tile varies fastest, then the n-tile.  The tiles
// that run at the same time (one per cluster, consecutive indices) then cover a block about
// kTileGroupM tall and (clusters / kTileGroupM) wide, so each operand panel they read is
// shared by several of them and stays in L2 while the group moves along n, instead of every
// wave touching almost every A panel once (m-fastest order).  The last group may be shorter.
constexpr int kTileGroupM = 8;
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb, int& nb) {
    const int per_group = kTileGroupM * n_tiles;
    const int grp = tile / per_group;
    const int local = tile - grp * per_group;
    const int m0 = grp * kTileGroupM;
    const int gm = m_tiles - m0 < kTileGroupM ? m_tiles - m0 : kTileGroupM;
    mb = m0 + local % gm;
    nb = local / gm;
}

// Work units of the 2-SM kernel.  The tiles that would make up a last, partial wave -- when
// there are at most half as many of them as clusters -- are each split into two 256 x 128
// halves (N = 128 MMAs, half the time), so the tail takes half a wave instead of a whole one
// while the other clusters idle.  Unit u < full_units is tile u; unit full_units + 2 j + h is
// half h (output columns [128 h, 128 h + 128) of the tile) of tile full_units + j.
struct Tc2Plan {
    int full_units, num_units;
};
__device__ __forceinline__ Tc2Plan tc2_plan(int num_tiles, int npairs) {
    const int tail = num_tiles % npairs;
    const bool split = tail != 0 && 2 * tail <= npairs;
    return Tc2Plan{split ? num_tiles - tail : num_tiles, split ? num_tiles + tail : num_tiles};
}
// unit -> tile coordinates and half (-1: the whole 256-column tile)
__device__ __forceinline__ void tc2_unit(int u, const Tc2Plan& pl, int m_tiles, int n_tiles, int& mb, int& nb,
                                         int& half) {
    int tile = u;
    half = -1;
    if (u >= pl.full_units) {
        const int v = u - pl.full_units;
        tile = pl.full_units + (v >> 1);
        half = v & 1;
    }
    tile_coords(tile, m_tiles, n_tiles, mb, nb);
}

template <bool kInt8, bool kAMN, bool kBMN, int kEpi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
    tc_gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmD, const TcGemmArgs args) {
    static_assert(!kInt8 || (!kAMN && !kBMN), "int8 operands are K-major here");
    constexpr int kBN = 256;                              // pair tile columns
    constexpr uint32_t kStageTxPair = 2u * 2u * kTc2HalfBytes;
    constexpr int kKbElems = kInt8 ? 128 : 64;
    constexpr int kInstrK = 4;
    constexpr uint32_t kIdesc = umma_idesc(kInt8, kAMN, kBMN, 256, kBN);
    constexpr uint32_t kTmemCols = 2 * kBN;
    constexpr int kChunkCols = epi_chunk_cols(kEpi);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kTc2Stages * kTc2HalfBytes;
    uint8_t* sE = sB + kTc2Stages * kTc2HalfBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + kEpiBytes);
    uint64_t* empty = full + kTc2Stages;
    uint64_t* tfull = empty + kTc2Stages;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTc2Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmD);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger_and_wait();

    const int num_tiles = args.m_tiles * args.n_tiles;   // m_tiles counts 256-row pair tiles
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const uint64_t lim = args.wait_ns;
    const Tc2Plan plan = tc2_plan(num_tiles, npairs);
    constexpr uint32_t kIdescHalf = umma_idesc(kInt8, kAMN, kBMN, 256, kBN / 2);

    if (warp == 0) {
        // ----------------------------------------------------------------- producer (both CTAs)
        if (elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int u = pair; u < plan.num_units && ok; u += npairs) {
                int mb, nb, half;
                tc2_unit(u, plan, args.m_tiles, args.n_tiles, mb, nb, half);
                const int arow = mb * 256 + static_cast<int>(rank) * 128;
                // CTA r supplies rows [128 r, 128 r + 128) of B for a whole tile, rows
                // [128 h + 64 r, 128 h + 64 r + 64) of it for half h (the same boxes are
                // loaded; the MMA reads their first 64 rows)
                const int brow = half < 0 ? nb * kBN + static_cast<int>(rank) * 128
                                          : nb * kBN + half * (kBN / 2) + static_cast<int>(rank) * 64;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, lim, abort_flag)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(&full[s], kStageTxPair);
                    const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
                    uint8_t* a_dst = sA + s * kTc2HalfBytes;
                    uint8_t* b_dst = sB + s * kTc2HalfBytes;
                    if constexpr (!kAMN) {
                        tma_load_2d_pair(a_dst, &tmA, fbar, kb * kKbElems, arow);
                    } else {
                        tma_load_2d_pair(a_dst, &tmA, fbar, arow, kb * 64);
                        tma_load_2d_pair(a_dst + 8192, &tmA, fbar, arow + 64, kb * 64);
                    }
                    if constexpr (!kBMN) {
                        tma_load_2d_pair(b_dst, &tmB, fbar, kb * kKbElems, brow);
                    } else {
                        tma_load_2d_pair(b_dst, &tmB, fbar, brow, kb * 64);
                        tma_load_2d_pair(b_dst + 8192, &tmB, fbar, brow + 64, kb * 64);
                    }
                    if (++s == kTc2Stages) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok && leader) {
                // the leader's full barriers count both CTAs' loads: wait (briefly) for them
                for (int i = 0; i < kTc2Stages; ++i) {
                    int ss = (s - 1 - i + 2 * kTc2Stages) % kTc2Stages;
                    uint32_t pp = (s - 1 - i < 0) ? (ph ^ 1u) : ph;
                    mbar_wait(&full[ss], pp, 100000000ull, nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA issuer (leader)
        if (leader && elect_one()) {
            int s = 0;
            uint32_t ph = 0;
            int tcount = 0;
            bool ok = true;
            for (int u = pair; u < plan.num_units && ok; u += npairs, ++tcount) {
                const int b = tcount & 1;
                const uint32_t tph = (tcount >> 1) & 1;
                const uint32_t idesc = u < plan.full_units ? kIdesc : kIdescHalf;
                if (!mbar_wait(&tempty[b], tph ^ 1u, lim, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kBN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(&full[s], ph, lim, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * kTc2HalfBytes);
                    const uint32_t b_base = smem_u32(sB + s * kTc2HalfBytes);
#pragma unroll
                    for (int kk = 0; kk < kInstrK; ++kk) {
                        uint64_t adesc, bdesc;
                        if constexpr (!kAMN) adesc = umma_desc_sw128(a_base + kk * 32, 16, 1024);
                        else adesc = umma_desc_sw128(a_base + kk * 2048, 8192, 1024);
                        if constexpr (!kBMN) bdesc = umma_desc_sw128(b_base + kk * 32, 16, 1024);
                        else bdesc = umma_desc_sw128(b_base + kk * 2048, 8192, 1024);
                        tc_mma_pair<kInt8>(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit_pair(&empty[s], 0x3);
                    if (++s == kTc2Stages) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(&tfull[b], 0x3);
            }
            if (!ok) {
                tc_commit_pair(&tfull[tcount & 1], 0x3);
                mbar_wait(&tfull[tcount & 1], ((tcount >> 1) & 1), 100000000ull, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;
        uint8_t* ebuf = sE + (warp - 2) * 2 * kEpiBufBytes;
        int buf = 0;
        int tcount = 0;
        float gm = 1.0f;
        if constexpr (kEpi != kEpiF32 && !epi_is_col(kEpi)) gm = __ldg(args.gamma);
        for (int u = pair; u < plan.num_units; u += npairs, ++tcount) {
            const int b = tcount & 1;
            const uint32_t tph = (tcount >> 1) & 1;
            if (!mbar_wait_warp(&tfull[b], tph, lim, abort_flag)) break;
            tc_fence_after();
            int mb, nb, half;
            tc2_unit(u, plan, args.m_tiles, args.n_tiles, mb, nb, half);
            const int ucols = half < 0 ? kBN : kBN / 2;             // accumulator columns of the unit
            const int col_base = nb * kBN + (half < 0 ? 0 : half * (kBN / 2));
            const int row0 = mb * 256 + static_cast<int>(rank) * 128 + quad * 32;
            const int row = row0 + lane;
            const bool row_ok = row < args.M;
            float cs = 1.0f;
            float cr = 1.0f;   // col epilogues: fl(1 / s_t)
            if constexpr (epi_is_col(kEpi)) {
                cs = row_ok ? __ldg(args.row_scale + row) : 1.0f;   // s_t
                cr = __frcp_rn(cs);
            }
            else if constexpr (epi_is_linear(kEpi)) cs = row_ok ? __fdiv_rn(gm, __ldg(args.row_scale + row)) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(b * kBN);
#pragma unroll 1
            for (int c0 = 0; c0 < ucols; c0 += kChunkCols) {
                const int col0 = col_base + c0;
                if (col0 >= args.N) break;                     // warp-uniform
                uint32_t ra[32], rb[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + c0, ra);
                if constexpr (kChunkCols == 64) {
                    tmem_ld_32x32b_x32(t_row + c0 + 32, rb);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rb[i] = 0u;
                }
                tmem_ld_wait();
                auto r = [&](int i) -> uint32_t { return i < 32 ? ra[i] : rb[i - 32]; };
                // the factor of chunk column i: gamma / s_t, or fl(gamma_n / s_t) per column
                // (correctly rounded from the row's reciprocal with two FMA corrections)
                auto fac = [&](int i) -> float {
                    if constexpr (epi_is_col(kEpi)) {
                        const int c = col0 + i < args.N ? col0 + i : args.N - 1;
                        return row_ok ? div_by_scale(__ldg(args.gamma + c), cs, cr) : 0.0f;
                    } else {
                        return cs;
                    }
                };
                uint4 v[8];
                if constexpr (epi_is_bf16(kEpi)) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float lo = __fmul_rn(static_cast<float>(static_cast<int32_t>(r(8 * j + 2 * e))), fac(8 * j + 2 * e));
                            const float hi = __fmul_rn(static_cast<float>(static_cast<int32_t>(r(8 * j + 2 * e + 1))), fac(8 * j + 2 * e + 1));
                            w[e] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
                        }
                        v[j] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float f[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t raw = r(4 * j + e);
                            if constexpr (kEpi == kEpiLinearF32 || kEpi == kEpiLinearColF32)
                                f[e] = __fmul_rn(static_cast<float>(static_cast<int32_t>(raw)), fac(4 * j + e));
                            else if constexpr (kEpi == kEpiScaleF32)
                                f[e] = __fmul_rn(gm, __uint_as_float(raw));
                            else
                                f[e] = __uint_as_float(raw);
                        }
                        v[j] = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                                          __float_as_uint(f[3]));
                    }
                }
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
                uint8_t* sb = ebuf + buf * kEpiBufBytes;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4*>(sb + lane * 128 + ((j ^ (lane & 7)) << 4)) = v[j];
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmD, sb, col0, row0);
                    bulk_commit_group();
                }
                buf ^= 1;
                if constexpr (epi_is_linear(kEpi)) {
                    if (args.acc_out != nullptr && row_ok) {
                        int32_t* dst = args.acc_out + static_cast<int64_t>(row) * args.N + col0;
#pragma unroll
                        for (int j = 0; j < kChunkCols / 4; ++j)
                            if (col0 + 4 * j < args.N)
                                reinterpret_cast<int4*>(dst)[j] = make_int4((int)r(4 * j), (int)r(4 * j + 1),
                                                                            (int)r(4 * j + 2), (int)r(4 * j + 3));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[b]), 0));
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync_all();   // both CTAs done with TMEM, with their barriers and with remote arrivals
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace bl

// gemm_packed2.cuh -- int8 x packed-ternary linear on CTA pairs (tcgen05.mma.cta_group::2 with
// the weight operand in tensor memory): 17 or more tokens, or fewer when their activation rows
// do not fit the decode GEMV's shared memory.
//
// P3 §3.1's linear on the 2-bit codes of P5 §4.1 / §5.1:
//   D[n, t] = sum_k W_q[n, k] x_q[t, k],   y[t, n] = fl(D * fl(gamma / s_t)),
// with the weight rows as the MMA's M dimension.  A cluster of two CTAs computes a tile of 256
// weight rows x bt tokens (bt = 32 ... 256) with one 2-SM instruction per 32 codes of K.
//
// The decoded weight never touches shared memory: each decoder thread owns one weight row,
// decodes the row's 128 codes of a k-block in registers and writes them with tcgen05.st into
// its CTA's tensor memory (lane = row, 4 codes per 32-bit column), where the MMA reads its A
// operand.  That saves the 2 bytes of shared-memory traffic per code of a staged int8 tile,
// and an M = 256 instruction with A in TMEM measured faster than with A in shared memory in
// the same issue loop (26.8 / 41 / 73 / 137 against 58.5 / 72.9 / 103.6 / 167.6 cycles at
// N = 32 / 64 / 128 / 256); issued without per-instruction overhead it runs at the full int8
// rate (16 / 32 cycles at N = 32 / 64).
//
// Per CTA r of a pair (rows [256 u + 128 r, +128) of weight tile u), 736 threads.  A "stage"
// of the activation and decoded-weight rings is two k-blocks (256 codes of K); a packed stage
// is four k-blocks.
//   warp 0     packed producer: TMA loads of the CTA's 128 rows' packed codes (512 codes per
//              row per stage, 128-byte swizzle) into its packed ring (its own barriers);
//   warp 22    activation producer: TMA loads of the CTA's half of the token tile (bt / 2 rows x
//              128 bytes per k-block) with the 2-SM TMA form, whose completion bytes count on the
//              leader's barrier of the stage -- the same barrier the decoders arrive on, so the
//              MMA issuer waits once and commits once per stage;
//   warps 6-21 decoders, four groups of four warps (one per TMEM lane quarter): group g decodes
//              the stages q = g mod 4 into its TMEM stage (64 columns): each thread owns one
//              weight row, decodes the row's codes in registers and writes them with tcgen05.st;
//              then tcgen05.wait::st, fence, and one arrival per warp on the LEADER's barrier of
//              that stage (9 arrivals: the group in both CTAs and the leader's activation
//              producer);
//   warp 1     leader only: one thread issues tcgen05.mma.cta_group::2.kind::i8 (eight per stage)
//              with A from both CTAs' TMEM stage and B from both CTAs' activation halves; its
//              commit frees the stage in both CTAs (TMEM and activation tile), after a unit's
//              last stage another arrives on both CTAs' accumulator-full barriers, and after
//              the pair's last unit a third arrives on a barrier used once;
//   warps 2-5  epilogue (both CTAs): TMEM lanes are the CTA's 128 weight rows; the unit's token
//              factors fl(gamma / s_t) are read before its accumulators are ready; per 32-token
//              chunk tcgen05.ld, y[t, n] = fl(acc * fl(gamma / s_t)) staged in shared memory as a
//              [token][row] tile and written with one TMA store (or the exact int32 partial sums
//              of K split sp into slice sp of a workspace, which pk_finalize_kernel adds in split
//              order); one arrival per warp on the leader's accumulator-empty barrier.  For the
//              pair's last unit the decoder warps, idle by then, take four of every five chunks;
//              they wait on the once-used barrier (they can run ahead of the accumulator-full
//              phases, where a parity wait would take an earlier unit's phase for the last's).
// The single-thread MMA loop's barrier waits (about 130 cycles each, measured, even on a completed
// phase) and commits cost about as much as the MMAs themselves at these widths: two k-blocks per
// stage and one barrier per stage keep them to one wait and one commit per 8 MMAs.
// TMEM (512 columns per CTA): accumulators in columns [0, 256) -- two 128-column buffers when
// bt <= 128 (a unit's epilogue overlaps the next unit's k-loop), one 256-column buffer
// otherwise -- and the decoded-weight ring (4 stages x 64 columns) in [256, 512).  Work units
// (weight tile, token tile, K split) are taken persistently, pair index + j * pairs.  Every wait
// is bounded; on a timeout each role unwinds as in the 2-SM GEMM.  No TMA load uses multicast.
#pragma once
#include "common.cuh"
#include "gemm_packed.cuh"

namespace bl {

constexpr int kPk2Rows = 128;          // weight rows per CTA (a pair tile: 256)
constexpr int kPk2Threads = kPkThreads + 32;   // + the activation producer warp
constexpr int kPk2DStages = 4;         // stages in flight: decoded weights in TMEM (one per decoder
                                       // group) and activation tiles in shared memory
constexpr int kPk2KbPerStage = 2;      // k-blocks per activation / decoded stage
constexpr uint32_t kPk2ACol = 256;     // first TMEM column of the decoded-weight ring
constexpr uint32_t kPk2StageCols = 64; // 256 int8 codes per row = 64 columns

constexpr uint32_t kPk2EpiBuf = 32 * 32 * 4;   // one 32-token x 32-row tile of 4-byte values
constexpr uint32_t kPk2EpiBytes = 4 * 2 * kPk2EpiBuf;   // two staging tiles per epilogue warp
constexpr int kPk2EpiHelpers = 5;      // warps per TMEM quarter sharing a pair's last epilogue:
                                       // its epilogue warp and its four decoder warps

__host__ __device__ inline size_t pk2_smem_bytes(int bt, int pstages) {
    return 1024 + static_cast<size_t>(pstages) * kPkPBytes + static_cast<size_t>(kPk2DStages) * static_cast<size_t>(bt) * 128 +
           kPk2EpiBytes + (2 * kPkMaxPStages + 2 * kPk2DStages + 5) * sizeof(uint64_t) + 16;
}

// TMA load of one 2-D box with an L2 evict-first policy: the packed weight is read once per
// launch, so it should not displace the activations (read by every weight tile) from L2.
__device__ __forceinline__ void tma_load_2d_evict_first(void* smem_dst, const void* desc, uint64_t* bar, int32_t x,
                                                        int32_t y) {
    asm volatile(
        "{\n\t.reg .b64 pol;\n\t"
        "createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n\t"
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], pol;\n\t}" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(desc)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// L2 prefetch of one 2-D box of a tensor map (no data returns to the SM, so it may run before
// the launch's dependency wait: L2 is the point of coherence for the previous kernel's writes).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* desc, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(desc)),
                 "r"(x), "r"(y)
                 : "memory");
}

// Arrive on a barrier of either CTA of the pair (address in the cluster window) with the
// default release at CTA scope; the waiter uses the default CTA-scope acquire.  The data the
// arrival publishes is decoded weights in TMEM, ordered by tcgen05 fences, or the release of
// accumulators read from TMEM -- not shared memory.  Measured on B200, an arrival with release at
// cluster scope cost 800-2500 cycles and a wait with acquire at cluster scope about 100 cycles,
// on the path of every stage.
__device__ __forceinline__ void pk2_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes from 32 registers per thread.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMA store (shared -> global) of one 3-D box; completion tracked with bulk groups.
__device__ __forceinline__ void tma_store_3d(const void* desc, const void* smem_src, int32_t x, int32_t y, int32_t z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(desc)),
                 "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T on the CTA pair (A: each CTA's 128 rows in its own TMEM).
__device__ __forceinline__ void tc_mma_pair_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "setp.ne.b32 P, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, P;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The eight MMAs of a full stage (two k-blocks x four 32-code steps) in one asm block.  A: 8
// TMEM columns per step from `a`.  B: the shared-memory descriptors b0 and b1 of the stage's
// two activation k-blocks, 32 bytes (2 in the descriptor's start-address field, which cannot
// carry: addresses stay below 256 KB) per step.  The first MMA accumulates iff `accumulate`,
// the other seven always.  One predicate set-up per stage instead of per MMA: measured on B200,
// a single thread issuing MMAs one C++ call at a time needed ~50 cycles per N = 64 instruction,
// which the tensor pipe runs in 32.
__device__ __forceinline__ void pk2_mma_stage(uint32_t d_tmem, uint32_t a, uint64_t b0, uint64_t b1, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred P, Q;\n\t.reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t.reg .b64 c1, c2, c3, c5, c6, c7;\n\t"
        "setp.ne.b32 P, %5, 0;\n\t"
        "setp.eq.b32 Q, %5, %5;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\tadd.u32 a4, %1, 32;\n\t"
        "add.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\tadd.u32 a7, %1, 56;\n\t"
        "add.s64 c1, %2, 2;\n\tadd.s64 c2, %2, 4;\n\tadd.s64 c3, %2, 6;\n\t"
        "add.s64 c5, %3, 2;\n\tadd.s64 c6, %3, 4;\n\tadd.s64 c7, %3, 6;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %4, P;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a1], c1, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a2], c2, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a3], c3, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a4], %3, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a5], c5, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a6], c6, %4, Q;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [a7], c7, %4, Q;\n\t}" ::"r"(d_tmem),
        "r"(a), "l"(b0), "l"(b1), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct Pk2Args {
    PkArgs pk;        // shapes, outputs, pstages; pk.bt is the pair tile's token count
};

template <bool kBf16Out>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPk2Threads, 1)
    tc_gemm_packed2_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmAcc,
                           const Pk2Args a2) {
    const PkArgs& args = a2.pk;
    constexpr int DS = kPk2DStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int PS = args.pstages;
    const int bt = args.bt;                                            // multiple of 32
    const int nacc = bt <= 128 ? 2 : 1;                                // accumulator buffers
    const uint32_t xh_bytes = static_cast<uint32_t>(bt) * 64u;         // one k-block: bt / 2 rows x 128 bytes
    // [packed: PS x 16 KB][activation halves: DS x 2 k-blocks x xh_bytes][epilogue staging]; 1024-aligned
    auto sP = [&](int p) { return smem + p * kPkPBytes; };
    uint8_t* sXbase = smem + PS * kPkPBytes;
    auto sX = [&](int x) { return sXbase + static_cast<uint32_t>(x) * (kPk2KbPerStage * xh_bytes); };
    uint8_t* sE = sXbase + static_cast<uint32_t>(DS) * (kPk2KbPerStage * xh_bytes);
    uint64_t* pfull = reinterpret_cast<uint64_t*>(sE + kPk2EpiBytes);
    uint64_t* pempty = pfull + kPkMaxPStages;    // this CTA's 16 decoder warps
    // stage d: dfull[d] (the leader's is used) completes when the group of d in both CTAs has
    // arrived (8 warps), the leader's activation producer has arrived with the stage's byte
    // count, and both CTAs' activation halves have landed; dempty[d] (each CTA) is the leader's
    // commit after the stage's MMAs (frees the TMEM stage and the activation stage)
    uint64_t* dfull = pempty + kPkMaxPStages;
    uint64_t* dempty = dfull + DS;
    uint64_t* tfull = dempty + DS;               // each CTA: the leader's commit after a unit
    uint64_t* tempty = tfull + 2;                // leader's is used: 4 epilogue warps per CTA
    // each CTA, used once: the leader's commit after the pair's last unit.  The decoder warps
    // wait on it, not on tfull: they may reach the last unit while a unit two or more commits
    // earlier is still open, and a parity wait cannot tell that phase from the one it wants.
    uint64_t* tlast = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tlast + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    if (threadIdx.x == 0) {
        for (int p = 0; p < PS; ++p) {
            mbar_init(&pfull[p], 1);
            mbar_init(&pempty[p], 4 * kPkDecGroups);
        }
        for (int d = 0; d < DS; ++d) {
            mbar_init(&dfull[d], 9);
            mbar_init(&dempty[d], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(tlast, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmP);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers initialised and TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    if (warp == 0 && lane == 0) {
        // the first unit's first packed stages into L2 while the previous kernel finishes
        // (its k-blocks [0, k_blocks / splits): the split index is 0 or the unit's own)
        const int nt = (pair / args.splits) / args.t_tiles;
        const int sp = pair % args.splits;
        const int kb0 = sp * args.k_blocks / args.splits;
        const int kb1 = (sp + 1) * args.k_blocks / args.splits;
        const int prow = nt * 2 * kPk2Rows + static_cast<int>(rank) * kPk2Rows;
        for (int i = 0, kb = kb0; i < PS && kb < kb1; ++i, kb += kPkKbPerP) tma_prefetch_l2_2d(&tmP, kb * 32, prow);
    }
    pdl_trigger_and_wait();

    const int units = args.n_tiles * args.t_tiles * args.splits;
    const uint64_t lim = args.wait_ns;
    // unit u -> (pair weight tile nt, token tile tt, K split sp) and its k-block range (32-bit
    // arithmetic: k_blocks < 2^24 and splits <= 8; a 64-bit division is a called routine whose
    // first, cold fetch measured 0.7 us at the start of every role)
    const int splits = args.splits, t_tiles = args.t_tiles, k_blocks = args.k_blocks;
    auto unit_of = [&](int u, int& nt, int& tt, int& kb0, int& kb1) {
        const int sp = splits == 1 ? 0 : u % splits;
        const int rest = splits == 1 ? u : u / splits;
        tt = t_tiles == 1 ? 0 : rest % t_tiles;
        nt = t_tiles == 1 ? rest : rest / t_tiles;
        kb0 = splits == 1 ? 0 : sp * k_blocks / splits;
        kb1 = splits == 1 ? k_blocks : (sp + 1) * k_blocks / splits;
    };
    // a bounded wait for the loads issued last, before the pair exits after a timeout
    auto drain = [&](uint64_t* full, int n_stages, int next, uint32_t ph, int issued) {
        for (int i = 0; i < n_stages && i < issued; ++i) {
            const int s = (next - 1 - i + 2 * n_stages) % n_stages;
            mbar_wait(&full[s], (next - 1 - i < 0) ? (ph ^ 1u) : ph, 100000000ull, nullptr);
        }
    };
    // ---- epilogue pieces: the epilogue warps run them for every unit; for the pair's last unit
    // the decoder warps take a share of the chunks (see the decoder role)
    // staging slots: four 2-byte tiles (bf16 Y alone) or two 4-byte tiles (f32 Y, int32 sums)
    const bool small_tiles = kBf16Out && args.splits == 1 && args.acc == nullptr;
    const uint32_t slot_bytes = small_tiles ? kPk2EpiBuf / 2 : kPk2EpiBuf;
    const int nslots = small_tiles ? 4 : 2;
    // fl(gamma / s_t) of token t (0 for the K-split partial sums, which are scaled later)
    auto token_factor = [&](float gm, int t) -> float {
        return (args.splits == 1 && t < args.T) ? __fdiv_rn(gm, __ldg(args.sx + t)) : 0.0f;
    };
    // chunk i of unit u: this warp's 32 TMEM lanes (weight rows) x 32 tokens, staged in shared
    // memory as [token][row] and written with one TMA store (rows beyond N and tokens beyond T are
    // clipped by the tensor map); cl = the factor of token t0 + 32 i + lane
    auto epi_chunk = [&](int u, int nt, int t0, uint32_t t_row, int i, float cl, uint8_t* ebuf, int& ebi) {
        const int c0 = 32 * i;
        const int n0 = nt * 2 * kPk2Rows + static_cast<int>(rank) * kPk2Rows + (warp & 3) * 32;
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row + c0, r);
        tmem_ld_wait();
        auto stage = [&]() -> uint8_t* {
            uint8_t* e = ebuf + ebi * slot_bytes;
            ebi = ebi + 1 == nslots ? 0 : ebi + 1;
            // the slot's previous store has read it
            if (lane == 0) {
                if (nslots == 4) bulk_wait_group_read<3>();
                else bulk_wait_group_read<1>();
            }
            __syncwarp();
            return e;
        };
        auto flush = [&](const CUtensorMap* tm, const uint8_t* e, bool three_d, int z) {
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) {
                if (three_d) tma_store_3d(tm, e, n0, t0 + c0, z);
                else tma_store_2d(tm, e, n0, t0 + c0);
                bulk_commit_group();
            }
        };
        if (args.splits > 1 || args.acc != nullptr) {
            uint8_t* e = stage();
#pragma unroll
            for (int j = 0; j < 32; ++j) reinterpret_cast<uint32_t*>(e + j * 128)[lane] = r[j];
            flush(&tmAcc, e, args.splits > 1, u % args.splits);
            if (args.splits > 1) return;
        }
        uint8_t* e = stage();
        if constexpr (kBf16Out) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                reinterpret_cast<uint16_t*>(e + j * 64)[lane] = float_to_bf16_bits(
                    __fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), __shfl_sync(0xffffffffu, cl, j)));
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                reinterpret_cast<float*>(e + j * 128)[lane] =
                    __fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), __shfl_sync(0xffffffffu, cl, j));
        }
        flush(&tmY, e, false, 0);
    };

    if (warp == 0) {
        // ----------------------------------------------------------------- packed producer (both CTAs)
        if (elect_one()) {
            int p = 0, issued = 0;
            uint32_t pph = 0;
            bool ok = true;
            for (int u = pair; u < units && ok; u += npairs) {
                int nt, tt, kb0, kb1;
                unit_of(u, nt, tt, kb0, kb1);
                const int prow = nt * 2 * kPk2Rows + static_cast<int>(rank) * kPk2Rows;
                for (int kb = kb0; kb < kb1; kb += kPkKbPerP) {
                    // the CTA's next packed stage: k-blocks kb .. kb + 3 of its 128 rows
                    if (!mbar_wait(&pempty[p], pph ^ 1u, lim, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&pfull[p], static_cast<uint32_t>(kPkPBytes));
                    tma_load_2d_evict_first(sP(p), &tmP, &pfull[p], kb * 32, prow);
                    ++issued;
                    if (++p == PS) { p = 0; pph ^= 1u; }
                }
            }
            if (!ok) drain(pfull, PS, p, pph, issued);
        }
        __syncwarp();
    } else if (warp == kPk2Threads / 32 - 1) {
        // ----------------------------------------------------------------- activation producer (both CTAs)
        if (elect_one()) {
            int d = 0;
            uint32_t dph = 0;
            bool ok = true;
            for (int u = pair; u < units && ok; u += npairs) {
                int nt, tt, kb0, kb1;
                unit_of(u, nt, tt, kb0, kb1);
                const int trow = tt * bt + static_cast<int>(rank) * (bt / 2);
                for (int kb = kb0; kb < kb1; kb += kPk2KbPerStage) {
                    const int nkb = min(kPk2KbPerStage, kb1 - kb);
                    // the stage's previous MMAs are done in both CTAs; the leader's barrier is in
                    // this stage's phase
                    if (!mbar_wait(&dempty[d], dph ^ 1u, lim, abort_flag)) { ok = false; break; }
                    if (leader) mbar_arrive_expect_tx(&dfull[d], 2u * static_cast<uint32_t>(nkb) * xh_bytes);
                    const uint32_t bar = mapa_shared(smem_u32(&dfull[d]), 0);
                    for (int j = 0; j < nkb; ++j)
                        tma_load_2d_pair(sX(d) + j * xh_bytes, &tmX, bar, (kb + j) * 128, trow);
                    if (++d == DS) { d = 0; dph ^= 1u; }
                }
            }
            // the loads issued last complete on a barrier that also waits for decoder arrivals:
            // after a timeout, give them time to land before the pair exits
            if (!ok) {
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 50000ull) __nanosleep(1000);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ----------------------------------------------------------------- decoders (both CTAs)
        const int grp = (warp - 6) >> 2;                // decodes stage sequence numbers q = grp mod 4
        const int row = 32 * (warp & 3) + lane;         // this thread's weight row = its TMEM lane
        const int sw = row & 7;                         // 128-byte swizzle of the packed row
        const uint32_t t_st = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + kPk2ACol +
                              static_cast<uint32_t>(grp) * kPk2StageCols;
        const uint32_t dfull_leader = mapa_shared(smem_u32(&dfull[grp]), 0);
        int p = 0;
        uint32_t pph = 0, dph = 0;
        int q = 0;                                      // stage sequence number
        bool ok = true;
        for (int u = pair; u < units && ok; u += npairs) {
            int nt, tt, kb0, kb1;
            unit_of(u, nt, tt, kb0, kb1);
            for (int kb = kb0; kb < kb1 && ok; kb += kPkKbPerP) {
                if (!mbar_wait_warp(&pfull[p], pph, lim, abort_flag)) { ok = false; break; }
                const uint8_t* src = sP(p) + row * 128;
                for (int h = 0; h < kPkKbPerP / kPk2KbPerStage; ++h) {
                    const int ks = kb + h * kPk2KbPerStage;
                    if (ks >= kb1) break;
                    if ((q & (kPkDecGroups - 1)) == grp) {
                        const int nkb = min(kPk2KbPerStage, kb1 - ks);
                        // the MMA has finished reading this stage in both CTAs (its previous use)
                        if (!mbar_wait_warp(&dempty[grp], dph ^ 1u, lim, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        for (int j = 0; j < nkb; ++j) {
                            // k-block 2 h + j of the packed stage: the row's 16-byte chunks 2 jj, 2 jj + 1
                            const int jj = h * kPk2KbPerStage + j;
                            const uint4 w0 = *reinterpret_cast<const uint4*>(src + (((2 * jj) ^ sw) << 4));
                            const uint4 w1 = *reinterpret_cast<const uint4*>(src + (((2 * jj + 1) ^ sw) << 4));
                            const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                            uint32_t v[32];
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const uint4 d = pk_decode_word(w[i]);   // codes 16 i .. 16 i + 15
                                v[4 * i] = d.x;
                                v[4 * i + 1] = d.y;
                                v[4 * i + 2] = d.z;
                                v[4 * i + 3] = d.w;
                            }
                            tmem_st_32x32b_x32(t_st + static_cast<uint32_t>(j) * 32u, v);
                        }
                        tmem_st_wait();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) pk2_arrive_remote(dfull_leader);
                        dph ^= 1u;
                    }
                    ++q;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&pempty[p]);
                if (++p == PS) { p = 0; pph ^= 1u; }
            }
        }
        // the pair's last unit: this warp takes epilogue chunks 1 + grp and 1 + grp + 5 of its TMEM
        // quarter (the quarter's epilogue warp takes chunks 0 and 5).  Its staging tiles lie in the
        // packed and activation rings, whose last loads have been consumed once the unit's
        // accumulators are complete.
        if (ok && pair < units) {
            const int last = (units - 1 - pair) / npairs;       // the unit's index among the pair's
            const int u = pair + last * npairs;
            int nt, tt, kb0, kb1;
            unit_of(u, nt, tt, kb0, kb1);
            const int t0 = tt * bt;
            const int i0 = 1 + grp, i1 = 1 + grp + kPk2EpiHelpers;
            if (32 * i0 < bt && t0 + 32 * i0 < args.T) {
                const float gm = __ldg(args.gamma);
                const float cl0 = token_factor(gm, t0 + 32 * i0 + lane);
                const float cl1 = 32 * i1 < bt ? token_factor(gm, t0 + 32 * i1 + lane) : 0.0f;
                const int b = last % nacc;
                if (mbar_wait_warp(tlast, 0, lim, abort_flag)) {
                    tc_fence_after();
                    uint8_t* hbuf = smem + (warp - 6) * 2 * kPk2EpiBuf;
                    int hbi = 0;
                    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * (warp & 3)) << 16) +
                                           static_cast<uint32_t>(b * 128);
                    epi_chunk(u, nt, t0, t_row, i0, cl0, hbuf, hbi);
                    if (32 * i1 < bt && t0 + 32 * i1 < args.T) epi_chunk(u, nt, t0, t_row, i1, cl1, hbuf, hbi);
                    if (lane == 0) bulk_wait_group<0>();
                    __syncwarp();
                }
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA issuer (leader)
        if (leader && elect_one()) {
            const uint32_t idesc = umma_idesc(true, false, false, 2 * kPk2Rows, bt);
            // B descriptors: stage d's first k-block at x_desc0 + d * x_stage16, its second
            // xh16 further (descriptor start addresses count 16-byte units)
            const uint64_t x_desc0 = umma_desc_sw128(smem_u32(sXbase), 16, 1024);
            const uint64_t x_stage16 = static_cast<uint64_t>((kPk2KbPerStage * xh_bytes) >> 4);
            const uint64_t xh16 = static_cast<uint64_t>(xh_bytes >> 4);
            int d = 0;
            uint32_t dph = 0;
            int tcount = 0;
            bool ok = true;
            for (int u = pair; u < units && ok; u += npairs, ++tcount) {
                int nt, tt, kb0, kb1;
                unit_of(u, nt, tt, kb0, kb1);
                const int b = tcount % nacc;
                const uint32_t tph = (tcount / nacc) & 1;
                if (!mbar_wait(&tempty[b], tph ^ 1u, lim, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * 128);
                for (int kb = kb0; kb < kb1; kb += kPk2KbPerStage) {
                    const int nkb = min(kPk2KbPerStage, kb1 - kb);
                    // both CTAs' decoded weights and activation halves
                    if (!mbar_wait(&dfull[d], dph, lim, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem_base + kPk2ACol + static_cast<uint32_t>(d) * kPk2StageCols;
                    const uint64_t b0 = x_desc0 + static_cast<uint64_t>(d) * x_stage16;
                    if (nkb == kPk2KbPerStage) {
                        pk2_mma_stage(d_tmem, a_tmem, b0, b0 + xh16, idesc, kb != kb0 ? 1u : 0u);
                    } else {   // a unit's last, single k-block
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_pair_i8_ts(d_tmem, a_tmem + kk * 8, b0 + static_cast<uint64_t>(2 * kk), idesc,
                                              (kb != kb0 || kk != 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&dempty[d], 0x3);
                    if (++d == DS) { d = 0; dph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(&tfull[b], 0x3);
            }
            // completes when every MMA of the pair is done (after a timeout too, so that the
            // bounded wait below outlasts the MMAs in flight before TMEM is freed)
            tc_commit_pair(tlast, 0x3);
            if (!ok) {
                tc_commit_pair(&tfull[tcount % nacc], 0x3);   // releases the epilogue warps
                mbar_wait(tlast, 0, 100000000ull, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;                 // TMEM lanes [32 quad, 32 quad + 32)
        const float gm = __ldg(args.gamma);
        uint8_t* ebuf = sE + (warp - 2) * 2 * kPk2EpiBuf;
        int ebi = 0;
        int tcount = 0;
        for (int u = pair; u < units; u += npairs, ++tcount) {
            int nt, tt, kb0, kb1;
            unit_of(u, nt, tt, kb0, kb1);
            const int b = tcount % nacc;
            const uint32_t tph = (tcount / nacc) & 1;
            const int t0 = tt * bt;
            // the pair's last unit: chunks i = 0 mod kPk2EpiHelpers here, the rest in the decoders
            const int step = u + npairs >= units ? kPk2EpiHelpers : 1;
            // lane l holds the factor of token t0 + 32 i + l, read before the accumulators are ready
            float fac[kPkMaxBT / 32];
#pragma unroll
            for (int i = 0; i < kPkMaxBT / 32; ++i)
                fac[i] = (32 * i < bt && i % step == 0) ? token_factor(gm, t0 + 32 * i + lane) : 0.0f;
            if (!mbar_wait_warp(&tfull[b], tph, lim, abort_flag)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(b * 128);
#pragma unroll 1
            for (int i = 0; i < kPkMaxBT / 32; i += step) {
                if (32 * i >= bt || t0 + 32 * i >= args.T) break;      // warp-uniform
                float cl = fac[0];
#pragma unroll
                for (int k = 1; k < kPkMaxBT / 32; ++k)
                    if (i == k) cl = fac[k];
                epi_chunk(u, nt, t0, t_row, i, cl, ebuf, ebi);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) pk2_arrive_remote(mapa_shared(smem_u32(&tempty[b]), 0));
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync_all();   // both CTAs done with TMEM, with their barriers and with remote arrivals
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}
}  // namespace bl

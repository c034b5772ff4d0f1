// gemm_packed.cuh -- int8 x packed-ternary tcgen05 GEMM for few tokens (prefill chunks and
// batched decode), reading the weight as its 2-bit codes.
//
// Restates the linear of P3 §3.1 (y = F.linear(x_q, W_q) * gamma / s_t) on the packed
// weight of P5 §4.1 (00 -> 0, 01 -> +1, 10 -> -1, 11 reserved -> 0) / §5.1: the weight
// bytes that cross HBM are a quarter of the int8 codes', which is what bounds a GEMM with
// few tokens.
//
// Operand roles are swapped so that the weight rows fill the 128-row tensor-core tile:
//   D[n, t] = sum_k W_q[n, k] x_q[t, k]     (UMMA M = 128 weight rows, N = bt tokens)
// so a batch of 16 tokens costs a 16-column MMA instead of a 128-row one.
//
// Warp roles (704 threads, one CTA per SM, persistent over work units), three rings:
//   packed ring (128 rows x 128 bytes = 512 codes per row per stage, 128-byte swizzle) and
//              activation ring (bt x 128-byte tiles per 128-code k-block, 4 stages in step with
//              the decoded ring): warp 0 keeps both full with TMA loads.  A packed box moves 128 bytes per
//              weight row: with 32-byte rows the copy engine's per-row rate, not HBM, was the
//              limit (measured);
//   decoded ring (DS = 4 or 8 stages of 128 rows x 128 int8 codes, 128-byte-swizzled
//              K-major): warps 6-21, four groups of four warps, group g decoding the k-blocks
//              q = g mod 4 into stage q mod DS (stage g, or stages g and g + 4 in turn), one
//              k-block of a packed stage into the int8 layout the MMA reads (what TMA would
//              have written for int8 codes), fence the writes to the async proxy and arrive;
//   warp 1     MMA issuer (tcgen05.mma kind::i8, one thread), accumulators in TMEM
//              (two 256-column buffers: the epilogue of one unit overlaps the next);
//   warps 2-5  epilogue: tcgen05.ld, then y[t, n] = fl(acc * fl(gamma / s_t)) (warp-wide
//              coalesced stores along n; each lane forms one token's factor and the warp
//              shares them by shuffle), or -- when K is split across units -- the exact int32
//              partial sums of split sp stored to slice sp of a workspace, which
//              pk_finalize_kernel adds in split order (exact) before the same epilogue.
// Every decoder warp waits on every packed stage and arrives on its empty barrier (16
// arrivals); each decoded stage is served by one group, which keeps one phase bit per stage
// it serves, so each barrier's phases are waited on strictly in order by each waiter (a
// parity wait cannot confuse a phase with the one two phases earlier); the producer and the
// MMA issuer walk all rings in order.
// Decode of one 32-bit word (16 codes): with a byte table TAB = {0, +1, -1, 0}, a byte
// permute whose selector nibbles are the codes looks all of them up at once:
//   even = prmt(TAB, sel = w & 0x33333333), odd = prmt(TAB, sel = (w >> 2) & 0x33333333)
// (and their upper halves), then two permutes interleave even and odd codes -- 13 integer
// operations per 16 codes.
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kPkDecGroups = 4;              // decoder groups of 4 warps
constexpr int kPkThreads = 192 + kPkDecGroups * 128;
constexpr int kPkBM = 128;                    // weight rows per tile (UMMA M)
constexpr int kPkMaxBT = 256;                 // tokens per tile (UMMA N)
constexpr int kPkMaxDStages = 2 * kPkDecGroups;   // decoded ring depth: 4 or 8 (one or two stages per group);
                                                // the activation ring moves in step with it, so one
                                                // commit per k-block frees both
constexpr int kPkMaxPStages = 12;             // packed ring depth
constexpr int kPkKbPerP = 4;                  // 128-code k-blocks per packed stage
constexpr int kPkABytes = kPkBM * 128;        // decoded weight tile per stage (int8, SW128 K-major)
constexpr int kPkPBytes = kPkBM * 128;        // packed weight tile per stage (512 codes per row)
constexpr uint32_t kPkTab = 0x00FF0100u;      // byte c = int8 value of code c

struct PkArgs {
    int T, N, K;
    int bt;                        // tokens per tile: multiple of 16, <= 256
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

__host__ __device__ inline size_t pk_smem_bytes(int bt, int pstages, int dstages) {
    return 1024 + static_cast<size_t>(dstages) * kPkABytes + static_cast<size_t>(dstages) * bt * 128 +
           static_cast<size_t>(pstages) * kPkPBytes + (2 * kPkMaxPStages + 3 * kPkMaxDStages + 4) * sizeof(uint64_t) + 16;
}

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

template <bool kBf16Out, int DS>
__global__ void __launch_bounds__(kPkThreads, 1)
    tc_gemm_packed_kernel(const __grid_constant__ CUtensorMap tmP, const __grid_constant__ CUtensorMap tmX,
                          const PkArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    static_assert(DS == kPkDecGroups || DS == 2 * kPkDecGroups, "decoded ring depth");
    constexpr int XS = DS;
    const int PS = args.pstages;
    const int bt = args.bt;
    const uint32_t x_bytes = static_cast<uint32_t>(bt) * 128u;
    // [decoded A: 4 x 16 KB][packed: PS x 16 KB][activations: XS x bt x 128]; all 1024-aligned
    auto sA = [&](int d) { return smem + d * kPkABytes; };
    uint8_t* sPbase = smem + DS * kPkABytes;
    auto sP = [&](int p) { return sPbase + p * kPkPBytes; };
    uint8_t* sXbase = sPbase + PS * kPkPBytes;
    auto sX = [&](int x) { return sXbase + x * x_bytes; };
    uint64_t* pfull = reinterpret_cast<uint64_t*>(sXbase + XS * x_bytes);
    uint64_t* pempty = pfull + kPkMaxPStages;
    uint64_t* xfull = pempty + kPkMaxPStages;
    uint64_t* dfull = xfull + XS;
    uint64_t* dempty = dfull + DS;             // frees decoded stage d and activation stage d
    uint64_t* tfull = dempty + DS;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int p = 0; p < PS; ++p) {
            mbar_init(&pfull[p], 1);
            mbar_init(&pempty[p], 4 * kPkDecGroups);   // every decoder warp
        }
        for (int x = 0; x < XS; ++x) {
            mbar_init(&xfull[x], 1);
        }
        for (int d = 0; d < DS; ++d) {
            mbar_init(&dfull[d], 4);     // the 4 decoder warps of the stage's group
            mbar_init(&dempty[d], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmP);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger_and_wait();

    const int units = args.n_tiles * args.t_tiles * args.splits;
    const uint64_t lim = args.wait_ns;
    // unit u -> (weight tile nt, token tile tt, K split sp) and its k-block range
    auto unit_of = [&](int u, int& nt, int& tt, int& kb0, int& kb1) {
        const int sp = u % args.splits;
        const int rest = u / args.splits;
        tt = rest % args.t_tiles;
        nt = rest / args.t_tiles;
        kb0 = static_cast<int>(static_cast<int64_t>(sp) * args.k_blocks / args.splits);
        kb1 = static_cast<int>(static_cast<int64_t>(sp + 1) * args.k_blocks / args.splits);
    };

    if (warp == 0) {
        // ----------------------------------------------------------------- producer (both load rings)
        if (elect_one()) {
            int p = 0, x = 0;
            uint32_t pph = 0, xph = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                int nt, tt, kb0, kb1;
                unit_of(u, nt, tt, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if ((kb - kb0) % kPkKbPerP == 0) {
                        // the unit's next packed stage: k-blocks kb .. kb + 3
                        if (!mbar_wait(&pempty[p], pph ^ 1u, lim, abort_flag)) { ok = false; break; }
                        mbar_arrive_expect_tx(&pfull[p], static_cast<uint32_t>(kPkPBytes));
                        tma_load_2d(sP(p), &tmP, &pfull[p], kb * 32, nt * kPkBM);
                        if (++p == PS) { p = 0; pph ^= 1u; }
                    }
                    if (!mbar_wait(&dempty[x], xph ^ 1u, lim, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(&xfull[x], x_bytes);
                    tma_load_2d(sX(x), &tmX, &xfull[x], kb * 128, tt * bt);
                    if (++x == XS) { x = 0; xph ^= 1u; }
                }
            }
            if (!ok) {
                // let the loads issued last land before the block exits (bounded)
                for (int i = 0; i < PS; ++i) {
                    const int pp = (p - 1 - i + 2 * PS) % PS;
                    mbar_wait(&pfull[pp], (p - 1 - i < 0) ? (pph ^ 1u) : pph, 100000000ull, nullptr);
                }
                for (int i = 0; i < XS; ++i) {
                    const int xx = (x - 1 - i + 2 * XS) % XS;
                    mbar_wait(&xfull[xx], (x - 1 - i < 0) ? (xph ^ 1u) : xph, 100000000ull, nullptr);
                }
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ----------------------------------------------------------------- decoders
        const int grp = (warp - 6) >> 2;           // decodes k-block sequence numbers q = grp mod 4
        const int dt = threadIdx.x - 192 - grp * 128;   // 0..127
        const int c = dt & 7;                      // word (16 codes) within a k-block's 32-byte row piece
        const int r0 = dt >> 3;                    // rows r0 + 16 i; r & 7 == r0 & 7 for all of them
        int p = 0;
        uint32_t pph = 0;
        uint32_t dph[DS / kPkDecGroups] = {};   // phase of each of the group's decoded stages
        int q = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            int nt, tt, kb0, kb1;
            unit_of(u, nt, tt, kb0, kb1);
            for (int kb = kb0; kb < kb1 && ok; kb += kPkKbPerP) {
                if (!mbar_wait_warp(&pfull[p], pph, lim, abort_flag)) { ok = false; break; }
                const uint8_t* src = sP(p);
                const int nkb = min(kPkKbPerP, kb1 - kb);
                for (int j = 0; j < nkb; ++j, ++q) {
                    if ((q & (kPkDecGroups - 1)) != grp) continue;
                    const int ds = q % DS;                      // grp, or grp + 4 on alternate turns
                    const int li = ds / kPkDecGroups;
                    // the MMA has finished with this decoded stage (its previous use)
                    if (!mbar_wait_warp(&dempty[ds], dph[li] ^ 1u, lim, abort_flag)) { ok = false; break; }
                    uint8_t* a = sA(ds);
                    // 16-byte chunk (2 j + c / 4) of row r sits at chunk (2 j + c / 4) ^ (r & 7)
                    const int src_off = ((((2 * j + (c >> 2)) ^ (r0 & 7)) << 4) | ((c & 3) << 2));
                    const int dst_off = (c ^ (r0 & 7)) << 4;
#pragma unroll
                    for (int i = 0; i < kPkBM / 16; ++i) {
                        const int r = r0 + 16 * i;
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(src + r * 128 + src_off);
                        *reinterpret_cast<uint4*>(a + r * 128 + dst_off) = pk_decode_word(w);
                    }
                    fence_proxy_async_shared();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&dfull[ds]);
                    dph[li] ^= 1u;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&pempty[p]);
                if (++p == PS) { p = 0; pph ^= 1u; }
            }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA issuer
        if (elect_one()) {
            const uint32_t idesc = umma_idesc(true, false, false, kPkBM, bt);
            int d = 0, x = 0;
            uint32_t dph = 0, xph = 0;
            int tcount = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tcount) {
                int nt, tt, kb0, kb1;
                unit_of(u, nt, tt, kb0, kb1);
                const int b = tcount & 1;
                const uint32_t tph = (tcount >> 1) & 1;
                if (!mbar_wait(&tempty[b], tph ^ 1u, lim, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kPkMaxBT);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&xfull[x], xph, lim, abort_flag) || !mbar_wait(&dfull[d], dph, lim, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA(d));
                    const uint32_t x_base = smem_u32(sX(x));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma<true>(d_tmem, umma_desc_sw128(a_base + kk * 32, 16, 1024),
                                     umma_desc_sw128(x_base + kk * 32, 16, 1024), idesc,
                                     (kb != kb0 || kk != 0) ? 1u : 0u);
                    tc_commit(&dempty[d]);     // d == x: the rings move in step
                    if (++d == DS) { d = 0; dph ^= 1u; }
                    if (++x == XS) { x = 0; xph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tfull[b]);
            }
            if (!ok) {
                tc_commit(&tfull[tcount & 1]);
                mbar_wait(&tfull[tcount & 1], ((tcount >> 1) & 1), 100000000ull, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------------- epilogue
        const int quad = warp & 3;                 // TMEM lanes [32 quad, 32 quad + 32)
        const float gm = __ldg(args.gamma);
        int tcount = 0;
        for (int u = blockIdx.x; u < units; u += gridDim.x, ++tcount) {
            int nt, tt, kb0, kb1;
            unit_of(u, nt, tt, kb0, kb1);
            const int b = tcount & 1;
            const uint32_t tph = (tcount >> 1) & 1;
            if (!mbar_wait_warp(&tfull[b], tph, lim, abort_flag)) break;
            tc_fence_after();
            const int n = nt * kPkBM + quad * 32 + lane;
            const bool n_ok = n < args.N;
            const int t0 = tt * bt;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(b * kPkMaxBT);
#pragma unroll 1
            for (int c0 = 0; c0 < bt; c0 += 32) {
                if (t0 + c0 >= args.T) break;                  // warp-uniform
                uint32_t r[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + c0, r);
                tmem_ld_wait();
                const int nj = min(32, min(bt - c0, args.T - t0 - c0));
                // lane l forms the factor of token t0 + c0 + l; the warp shares them by shuffle
                const float cl = (args.splits == 1 && lane < nj) ? __fdiv_rn(gm, __ldg(args.sx + t0 + c0 + lane)) : 0.0f;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (j >= nj) break;                            // warp-uniform
                    const float cj = __shfl_sync(0xffffffffu, cl, j);
                    if (!n_ok) continue;
                    const int t = t0 + c0 + j;
                    const int64_t o = static_cast<int64_t>(t) * args.N + n;
                    const int32_t v = static_cast<int32_t>(r[j]);
                    if (args.splits > 1) {
                        const int sp = u % args.splits;
                        args.acc[static_cast<int64_t>(sp) * args.T * args.N + o] = v;
                    } else {
                        const float y = __fmul_rn(static_cast<float>(v), cj);
                        if constexpr (kBf16Out)
                            static_cast<uint16_t*>(args.y)[o] = float_to_bf16_bits(y);
                        else
                            static_cast<float*>(args.y)[o] = y;
                        if (args.acc != nullptr) args.acc[o] = v;
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
        tmem_dealloc(tmem_base, 512);
    }
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

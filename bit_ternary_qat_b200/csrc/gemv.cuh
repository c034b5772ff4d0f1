// gemv.cuh -- K7: decode GEMV over 2-bit packed ternary weights.
//
// P5 ("1.58-bit量化技术…") §3.1: a ternary weight turns the multiply-accumulate into
// add (W = +1), subtract (W = -1) or skip (W = 0); §4.1: codes 00 -> 0, 01 -> +1,
// 10 -> -1, 11 reserved (decodes to 0 here).  Output y = acc * (gamma / s_b), the factor
// formed once per activation row.
//
// The weights are streamed from HBM exactly once (N x K/4 bytes, one warp per output row,
// lanes on consecutive 8-byte chunks so any K % 32 == 0 row is aligned).  No code is ever decoded to a
// value: for each 32-bit word of 16 codes, the bit-planes lo_j = (w >> 2j) & 0x01010101
// and hi_j = (w >> 2j+1) & 0x01010101 (j = 0..3) are 0/1 bytes, and
//   sum_k dec(c_k) x_k = sum_j dp4a(lo_j, x_j) - dp4a(hi_j, x_j),
// which also maps the reserved 11 to 0.  Byte i of lo_j holds the code of element
// 16g + 4i + j, so the activation words are staged once per block in shared memory in
// that interleaved order: x_j = (x[16g+j], x[16g+4+j], x[16g+8+j], x[16g+12+j]).
#pragma once
#include "common.cuh"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;

// Shared-memory activation layout: element (b, h, c) = the 4 interleaved words of
// group g = 2c + h (c = 8-byte chunk index of a packed row, h = word within the chunk),
// so consecutive lanes read consecutive 16-byte entries (no bank conflicts).
// sum_i a.u8[i] * b.s8[i] + c
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int gemv_xs_index(int b, int h, int c, int nchunk) {
    return (b * 2 + h) * nchunk + c;
}

// NB <= 4: the bit-planes are masked in place (w & (0x01010101 << 2j)), which needs no
// shifts but leaves plane j scaled by 2^(2j) (lo) or 2^(2j+1) (hi); one accumulator per
// plane, unscaled exactly at the end.  NB > 4: planes are shifted down first so a batch
// row needs only two accumulators.
template <int NB>
__global__ void __launch_bounds__(kGemvThreads) ternary_gemv_kernel(const uint8_t* __restrict__ packed,
                                                                    const float* __restrict__ gamma, int N, int K,
                                                                    const int8_t* __restrict__ xq,
                                                                    const float* __restrict__ sx, int B,
                                                                    float* __restrict__ y,
                                                                    int32_t* __restrict__ acc_out) {
    extern __shared__ int4 xs[];       // [B][2][K/32]
    const int G = K / 16;
    const int nchunk = K / 32;          // 8-byte chunks (32 codes) per packed row
    for (int idx = threadIdx.x; idx < B * G; idx += kGemvThreads) {
        const int b = idx / G, g = idx - b * G;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(b) * K) + g);
        int4 o;
        int* ov = reinterpret_cast<int*>(&o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t t01 = __byte_perm(raw.x, raw.y, j | ((4 + j) << 4));
            const uint32_t t23 = __byte_perm(raw.z, raw.w, j | ((4 + j) << 4));
            ov[j] = static_cast<int>(__byte_perm(t01, t23, 0x5410));
        }
        xs[gemv_xs_index(b, g & 1, g >> 1, nchunk)] = o;
    }
    __syncthreads();

    const float gm = __ldg(gamma);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool kInPlace = NB <= 4;
    constexpr int kAcc = kInPlace ? 8 : 2;
    for (int n = blockIdx.x * kGemvWarps + warp; n < N; n += gridDim.x * kGemvWarps) {
        int acc[NB][kAcc];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int a = 0; a < kAcc; ++a) acc[b][a] = 0;
        const uint2* row = reinterpret_cast<const uint2*>(packed + static_cast<int64_t>(n) * (K / 4));
        constexpr int kU = 8;   // 8-byte chunks per lane loaded before any math (64 codes x 8)
        for (int cb = 0; cb < nchunk; cb += 32 * kU) {
            uint2 pw[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int c = cb + lane + 32 * u;
                pw[u] = c < nchunk ? __ldcs(row + c) : make_uint2(0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int c = cb + lane + 32 * u;
                if (c >= nchunk) continue;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w = h == 0 ? pw[u].x : pw[u].y;
                    int lo[4], hi[4];
                    if constexpr (kInPlace) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            lo[j] = static_cast<int>(w & (0x01010101u << (2 * j)));
                            hi[j] = static_cast<int>(w & (0x02020202u << (2 * j)));
                        }
                    } else {
                        const uint32_t w1 = w >> 1;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            lo[j] = static_cast<int>((w >> (2 * j)) & 0x01010101u);
                            hi[j] = static_cast<int>((w1 >> (2 * j)) & 0x01010101u);
                        }
                    }
#pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        if (b < B) {
                            const int4 xv = xs[gemv_xs_index(b, h, c, nchunk)];
                            const int xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if constexpr (kInPlace) {
                                    // bytes of lo[j]/hi[j] are 0 or 2^(2j) / 2^(2j+1): read them as
                                    // unsigned (2^7 does not fit a signed byte)
                                    acc[b][2 * j] = dp4a_us(static_cast<uint32_t>(lo[j]), xw[j], acc[b][2 * j]);
                                    acc[b][2 * j + 1] =
                                        dp4a_us(static_cast<uint32_t>(hi[j]), xw[j], acc[b][2 * j + 1]);
                                } else {
                                    acc[b][0] = __dp4a(lo[j], xw[j], acc[b][0]);
                                    acc[b][1] = __dp4a(hi[j], xw[j], acc[b][1]);
                                }
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            if (b < B) {
                int part;
                if constexpr (kInPlace) {
                    part = 0;
#pragma unroll
                    for (int j = 0; j < 4; ++j) part += (acc[b][2 * j] >> (2 * j)) - (acc[b][2 * j + 1] >> (2 * j + 1));
                } else {
                    part = acc[b][0] - acc[b][1];
                }
                const int tot = warp_sum(part);
                if (lane == 0) {
                    const int64_t o = static_cast<int64_t>(b) * N + n;
                    y[o] = __fmul_rn(static_cast<float>(tot), __fdiv_rn(gm, __ldg(sx + b)));
                    if (acc_out != nullptr) acc_out[o] = tot;
                }
            }
        }
    }
}

// ------------------------------------------------------------------------------------
// Tensor-core variant (mma.sync m16n8k32, u8 x s8 -> s32).
//
// A warp owns 16 weight rows.  For a "super-chunk" of 8 packed words per row (128 codes),
// lane (g = lane/4, t = lane%4) holds words 2t and 2t+1 of rows g and g+8.  For a bit
// plane p (lo = bit 0, hi = bit 1) and a position j (code j of each byte), masking a word
// in place, w & (0x01010101 << (2j + p)), gives 4 bytes that are 0 or 2^(2j+p): exactly
// the 4 int8 entries one mma A register holds.  So with logical k = 4t + i (word 2t) and
// 16 + 4t + i (word 2t+1), the A fragment of (j, p) is 4 masked words, and the matching B
// fragment is the interleaved activation word x_j of groups 2t and 2t+1 (already staged in
// shared memory), for batch column g.  Eight mma per n-tile per super-chunk (4 j x 2
// planes) accumulate into D[j][p]; the result is sum_j D_lo[j] / 4^j - D_hi[j] / (2 4^j),
// exact since every term of D[j][p] is a multiple of its scale.  The K reduction happens
// inside the mma, so no cross-lane reduction is needed; 16 rows x 128 codes cost 32
// masking instructions per lane.
// ------------------------------------------------------------------------------------
constexpr int kGemvMmaWarps = 8;
constexpr int kGemvMmaThreads = kGemvMmaWarps * 32;

__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Work split: a block keeps the staged activations and loops over row groups (16 rows).
// Its 8 warps form RS = 8 / KS row slots of KS warps; the KS warps of a slot split the
// row's super-chunks, and their exact int32 partial sums are added in shared memory.
// NTILES n-tiles of 8 batch columns (B <= 8 * NTILES).
template <int NTILES>
__global__ void __launch_bounds__(kGemvMmaThreads, 2) ternary_gemv_mma_kernel(
    const uint8_t* __restrict__ packed, const float* __restrict__ gamma, int N, int K,
    const int8_t* __restrict__ xq, const float* __restrict__ sx, int B, int KS, float* __restrict__ y,
    int32_t* __restrict__ acc_out) {
    constexpr int kU = NTILES == 1 ? 8 : 4;      // super-chunks (8 bytes per lane each) loaded at once
    constexpr int BP = 8 * NTILES;
    extern __shared__ int4 xs[];                 // [BP][G + 1]: interleaved words per group
    __shared__ int red[kGemvMmaWarps][NTILES * 4][32];
    const int G = K / 16;                        // groups of 16 codes (one packed word) per row
    const int ld = G + 1;                        // padded row stride (int4) -> conflict-free reads
    for (int idx = threadIdx.x; idx < BP * G; idx += kGemvMmaThreads) {
        const int b = idx / G, gg = idx - b * G;
        int4 o = make_int4(0, 0, 0, 0);
        if (b < B) {
            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(b) * K) + gg);
            int* ov = reinterpret_cast<int*>(&o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t t01 = __byte_perm(raw.x, raw.y, j | ((4 + j) << 4));
                const uint32_t t23 = __byte_perm(raw.z, raw.w, j | ((4 + j) << 4));
                ov[j] = static_cast<int>(__byte_perm(t01, t23, 0x5410));
            }
        }
        xs[b * ld + gg] = o;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int RS = kGemvMmaWarps / KS;
    const int ks = warp % KS, rs = warp / KS;
    const int nsc = (G + 7) / 8;                 // super-chunks of 8 words per row
    const int per = (nsc + KS - 1) / KS;         // super-chunks per warp
    const int sc_begin = ks * per;
    const int sc_end = min(nsc, sc_begin + per);
    const int row_words = K / 16;
    const float gm = __ldg(gamma);
    const int n_rg = N / 16;
    for (int rg = blockIdx.x * RS + rs; rg < n_rg; rg += gridDim.x * RS) {
        const int r0 = rg * 16 + g, r1 = r0 + 8;
        const uint32_t* w0 = reinterpret_cast<const uint32_t*>(packed + static_cast<int64_t>(r0) * (K / 4));
        const uint32_t* w1 = reinterpret_cast<const uint32_t*>(packed + static_cast<int64_t>(r1) * (K / 4));
        int d[4][2][NTILES][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[j][p][nt][i] = 0;
        for (int sc0 = sc_begin; sc0 < sc_end; sc0 += kU) {
            uint2 wa[kU], wb[kU];                // words (2t, 2t+1) of rows r0 and r1
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int wi = (sc0 + u) * 8 + 2 * t;
                if (sc0 + u < sc_end && wi < row_words) {     // row_words is even: wi + 1 < row_words too
                    wa[u] = __ldcs(reinterpret_cast<const uint2*>(w0 + wi));
                    wb[u] = __ldcs(reinterpret_cast<const uint2*>(w1 + wi));
                } else {
                    wa[u] = make_uint2(0u, 0u);
                    wb[u] = make_uint2(0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int sc = sc0 + u;
                if (sc >= sc_end) break;
                const int grp = sc * 8 + 2 * t;  // group of word 2t; word 2t+1 is grp + 1
                int4 xb0[NTILES], xb1[NTILES];
#pragma unroll
                for (int nt = 0; nt < NTILES; ++nt) {
                    const int n = nt * 8 + g;
                    xb0[nt] = grp < G ? xs[n * ld + grp] : make_int4(0, 0, 0, 0);
                    xb1[nt] = grp + 1 < G ? xs[n * ld + grp + 1] : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const uint32_t m = 0x01010101u << (2 * j + p);
                        const uint32_t a[4] = {wa[u].x & m, wb[u].x & m, wa[u].y & m, wb[u].y & m};
#pragma unroll
                        for (int nt = 0; nt < NTILES; ++nt) {
                            const int* x0 = reinterpret_cast<const int*>(&xb0[nt]);
                            const int* x1 = reinterpret_cast<const int*>(&xb1[nt]);
                            mma_u8s8_16832(d[j][p][nt], a, static_cast<uint32_t>(x0[j]), static_cast<uint32_t>(x1[j]));
                        }
                    }
                }
            }
        }
        // this warp's exact partial sums: D[i] is rows (r0, r0, r1, r1) x batch columns
        // (2t, 2t+1, 2t, 2t+1) of each n-tile
        int tot[NTILES][4];
#pragma unroll
        for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int v = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) v += (d[j][0][nt][i] >> (2 * j)) - (d[j][1][nt][i] >> (2 * j + 1));
                tot[nt][i] = v;
            }
        if (KS > 1) {
#pragma unroll
            for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[warp][nt * 4 + i][lane] = tot[nt][i];
            named_barrier(1 + rs, KS * 32);
            if (ks == 0) {
                for (int o = 1; o < KS; ++o)
#pragma unroll
                    for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) tot[nt][i] += red[warp + o][nt * 4 + i][lane];
            }
        }
        if (ks == 0) {
#pragma unroll
            for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int b = nt * 8 + 2 * t + (i & 1);
                    const int row = (i < 2) ? r0 : r1;
                    if (b < B) {
                        const int64_t o = static_cast<int64_t>(b) * N + row;
                        y[o] = __fmul_rn(static_cast<float>(tot[nt][i]), __fdiv_rn(gm, __ldg(sx + b)));
                        if (acc_out != nullptr) acc_out[o] = tot[nt][i];
                    }
                }
        }
        if (KS > 1) named_barrier(1 + rs, KS * 32);   // red[] is reused by the next row group
    }
}

// Bounded-wait self test: one thread waits on an mbarrier that nothing arrives on.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns, &abort_flag);
}

}  // namespace bl

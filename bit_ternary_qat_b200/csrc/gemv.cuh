// gemv.cuh -- K7: decode GEMV over 2-bit packed ternary weights.
//
// P5 ("1.58-bit量化技术…") §3.1: a ternary weight turns the multiply-accumulate into
// add (W = +1), subtract (W = -1) or skip (W = 0); §4.1: codes 00 -> 0, 01 -> +1,
// 10 -> -1, 11 reserved (decodes to 0 here).  Output y = acc * (gamma / s_b), the factor
// formed once per activation row.
//
// The weights are streamed from HBM exactly once, by TMA, and no code is ever decoded to a
// value: for a 32-bit word of 16 codes (code 16g + 4i + j at bits 8i + 2j), the in-place
// mask w & (0x01010101 << (2j + p)) keeps bit p of code j of each byte, i.e. four bytes
// that are 0 or 2^(2j+p).  With the activations staged once per block as interleaved words
// x_j = (x[16g+j], x[16g+4+j], x[16g+8+j], x[16g+12+j]),
//   sum_k dec(c_k) x_k = sum_j (lo-plane . x_j) / 4^j - (hi-plane . x_j) / (2 4^j),
// which also maps the reserved 11 to 0.  The dot products run on the tensor cores
// (mma.sync m16n8k32, u8 x s8 -> s32).
#pragma once
#include "common.cuh"

namespace bl {

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
__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kGemvTileBytes = 16 * 128;   // one TMA box: 16 weight rows x 128 bytes (512 codes)

template <int WB, int S>
__host__ __device__ constexpr size_t gemv_ring_bytes() { return (size_t)WB * S * kGemvTileBytes; }

// Weights reach shared memory through TMA: every warp streams its own row groups through a
// private ring of S boxes (16 rows x 128 bytes, 128-byte swizzle) and keeps S boxes in
// flight; a per-slot mbarrier (bounded wait) says when a box has landed.  Within a box,
// lane (g, t) reads words (2t, 2t+1) of each 32-byte super-chunk of rows g and g+8 from
// the swizzled layout -- conflict free -- and runs the mma of the comment above.  A warp
// owns whole row groups, so its accumulators are final when the row group ends.
// NTILES n-tiles of 8 batch columns (B <= 8 * NTILES); only the first B batch rows of the
// activations are staged.
template <int NTILES, int WB, int S>
__global__ void __launch_bounds__(WB * 32) ternary_gemv_tma_kernel(
    const __grid_constant__ CUtensorMap tmW, const float* __restrict__ gamma, int N, int K,
    const int8_t* __restrict__ xq, const float* __restrict__ sx, int B, float* __restrict__ y,
    int32_t* __restrict__ acc_out, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* rings = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int G = K / 16;                        // groups of 16 codes (one packed word) per row
    const int ld = G + 1;                        // padded row stride (int4) -> conflict-free reads
    int4* xs = reinterpret_cast<int4*>(rings + gemv_ring_bytes<WB, S>());   // [B][G + 1]
    uint64_t* bars = reinterpret_cast<uint64_t*>(xs + static_cast<size_t>(B) * ld);

    for (int idx = threadIdx.x; idx < B * G; idx += WB * 32) {
        const int b = idx / G, gg = idx - b * G;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(b) * K) + gg);
        int4 o;
        int* ov = reinterpret_cast<int*>(&o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t t01 = __byte_perm(raw.x, raw.y, j | ((4 + j) << 4));
            const uint32_t t23 = __byte_perm(raw.z, raw.w, j | ((4 + j) << 4));
            ov[j] = static_cast<int>(__byte_perm(t01, t23, 0x5410));
        }
        xs[b * ld + gg] = o;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < WB * S; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int KT = (K / 4 + 127) / 128;          // boxes per row
    const int n_rg = N / 16;
    const int first_rg = blockIdx.x * WB + warp;
    const int rg_step = gridDim.x * WB;
    const int my_rgs = first_rg < n_rg ? (n_rg - first_rg + rg_step - 1) / rg_step : 0;
    const int total = my_rgs * KT;
    uint8_t* ring = rings + static_cast<size_t>(warp) * S * kGemvTileBytes;
    uint64_t* bar = bars + warp * S;
    const float gm = __ldg(gamma);

    auto issue = [&](int i, int rg, int kt) {
        const int slot = i % S;
        mbar_arrive_expect_tx(&bar[slot], kGemvTileBytes);
        tma_load_2d(ring + slot * kGemvTileBytes, &tmW, &bar[slot], kt * 128, rg * 16);
    };
    // producer position (lane 0 only): the box S tiles ahead of the consumer
    int p_rg = first_rg, p_kt = 0;
    auto advance = [&](int& rg, int& kt) {
        if (++kt == KT) { kt = 0; rg += rg_step; }
    };
    if (lane == 0)
        for (int i = 0; i < S && i < total; ++i) { issue(i, p_rg, p_kt); advance(p_rg, p_kt); }

    // per-lane constants: swizzled offsets of words (2t, 2t+1) of super-chunk sc in rows g and
    // g+8 (same chunk permutation, since (g + 8) % 8 == g) and the activation-word indices
    int off[4];
#pragma unroll
    for (int sc = 0; sc < 4; ++sc) off[sc] = g * 128 + (((2 * sc + (t >> 1)) ^ g) << 4) + 8 * (t & 1);
    int xbase[NTILES];
    bool xlive[NTILES];
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt) {
        xlive[nt] = nt * 8 + g < B;
        xbase[nt] = (nt * 8 + g) * ld + 2 * t;
    }

    constexpr bool kShift = NTILES == 2;
    constexpr int kJ = kShift ? 1 : 4;
    int d[kJ][2][NTILES][4];
    bool ok = true;
    int i = 0;
    int c_rg = first_rg, c_kt = 0;               // consumer position
    for (; i < total; ++i) {
        const int slot = i % S;
        if (c_kt == 0) {
#pragma unroll
            for (int j = 0; j < kJ; ++j)
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                        for (int q = 0; q < 4; ++q) d[j][p][nt][q] = 0;
        }
        if (!mbar_wait(&bar[slot], (i / S) & 1, wait_ns, nullptr)) { ok = false; break; }
        const uint8_t* tile = ring + slot * kGemvTileBytes;
        const int gbase = c_kt * 32;             // first group of this box
#pragma unroll
        for (int sc = 0; sc < 4; ++sc) {
            // NTILES == 1: planes masked in place (scale 2^(2j+p), one accumulator set per
            // (j, p)).  NTILES == 2: planes shifted down to scale 1 first (one more instruction
            // per register, two accumulator sets instead of eight).
            const uint2 wa = *reinterpret_cast<const uint2*>(tile + off[sc]);
            const uint2 wb = *reinterpret_cast<const uint2*>(tile + off[sc] + 8 * 128);
            const int grp = gbase + sc * 8;      // + 2t (in xbase): group of word 2t
            int4 xb0[NTILES], xb1[NTILES];
#pragma unroll
            for (int nt = 0; nt < NTILES; ++nt) {
                const bool live = xlive[nt] && grp + 2 * t < G;   // G is even: grp + 2t + 1 < G too
                xb0[nt] = live ? xs[xbase[nt] + grp] : make_int4(0, 0, 0, 0);
                xb1[nt] = live ? xs[xbase[nt] + grp + 1] : make_int4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    uint32_t a[4];
                    if constexpr (kShift) {
                        const int sh = 2 * j + p;
                        a[0] = (wa.x >> sh) & 0x01010101u; a[1] = (wb.x >> sh) & 0x01010101u;
                        a[2] = (wa.y >> sh) & 0x01010101u; a[3] = (wb.y >> sh) & 0x01010101u;
                    } else {
                        const uint32_t m = 0x01010101u << (2 * j + p);
                        a[0] = wa.x & m; a[1] = wb.x & m; a[2] = wa.y & m; a[3] = wb.y & m;
                    }
                    const int jj = kShift ? 0 : j;
#pragma unroll
                    for (int nt = 0; nt < NTILES; ++nt) {
                        const int* x0 = reinterpret_cast<const int*>(&xb0[nt]);
                        const int* x1 = reinterpret_cast<const int*>(&xb1[nt]);
                        mma_u8s8_16832(d[jj][p][nt], a, static_cast<uint32_t>(x0[j]), static_cast<uint32_t>(x1[j]));
                    }
                }
            }
        }
        __syncwarp();                            // every lane is done with this slot
        if (lane == 0 && i + S < total) { issue(i + S, p_rg, p_kt); advance(p_rg, p_kt); }
        if (c_kt == KT - 1) {
            // D[q]: rows (r0, r0, r1, r1) x batch columns (2t, 2t+1, 2t, 2t+1) of each n-tile
            const int r0 = c_rg * 16 + g, r1 = r0 + 8;
#pragma unroll
            for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    int tot = 0;
                    if constexpr (kShift) {
                        tot = d[0][0][nt][q] - d[0][1][nt][q];
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tot += (d[j][0][nt][q] >> (2 * j)) - (d[j][1][nt][q] >> (2 * j + 1));
                    }
                    const int b = nt * 8 + 2 * t + (q & 1);
                    if (b < B) {
                        const int64_t o = static_cast<int64_t>(b) * N + ((q < 2) ? r0 : r1);
                        y[o] = __fmul_rn(static_cast<float>(tot), __fdiv_rn(gm, __ldg(sx + b)));
                        if (acc_out != nullptr) acc_out[o] = tot;
                    }
                }
        }
        advance(c_rg, c_kt);
    }
    if (!ok && lane == 0) {
        // drain the boxes still in flight into this warp's ring before the block can exit
        for (int k = i + 1; k < total && k < i + S; ++k) mbar_wait(&bar[k % S], (k / S) & 1, 100000000ull, nullptr);
    }
    __syncwarp();
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

// gemv.cuh -- K7: decode GEMV over 2-bit packed ternary weights.
//
// P5 ("1.58-bit量化技术…") §3.1: a ternary weight turns the multiply-accumulate into
// add (W = +1), subtract (W = -1) or skip (W = 0); §4.1: codes 00 -> 0, 01 -> +1,
// 10 -> -1, 11 reserved (decodes to 0 here).  Output y = acc * (gamma / s_b), the factor
// formed once per activation row.
//
// The weights are streamed from HBM exactly once, into registers, and no code is ever decoded to a
// separate value.  Two identities do the decoding inside 32-bit words of 16 codes (code
// 16g + 4i + j of row n at bits 8i + 2j of word g):
//   (1) with L = w & 0x5555..., H = (w >> 1) & 0x5555..., the word
//         F = (L | 0xAAAA...) - H
//       holds in every 2-bit field f = 2 + lo - hi = dec(c) + 2, in {1, 2, 3} (no borrow
//       crosses a field because 2 + lo >= 1 + hi), and the reserved code 11 gives f = 2,
//       i.e. dec = 0;
//   (2) F & (0x03030303 << 2j) keeps field j of each byte in place: four bytes f * 4^j,
//       exactly the four u8 entries of one mma A register.
// With the activations staged once per block as interleaved words
// x_j = (x[16g+j], x[16g+4+j], x[16g+8+j], x[16g+12+j]),
//   sum_k dec(c_k) x_k = sum_j D_j / 4^j - 2 sum_k x_k,   D_j = sum (F & mask_j) . x_j,
// where every D_j is an exact multiple of 4^j and sum_k x_k is a property of the
// activation row alone.  The dot products D_j run on the tensor cores (mma.sync m16n8k32,
// u8 x s8 -> s32): one byte slot per code.
#pragma once
#include "common.cuh"

namespace bl {

__device__ __forceinline__ void mma_u8s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// identity (1): fields dec(c) + 2
__device__ __forceinline__ uint32_t ternary_fields(uint32_t w) {
    return ((w & 0x55555555u) | 0xAAAAAAAAu) - ((w >> 1) & 0x55555555u);
}

constexpr int kGemvStepBytes = 64;          // one step: 64 bytes (256 codes) of each of 16 rows
constexpr int kGemvU = 4;                   // steps per batch of loads (software pipelined)

// Shared memory of one block: staged activations (+1 int4 of padding per row), int32
// row-group accumulators (+ activation row sums), one mbarrier.  `max_rgs` row groups.
__host__ __device__ inline size_t gemv_smem_bytes(int B, int K, int max_rgs) {
    const int spr = (K / 16 + 15) / 16;     // steps per row
    const size_t ld = (size_t)spr * 16 + 1;
    const size_t acc_ints = ((size_t)max_rgs * 16 * B + B + 1) & ~(size_t)1;
    return 16 + (size_t)B * ld * 16 + acc_ints * 4 + sizeof(uint64_t) + 16;
}

// ------------------------------------------------------------------------------------
// Block b owns the row groups (16 rows each) [rg0, rg1) of a balanced partition of the
// N/16 row groups; its work is split into steps (row group, 64-byte column block) numbered
// row-group-major, and warp w takes one contiguous, equally long run of them (+-1), so a
// warp's run touches one or two row groups and all warps stream the same number of bytes.
// A warp reads its weights straight from HBM into registers: per step, lane (g = lane/4,
// t = lane%4) loads words 4t..4t+3 of the step's 64 bytes of rows g and g+8 (one 16-byte
// load each; 8 rows x 64 contiguous bytes per warp instruction), kGemvU steps per batch,
// two batches in registers (the next loading while the current one is multiplied), with
// the load and compute positions advanced incrementally (no division in the loop).
// Words 4t, 4t+1 feed one m16n8k32 k-block and words 4t+2, 4t+3 the next: byte i of word q
// holds codes 16q + 4i + j,
// so k-slot 4t + i (16 + 4t + i) of a k-block pairs with activation word x_j of group q =
// 4t (4t + 1), etc.  When its run leaves a row group the warp folds its accumulators and
// adds them into the block's shared int32 sums of that row group (shared-memory integer
// atomics: exact, order free); after a block barrier the block writes y for its rows.
// The activation rows reach shared memory by bulk copy (one bounded mbarrier wait) while
// the first weight batch is already in flight, and are interleaved in place.
// ------------------------------------------------------------------------------------
template <int NTILES, int WB, bool kBf16Out = false>
__global__ void __launch_bounds__(WB * 32, 1) ternary_gemv_kernel(
    const uint8_t* __restrict__ W, const float* __restrict__ gamma, int gamma_stride, int N, int K,
    const int8_t* __restrict__ xq, const float* __restrict__ sx, int B, void* __restrict__ y,
    int32_t* __restrict__ acc_out, uint64_t wait_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((16u - (smem_u32(smem_raw) & 15u)) & 15u);
    const int row_bytes = K / 4;
    const int G = K / 16;                        // packed words per weight row
    const int spr = (G + 15) / 16;               // steps per row (16 words each)
    const int Gp = spr * 16;                     // staged activation groups per row (zero past G)
    const int ld = Gp + 1;
    const int n_rg = N / 16;
    const int rg0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * n_rg / gridDim.x);
    const int rg1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * n_rg / gridDim.x);
    const int nrg = rg1 - rg0;
    int4* xs = reinterpret_cast<int4*>(base);                                  // [B][ld]
    int* accs = reinterpret_cast<int*>(xs + static_cast<size_t>(B) * ld);      // [nrg*16][B]
    int* xsum = accs + nrg * 16 * B;                                          // [B]
    uint64_t* xbar = reinterpret_cast<uint64_t*>(accs + ((nrg * 16 * B + B + 1) & ~1));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    if (threadIdx.x == 0) {
        mbar_init(xbar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger_and_wait();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(B * K));
        for (int b = 0; b < B; ++b)
            bulk_load(xs + static_cast<size_t>(b) * ld, xq + static_cast<int64_t>(b) * K, static_cast<uint32_t>(K), xbar);
    }

    // this warp's run of steps [i0, i1) of the block's row-group-major sequence
    const int nsteps = nrg * spr;
    const int i0 = static_cast<int>(static_cast<int64_t>(warp) * nsteps / WB);
    const int i1 = static_cast<int>(static_cast<int64_t>(warp + 1) * nsteps / WB);
    // Load cursor: the next step to load, its position in its row, and this lane's address of
    // its 16-byte slice of row g (row g+8 is 8 rows further).  A slice past the row end (the
    // last step of a row when K/4 is not a multiple of 64) loads as zeros.
    const int64_t r8 = 8 * static_cast<int64_t>(row_bytes);
    const int64_t rg_jump = 16 * static_cast<int64_t>(row_bytes) - static_cast<int64_t>(spr) * kGemvStepBytes;
    const bool tail_ok = (spr - 1) * kGemvStepBytes + 16 * t < row_bytes;
    int li = i0, l_s = i0 % spr;
    const uint8_t* lp = W + (static_cast<int64_t>(rg0 + i0 / spr) * 16 + g) * row_bytes +
                        static_cast<int64_t>(l_s) * kGemvStepBytes + 16 * t;
    auto load_next = [&](uint4& ra, uint4& rb) {
        ra = make_uint4(0u, 0u, 0u, 0u);
        rb = ra;
        if (li < i1 && (l_s != spr - 1 || tail_ok)) {
            ra = __ldcs(reinterpret_cast<const uint4*>(lp));
            rb = __ldcs(reinterpret_cast<const uint4*>(lp + r8));
        }
        ++li;
        lp += kGemvStepBytes;
        if (++l_s == spr) {
            l_s = 0;
            lp += rg_jump;
        }
    };
    // two batches of kGemvU steps in registers: one multiplied while the other loads
    uint4 Aa[kGemvU], Ab[kGemvU], Ba[kGemvU], Bb[kGemvU];
#pragma unroll
    for (int u = 0; u < kGemvU; ++u) load_next(Aa[u], Ab[u]);

    // activations: wait for the copies, interleave in place (zero past K), clear the sums
    for (int idx = threadIdx.x; idx < nrg * 16 * B; idx += WB * 32) accs[idx] = 0;
    mbar_wait(xbar, 0, wait_ns, nullptr);
    for (int idx = threadIdx.x; idx < B * Gp; idx += WB * 32) {
        const int b = idx / Gp, gg = idx - b * Gp;
        int4 o = make_int4(0, 0, 0, 0);
        if (gg < G) {
            const int4 raw = xs[b * ld + gg];
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
    // sum_k x[b][k] (the "- 2 sum x" term), one warp per activation row
    for (int b = warp; b < B; b += WB) {
        int sacc = 0;
        for (int gg = lane; gg < Gp; gg += 32) {
            const int4 v = xs[b * ld + gg];
            sacc = __dp4a(v.x, 0x01010101, sacc);
            sacc = __dp4a(v.y, 0x01010101, sacc);
            sacc = __dp4a(v.z, 0x01010101, sacc);
            sacc = __dp4a(v.w, 0x01010101, sacc);
        }
        sacc = warp_sum(sacc);
        if (lane == 0) xsum[b] = sacc;
    }

    // batch column of this lane in n-tile nt (columns past B read row B-1; never written)
    int xbase[NTILES];
#pragma unroll
    for (int nt = 0; nt < NTILES; ++nt) xbase[nt] = min(nt * 8 + g, B - 1) * ld + 4 * t;

    int d[4][NTILES][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) d[j][nt][q] = 0;
    auto flush = [&](int rgl) {
#pragma unroll
        for (int nt = 0; nt < NTILES; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int tot = d[0][nt][q] + (d[1][nt][q] >> 2) + (d[2][nt][q] >> 4) + (d[3][nt][q] >> 6);
                const int b = nt * 8 + 2 * t + (q & 1);
                const int r = (q < 2) ? g : g + 8;
                if (b < B) atomicAdd(&accs[(rgl * 16 + r) * B + b], tot);
                d[0][nt][q] = d[1][nt][q] = d[2][nt][q] = d[3][nt][q] = 0;
            }
    };
    // one step: two k-blocks (words 4t, 4t+1 and 4t+2, 4t+3 of rows g and g+8)
    auto mma_step = [&](const uint4& ra, const uint4& rb, int s) {
        const uint32_t fa[4] = {ternary_fields(ra.x), ternary_fields(ra.y), ternary_fields(ra.z), ternary_fields(ra.w)};
        const uint32_t fb[4] = {ternary_fields(rb.x), ternary_fields(rb.y), ternary_fields(rb.z), ternary_fields(rb.w)};
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            int4 x0[NTILES], x1[NTILES];
#pragma unroll
            for (int nt = 0; nt < NTILES; ++nt) {
                x0[nt] = xs[xbase[nt] + s * 16 + 2 * kb];
                x1[nt] = xs[xbase[nt] + s * 16 + 2 * kb + 1];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t m = 0x03030303u << (2 * j);
                const uint32_t a[4] = {fa[2 * kb] & m, fb[2 * kb] & m, fa[2 * kb + 1] & m, fb[2 * kb + 1] & m};
#pragma unroll
                for (int nt = 0; nt < NTILES; ++nt) {
                    const int* p0 = reinterpret_cast<const int*>(&x0[nt]);
                    const int* p1 = reinterpret_cast<const int*>(&x1[nt]);
                    mma_u8s8_16832(d[j][nt], a, static_cast<uint32_t>(p0[j]), static_cast<uint32_t>(p1[j]));
                }
            }
        }
    };

    int ci = i0, c_s = i0 % spr, c_rgl = i0 / spr;   // compute cursor
    auto process = [&](uint4 (&pa)[kGemvU], uint4 (&pb)[kGemvU]) {
#pragma unroll
        for (int u = 0; u < kGemvU; ++u) {
            if (ci < i1) {
                mma_step(pa[u], pb[u], c_s);
                if (c_s == spr - 1 || ci == i1 - 1) flush(c_rgl);
                ++ci;
                if (++c_s == spr) {
                    c_s = 0;
                    ++c_rgl;
                }
            }
        }
    };
    while (ci < i1) {
#pragma unroll
        for (int u = 0; u < kGemvU; ++u) load_next(Ba[u], Bb[u]);
        process(Aa, Ab);
        if (ci >= i1) break;
#pragma unroll
        for (int u = 0; u < kGemvU; ++u) load_next(Aa[u], Ab[u]);
        process(Ba, Bb);
    }
    __syncthreads();

    // y[b][n] = (acc - 2 sum x_b) * fl(gamma_n / s_b) for this block's rows, row-fastest
    // (gamma_n = gamma[n * gamma_stride]: one scale, or one per weight row), stored as fp32
    // or rounded to bf16
    const int rows = nrg * 16;
    for (int idx = threadIdx.x; idx < rows * B; idx += WB * 32) {
        const int b = idx / rows, r = idx - b * rows;
        const int acc = accs[r * B + b] - 2 * xsum[b];
        const int n = rg0 * 16 + r;
        const int64_t o = static_cast<int64_t>(b) * N + n;
        const float gm = __ldg(gamma + static_cast<int64_t>(n) * gamma_stride);
        const float yv = __fmul_rn(static_cast<float>(acc), __fdiv_rn(gm, __ldg(sx + b)));
        if constexpr (kBf16Out)
            static_cast<uint16_t*>(y)[o] = float_to_bf16_bits(yv);
        else
            static_cast<float*>(y)[o] = yv;
        if (acc_out != nullptr) acc_out[o] = acc;
    }
}

// Bounded-wait self test: one thread waits on an mbarrier that nothing arrives on.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    pdl_trigger_and_wait();
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

// bitlinear.cu -- C ABI of the BitLinear hot path (declared in include/bitlinear.h).
//
// Host side only: argument validation (before any CUDA call, so a bad call launches
// nothing), TMA tensor-map encoding, grid sizing and kernel launches.  All arithmetic
// of the path happens in the kernels included below; nothing here touches the data.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/bitlinear.h"
#include "common.cuh"
#include "act_quant.cuh"
#include "weight_quant.cuh"
#include "gemm_tc.cuh"
#include "gemm_simt.cuh"
#include "rmsnorm_bwd.cuh"
#include "gemv.cuh"
#include "optim.cuh"
#include "gemm_packed.cuh"
#include "gemm_packed2.cuh"
#include "mma_peak.cuh"
#include "read_peak.cuh"

// Scratch of bitlinear_quant_weight_noalloc: the pass-1 partial sums of |W| live in this
// file-scope device array instead of a caller workspace.  Every device that loads the
// library holds it until the process exits.  Host code must not pass the symbol itself to
// a kernel (on the host it names a host-side shadow, not device memory): the device
// address is looked up with cudaGetSymbolAddress once per device and passed instead.
static __device__ __align__(256) double g_quant_scratch[bl::kWqMaxPartials];

namespace {

thread_local std::string g_last_error = "no error";
std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_ns{2000000000ull};

bl_status fail(bl_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

#define BL_REQUIRE(cond, status, ...)                  \
    do {                                               \
        if (!(cond)) return fail(status, __VA_ARGS__); \
    } while (0)

#define BL_TRY(expr)                     \
    do {                                 \
        bl_status _s = (expr);           \
        if (_s != BL_OK) return _s;      \
    } while (0)

bl_status check_dims(int64_t T, int64_t N, int64_t K) {
    BL_REQUIRE(T >= 1 && N >= 1 && K >= 1, BL_ERR_INVALID_ARG, "sizes must be positive (T=%lld N=%lld K=%lld)",
               (long long)T, (long long)N, (long long)K);
    BL_REQUIRE(T <= kMaxDim && N <= kMaxDim && K <= kMaxDim, BL_ERR_UNSUPPORTED_SHAPE, "sizes must be < 2^31");
    BL_REQUIRE(K % 32 == 0, BL_ERR_UNSUPPORTED_SHAPE, "K (d_in) must be a multiple of 32, got %lld", (long long)K);
    BL_REQUIRE(N % 16 == 0, BL_ERR_UNSUPPORTED_SHAPE, "N (d_out) must be a multiple of 16, got %lld", (long long)N);
    return BL_OK;
}

bl_status check_ptr(const void* p, const char* name, bool required) {
    if (p == nullptr) {
        BL_REQUIRE(!required, BL_ERR_INVALID_ARG, "%s must not be NULL", name);
        return BL_OK;
    }
    BL_REQUIRE(aligned16(p), BL_ERR_MISALIGNED, "%s must be 16-byte aligned", name);
    return BL_OK;
}

bl_status check_dtype(bl_dtype dt) {
    BL_REQUIRE(dt == BL_F32 || dt == BL_BF16, BL_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    return BL_OK;
}

// ------------------------------------------------------------------------------------
// device checks
// ------------------------------------------------------------------------------------
struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int max_smem_optin = 0;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];
bool g_dev_ok[64] = {};

bl_status current_device(DeviceInfo* out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    BL_REQUIRE(dev >= 0 && dev < 64, BL_ERR_DEVICE, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev_ok[dev]) {
        DeviceInfo d;
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        e = cudaGetLastError();
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
        if (d.major != 10) return fail(BL_ERR_DEVICE, "device %d is sm_%d0; this library is built for sm_100a", dev, d.major);
        g_dev[dev] = d;
        g_dev_ok[dev] = true;
    }
    *out = g_dev[dev];
    return BL_OK;
}

bl_status launched(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return BL_OK;
}

// Every kernel is launched with programmatic dependent launch: its blocks may be scheduled
// while the previous kernel in the stream drains (each kernel signals this at its start),
// and each kernel runs its set-up (barriers, TMEM, descriptor prefetch) and then waits
// (griddepcontrol.wait) for the previous grid's completion and memory before it touches
// global memory.  After a kernel launched without the attribute the wait is a no-op.
template <typename... KArgs, typename... Args>
void pdl_launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);   // errors surface in launched()
}

// ------------------------------------------------------------------------------------
// TMA tensor maps
// ------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

enum TmType { kTmU8 = 0, kTmBf16 = 1, kTmF32 = 2, kTmI32 = 3 };

// 2-D row-major tensor [outer x inner] with 128-byte swizzled boxes [box_outer x box_inner]
// (box_inner * element size == 128 bytes).
bl_status make_tmap(CUtensorMap* tm, const void* base, TmType t, uint64_t inner, uint64_t outer,
                    uint32_t box_inner, uint32_t box_outer, bool swizzle128 = true) {
    EncodeTiledFn fn = encode_fn();
    BL_REQUIRE(fn != nullptr, BL_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const uint64_t esize = t == kTmU8 ? 1 : (t == kTmBf16 ? 2 : 4);
    const CUtensorMapDataType dt = t == kTmU8    ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : t == kTmBf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                   : t == kTmI32  ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * esize};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    BL_REQUIRE(r == CUDA_SUCCESS, BL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return BL_OK;
}

// 3-D map over int32 slices [outer][middle][inner] (no swizzle): the K-split partial sums,
// one box of box_inner x box_middle elements in one slice.
bl_status make_tmap3_i32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t middle, uint64_t outer,
                         uint32_t box_inner, uint32_t box_middle) {
    EncodeTiledFn fn = encode_fn();
    BL_REQUIRE(fn != nullptr, BL_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[3] = {inner, middle, outer};
    cuuint64_t strides[2] = {inner * 4, inner * middle * 4};
    cuuint32_t box[3] = {box_inner, box_middle, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    BL_REQUIRE(r == CUDA_SUCCESS, BL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return BL_OK;
}

// ------------------------------------------------------------------------------------
// tcgen05 GEMM launcher
// ------------------------------------------------------------------------------------
constexpr int kBN = 256;

template <bool kInt8, bool kAMN, bool kBMN, int kEpi>
bl_status launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td, bl::TcGemmArgs a,
                    cudaStream_t st, const DeviceInfo& dev) {
    auto kern = bl::tc_gemm_kernel<kInt8, kAMN, kBMN, kBN, kEpi>;
    const size_t smem = bl::tc_smem_bytes<kBN>();
    BL_REQUIRE((int)smem <= dev.max_smem_optin, BL_ERR_DEVICE, "GEMM needs %zu bytes of shared memory", smem);
    static std::atomic<uint64_t> attr_set{0};   // bit d: attribute set on device d
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    if (!(attr_set.load() & (1ull << dev_id))) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_set.fetch_or(1ull << dev_id);
    }
    a.m_tiles = (a.M + bl::kTcBM - 1) / bl::kTcBM;
    a.n_tiles = (a.N + kBN - 1) / kBN;
    const int kb_elems = kInt8 ? 128 : 64;
    a.k_blocks = (a.K + kb_elems - 1) / kb_elems;
    a.wait_ns = g_wait_ns.load();
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = tiles < dev.sms ? tiles : dev.sms;
    pdl_launch(kern, dim3(grid), dim3(bl::kTcThreads), smem, st, ta, tb, td, a);
    return launched("tc_gemm");
}

// 2-SM variant: clusters of two CTAs, 256 x 256 tiles.  The grid is as many clusters as
// fit on the device at once (queried once per device and kernel), at most one per tile.
template <bool kInt8, bool kAMN, bool kBMN, int kEpi>
bl_status launch_tc2(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td, bl::TcGemmArgs a,
                     cudaStream_t st, const DeviceInfo& dev) {
    auto kern = bl::tc_gemm2_kernel<kInt8, kAMN, kBMN, kEpi>;
    const size_t smem = bl::tc2_smem_bytes();
    BL_REQUIRE((int)smem <= dev.max_smem_optin, BL_ERR_DEVICE, "GEMM needs %zu bytes of shared memory", smem);
    static std::atomic<int> max_clusters[64] = {};
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    if (dev_id < 0 || dev_id >= 64) return fail(BL_ERR_DEVICE, "device ordinal %d out of range", dev_id);
    int mc = max_clusters[dev_id].load();
    if (mc == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(dev.sms / 2));
        cfg.blockDim = dim3(bl::kTcThreads);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s", cudaGetErrorString(e));
        if (n < 1) return fail(BL_ERR_DEVICE, "no 2-CTA cluster of the GEMM fits on the device");
        mc = n;
        max_clusters[dev_id].store(mc);
    }
    a.m_tiles = (a.M + 255) / 256;
    a.n_tiles = (a.N + 255) / 256;
    const int kb_elems = kInt8 ? 128 : 64;
    a.k_blocks = (a.K + kb_elems - 1) / kb_elems;
    a.wait_ns = g_wait_ns.load();
    const int tiles = a.m_tiles * a.n_tiles;
    const int clusters = tiles < mc ? tiles : mc;
    pdl_launch(kern, dim3(2 * clusters), dim3(bl::kTcThreads), smem, st, ta, tb, td, a);
    return launched("tc_gemm2");
}

// The 2-SM kernel computes 256-row tiles; for a single 128-row tile the 1-SM kernel wastes
// nothing and needs no partner CTA.
inline bool use_2sm(int64_t M) { return M > bl::kTcBM; }

// ------------------------------------------------------------------------------------
// pieces shared by the entry points (validation already done by the caller)
// ------------------------------------------------------------------------------------
// One row per block (the kernel can take R adjacent rows per block; measured slower here).
template <bool kBf16, int VPT>
void launch_act_quant_v(const void* X, int64_t T, int64_t K, int apply_norm, const float* g, float eps, int8_t* Xq,
                        float* sx, float* rinv, void* Xdq, cudaStream_t st) {
    constexpr int NT = bl::act_threads<kBf16>();
    constexpr int R = 1;
    const unsigned grid = (unsigned)((T + R - 1) / R);
    pdl_launch(bl::act_quant_kernel<kBf16, NT, VPT, R>, dim3(grid), dim3(NT), 0, st, X, (int)T, (int)K, apply_norm, g,
               eps, Xq, sx, rinv, Xdq);
}

// SM count of the current device (cached per device).
int sm_count() {
    static std::atomic<int> cache[64] = {};
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    if (dev_id < 0 || dev_id >= 64) return 148;
    int n = cache[dev_id].load();
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev_id) != cudaSuccess || n <= 0) n = 148;
        cache[dev_id].store(n);
    }
    return n;
}

// Persistent: two blocks of 8 row-warps per SM at most.
template <bool kBf16, int VPL>
void launch_act_quant_w(const void* X, int64_t T, int64_t K, int apply_norm, const float* g, float eps, int8_t* Xq,
                        float* sx, float* rinv, void* Xdq, cudaStream_t st) {
    const int64_t blocks = std::min<int64_t>((T + 7) / 8, 2 * (int64_t)sm_count());
    pdl_launch(bl::act_quant_warp_kernel<kBf16, VPL>, dim3((unsigned)blocks), dim3(256), 0, st, X, (int)T,
               (int)K, apply_norm, g, eps, Xq, sx, rinv, Xdq);
}

// Rows of at most 256 vectors (2048 bf16 / 1024 fp32 elements): warp per row; longer rows:
// block per row.
template <bool kBf16>
void launch_act_quant(const void* X, int64_t T, int64_t K, int apply_norm, const float* g, float eps, int8_t* Xq,
                      float* sx, float* rinv, void* Xdq, cudaStream_t st) {
    constexpr int NT = bl::act_threads<kBf16>();
    const int64_t nvec = K / (kBf16 ? 8 : 4);
    if (nvec <= 32) return launch_act_quant_w<kBf16, 1>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    if (nvec <= 64) return launch_act_quant_w<kBf16, 2>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    if (nvec <= 128) return launch_act_quant_w<kBf16, 4>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    // rows of 129-256 vectors: the warp-per-row kernel, except bf16 rows when there are at
    // most 8192 of them, where the block-per-row kernel's wider concurrency measured faster
    // (4096 x 2048 bf16: 10.0 against 11.2 us back to back; 16384 rows: 36.0 against 34.4 us;
    // fp32 4096 x 1024: 10.9 against 8.0 us)
    if (nvec <= 256 && (!kBf16 || T > 8192))
        return launch_act_quant_w<kBf16, 8>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    const int64_t vpt = (nvec + NT - 1) / NT;
    if (vpt <= 1) launch_act_quant_v<kBf16, 1>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else if (vpt <= 2) launch_act_quant_v<kBf16, 2>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else if (vpt <= 4) launch_act_quant_v<kBf16, 4>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else if (vpt <= 8) launch_act_quant_v<kBf16, 8>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else if (vpt <= 12) launch_act_quant_v<kBf16, 12>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else launch_act_quant_v<kBf16, 16>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
}

bl_status run_act_quant(const void* X, bl_dtype x_dt, int64_t T, int64_t K, int apply_norm, const float* g,
                        float eps, int8_t* Xq, float* sx, float* rinv, void* Xdq, cudaStream_t st) {
    if (x_dt == BL_BF16)
        launch_act_quant<true>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    else
        launch_act_quant<false>(X, T, K, apply_norm, g, eps, Xq, sx, rinv, Xdq, st);
    return launched("act_quant");
}

bl_status run_linear(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const int8_t* Wq, const float* gamma,
                     int64_t N, void* Y, bl_dtype y_dt, int32_t* acc, cudaStream_t st, const DeviceInfo& dev) {
    CUtensorMap ta, tb, td;
    const bool two = use_2sm(T);
    BL_TRY(make_tmap(&ta, Xq, kTmU8, (uint64_t)K, (uint64_t)T, 128, 128));
    BL_TRY(make_tmap(&tb, Wq, kTmU8, (uint64_t)K, (uint64_t)N, 128, two ? 128 : kBN));
    bl::TcGemmArgs a{};
    a.M = (int)T; a.N = (int)N; a.K = (int)K;
    a.acc_out = acc; a.row_scale = sx; a.gamma = gamma;
    if (y_dt == BL_BF16) {
        BL_TRY(make_tmap(&td, Y, kTmBf16, (uint64_t)N, (uint64_t)T, 64, 32));
        if (two) return launch_tc2<true, false, false, bl::kEpiLinearBf16>(ta, tb, td, a, st, dev);
        return launch_tc<true, false, false, bl::kEpiLinearBf16>(ta, tb, td, a, st, dev);
    }
    BL_TRY(make_tmap(&td, Y, kTmF32, (uint64_t)N, (uint64_t)T, 32, 32));
    if (two) return launch_tc2<true, false, false, bl::kEpiLinearF32>(ta, tb, td, a, st, dev);
    return launch_tc<true, false, false, bl::kEpiLinearF32>(ta, tb, td, a, st, dev);
}

// Per-column scales gamma_n: the 2-SM kernel at every T (its rows past T are zero-filled
// loads and clipped stores).
bl_status run_linear_rows(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const int8_t* Wq,
                          const float* gamma_rows, int64_t N, void* Y, bl_dtype y_dt, int32_t* acc, cudaStream_t st,
                          const DeviceInfo& dev) {
    CUtensorMap ta, tb, td;
    BL_TRY(make_tmap(&ta, Xq, kTmU8, (uint64_t)K, (uint64_t)T, 128, 128));
    BL_TRY(make_tmap(&tb, Wq, kTmU8, (uint64_t)K, (uint64_t)N, 128, 128));
    bl::TcGemmArgs a{};
    a.M = (int)T; a.N = (int)N; a.K = (int)K;
    a.acc_out = acc; a.row_scale = sx; a.gamma = gamma_rows;
    if (y_dt == BL_BF16) {
        BL_TRY(make_tmap(&td, Y, kTmBf16, (uint64_t)N, (uint64_t)T, 64, 32));
        return launch_tc2<true, false, false, bl::kEpiLinearColBf16>(ta, tb, td, a, st, dev);
    }
    BL_TRY(make_tmap(&td, Y, kTmF32, (uint64_t)N, (uint64_t)T, 32, 32));
    return launch_tc2<true, false, false, bl::kEpiLinearColF32>(ta, tb, td, a, st, dev);
}

bl_status run_grad_input_gemm(const void* dY, bl_dtype dt, const uint16_t* Wq_bf16, const float* gamma, int64_t T,
                              int64_t K, int64_t N, float* dXhat, cudaStream_t st, const DeviceInfo& dev) {
    if (dt == BL_BF16) {
        CUtensorMap ta, tb, td;
        BL_TRY(make_tmap(&ta, dY, kTmBf16, (uint64_t)N, (uint64_t)T, 64, 128));      // dY, K-major (contraction N)
        BL_TRY(make_tmap(&tb, Wq_bf16, kTmBf16, (uint64_t)K, (uint64_t)N, 64, 64));  // W_q, MN-major (rows = N)
        BL_TRY(make_tmap(&td, dXhat, kTmF32, (uint64_t)K, (uint64_t)T, 32, 32));
        bl::TcGemmArgs a{};
        a.M = (int)T; a.N = (int)K; a.K = (int)N;
        a.gamma = gamma;
        if (use_2sm(T)) return launch_tc2<false, false, true, bl::kEpiScaleF32>(ta, tb, td, a, st, dev);
        return launch_tc<false, false, true, bl::kEpiScaleF32>(ta, tb, td, a, st, dev);
    }
    // fp32 layer: CUDA-core fp32 contraction, C[t,k] = gamma * sum_n dY[t,n] W_q[n,k]
    dim3 grid((unsigned)((K + 63) / 64), (unsigned)((T + 63) / 64));
    pdl_launch(bl::simt_gemm_kernel<float, uint16_t>, grid, dim3(256), 0, st, (int)T, (int)K, (int)N,
               static_cast<const float*>(dY), N, (int64_t)1, Wq_bf16, (int64_t)1, K, gamma, dXhat, K);
    return launched("simt_gemm(grad_input)");
}

bl_status run_grad_weight_gemm(const void* dY, const void* Xdq, bl_dtype dt, int64_t T, int64_t K, int64_t N,
                               float* dW, cudaStream_t st, const DeviceInfo& dev) {
    if (dt == BL_BF16) {
        CUtensorMap ta, tb, td;
        BL_TRY(make_tmap(&ta, dY, kTmBf16, (uint64_t)N, (uint64_t)T, 64, 64));    // dY^T: MN-major (n contiguous)
        BL_TRY(make_tmap(&tb, Xdq, kTmBf16, (uint64_t)K, (uint64_t)T, 64, 64));   // X_dq: MN-major (k contiguous)
        BL_TRY(make_tmap(&td, dW, kTmF32, (uint64_t)K, (uint64_t)N, 32, 32));
        bl::TcGemmArgs a{};
        a.M = (int)N; a.N = (int)K; a.K = (int)T;
        if (use_2sm(N)) return launch_tc2<false, true, true, bl::kEpiF32>(ta, tb, td, a, st, dev);
        return launch_tc<false, true, true, bl::kEpiF32>(ta, tb, td, a, st, dev);
    }
    dim3 grid((unsigned)((K + 63) / 64), (unsigned)((N + 63) / 64));
    pdl_launch(bl::simt_gemm_kernel<float, float>, grid, dim3(256), 0, st, (int)N, (int)K, (int)T,
               static_cast<const float*>(dY), (int64_t)1, N, static_cast<const float*>(Xdq), (int64_t)1, K,
               static_cast<const float*>(nullptr), dW, K);
    return launched("simt_gemm(grad_weight)");
}

size_t quant_ws_bytes() { return sizeof(double) * bl::kWqMaxPartials; }

// Weight quantiser pass 2: gamma, threshold and codes (one round of kTqGroups groups per
// thread when the grid covers W).
// tau_factor < 0: the round/clamp threshold; else the zero threshold fl32(tau_factor * gamma).
bl_status run_ternary(const float* W, int64_t n, const double* partials, int parts, int8_t* Wq_i8, uint16_t* Wq_bf16,
                      uint8_t* Wpacked, float* gamma, cudaStream_t st, const DeviceInfo& dev,
                      float tau_factor = -1.0f) {
    const int64_t groups = n / 16;
    const int64_t per_block = (int64_t)bl::kWqThreads * bl::kTqGroups;
    int64_t blocks = (groups + per_block - 1) / per_block;
    const int64_t cap = (int64_t)dev.sms * 4;
    if (blocks > cap) blocks = cap;
    if (tau_factor >= 0.0f) {
        pdl_launch(bl::ternary_quant_kernel<true>, dim3((unsigned)blocks), dim3(bl::kWqThreads), 0, st, W, n,
                   partials, parts, Wq_i8, Wq_bf16, Wpacked, gamma, tau_factor);
        return launched("ternary_quant(tau)");
    }
    pdl_launch(bl::ternary_quant_kernel<false>, dim3((unsigned)blocks), dim3(bl::kWqThreads), 0, st, W, n, partials,
               parts, Wq_i8, Wq_bf16, Wpacked, gamma, 0.0f);
    return launched("ternary_quant");
}

// Weight quantiser: fp64 partial sums of |W| (pass 1), then pass 2.
bl_status run_quant_weight(const float* W, int64_t n, void* scratch, int8_t* Wq_i8, uint16_t* Wq_bf16,
                           uint8_t* Wpacked, float* gamma, cudaStream_t st, const DeviceInfo& dev,
                           float tau_factor = -1.0f) {
    double* partials = static_cast<double*>(scratch);
    const int parts = bl::wq_num_partials(n);
    pdl_launch(bl::absmean_partial_kernel, dim3(parts), dim3(bl::kWqThreads), 0, st, W, n, partials);
    BL_TRY(launched("absmean_partial"));
    return run_ternary(W, n, partials, parts, Wq_i8, Wq_bf16, Wpacked, gamma, st, dev, tau_factor);
}

// Optimizer scratch: dW^2 partials, |W_new| partials, the published step index.
constexpr size_t kOptWpartOffset = sizeof(double) * bl::kWqMaxPartials;
constexpr size_t kOptStepOffset = 2 * sizeof(double) * bl::kWqMaxPartials;
size_t opt_ws_bytes() { return kOptStepOffset + 16; }

size_t dg_ws_bytes(int64_t K) { return sizeof(float) * (size_t)bl::kBwdMaxBlocks * (size_t)K; }

// Persistent grid: as many blocks as are resident at once (queried once per device and
// instantiation), at most kBwdMaxBlocks and at most one per row.
template <bool kBf16X, int NT, int VPT, bool kGain>
int launch_rmsnorm_bwd_v(const void* X, const float* rinv, const float* g, float* dX, int64_t T, int64_t K,
                         float* partial, int sms, cudaStream_t st) {
    auto kern = bl::rmsnorm_bwd_kernel<kBf16X, NT, VPT, kGain>;
    static std::atomic<int> per_sm[64] = {};
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    int b = (dev_id >= 0 && dev_id < 64) ? per_sm[dev_id].load() : 0;
    if (b == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, NT, 0) != cudaSuccess || b < 1) b = 1;
        if (dev_id >= 0 && dev_id < 64) per_sm[dev_id].store(b);
    }
    int64_t grid = (int64_t)b * sms;
    if (grid > bl::kBwdMaxBlocks) grid = bl::kBwdMaxBlocks;
    if (grid > T) grid = T;
    pdl_launch(kern, dim3((unsigned)grid), dim3(NT), 0, st, X, rinv, g, dX, (int)T, (int)K, partial);
    return (int)grid;
}

// Block size: the smallest of 128 / 256 / 512 / 1024 threads that covers a row with at most
// four 16-byte column vectors per thread (K <= 16384).
template <bool kBf16X, bool kGain>
int launch_rmsnorm_bwd_g(const void* X, const float* rinv, const float* g, float* dX, int64_t T, int64_t K,
                         float* partial, int sms, cudaStream_t st) {
    const int64_t nvec = K / 4;
#define BL_BWD(NT)                                                                                              \
    if (nvec <= 4 * (NT)) {                                                                                     \
        const int64_t vpt = (nvec + (NT) - 1) / (NT);                                                          \
        if (vpt <= 1) return launch_rmsnorm_bwd_v<kBf16X, NT, 1, kGain>(X, rinv, g, dX, T, K, partial, sms, st); \
        if (vpt <= 2) return launch_rmsnorm_bwd_v<kBf16X, NT, 2, kGain>(X, rinv, g, dX, T, K, partial, sms, st); \
        if (vpt <= 3) return launch_rmsnorm_bwd_v<kBf16X, NT, 3, kGain>(X, rinv, g, dX, T, K, partial, sms, st); \
        return launch_rmsnorm_bwd_v<kBf16X, NT, 4, kGain>(X, rinv, g, dX, T, K, partial, sms, st);               \
    }
    BL_BWD(128)
    BL_BWD(256)
    BL_BWD(512)
    BL_BWD(1024)
#undef BL_BWD
    return 0;
}

template <bool kBf16X>
int launch_rmsnorm_bwd(const void* X, const float* rinv, const float* g, float* dX, int64_t T, int64_t K,
                       float* partial, int sms, cudaStream_t st) {
    if (g != nullptr) return launch_rmsnorm_bwd_g<kBf16X, true>(X, rinv, g, dX, T, K, partial, sms, st);
    return launch_rmsnorm_bwd_g<kBf16X, false>(X, rinv, g, dX, T, K, partial, sms, st);
}

bl_status run_rmsnorm_bwd(const void* X, bl_dtype dt, const float* rinv, const float* g, float* dX, int64_t T,
                          int64_t K, float* dg, void* ws, int sms, cudaStream_t st) {
    float* partial = dg != nullptr ? static_cast<float*>(ws) : nullptr;
    const int grid = dt == BL_BF16 ? launch_rmsnorm_bwd<true>(X, rinv, g, dX, T, K, partial, sms, st)
                                   : launch_rmsnorm_bwd<false>(X, rinv, g, dX, T, K, partial, sms, st);
    BL_TRY(launched("rmsnorm_bwd"));
    if (dg != nullptr) {
        pdl_launch(bl::dg_reduce_kernel, dim3((unsigned)((K + 31) / 32)), dim3(1024), 0, st,
                   static_cast<const float*>(partial), grid, (int)K, dg);
        BL_TRY(launched("dg_reduce"));
    }
    return BL_OK;
}

// ------------------------------------------------------------------------------------
// packed-weight GEMM: tile shape, K split and launch
// ------------------------------------------------------------------------------------
// Packed-weight GEMM on CTA pairs: 256-row weight tiles x bt tokens
// (bt = T rounded up to 32, at most 256), a K split when the tiles fill at most half the
// pairs, the activation ring, and the packed ring in the rest of shared memory.  The grid is
// as many pairs as fit at once, at most one per unit.
template <bool kBf16Out>
bl_status launch_packed2(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const uint8_t* Wpacked,
                         const float* gamma, int64_t N, void* Y, int32_t* acc, int32_t* scratch,
                         size_t scratch_bytes, cudaStream_t st, const DeviceInfo& dev) {
    bl::Pk2Args a2{};
    bl::PkArgs& a = a2.pk;
    a.T = (int)T; a.N = (int)N; a.K = (int)K;
    int64_t bt = (T + 31) / 32 * 32;
    if (bt > bl::kPkMaxBT) bt = bl::kPkMaxBT;
    a.bt = (int)bt;
    a.t_tiles = (int)((T + bt - 1) / bt);
    a.n_tiles = (int)((N + 2 * bl::kPk2Rows - 1) / (2 * bl::kPk2Rows));
    a.k_blocks = (int)((K + 127) / 128);
    const size_t budget = (size_t)dev.max_smem_optin;
    int pstages = (int)((budget - bl::pk2_smem_bytes((int)bt, 0)) / bl::kPkPBytes);
    pstages = std::min(pstages, bl::kPkMaxPStages);
    // the decoder warps stage their share of the last epilogue (16 x 8 KB) in the packed and
    // activation rings
    BL_REQUIRE(pstages >= 2 && (size_t)pstages * bl::kPkPBytes + (size_t)bl::kPk2DStages * bt * 128 >=
                                   16 * 2 * (size_t)bl::kPk2EpiBuf,
               BL_ERR_DEVICE, "packed GEMM: shared memory too small");
    a.pstages = pstages;
    auto kern = bl::tc_gemm_packed2_kernel<kBf16Out>;
    const size_t smem = bl::pk2_smem_bytes((int)bt, pstages);
    // pairs resident at once, per device and token-tile width (the shared memory differs)
    static std::atomic<int> max_clusters[64][bl::kPkMaxBT / 32] = {};
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    if (dev_id < 0 || dev_id >= 64) return fail(BL_ERR_DEVICE, "device ordinal %d out of range", dev_id);
    std::atomic<int>& mc_slot = max_clusters[dev_id][bt / 32 - 1];
    int mc = mc_slot.load();
    if (mc == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dev.max_smem_optin);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(dev.sms / 2));
        cfg.blockDim = dim3(bl::kPk2Threads);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s", cudaGetErrorString(e));
        if (n < 1) return fail(BL_ERR_DEVICE, "no 2-CTA cluster of the packed GEMM fits on the device");
        mc = n;
        mc_slot.store(mc);
    }
    const int64_t base = (int64_t)a.n_tiles * a.t_tiles;
    int splits = 1;
    if (2 * base <= mc) {
        // the partial sums and their second launch cost more than a second wave of units
        // returns, so K is split only when the tiles fill at most half the pairs, into as many
        // units as one wave holds, each at least 8 k-blocks (4 stages) long
        int64_t sp = std::min<int64_t>(8, (int64_t)mc / base);
        sp = std::min<int64_t>(sp, a.k_blocks / 8);
        sp = std::min<int64_t>(sp, (int64_t)(scratch_bytes / ((size_t)T * N * sizeof(int32_t))));
        splits = (int)std::max<int64_t>(1, sp);
    }
    a.splits = splits;
    a.sx = sx; a.gamma = gamma; a.y = Y;
    a.acc = splits > 1 ? scratch : acc;
    a.wait_ns = g_wait_ns.load();
    CUtensorMap tp, tx, ty, tacc;
    BL_TRY(make_tmap(&tp, Wpacked, kTmU8, (uint64_t)(K / 4), (uint64_t)N, 128, bl::kPk2Rows));
    BL_TRY(make_tmap(&tx, Xq, kTmU8, (uint64_t)K, (uint64_t)T, 128, (uint32_t)(bt / 2)));
    // the epilogue's TMA stores: 32 rows x 32 tokens per box, no swizzle
    BL_TRY(make_tmap(&ty, Y, kBf16Out ? kTmBf16 : kTmF32, (uint64_t)N, (uint64_t)T, 32, 32, false));
    std::memset(&tacc, 0, sizeof(tacc));
    if (splits > 1)
        BL_TRY(make_tmap3_i32(&tacc, scratch, (uint64_t)N, (uint64_t)T, (uint64_t)splits, 32, 32));
    else if (acc != nullptr)
        BL_TRY(make_tmap(&tacc, acc, kTmI32, (uint64_t)N, (uint64_t)T, 32, 32, false));
    const int64_t units = base * splits;
    const unsigned clusters = (unsigned)std::min<int64_t>(units, mc);
    pdl_launch(kern, dim3(2 * clusters), dim3(bl::kPk2Threads), smem, st, tp, tx, ty, tacc, a2);
    BL_TRY(launched("tc_gemm_packed2"));
    if (splits > 1) {
        const int64_t nv = T * N / 4;
        pdl_launch(bl::pk_finalize_kernel<kBf16Out>, dim3((unsigned)std::min<int64_t>((nv + 255) / 256, (int64_t)dev.sms * 8)),
                   dim3(256), 0, st, static_cast<const int32_t*>(scratch), splits, sx, gamma, (int)T, (int)N, Y, acc);
        BL_TRY(launched("pk_finalize"));
    }
    return BL_OK;
}

// Row kernels keep a whole row in registers: d_in is limited to 16384.
constexpr int64_t kMaxRowK = 16384;

// One block per SM (at most one per row group) of 16 warps (12 for two n-tiles, whose
// accumulators need more registers).
template <int NTILES, bool kBf16Out = false>
bl_status launch_gemv(const uint8_t* Wpacked, const float* gamma, int gamma_stride, int64_t N, int64_t K,
                      const int8_t* xq, const float* sx, int64_t B, void* y, int32_t* acc, cudaStream_t st,
                      const DeviceInfo& dev) {
    constexpr int WB = NTILES == 1 ? 16 : 12;
    const int64_t n_rg = N / 16;
    const int64_t nb = n_rg < dev.sms ? n_rg : dev.sms;
    const int max_rgs = (int)((n_rg + nb - 1) / nb);
    const size_t smem = bl::gemv_smem_bytes((int)B, (int)K, max_rgs);
    BL_REQUIRE(smem <= (size_t)dev.max_smem_optin, BL_ERR_UNSUPPORTED_SHAPE,
               "GEMV needs %zu bytes of shared memory for B = %lld, K = %lld; at most %d fit", smem, (long long)B,
               (long long)K, dev.max_smem_optin);
    auto kern = bl::ternary_gemv_kernel<NTILES, WB, kBf16Out>;
    static std::atomic<uint64_t> attr_set{0};   // bit d: attribute set on device d
    int dev_id = 0;
    cudaGetDevice(&dev_id);
    if (dev_id < 0 || dev_id >= 64) return fail(BL_ERR_DEVICE, "device ordinal %d out of range", dev_id);
    if (!(attr_set.load() & (1ull << dev_id))) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dev.max_smem_optin);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        attr_set.fetch_or(1ull << dev_id);
    }
    pdl_launch(kern, dim3((unsigned)nb), dim3(WB * 32), smem, st, Wpacked, gamma, gamma_stride, (int)N, (int)K, xq,
               sx, (int)B, y, acc, g_wait_ns.load());
    return launched("ternary_gemv");
}

}  // namespace

// ====================================================================================
// exported C ABI
// ====================================================================================
extern "C" {

int bl_abi_version(void) { return BITLINEAR_ABI_VERSION; }

const char* bl_last_error(void) { return g_last_error.c_str(); }

size_t bitlinear_workspace_bytes(int64_t T, int64_t N, int64_t K) {
    (void)T;
    (void)N;
    if (K < 0) K = 0;
    size_t a = quant_ws_bytes();
    size_t b = dg_ws_bytes(K);
    size_t m = a > b ? a : b;
    if (opt_ws_bytes() > m) m = opt_ws_bytes();
    return (m + 255) & ~size_t(255);
}

void bl_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns == 0 ? 2000000000ull : ns); }

uint64_t bl_launch_count(void) { return g_launches.load(); }

bl_status bl_check_device_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, bl::g_bl_status, sizeof(int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(bl::g_bl_status, &zero, sizeof(int));
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
    if (v != 0) return fail((bl_status)v, "a kernel reported status %d (bounded wait expired)", v);
    return BL_OK;
}

bl_status bitlinear_quant_weight(const float* W, int64_t N, int64_t K, int8_t* Wq_i8, uint16_t* Wq_bf16,
                                 uint8_t* Wpacked, float* gamma, void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", false));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_ptr(ws, "ws", true));
    BL_TRY(check_dims(1, N, K));
    BL_REQUIRE(ws_bytes >= quant_ws_bytes(), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu",
               quant_ws_bytes(), ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return run_quant_weight(W, N * K, ws, Wq_i8, Wq_bf16, Wpacked, gamma, st, dev);
}

bl_status bitlinear_act_quant(const void* X, bl_dtype x_dt, int64_t T, int64_t K, int apply_rmsnorm, const float* g,
                              float eps, int8_t* Xq, float* sx, float* rinv, void* Xdq, void* stream) {
    BL_TRY(check_dtype(x_dt));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(rinv, "rinv", apply_rmsnorm != 0));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(Xdq, "Xdq", false));
    BL_TRY(check_dims(T, 16, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    BL_REQUIRE(!(eps < 0.0f) && eps == eps, BL_ERR_INVALID_ARG, "eps must be >= 0");
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_act_quant(X, x_dt, T, K, apply_rmsnorm, g, eps, Xq, sx, rinv, Xdq, static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_linear(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const int8_t* Wq_i8,
                           const float* gamma, int64_t N, void* Y, bl_dtype y_dt, int32_t* acc, void* stream) {
    BL_TRY(check_dtype(y_dt));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Y, "Y", true));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_dims(T, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_linear(Xq, sx, T, K, Wq_i8, gamma, N, Y, y_dt, acc, static_cast<cudaStream_t>(stream), dev);
}

bl_status bitlinear_forward(const void* X, bl_dtype x_dt, int64_t T, int64_t K, const float* g, float eps,
                            const int8_t* Wq_i8, const float* gamma, int64_t N, void* Y, int8_t* Xq, float* sx,
                            float* rinv, void* Xdq, int32_t* acc, void* stream) {
    BL_TRY(check_dtype(x_dt));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Y, "Y", true));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(rinv, "rinv", true));
    BL_TRY(check_ptr(Xdq, "Xdq", false));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_dims(T, N, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    BL_REQUIRE(!(eps < 0.0f) && eps == eps, BL_ERR_INVALID_ARG, "eps must be >= 0");
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    BL_TRY(run_act_quant(X, x_dt, T, K, 1, g, eps, Xq, sx, rinv, Xdq, st));
    return run_linear(Xq, sx, T, K, Wq_i8, gamma, N, Y, x_dt, acc, st, dev);
}

bl_status bitlinear_forward_qat(const void* X, bl_dtype x_dt, int64_t T, int64_t K, const float* g, float eps,
                                const float* W, int64_t N, int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                float* gamma, void* Y, int8_t* Xq, float* sx, float* rinv, void* Xdq, int32_t* acc,
                                void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_dtype(x_dt));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", true));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Y, "Y", true));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(rinv, "rinv", true));
    BL_TRY(check_ptr(Xdq, "Xdq", false));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_ptr(ws, "ws", true));
    BL_TRY(check_dims(T, N, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    BL_REQUIRE(!(eps < 0.0f) && eps == eps, BL_ERR_INVALID_ARG, "eps must be >= 0");
    BL_REQUIRE(ws_bytes >= quant_ws_bytes(), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu",
               quant_ws_bytes(), ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the |W| partial sums, the ternary codes (their second read of W follows the first
    // directly, so it hits L2 when W fits there), the activation quantiser, then the GEMM
    const int64_t n = N * K;
    const int parts = bl::wq_num_partials(n);
    double* partials = static_cast<double*>(ws);
    pdl_launch(bl::absmean_partial_kernel, dim3(parts), dim3(bl::kWqThreads), 0, st, W, n, partials);
    BL_TRY(launched("absmean_partial"));
    BL_TRY(run_ternary(W, n, partials, parts, Wq_i8, Wq_bf16, Wpacked, gamma, st, dev));
    BL_TRY(run_act_quant(X, x_dt, T, K, 1, g, eps, Xq, sx, rinv, Xdq, st));
    return run_linear(Xq, sx, T, K, Wq_i8, gamma, N, Y, x_dt, acc, st, dev);
}

bl_status bitlinear_backward_input(const void* dY, const void* X, bl_dtype dt, int64_t T, int64_t K, int64_t N,
                                   const float* g, const float* rinv, const uint16_t* Wq_bf16, const float* gamma,
                                   float* dX, float* dg, void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_dtype(dt));
    BL_TRY(check_ptr(dY, "dY", true));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(rinv, "rinv", true));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(dX, "dX", true));
    BL_TRY(check_ptr(dg, "dg", false));
    BL_TRY(check_ptr(ws, "ws", dg != nullptr));
    BL_TRY(check_dims(T, N, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    if (dg != nullptr)
        BL_REQUIRE(ws_bytes >= dg_ws_bytes(K), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", dg_ws_bytes(K),
                   ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    BL_TRY(run_grad_input_gemm(dY, dt, Wq_bf16, gamma, T, K, N, dX, st, dev));
    return run_rmsnorm_bwd(X, dt, rinv, g, dX, T, K, dg, ws, dev.sms, st);
}

bl_status bitlinear_grad_input(const void* dY, bl_dtype dt, int64_t T, int64_t K, int64_t N, const uint16_t* Wq_bf16,
                               const float* gamma, float* dXhat, void* stream) {
    BL_TRY(check_dtype(dt));
    BL_TRY(check_ptr(dY, "dY", true));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(dXhat, "dXhat", true));
    BL_TRY(check_dims(T, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_grad_input_gemm(dY, dt, Wq_bf16, gamma, T, K, N, dXhat, static_cast<cudaStream_t>(stream), dev);
}

bl_status bitlinear_rmsnorm_backward(const void* X, bl_dtype dt, int64_t T, int64_t K, const float* g,
                                     const float* rinv, float* dX_inout, float* dg, void* ws, size_t ws_bytes,
                                     void* stream) {
    BL_TRY(check_dtype(dt));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(rinv, "rinv", true));
    BL_TRY(check_ptr(dX_inout, "dX", true));
    BL_TRY(check_ptr(dg, "dg", false));
    BL_TRY(check_ptr(ws, "ws", dg != nullptr));
    BL_TRY(check_dims(T, 16, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    if (dg != nullptr)
        BL_REQUIRE(ws_bytes >= dg_ws_bytes(K), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", dg_ws_bytes(K),
                   ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_rmsnorm_bwd(X, dt, rinv, g, dX_inout, T, K, dg, ws, dev.sms, static_cast<cudaStream_t>(stream));
}

bl_status bitlinear_backward_weight(const void* dY, const void* Xdq, bl_dtype dt, int64_t T, int64_t K, int64_t N,
                                    float* dW, void* stream) {
    BL_TRY(check_dtype(dt));
    BL_TRY(check_ptr(dY, "dY", true));
    BL_TRY(check_ptr(Xdq, "Xdq", true));
    BL_TRY(check_ptr(dW, "dW", true));
    BL_TRY(check_dims(T, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_grad_weight_gemm(dY, Xdq, dt, T, K, N, dW, static_cast<cudaStream_t>(stream), dev);
}

bl_status bitlinear_backward(const void* dY, const void* X, const void* Xdq, bl_dtype dt, int64_t T, int64_t K,
                             int64_t N, const float* g, const float* rinv, const uint16_t* Wq_bf16, const float* gamma,
                             float* dX, float* dW, float* dg, void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_ptr(Xdq, "Xdq", true));
    BL_TRY(check_ptr(dW, "dW", true));
    BL_TRY(bitlinear_backward_input(dY, X, dt, T, K, N, g, rinv, Wq_bf16, gamma, dX, dg, ws, ws_bytes, stream));
    return bitlinear_backward_weight(dY, Xdq, dt, T, K, N, dW, stream);
}

bl_status ternary_pack(const int8_t* Wq_i8, int64_t N, int64_t K, uint8_t* Wpacked, void* stream) {
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", true));
    BL_TRY(check_ptr(Wpacked, "Wpacked", true));
    BL_TRY(check_dims(1, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    const int64_t groups = N * K / 16;
    int64_t blocks = (groups + 255) / 256;
    if (blocks > (int64_t)dev.sms * 8) blocks = (int64_t)dev.sms * 8;
    pdl_launch(bl::ternary_pack_kernel, dim3((unsigned)blocks), dim3(256), 0, static_cast<cudaStream_t>(stream), Wq_i8,
               N * K, Wpacked);
    return launched("ternary_pack");
}

bl_status gemv_entry(const uint8_t* Wpacked, const float* gamma, int gamma_stride, int64_t N, int64_t K,
                     const int8_t* xq, const float* sx, int64_t B, float* y, int32_t* acc, void* stream);

bl_status ternary_gemv(const uint8_t* Wpacked, const float* gamma, int64_t N, int64_t K, const int8_t* xq,
                       const float* sx, int64_t B, float* y, int32_t* acc, void* stream) {
    return gemv_entry(Wpacked, gamma, 0, N, K, xq, sx, B, y, acc, stream);
}

bl_status ternary_gemv_rows(const uint8_t* Wpacked, const float* gamma_rows, int64_t N, int64_t K, const int8_t* xq,
                            const float* sx, int64_t B, float* y, int32_t* acc, void* stream) {
    return gemv_entry(Wpacked, gamma_rows, 1, N, K, xq, sx, B, y, acc, stream);
}

bl_status gemv_entry(const uint8_t* Wpacked, const float* gamma, int gamma_stride, int64_t N, int64_t K,
                     const int8_t* xq, const float* sx, int64_t B, float* y, int32_t* acc, void* stream) {
    BL_TRY(check_ptr(Wpacked, "Wpacked", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(xq, "xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(y, "y", true));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_dims(1, N, K));
    BL_REQUIRE(K % 64 == 0, BL_ERR_UNSUPPORTED_SHAPE,
               "the GEMV reads packed rows in 16-byte pieces: K must be a multiple of 64, got %lld", (long long)K);
    BL_REQUIRE(B >= 1 && B <= 16, BL_ERR_UNSUPPORTED_SHAPE, "batch must be in [1, 16], got %lld", (long long)B);
    BL_REQUIRE(K <= 65536, BL_ERR_UNSUPPORTED_SHAPE, "K must be <= 65536 for the GEMV, got %lld", (long long)K);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (B <= 8) return launch_gemv<1>(Wpacked, gamma, gamma_stride, N, K, xq, sx, B, y, acc, st, dev);
    return launch_gemv<2>(Wpacked, gamma, gamma_stride, N, K, xq, sx, B, y, acc, st, dev);
}

namespace {
// cuCtxGetCurrent through the runtime's driver entry point (the library does not link libcuda)
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

constexpr int kScratchDevices = 64;
struct ScratchAddr {
    CUcontext ctx;
    void* addr;
};
}  // namespace

bl_status bitlinear_quant_weight_noalloc(const float* W, int64_t N, int64_t K, int8_t* Wq_i8, uint16_t* Wq_bf16,
                                         uint8_t* Wpacked, float* gamma, void* stream) {
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", false));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_dims(1, N, K));
    const int64_t n = N * K;
    const int parts = bl::wq_num_partials(n);
    BL_REQUIRE(parts <= bl::kWqMaxPartials, BL_ERR_UNSUPPORTED_SHAPE,
               "the built-in scratch holds %d partial sums, this weight needs %d", bl::kWqMaxPartials, parts);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    // set-up, once per device and context: the device address of the scratch array.  The
    // address belongs to the context that loaded this module, so it is cached together with
    // that context and looked up again when the current context differs (after a
    // cudaDeviceReset the device gets a new primary context and the old address is gone).
    int dev_id = -1;
    cudaError_t e = cudaGetDevice(&dev_id);
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    BL_REQUIRE(dev_id >= 0 && dev_id < kScratchDevices, BL_ERR_INVALID_ARG,
               "device index %d is beyond the %d devices the scratch table covers", dev_id, kScratchDevices);
    CtxGetCurrentFn ctx_fn = ctx_get_current_fn();
    BL_REQUIRE(ctx_fn != nullptr, BL_ERR_CUDA, "cuCtxGetCurrent is unavailable");
    CUcontext ctx = nullptr;
    CUresult cr = ctx_fn(&ctx);
    BL_REQUIRE(cr == CUDA_SUCCESS && ctx != nullptr, BL_ERR_CUDA, "cuCtxGetCurrent failed (%d)", (int)cr);
    void* scratch = nullptr;
    {
        static std::mutex mu;
        static ScratchAddr cache[kScratchDevices] = {};
        std::lock_guard<std::mutex> lk(mu);
        if (cache[dev_id].addr == nullptr || cache[dev_id].ctx != ctx) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_quant_scratch);
            if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
            cache[dev_id].addr = p;
            cache[dev_id].ctx = ctx;
        }
        scratch = cache[dev_id].addr;
    }
    // pass 1 writes every partial that pass 2 reads, so nothing in the scratch needs clearing
    return run_quant_weight(W, n, scratch, Wq_i8, Wq_bf16, Wpacked, gamma, static_cast<cudaStream_t>(stream), dev);
}

// ------------------------------------------------------------------------------------
// quantiser variants
// ------------------------------------------------------------------------------------
bl_status bitlinear_quant_weight_rows(const float* W, int64_t N, int64_t K, int8_t* Wq_i8, uint16_t* Wq_bf16,
                                      uint8_t* Wpacked, float* gamma_rows, void* stream) {
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(gamma_rows, "gamma_rows", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", false));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_dims(1, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    pdl_launch(bl::ternary_quant_rows_kernel, dim3((unsigned)((N + 7) / 8)), dim3(256), 0,
               static_cast<cudaStream_t>(stream), W, (int)N, (int)K, Wq_i8, Wq_bf16, Wpacked, gamma_rows);
    return launched("ternary_quant_rows");
}

bl_status bitlinear_quant_weight_tau(const float* W, int64_t N, int64_t K, float tau_factor, int8_t* Wq_i8,
                                     uint16_t* Wq_bf16, uint8_t* Wpacked, float* gamma, void* ws, size_t ws_bytes,
                                     void* stream) {
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", false));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_ptr(ws, "ws", true));
    BL_TRY(check_dims(1, N, K));
    BL_REQUIRE(tau_factor >= 0.0f && tau_factor <= 1e30f, BL_ERR_INVALID_ARG,
               "tau_factor must be finite and >= 0, got %g", (double)tau_factor);
    BL_REQUIRE(ws_bytes >= quant_ws_bytes(), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu",
               quant_ws_bytes(), ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_quant_weight(W, N * K, ws, Wq_i8, Wq_bf16, Wpacked, gamma, static_cast<cudaStream_t>(stream), dev,
                            tau_factor);
}

bl_status bitlinear_act_quant_tensor(const void* X, bl_dtype x_dt, int64_t T, int64_t K, int apply_rmsnorm,
                                     const float* g, float eps, int8_t* Xq, float* sx, float* rinv, void* Xdq,
                                     void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_dtype(x_dt));
    BL_TRY(check_ptr(X, "X", true));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(rinv, "rinv", apply_rmsnorm != 0));
    BL_TRY(check_ptr(g, "g", false));
    BL_TRY(check_ptr(Xdq, "Xdq", false));
    BL_TRY(check_ptr(ws, "ws", true));
    BL_TRY(check_dims(T, 16, K));
    BL_REQUIRE(K <= kMaxRowK, BL_ERR_UNSUPPORTED_SHAPE, "d_in must be <= %lld for the row kernels, got %lld",
               (long long)kMaxRowK, (long long)K);
    BL_REQUIRE(!(eps < 0.0f) && eps == eps, BL_ERR_INVALID_ARG, "eps must be >= 0");
    BL_REQUIRE(ws_bytes >= sizeof(float) * bl::kActMaxPartials, BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu",
               sizeof(float) * bl::kActMaxPartials, ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t row_blocks = (T + 7) / 8;
    const int grid = (int)(row_blocks < bl::kActMaxPartials ? row_blocks : bl::kActMaxPartials);
    float* partials = static_cast<float*>(ws);
    if (x_dt == BL_BF16) {
        pdl_launch(bl::act_tensor_max_kernel<true>, dim3(grid), dim3(256), 0, st, X, (int)T, (int)K, apply_rmsnorm, g,
                   eps, rinv, partials);
        BL_TRY(launched("act_tensor_max"));
        pdl_launch(bl::act_tensor_quant_kernel<true>, dim3(grid), dim3(256), 0, st, X, (int)T, (int)K, apply_rmsnorm,
                   g, static_cast<const float*>(partials), grid, Xq, sx, static_cast<const float*>(rinv), Xdq);
    } else {
        pdl_launch(bl::act_tensor_max_kernel<false>, dim3(grid), dim3(256), 0, st, X, (int)T, (int)K, apply_rmsnorm,
                   g, eps, rinv, partials);
        BL_TRY(launched("act_tensor_max"));
        pdl_launch(bl::act_tensor_quant_kernel<false>, dim3(grid), dim3(256), 0, st, X, (int)T, (int)K, apply_rmsnorm,
                   g, static_cast<const float*>(partials), grid, Xq, sx, static_cast<const float*>(rinv), Xdq);
    }
    return launched("act_tensor_quant");
}

bl_status bitlinear_linear_rows(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const int8_t* Wq_i8,
                                const float* gamma_rows, int64_t N, void* Y, bl_dtype y_dt, int32_t* acc,
                                void* stream) {
    BL_TRY(check_dtype(y_dt));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", true));
    BL_TRY(check_ptr(gamma_rows, "gamma_rows", true));
    BL_TRY(check_ptr(Y, "Y", true));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_dims(T, N, K));
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    return run_linear_rows(Xq, sx, T, K, Wq_i8, gamma_rows, N, Y, y_dt, acc, static_cast<cudaStream_t>(stream), dev);
}

// ------------------------------------------------------------------------------------
// int8 x packed-ternary GEMM (few tokens)
// ------------------------------------------------------------------------------------
bl_status bitlinear_linear_packed(const int8_t* Xq, const float* sx, int64_t T, int64_t K, const uint8_t* Wpacked,
                                  const float* gamma, int64_t N, void* Y, bl_dtype y_dt, int32_t* acc, void* ws,
                                  size_t ws_bytes, void* stream) {
    BL_TRY(check_dtype(y_dt));
    BL_TRY(check_ptr(Xq, "Xq", true));
    BL_TRY(check_ptr(sx, "sx", true));
    BL_TRY(check_ptr(Wpacked, "Wpacked", true));
    BL_TRY(check_ptr(gamma, "gamma", true));
    BL_TRY(check_ptr(Y, "Y", true));
    BL_TRY(check_ptr(acc, "acc", false));
    BL_TRY(check_ptr(ws, "ws", false));
    BL_TRY(check_dims(T, N, K));
    BL_REQUIRE(K % 64 == 0, BL_ERR_UNSUPPORTED_SHAPE,
               "packed rows are read in 16-byte pieces: K must be a multiple of 64, got %lld", (long long)K);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    int32_t* scratch = static_cast<int32_t*>(ws);
    const size_t scratch_bytes = ws != nullptr ? ws_bytes : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Up to 16 tokens whose activation rows fit a block's shared memory: the decode GEMV's
    // kernel (codes decoded in registers, warp-level int8 MMA), which streams the packed
    // weight faster than the tensor-core tile with 16-column MMAs.
    if (T <= 16 && K <= 65536) {
        const int64_t n_rg = N / 16;
        const int64_t nb = n_rg < dev.sms ? n_rg : dev.sms;
        const int max_rgs = (int)((n_rg + nb - 1) / nb);
        if (bl::gemv_smem_bytes((int)T, (int)K, max_rgs) <= (size_t)dev.max_smem_optin) {
            if (y_dt == BL_BF16)
                return T <= 8 ? launch_gemv<1, true>(Wpacked, gamma, 0, N, K, Xq, sx, T, Y, acc, st, dev)
                              : launch_gemv<2, true>(Wpacked, gamma, 0, N, K, Xq, sx, T, Y, acc, st, dev);
            return T <= 8 ? launch_gemv<1, false>(Wpacked, gamma, 0, N, K, Xq, sx, T, Y, acc, st, dev)
                          : launch_gemv<2, false>(Wpacked, gamma, 0, N, K, Xq, sx, T, Y, acc, st, dev);
        }
    }
    // Otherwise (17 tokens or more, or rows too long for the GEMV): 2-SM tiles of 256 weight
    // rows with the decoded codes in tensor memory
    if (y_dt == BL_BF16)
        return launch_packed2<true>(Xq, sx, T, K, Wpacked, gamma, N, Y, acc, scratch, scratch_bytes, st, dev);
    return launch_packed2<false>(Xq, sx, T, K, Wpacked, gamma, N, Y, acc, scratch, scratch_bytes, st, dev);
}

// ------------------------------------------------------------------------------------
// optimizer step
// ------------------------------------------------------------------------------------
bl_status bitlinear_optimizer_step(float* W, const float* dW, float* m, float* v, int64_t N, int64_t K, float lr,
                                   float beta1, float beta2, float eps, float weight_decay, float max_norm,
                                   int32_t* step, int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked, float* gamma,
                                   void* ws, size_t ws_bytes, void* stream) {
    BL_TRY(check_ptr(W, "W", true));
    BL_TRY(check_ptr(dW, "dW", true));
    BL_TRY(check_ptr(m, "m", true));
    BL_TRY(check_ptr(v, "v", true));
    BL_TRY(check_ptr(step, "step", true));
    BL_TRY(check_ptr(gamma, "gamma", false));
    BL_TRY(check_ptr(Wq_i8, "Wq_i8", false));
    BL_TRY(check_ptr(Wq_bf16, "Wq_bf16", false));
    BL_TRY(check_ptr(Wpacked, "Wpacked", false));
    BL_TRY(check_ptr(ws, "ws", true));
    BL_TRY(check_dims(1, N, K));
    BL_REQUIRE(gamma != nullptr || (Wq_i8 == nullptr && Wq_bf16 == nullptr && Wpacked == nullptr), BL_ERR_INVALID_ARG,
               "the next step's codes need gamma");
    BL_REQUIRE(lr >= 0.0f && lr <= 1e30f, BL_ERR_INVALID_ARG, "lr must be finite and >= 0");
    BL_REQUIRE(beta1 >= 0.0f && beta1 < 1.0f && beta2 >= 0.0f && beta2 < 1.0f, BL_ERR_INVALID_ARG,
               "betas must be in [0, 1)");
    BL_REQUIRE(eps > 0.0f && eps <= 1e30f, BL_ERR_INVALID_ARG, "eps must be finite and > 0");
    BL_REQUIRE(weight_decay >= 0.0f && weight_decay <= 1e30f, BL_ERR_INVALID_ARG,
               "weight_decay must be finite and >= 0");
    BL_REQUIRE(max_norm == max_norm && max_norm <= 1e30f, BL_ERR_INVALID_ARG, "max_norm must be finite");
    BL_REQUIRE(ws_bytes >= opt_ws_bytes(), BL_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", opt_ws_bytes(),
               ws_bytes);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n = N * K;
    const int parts = bl::wq_num_partials(n);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    double* gpart = reinterpret_cast<double*>(wsb);
    double* wpart = reinterpret_cast<double*>(wsb + kOptWpartOffset);
    int32_t* step_next = reinterpret_cast<int32_t*>(wsb + kOptStepOffset);
    bl::AdamwArgs a{};
    a.lr = lr;
    a.beta1 = beta1;
    a.beta2 = beta2;
    a.eps = eps;
    a.decay = (float)(1.0 - (double)lr * (double)weight_decay);
    a.omb1 = (float)(1.0 - (double)beta1);
    a.omb2 = (float)(1.0 - (double)beta2);
    a.max_norm = max_norm;
    pdl_launch(bl::grad_sumsq_partial_kernel, dim3(parts), dim3(bl::kWqThreads), 0, st, dW, n, gpart,
               static_cast<const int32_t*>(step), step_next);
    BL_TRY(launched("grad_sumsq_partial"));
    pdl_launch(bl::adamw_clamp_kernel, dim3(parts), dim3(bl::kWqThreads), 0, st, W, dW, m, v, n,
               static_cast<const double*>(gpart), parts, a, static_cast<const int32_t*>(step_next), step,
               gamma != nullptr ? wpart : static_cast<double*>(nullptr));
    BL_TRY(launched("adamw_clamp"));
    if (gamma == nullptr) return BL_OK;
    // the next step's codes from the |W_new| partials written above (the quantiser's pass 2)
    return run_ternary(W, n, wpart, parts, Wq_i8, Wq_bf16, Wpacked, gamma, st, dev);
}

bl_status bl_mma_peak_probe(int kind, int pair, int iters, double* ops_out, void* stream) {
    BL_REQUIRE(kind >= 0 && kind <= 2, BL_ERR_INVALID_ARG, "kind must be 0 (int8), 1 (bf16) or 2 (mma.sync int8), got %d",
               kind);
    BL_REQUIRE(pair == 0 || pair == 1, BL_ERR_INVALID_ARG, "pair must be 0 or 1, got %d", pair);
    BL_REQUIRE(iters >= 1 && iters <= (1 << 20), BL_ERR_INVALID_ARG, "iters must be in [1, 2^20], got %d", iters);
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    if (kind == 2) {
        // per instruction 16 x 8 x 32 multiply-adds; every warp of every SM runs kImmaChains per iteration
        if (ops_out)
            *ops_out = 2.0 * 16 * 8 * 32 * (double)bl::kImmaChains * bl::kImmaWarps * dev.sms * (double)iters;
        pdl_launch(bl::imma_sync_peak_kernel, dim3((unsigned)dev.sms), dim3(bl::kImmaWarps * 32), 0,
                   static_cast<cudaStream_t>(stream), iters);
        return launched("imma_sync_peak");
    }
    BL_REQUIRE(bl::kPeakSmemBytes <= dev.max_smem_optin, BL_ERR_DEVICE, "probe needs %d bytes of shared memory",
               bl::kPeakSmemBytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint64_t wait_ns = g_wait_ns.load();
    int ctas = pair ? 2 * (dev.sms / 2) : dev.sms;
    void (*kern)(int, uint64_t) = nullptr;
    if (pair) kern = kind == 0 ? bl::mma_peak2_kernel<true> : bl::mma_peak2_kernel<false>;
    else kern = kind == 0 ? bl::mma_peak_kernel<true> : bl::mma_peak_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bl::kPeakSmemBytes);
    if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    if (pair) {
        // no more clusters than can be resident at once: every pair runs in the same wave
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ctas);
        cfg.blockDim = dim3(bl::kPeakThreads);
        cfg.dynamicSmemBytes = bl::kPeakSmemBytes;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return fail(BL_ERR_CUDA, "cudaOccupancyMaxActiveClusters: %s", cudaGetErrorString(e));
        if (n < 1) return fail(BL_ERR_DEVICE, "no 2-CTA cluster of the probe fits on the device");
        ctas = std::min(ctas, 2 * n);
    }
    // multiply-adds x 2 of the launch: per instruction M x N x (32 bytes of K)
    const double k_per_instr = kind == 0 ? 32.0 : 16.0;
    const double per_instr = 2.0 * (pair ? 256.0 * 256.0 : 128.0 * 256.0) * k_per_instr;
    const double units = pair ? ctas / 2 : ctas;
    if (ops_out) *ops_out = units * 4.0 * (double)iters * per_instr;
    pdl_launch(kern, dim3((unsigned)ctas), dim3(bl::kPeakThreads), (size_t)bl::kPeakSmemBytes, st, iters, wait_ns);
    return launched("mma_peak");
}

bl_status bl_read_peak_probe(const uint8_t* buf, int64_t rows, int64_t row_bytes, int pattern, uint32_t* sink,
                             void* stream) {
    BL_TRY(check_ptr(buf, "buf", true));
    BL_TRY(check_ptr(sink, "sink", true));
    BL_REQUIRE(pattern == 0 || pattern == 1, BL_ERR_INVALID_ARG, "pattern must be 0 (GEMV) or 1 (coalesced), got %d",
               pattern);
    BL_REQUIRE(rows >= 16 && rows % 16 == 0 && rows <= (1 << 30), BL_ERR_UNSUPPORTED_SHAPE,
               "rows must be a positive multiple of 16 (at most 2^30), got %lld", (long long)rows);
    BL_REQUIRE(row_bytes >= 64 && row_bytes % 64 == 0 && row_bytes <= (1 << 24), BL_ERR_UNSUPPORTED_SHAPE,
               "row_bytes must be a positive multiple of 64 (at most 2^24), got %lld", (long long)row_bytes);
    // keeps a block's step count (32-bit in the kernel) in range
    BL_REQUIRE(rows * row_bytes <= (int64_t(1) << 40), BL_ERR_UNSUPPORTED_SHAPE, "buffer larger than 2^40 bytes");
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n_rg = rows / 16;
    if (pattern == 0) {
        // as the GEMV: one block per SM, at most one per row group
        const unsigned nb = (unsigned)std::min<int64_t>(n_rg, dev.sms);
        pdl_launch(bl::read_peak_gemv_kernel, dim3(nb), dim3(bl::kReadWarps * 32), 0, st, buf, (int)rows,
                   (int)row_bytes, sink);
    } else {
        pdl_launch(bl::read_peak_coalesced_kernel, dim3((unsigned)dev.sms), dim3(bl::kReadWarps * 32), 0, st,
                   reinterpret_cast<const uint4*>(buf), rows * row_bytes / 16, sink);
    }
    return launched("read_peak");
}

bl_status bl_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
    BL_REQUIRE(limit_ns > 0 && limit_ns <= 10000000000ull, BL_ERR_INVALID_ARG, "limit must be in (0, 10 s]");
    DeviceInfo dev;
    BL_TRY(current_device(&dev));
    pdl_launch(bl::selftest_wait_kernel, dim3(1), dim3(32), 0, static_cast<cudaStream_t>(stream), limit_ns);
    return launched("selftest_wait");
}

}  // extern "C"

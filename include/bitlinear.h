/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitNet b1.58 BitLinear hot path.
 *
 * Source pages (titles), cited per entry point below:
 *   P1 = "BitNet量化感知训练中的梯度传播优化：解决符号函数不可微性的工程实践" (blog.hotdry.top)
 *   P2 = "BitNet 三元权重量化训练工程：直通估计器与梯度裁剪实践" (blog.hotdry.top)
 *   P3 = "BitNet 1.5技术解析：2比特量化在神经网络中的应用与挑战" (intelliparadigm.com)
 *   P4 = "BitNet b1.58：三元权重下的STE设计与优化" (zyxy.net)
 *   P5 = "1.58-bit量化技术突破AI算力与内存墙限制" (intelliparadigm.com)
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * Shapes follow nn.Linear (P3 §3.1): the latent weight W is [N x K] row-major
 * (N = d_out, K = d_in), activations X are [T x K] row-major (T tokens), the output
 * Y is [T x N].  All matrices are dense row-major with no padding.
 *
 * Memory and ownership: every pointer is DEVICE memory owned by the caller and must
 * stay valid until the work queued on `stream` has finished.  The library allocates
 * no device or host memory.  Entry points that need scratch take a caller workspace
 * (`ws`, `ws_bytes`); `bitlinear_workspace_bytes()` gives a size that suffices.
 * gamma, s_x and r live on the device so a training step never syncs to the host.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 * Every entry point is asynchronous on that stream.
 *
 * Sizes and alignment (validated on the host before anything is launched):
 *   - T >= 1, N >= 1, K >= 1; K % 32 == 0 (whole 64-bit words of 2-bit codes per row,
 *     P5 §5.1); N % 16 == 0 (16-byte aligned rows of Y and dY for TMA and vector
 *     stores); every pointer 16-byte aligned; T, N, K < 2^31;
 *   - K <= 16384 for the entry points with a per-token row kernel (act quant, forward,
 *     backward input, RMSNorm backward): those kernels hold a whole row in registers.
 * Numerics: fp32 quantiser arithmetic with round-half-to-even (torch.round in the
 * pages' snippets), fp64 reductions, exact int32 accumulation for the int8 x ternary
 * contraction.  Inputs must be finite.
 *
 * Errors: every entry point returns a bl_status.  A non-OK status from validation
 * means nothing was launched.  BL_ERR_CUDA reports a launch error (the message,
 * retrievable with bl_last_error(), names the CUDA error).  Kernels never trap:
 * every wait inside a kernel is bounded, and a wait that runs out records
 * BL_ERR_TIMEOUT in a device status word that bl_check_device_status() reads.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BL_API __attribute__((visibility("default")))
#else
#define BL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BL_OK = 0,
    BL_ERR_INVALID_ARG = 1,        /* null required pointer, non-positive size, bad dtype */
    BL_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 32, N % 16, or a size beyond the limits above  */
    BL_ERR_MISALIGNED = 3,         /* a pointer not 16-byte aligned                       */
    BL_ERR_WORKSPACE = 4,          /* ws too small (or NULL with ws_bytes needed)          */
    BL_ERR_CUDA = 5,               /* CUDA runtime / driver error                          */
    BL_ERR_TIMEOUT = 6,            /* a bounded device wait expired                        */
    BL_ERR_DEVICE = 7              /* the current device is not an sm_100 (B200) GPU        */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1 } bl_dtype;

/* ABI version of this header (bumped on any signature change). */
#define BITLINEAR_ABI_VERSION 1
BL_API int bl_abi_version(void);

/* Message of the last non-OK status returned on this host thread (never NULL). */
BL_API const char* bl_last_error(void);

/* Bytes of workspace that suffice for every entry point on a layer of this size. */
BL_API size_t bitlinear_workspace_bytes(int64_t T, int64_t N, int64_t K);

/* Synchronises `stream`, then reads and clears the device status word written by
 * bounded waits on the current device.  Returns BL_OK, BL_ERR_TIMEOUT or BL_ERR_CUDA. */
BL_API bl_status bl_check_device_status(void* stream);

/* Upper bound, in nanoseconds, of any single wait inside a kernel launched after this
 * call (default 2e9).  0 restores the default. */
BL_API void bl_set_wait_limit_ns(uint64_t ns);

/* Number of kernels this library has launched in this process (all devices). */
BL_API uint64_t bl_launch_count(void);

/* ------------------------------------------------------------------------------
 * Weight quantiser: per-tensor absmean ternary (P3 §2.1 weight_quant; P5 §2.2
 * ternary_quantize; P2 "直通估计器在三元权重量化中的作用").
 *   gamma = max( mean_{n,k} |W[n,k]|, 1e-5 )        (mean accumulated in fp64)
 *   W_q   = clamp( round( W / gamma ), -1, 1 )        (fp32 division, half-to-even)
 * Outputs (each optional, may be NULL):
 *   Wq_i8    int8  [N x K]   codes -1/0/+1 (operand of the forward GEMM)
 *   Wq_bf16  bf16  [N x K]   the same codes as bf16 bits (operand of the backward)
 *   Wpacked  uint8 [N x K/4] 2-bit codes 00->0, 01->+1, 10->-1 (P5 §4.1); element k
 *            of row n at byte n*K/4 + k/4, bits 2*(k%4)+{0,1}
 *   gamma    fp32  [1]       required
 * W: fp32 [N x K].  ws: at least bitlinear_workspace_bytes(1, N, K) bytes.
 * Deterministic: the same W gives bit-identical outputs on every call. */
BL_API bl_status bitlinear_quant_weight(const float* W, int64_t N, int64_t K,
                                 int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                 float* gamma, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------
 * bitlinear_quant_weight without a workspace.  (Not from the pages: they have no
 * counterpart; it exists for callers.)  Some callers cannot allocate device memory at
 * all -- for example a serving process whose device memory is handed out by another
 * allocator that owns the whole pool -- so they cannot pass the workspace that
 * bitlinear_quant_weight needs for its per-block partial sums of |W|.  This variant
 * computes exactly the same gamma and codes (bit-identical outputs), but keeps those
 * partial sums in a scratch array compiled into the library: 1184 fp64 values
 * (9,472 bytes) per device, held by every GPU that loads the library until the process
 * exits.  It allocates nothing and calls no allocating routine.
 *   - Sizes: any N x K accepted by bitlinear_quant_weight fits (the number of partial
 *     sums is capped at 1184); a weight that needed more would be rejected with
 *     BL_ERR_UNSUPPORTED_SHAPE.
 *   - Set-up: the first call on each device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with the device's
 *     current context; a call that finds another context current (after cudaDeviceReset)
 *     looks it up again.  Make the first call on a device, and the first after a reset,
 *     before any stream capture.  Device ordinals 0..63 are covered; a call on a device
 *     beyond them returns BL_ERR_INVALID_ARG.
 *   - Sharing: all calls on a device share the one array and it keeps the last call's
 *     contents.  Nothing in it needs to start at zero (every partial a call reads was
 *     written by that call), but calls that overlap on the GPU (for example on two
 *     streams) race on it: serialise them. */
BL_API bl_status bitlinear_quant_weight_noalloc(const float* W, int64_t N, int64_t K,
                                         int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                         float* gamma, void* stream);

/* ------------------------------------------------------------------------------
 * Activation quantiser with optional RMSNorm in front (P3 §3.1 RMSNorm before
 * activation_quant; P3 §2.2 activation_quant; P2 per-token absmax 8-bit).
 *   r_t   = 1 / sqrt( mean_k X[t,k]^2 + eps )        (fp64 sum; only if apply_rmsnorm)
 *   x_hat = X * r_t * g_k                            (x_hat = X if !apply_rmsnorm)
 *   s_t   = 127 / max( max_k |x_hat[t,k]|, 1e-5 )
 *   X_q   = clamp( round( x_hat * s_t ), -128, 127 )
 *   X_dq  = X_q / s_t   (rounded to x_dt; the value the straight-through estimator
 *                        forwards, saved for the weight gradient)
 * X: [T x K] of x_dt.  g: fp32 [K] or NULL (gain 1).  Outputs: Xq int8 [T x K],
 * sx fp32 [T] (required); rinv fp32 [T] (required iff apply_rmsnorm); Xdq [T x K]
 * of x_dt (optional). */
BL_API bl_status bitlinear_act_quant(const void* X, bl_dtype x_dt, int64_t T, int64_t K,
                              int apply_rmsnorm, const float* g, float eps,
                              int8_t* Xq, float* sx, float* rinv, void* Xdq, void* stream);

/* ------------------------------------------------------------------------------
 * The int8 x ternary contraction with its rescale (P3 §3.1 F.linear(x_quant, w_quant)
 * * scale; P5 §3.1 add / subtract / skip):
 *   acc[t,n] = sum_k X_q[t,k] * W_q[n,k]          exact int32 (tcgen05 kind::i8)
 *   Y[t,n]   = acc[t,n] * (gamma / s_t)            fp32 (the factor formed once per token),
 *                                                  then rounded to y_dt
 * Xq int8 [T x K], sx fp32 [T], Wq_i8 int8 [N x K], gamma fp32 [1] (device).
 * Y [T x N] of y_dt.  acc int32 [T x N] optional (debug / parity). */
BL_API bl_status bitlinear_linear(const int8_t* Xq, const float* sx, int64_t T, int64_t K,
                           const int8_t* Wq_i8, const float* gamma, int64_t N,
                           void* Y, bl_dtype y_dt, int32_t* acc, void* stream);

/* ------------------------------------------------------------------------------
 * BitLinear forward (P3 §3.1): bitlinear_act_quant(apply_rmsnorm = 1) followed by
 * bitlinear_linear with y_dt = x_dt.  Saves Xq, sx, rinv (required) and Xdq
 * (optional, needed by bitlinear_backward_weight) for the backward. */
BL_API bl_status bitlinear_forward(const void* X, bl_dtype x_dt, int64_t T, int64_t K,
                            const float* g, float eps,
                            const int8_t* Wq_i8, const float* gamma, int64_t N,
                            void* Y, int8_t* Xq, float* sx, float* rinv, void* Xdq,
                            int32_t* acc, void* stream);

/* ------------------------------------------------------------------------------
 * Quantisation-aware forward from the fp32 latent weight: what P3 §3.1's BitLinear.forward
 * computes (RMSNorm, activation_quant, weight_quant, then the linear), A1-A6 in one call:
 * the weight quantiser's fp64 partial sums of |W|, the ternary codes, the activation
 * quantiser, then the GEMM.
 * Outputs: those of bitlinear_quant_weight (Wq_i8 required here -- the GEMM operand --,
 * Wq_bf16 and Wpacked optional, gamma) and of bitlinear_forward; all bit-identical to
 * bitlinear_quant_weight followed by bitlinear_forward.
 * ws: at least bitlinear_workspace_bytes(T, N, K) bytes (no initialisation needed). */
BL_API bl_status bitlinear_forward_qat(const void* X, bl_dtype x_dt, int64_t T, int64_t K,
                                const float* g, float eps, const float* W, int64_t N,
                                int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked, float* gamma,
                                void* Y, int8_t* Xq, float* sx, float* rinv, void* Xdq,
                                int32_t* acc, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------
 * Straight-through backward, input side (P3 §3.2; P5 §3.2 TernarySTE returns
 * grad_output unchanged; P4 §3.2 grad_w = grad_output), then the RMSNorm backward:
 *   dX_hat[t,k] = gamma * sum_n dY[t,n] * W_q[n,k]            (fp32 accumulation)
 *   u = X * r,  h = g * dX_hat,  c_t = (1/K) sum_k h u
 *   dX[t,k]     = r_t * ( h - u * c_t )
 *   dg[k]       = sum_t dX_hat[t,k] * u[t,k]                  (optional)
 * dY [T x N] and X [T x K] of dt; g fp32 [K] or NULL; rinv fp32 [T] from the forward;
 * Wq_bf16 bf16 [N x K] codes; gamma fp32 [1].  dX fp32 [T x K] (gradients in fp32,
 * P2 "bf16 for forward, fp32 for gradients"); dg fp32 [K] or NULL.
 * ws: at least bitlinear_workspace_bytes(T, N, K) bytes when dg != NULL. */
BL_API bl_status bitlinear_backward_input(const void* dY, const void* X, bl_dtype dt,
                                   int64_t T, int64_t K, int64_t N,
                                   const float* g, const float* rinv,
                                   const uint16_t* Wq_bf16, const float* gamma,
                                   float* dX, float* dg, void* ws, size_t ws_bytes,
                                   void* stream);

/* The two halves of bitlinear_backward_input, callable on their own:
 *   bitlinear_grad_input:       dX_hat = gamma * dY . W_q   -> fp32 [T x K]
 *   bitlinear_rmsnorm_backward: dX = RMSNorm backward of dX_hat, computed IN PLACE over
 *                               the fp32 buffer that holds dX_hat; dg optional. */
BL_API bl_status bitlinear_grad_input(const void* dY, bl_dtype dt, int64_t T, int64_t K, int64_t N,
                               const uint16_t* Wq_bf16, const float* gamma, float* dXhat,
                               void* stream);
BL_API bl_status bitlinear_rmsnorm_backward(const void* X, bl_dtype dt, int64_t T, int64_t K,
                                     const float* g, const float* rinv, float* dX_inout,
                                     float* dg, void* ws, size_t ws_bytes, void* stream);

/* Straight-through backward, weight side (P3 §3.2: the gradient reaches the fp32
 * latent weight):  dW[n,k] = sum_t dY[t,n] * X_dq[t,k]   (fp32 accumulation).
 * dY [T x N] and Xdq [T x K] of dt; dW fp32 [N x K]. */
BL_API bl_status bitlinear_backward_weight(const void* dY, const void* Xdq, bl_dtype dt,
                                    int64_t T, int64_t K, int64_t N, float* dW,
                                    void* stream);

/* Both halves of the backward on one stream. */
BL_API bl_status bitlinear_backward(const void* dY, const void* X, const void* Xdq, bl_dtype dt,
                             int64_t T, int64_t K, int64_t N,
                             const float* g, const float* rinv,
                             const uint16_t* Wq_bf16, const float* gamma,
                             float* dX, float* dW, float* dg,
                             void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------
 * 2-bit packing of ternary codes (P5 §4.1; P5 §5.1 64-bit boundaries): Wq_i8 int8
 * [N x K] with values in {-1,0,1} -> Wpacked uint8 [N x K/4], layout as in
 * bitlinear_quant_weight.  Values outside {-1,0,1} are packed as 0. */
BL_API bl_status ternary_pack(const int8_t* Wq_i8, int64_t N, int64_t K, uint8_t* Wpacked,
                       void* stream);

/* ------------------------------------------------------------------------------
 * Decode GEMV over packed ternary weights (P5 §3.1 W=+1 -> y += x, W=-1 -> y -= x,
 * W=0 -> skip; P5 §4.1 codes, reserved 11 decodes to 0):
 *   acc[b,n] = sum_k decode(Wpacked[n,k]) * xq[b,k]   exact int32
 *   y[b,n]   = acc[b,n] * (gamma / sx[b])              fp32
 * Wpacked uint8 [N x K/4]; gamma fp32 [1]; xq int8 [B x K]; sx fp32 [B];
 * y fp32 [B x N]; acc int32 [B x N] optional.  1 <= B <= 16, K <= 65536, and K % 64 == 0
 * (packed rows are read in 16-byte pieces and activation rows are bulk-copied, both of
 * which need 16-byte aligned rows).
 * A block keeps B activation rows (B * K bytes) in shared memory: shapes whose rows do not
 * fit (e.g. B * K well above 160 KB) return BL_ERR_UNSUPPORTED_SHAPE. */
BL_API bl_status ternary_gemv(const uint8_t* Wpacked, const float* gamma, int64_t N, int64_t K,
                       const int8_t* xq, const float* sx, int64_t B,
                       float* y, int32_t* acc, void* stream);

/* ==============================================================================
 * Quantiser variants the pages print beside the b1.58 defaults.  Same conventions,
 * sizes, rounding and error behaviour as the entry points above.
 * ============================================================================== */

/* Per-row weight scale (P4 §9 "Quantizer": scale = mean |W| over each output row),
 * with the b1.58 round/clamp (P3 §2.1, P5 §2.2):
 *   gamma_rows[n] = max( (float)(sum_k |W[n,k]| / K), 1e-5 )   fp64 sum
 *   W_q[n,k]      = clamp(round(fl32(W[n,k] / gamma_rows[n])), -1, 1)
 * Outputs as bitlinear_quant_weight, except that Wq_bf16 holds the dequantised weight
 * W_q[n,k] * bf16(gamma_rows[n]) (bf16 bits; the operand of the backward contraction, to
 * be used with a gamma of 1.0), and gamma_rows is fp32 [N].  No workspace. */
BL_API bl_status bitlinear_quant_weight_rows(const float* W, int64_t N, int64_t K,
                                      int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                      float* gamma_rows, void* stream);

/* Zero threshold (P2, "直通估计器在三元权重量化中的作用": tau = 0.7 x scale, |W| < tau
 * quantises to 0), with the per-tensor gamma of bitlinear_quant_weight:
 *   tau = fl32(tau_factor * gamma);  W_q = 0 if |W| < tau, else sign(W)  (sign(0) = 0)
 * tau_factor finite and >= 0 (0.7 on the page; 0.5 reproduces the round rule except at
 * exact ties), else BL_ERR_INVALID_ARG.  Outputs and workspace as bitlinear_quant_weight. */
BL_API bl_status bitlinear_quant_weight_tau(const float* W, int64_t N, int64_t K, float tau_factor,
                                     int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                     float* gamma, void* ws, size_t ws_bytes, void* stream);

/* Per-tensor activation scale (P5 §5.1 quantize_activation: one 127 / max|x| for the
 * whole tensor), applied to x_hat as in bitlinear_act_quant:
 *   s    = fl32(127 / max(max_{t,k} |x_hat[t,k]|, 1e-5)),  written to sx[t] for every t
 *   X_q  = clamp(round(fl32(x_hat * s)), -128, 127),  X_dq = fl32(X_q / s)
 * Arguments as bitlinear_act_quant plus ws: at least bitlinear_workspace_bytes(T, N, K)
 * bytes (block maxima).  Two launches; X is read twice. */
BL_API bl_status bitlinear_act_quant_tensor(const void* X, bl_dtype x_dt, int64_t T, int64_t K,
                                     int apply_rmsnorm, const float* g, float eps,
                                     int8_t* Xq, float* sx, float* rinv, void* Xdq,
                                     void* ws, size_t ws_bytes, void* stream);

/* The int8 x ternary linear with a per-row weight scale (the weight rows are the output
 * columns):  y[t,n] = fl32( (float)acc[t,n] * fl32(gamma_rows[n] / sx[t]) ).
 * Arguments as bitlinear_linear with gamma_rows fp32 [N]. */
BL_API bl_status bitlinear_linear_rows(const int8_t* Xq, const float* sx, int64_t T, int64_t K,
                                const int8_t* Wq_i8, const float* gamma_rows, int64_t N,
                                void* Y, bl_dtype y_dt, int32_t* acc, void* stream);

/* The decode GEMV with a per-row weight scale: y[b,n] = acc[b,n] * fl32(gamma_rows[n] / sx[b]).
 * Arguments and limits as ternary_gemv with gamma_rows fp32 [N]. */
BL_API bl_status ternary_gemv_rows(const uint8_t* Wpacked, const float* gamma_rows, int64_t N, int64_t K,
                            const int8_t* xq, const float* sx, int64_t B,
                            float* y, int32_t* acc, void* stream);

/* ==============================================================================
 * int8 x packed-ternary linear for few tokens (prefill chunks, batched decode): the
 * linear of bitlinear_linear computed from the 2-bit packed weight (P5 §4.1 codes, §5.1
 * packing; a quarter of the int8 weight bytes cross HBM), decoded to int8 on chip and
 * multiplied on the tensor cores (P3 §3.1):
 *   acc[t,n] = sum_k decode(Wpacked[n,k]) * Xq[t,k]     exact int32 (reserved 11 -> 0)
 *   Y[t,n]   = fl32(acc[t,n] * fl32(gamma / sx[t]))     in y_dt
 * Xq int8 [T x K]; sx fp32 [T]; Wpacked uint8 [N x K/4]; gamma fp32 [1]; Y [T x N];
 * acc int32 [T x N] optional.  K % 64 == 0.  Meant for T up to a few hundred tokens
 * (beyond that bitlinear_linear on the int8 codes is compute-bound and faster).
 * Kernels by token count:
 *   up to 16 tokens, when their activation rows fit one block's shared memory: the decode
 *     GEMV's kernel (codes decoded in registers, warp-level int8 MMA; ws unused);
 *   otherwise: CTA pairs with 256 weight rows x up to 256 tokens per tile (codes decoded
 *     into tensor memory, 2-SM tcgen05 MMAs, TMA-stored output).
 * When the weight tiles fill at most half of the CTA pairs, K may be split: split sp stores
 * its exact int32 partial sums to slice sp of ws (int32 [splits x T x N]) and a second launch
 * adds the slices in split order and applies the scale.  The split count is limited by
 * ws_bytes / (4 T N) (ws NULL: no split), by 8, by K / 1024 and by one wave of pairs.
 * One or two launches. */
BL_API bl_status bitlinear_linear_packed(const int8_t* Xq, const float* sx, int64_t T, int64_t K,
                                  const uint8_t* Wpacked, const float* gamma, int64_t N,
                                  void* Y, bl_dtype y_dt, int32_t* acc, void* ws, size_t ws_bytes,
                                  void* stream);

/* ==============================================================================
 * Optimizer step of the latent weight, fused with the next step's weight quantiser
 * (clip -> AdamW -> clamp, in the pages' order):
 *   gradient clipping per weight matrix (P5 §6.2: clip_grad_norm_(p, 1.0)):
 *     c = min(1, max_norm / (||dW||_2 + 1e-6)), c = 1 when max_norm <= 0;  g = c dW
 *   AdamW (P1 optimizer configuration: lr 1e-3, betas (0.9, 0.95), weight decay 0.01,
 *   eps 1e-6), decoupled decay, bias-corrected moments, step t:
 *     m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
 *     W <- W (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 *   clamp (P1 "梯度裁剪与权重约束"): W <- clamp(W, -1, 1).
 * W, m, v fp32 [N x K] are updated in place; dW fp32 [N x K] (after any all-reduce) is
 * read only.  step: device int32 holding the number of steps taken so far; this call uses
 * t = *step + 1 and stores t back (so the call can be replayed in a CUDA graph).
 * Element arithmetic is fp32 (one rounding per operation); the norm is an fp64 sum.
 * If gamma is not NULL the call also produces the NEXT step's ternary weights from the
 * updated W exactly as bitlinear_quant_weight would (same partial sums, same gamma, same
 * codes; Wq_i8 / Wq_bf16 / Wpacked optional), reusing |W| sums taken during the update.
 * Hyper-parameters must be finite with lr >= 0, 0 <= betas < 1, eps > 0, wd >= 0, else
 * BL_ERR_INVALID_ARG.  ws: at least bitlinear_workspace_bytes(T, N, K) bytes.
 * Three launches with gamma, two without; all HBM-bound. */
BL_API bl_status bitlinear_optimizer_step(float* W, const float* dW, float* m, float* v,
                                   int64_t N, int64_t K, float lr, float beta1, float beta2,
                                   float eps, float weight_decay, float max_norm, int32_t* step,
                                   int8_t* Wq_i8, uint16_t* Wq_bf16, uint8_t* Wpacked,
                                   float* gamma, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------------
 * Tensor-pipe peak probe (a measurement kernel with no counterpart on the pages): one
 * launch in which every CTA (or CTA pair) issues iters x 4 tcgen05.mma from fixed
 * pseudo-random shared-memory operands into one TMEM accumulator, with no global-memory
 * traffic, so the achieved rate is the tensor pipe's ceiling for the GEMMs' instruction
 * shapes.  kind 0 = kind::i8 (s8 x s8 -> s32, 32 values of K per instruction), 1 = kind::f16
 * (bf16 x bf16 -> f32, 16 values).  pair 0 = cta_group::1, M = 128 x N = 256 on every SM;
 * pair 1 = cta_group::2, M = 256 x N = 256 on every resident pair of SMs.  kind 2 = the
 * warp-level mma.sync m16n8k32 (u8 x s8 -> s32) of the decode GEMV, from registers, 16 warps
 * per SM with 8 independent accumulators each (pair ignored).  iters in [1, 2^20].  ops_out (host pointer, may be NULL) receives 2 x the multiply-adds of the
 * launch; divide by the launch's duration (CUDA events on `stream`) for the rate. */
BL_API bl_status bl_mma_peak_probe(int kind, int pair, int iters, double* ops_out, void* stream);

/* ------------------------------------------------------------------------------
 * Read-bandwidth probe (a measurement kernel with no counterpart on the pages): one launch
 * that reads every byte of buf, a [rows x row_bytes] uint8 device array, once and does no
 * arithmetic with it, giving the read-only ceiling against which the decode GEMV's weight
 * stream is judged.  pattern 0 reads it as the decode GEMV reads a packed weight (one block
 * per SM, balanced 16-row groups, 64-byte column steps, 8 rows x 64 bytes per warp load);
 * pattern 1 reads contiguous equal spans per block, 512 bytes per warp load.  rows: a
 * positive multiple of 16 (at most 2^30); row_bytes: a positive multiple of 64 (at most
 * 2^24); rows x row_bytes at most 2^40; buf 16-byte aligned.  sink: one device uint32 that the kernel writes only if the
 * XOR of all loads equals a fixed constant (the buffer's owner may ignore it).  Launched with
 * programmatic dependent launch like the GEMV; time it with CUDA events on `stream`. */
BL_API bl_status bl_read_peak_probe(const uint8_t* buf, int64_t rows, int64_t row_bytes, int pattern, uint32_t* sink,
                                    void* stream);

/* ------------------------------------------------------------------------------
 * Self-test of the bounded-wait machinery: launches one block that waits on an
 * mbarrier nothing arrives on, with the given limit (ns), and returns.  Afterwards
 * bl_check_device_status() must report BL_ERR_TIMEOUT.  No counterpart on the pages. */
BL_API bl_status bl_selftest_bounded_wait(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */

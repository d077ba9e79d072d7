/*
 * bitlinear.h -- C ABI of libbitlinear.so: binarized linear layers on
 * NVIDIA B200 (sm_100a).
 *
 * Two layers and the step that feeds them:
 *   - FBI-linear (W1A16): "FBI-LLM: Fully Binarized Large Language Model"
 *     (MarkTechPost article as rewritten on cloudsagepro.com), the paragraph
 *     defining FBI-linear and the experiments paragraph (W1A16).
 *   - BitLinear (W1A8): "BitNet b1.58: 1bit LLM 时代" (coreui.cn), section 1
 *     (BitNet), Eq.(1)-(8).
 *   - bin_pack: the binarisation of those two passages (sign of W, or of
 *     W minus its mean) written as 1-bit planes plus the scales.
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or equivalent)
 *     unless a parameter says otherwise. The caller owns every buffer; the
 *     library allocates nothing on any call path.
 *   - Layouts are row-major and dense. Activations x are bf16, passed as raw
 *     16-bit patterns (uint16_t). Weights W are fp32.
 *   - Packed sign planes: row j of an N x K sign matrix is K/32 uint32 words;
 *     element (j,k) is bit (k mod 32) of word [j*(K/32) + k/32]; a set bit is
 *     +1, a clear bit -1. (The pages give no layout; this is the library's.)
 *   - Shapes: M >= 0 tokens, N >= 1 output channels, K >= 128 inputs with
 *     K % 128 == 0 (so a packed row is a whole number of 16-byte chunks).
 *     M == 0 is a valid no-op. Every pointer must be 16-byte aligned.
 *     M*K, N*K and M*N must each be below 2^40.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronise it. Argument errors are returned
 *     before anything is enqueued. Launch errors are returned as
 *     BL_ERR_CUDA. Faults detected inside a kernel (a bounded wait that ran
 *     out) are recorded in a per-device error word, read by bl_device_error.
 *   - No C++ exception crosses this boundary. Thread-safe: the library keeps
 *     no mutable host state apart from per-device one-time set-up.
 *   - Buffers passed to one call must not overlap, except that inputs may
 *     alias other inputs.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define BL_OK 0
#define BL_ERR_INVALID_ARG (-1) /* null pointer, negative size, misalignment    */
#define BL_ERR_UNSUPPORTED (-2) /* shape outside the supported set (K % 128)     */
#define BL_ERR_CUDA (-3)        /* a CUDA runtime/driver call or launch failed   */
#define BL_ERR_TIMEOUT (-4)     /* a kernel's bounded wait ran out (device word) */
#define BL_ERR_NO_DEVICE (-5)   /* no usable sm_100 device is current            */
#define BL_ERR_SCRATCH_LIMIT (-6) /* problem too big for the fixed scratch of       */
                                  /* bitlinear_w1a8_noalloc                         */

/* ---- bin_pack modes ----------------------------------------------------- */
#define BL_PACK_FBI 0     /* sign(W), per-output-channel alpha                */
#define BL_PACK_BITNET 1  /* sign(W - mean W), global alpha and beta          */
#define BL_PACK_TERNARY 2 /* b1.58: RoundClip(W / (mean|W| + eps)), two planes */

/* ---- ops for bl_workspace_bytes ----------------------------------------- */
#define BL_OP_PACK_FBI 0
#define BL_OP_PACK_BITNET 1
#define BL_OP_W1A16 2
#define BL_OP_W1A8 3
#define BL_OP_PACK_TERNARY 4
#define BL_OP_W158A8 5
#define BL_OP_W1A8_EX 6 /* bitlinear_w1a8_ex with a per-tensor quantiser */
#define BL_OP_W1A16_STACK 7 /* bin_linear_w1a16_stack(_batch) (M tokens, N = total outputs; K ignored) */
#define BL_OP_W1A16_BACKWARD 8 /* bin_linear_w1a16_backward */

/* Library ABI version (this header: 1). */
int bl_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* bl_status_string(int status);

/* Bytes of device workspace the call `op` needs for the given shape (0 when
 * it needs none). Host-only: touches no device. Returns 0 for invalid
 * shapes too; the call itself reports those. */
size_t bl_workspace_bytes(int op, int64_t M, int64_t N, int64_t K);

/*
 * bin_pack -- binarise W [N x K] fp32 into packed sign planes plus scales.
 *
 * mode BL_PACK_FBI ("FBI-LLM" page, FBI-linear paragraph):
 *   s_jk = Sign(W_jk) with Sign(v) = +1 if v > 0 else -1 (BitNet Eq.(2));
 *   alpha[j] = (1/K) * sum_k |W_jk|  -- one scale per output channel,
 *   accumulated in fp64 and rounded once to fp32. `alpha` has N floats.
 *   `beta` is unused (may be NULL). No workspace (ws may be NULL).
 * mode BL_PACK_BITNET ("BitNet b1.58" page, section 1, Eq.(1)-(3), (8)):
 *   a = (1/NK) * sum W (fp64);  s_jk = Sign(W_jk - a) compared in fp64;
 *   beta = (1/NK) * sum |W| (fp64, unshifted W).
 *   alpha[0] = (float)a (informational), beta[0] = (float)beta.
 *   Needs ws of bl_workspace_bytes(BL_OP_PACK_BITNET, 0, N, K) bytes.
 * mode BL_PACK_TERNARY ("BitNet b1.58" page, section 2, Eq.(9)-(11)):
 *   g = (1/NK) * sum |W| (fp64);  W~_jk = RoundClip(W_jk / (g + 1e-5), -1, 1)
 *   with round half to even and the division in fp64 (so +1 iff the quotient
 *   exceeds 1/2, -1 iff it is below -1/2, else 0). beta[0] = (float)g, the
 *   scale of the forward; `alpha` is unused (may be NULL). packed is
 *   [N x K/16] uint32: per row, per 128-k block, 4 words of the +1 plane then
 *   4 words of the -1 plane (element k at bit k mod 32 of word (k mod 128)/32
 *   of each plane; never both bits). Needs ws of
 *   bl_workspace_bytes(BL_OP_PACK_TERNARY, 0, N, K) bytes.
 * Outputs: packed [N x K/32] uint32 (layout above; [N x K/16] for
 * BL_PACK_TERNARY). All device pointers.
 */
int bin_pack(const float* W, int64_t N, int64_t K, int mode, uint32_t* packed, float* alpha,
             float* beta, void* ws, size_t ws_bytes, void* stream);

/*
 * bin_linear_w1a16 -- FBI-linear forward, 1-bit weights, bf16 activations
 * ("FBI-LLM" page: sign(W) times a full-precision per-output-channel scale;
 * W1A16 configuration of its experiments paragraph):
 *   y[m][j] = bf16( alpha[j] * sum_k s_jk * x[m][k] )
 * x [M x K] bf16, packed [N x K/32], alpha [N] fp32 (any values: the page
 * only initialises them), y [M x N] bf16 (round to nearest even).
 * Accumulation is fp32. A single token uses a lookup-table GEMV (a cluster
 * of CTAs splits K; signed byte sums of x are tabulated in shared memory);
 * 2 to 16 tokens with K % 256 == 0 and K <= 12288 a GEMV whose products run
 * on the warp-level MMA; other shapes of up to 4 tokens a predicated-add
 * GEMV; more tokens a tcgen05 tensor-core GEMM. No workspace.
 */
int bin_linear_w1a16(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y,
                     int64_t M, int64_t N, int64_t K, void* stream);

/*
 * bin_linear_w1a16_ex -- bin_linear_w1a16 with launch flags.
 *   BL_FLAG_OVERLAP_PREVIOUS: the caller promises that `packed` and `alpha`
 *   are not written by the kernel enqueued immediately before this call on
 *   `stream` (true for a chain of inference layers). The lookup-table and
 *   warp-MMA GEMVs (1 to 16 tokens) may then start streaming the weights
 *   before that kernel has finished (programmatic dependent launch); they
 *   still wait for it before reading x or writing y. Other kernels ignore the flag. flags = 0 is exactly
 *   bin_linear_w1a16.
 */
#define BL_FLAG_OVERLAP_PREVIOUS 1u
int bin_linear_w1a16_ex(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y,
                        int64_t M, int64_t N, int64_t K, unsigned flags, void* stream);

/*
 * bin_linear_w1a16_backward -- gradients of the FBI-linear forward with the
 * straight-through estimator ("FBI-LLM" page, FBI-linear paragraph: the
 * estimator carries the gradient through the sign function; no clipping
 * window is given, so ds/dW is taken as 1). With z = S x (before alpha) and
 * the incoming gradient dy [M x N] bf16:
 *   dx[m][k]  = bf16( sum_j dy[m][j] * alpha[j] * s_jk )
 *   dw[j][k]  = alpha[j] * sum_m dy[m][j] * x[m][k]          (fp32)
 *   dalpha[j] = sum_m dy[m][j] * z[m][j] = sum_k s_jk * sum_m dy[m][j] x[m][k]   (fp32)
 * x [M x K] bf16, packed [N x K/32] and alpha [N] as in the forward. dx may
 * be NULL (not computed); dw and dalpha are both given or both NULL. dx
 * takes dy * alpha split into two bf16 parts through the forward kernels;
 * the products over m run on the tensor cores with fp32 accumulation.
 * K % 128 == 0 and N % 128 == 0. ws: bl_workspace_bytes(BL_OP_W1A16_BACKWARD,
 * M, N, K) bytes of device memory, 16-byte aligned. M == 0 zero-fills dw and
 * dalpha.
 */
int bin_linear_w1a16_backward(const uint16_t* x, const uint32_t* packed, const float* alpha,
                              const uint16_t* dy, uint16_t* dx, float* dw, float* dalpha, int64_t M,
                              int64_t N, int64_t K, void* ws, size_t ws_bytes, void* stream);

/*
 * bin_linear_w1a16_stack -- single-token decode through a stack of FBI-linear
 * layers in one persistent launch (the same y = bf16(alpha * sum s x) as
 * bin_linear_w1a16 at M = 1, for every linear of the stack).
 *
 * The stack is a sequence of levels. Level i reads one input vector
 * levels[i].x (K bf16) and runs the linears jobs[first_job .. first_job +
 * num_jobs), each writing its own y (N bf16). levels[i].x is either exactly
 * the y of one linear of an earlier level (same pointer, N == K) or a buffer
 * written before the call that no linear of the stack writes; every linear's
 * y is a buffer of its own (no two overlap). Other stacks are rejected with
 * BL_ERR_INVALID_ARG. A level starts as soon as its own input is complete.
 * Limits: K a multiple of 256, 256 <= K <= 12288; 1 <= N < 2^31; x and
 * packed 16-byte aligned. Results are bit-identical to bin_linear_w1a16
 * whenever that call splits K eight ways (K/32 words a multiple of 8, 128..384
 * of them, e.g. K = 4096 and 11008).
 * The weights of the levels ahead stream into shared memory while a level
 * waits for its input. The call enqueues at most one zero-fill of ws and one
 * kernel per 96 levels (or per 144 linears) on `stream`. ws:
 * bl_workspace_bytes(BL_OP_W1A16_STACK, 0, total_N, 0) bytes of device
 * memory, 16-byte aligned, not shared with a call still running, where
 * total_N is the sum of N over the stack's linears. The kernel needs every
 * one of its CTAs resident at once (one per SM in clusters of 8): if the GPU
 * cannot host them all it records BL_ERR_TIMEOUT (bl_device_error) instead of
 * waiting forever.
 */
typedef struct bl_stack_job {
  const uint32_t* packed; /* [N x K/32] */
  const float* alpha;     /* [N] */
  uint16_t* y;            /* [N] bf16 */
  int64_t N;
} bl_stack_job;
typedef struct bl_stack_level {
  const uint16_t* x; /* [K] bf16 */
  int64_t K;
  int32_t first_job;
  int32_t num_jobs;
} bl_stack_level;
int bin_linear_w1a16_stack(const bl_stack_level* levels, int num_levels, const bl_stack_job* jobs,
                           int num_jobs, void* ws, size_t ws_bytes, void* stream);

/*
 * bin_linear_w1a16_stack_batch -- bin_linear_w1a16_stack for a decode batch
 * of M tokens (1 <= M <= 16): every level's x is [M x K] and every linear's y
 * [M x N] (bf16, row-major), y[m][j] = bf16(alpha[j] * sum_k s_jk x[m][k])
 * for each token. The rules on inputs and outputs are those of
 * bin_linear_w1a16_stack, with buffers of M rows. M == 1 is exactly
 * bin_linear_w1a16_stack; for M >= 2 the products run on the warp-level
 * tensor-core MMA (fp32 accumulation), with the same weight streaming. ws:
 * bl_workspace_bytes(BL_OP_W1A16_STACK, M, total_N, 0) bytes.
 */
int bin_linear_w1a16_stack_batch(const bl_stack_level* levels, int num_levels, const bl_stack_job* jobs,
                                 int num_jobs, int64_t M, void* ws, size_t ws_bytes, void* stream);

/*
 * bitlinear_w1a8 -- BitNet BitLinear forward ("BitNet b1.58" page,
 * section 1, Eq.(4)-(5), (7)-(8)), per token m:
 *   mu = mean_k x,  var = mean_k (x - mu)^2,  ln_k = (x_k - mu)/sqrt(var + 1e-5)
 *   gamma_m = max_k |ln_k|
 *   q_mk = clamp(round_half_even(ln_k * 128 / gamma_m), -127, 127)  (0 if gamma_m == 0)
 *   acc[m][j] = sum_k s_jk * q_mk        (exact int32)
 *   y[m][j] = fp32( acc * beta * gamma_m / 128 )   (the exact value rounded once; within 1 ulp
 *                                                 of that rounding near rounding midpoints)
 * LN statistics and the quantisation decision are taken in fp64.
 * x [M x K] bf16, packed [N x K/32] (from BL_PACK_BITNET), beta: DEVICE
 * pointer to one float (so pack -> forward needs no host round trip),
 * y [M x N] fp32. Needs ws of bl_workspace_bytes(BL_OP_W1A8, M, N, K) bytes
 * (the int8 codes and per-token gamma live there between the two kernels).
 * Kernels: for M <= 16 with K <= 1024 and M * K <= 16384 one launch does
 * everything; otherwise the LN + quantisation kernel, then for up to 16
 * tokens a GEMV on the warp-level int8 MMA (K % 256 == 0, K <= 12288) or on
 * dp4a (other K), for more tokens the tcgen05 int8 GEMM.
 */
int bitlinear_w1a8(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                   int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes, void* stream);

/*
 * bitlinear_w1a8_debug -- the same kernels as bitlinear_w1a8, also exporting
 * the intermediates for two-level parity checks. Any of the extra outputs
 * may be NULL. xq_out [M x K] int8 codes, gamma_out [M] fp64, acc_out
 * [M x N] int32 accumulators. If xq_in is non-NULL the LN/quantisation step
 * is skipped and (xq_in [M x K] int8, gamma_in [M] fp64) are used instead.
 */
int bitlinear_w1a8_debug(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                         int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                         int8_t* xq_out, double* gamma_out, int32_t* acc_out,
                         const int8_t* xq_in, const double* gamma_in, void* stream);

/*
 * bitlinear_w158a8 -- BitNet b1.58 BitLinear forward ("BitNet b1.58" page,
 * section 2: the ternary weights of Eq.(9)-(11) in the forward of section 1,
 * whose LN and activation quantisation b1.58 keeps). Exactly bitlinear_w1a8
 * with acc[m][j] = sum_k W~_jk * q_mk (W~ in {-1, 0, +1}, exact int32) and
 * beta = the mean |W| from bin_pack(BL_PACK_TERNARY). packed [N x K/16]
 * (two planes, layout of BL_PACK_TERNARY). Needs ws of
 * bl_workspace_bytes(BL_OP_W158A8, M, N, K) bytes (same as BL_OP_W1A8).
 */
int bitlinear_w158a8(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                     int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes, void* stream);

/* bitlinear_w158a8_debug -- bitlinear_w158a8 with the extra outputs and
 * inputs of bitlinear_w1a8_debug. */
int bitlinear_w158a8_debug(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                           int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                           int8_t* xq_out, double* gamma_out, int32_t* acc_out,
                           const int8_t* xq_in, const double* gamma_in, void* stream);

/*
 * bitlinear_w1a8_ex -- bitlinear_w1a8 / bitlinear_w158a8 with the other
 * activation quantisers of the "BitNet b1.58" page, section 1:
 *   BL_W1A8_PER_TENSOR  Eq.(5) as printed, gamma = ||LN(x)||_inf over the
 *                       whole M x K matrix (shared by every token); codes
 *                       clamp(rne(LN * 128 / gamma), -127, 127).
 *   BL_W1A8_NONNEG      Eq.(6), for activations before a nonlinearity:
 *                       eta = smallest LN value of the matrix, gamma =
 *                       max(LN - eta), codes clamp(rne((LN - eta) * 128 /
 *                       gamma), 0, 127); the output is Eq.(7) as printed,
 *                       y = acc * beta * gamma / 128 (no eta term appears on
 *                       the page). So y estimates beta * W~ (LN - eta), not
 *                       beta * W~ LN: the eta * beta * sum_k W~_jk term is
 *                       not added back. Implies per tensor.
 *   BL_W1A8_TERNARY     packed holds b1.58 ternary weights (BL_PACK_TERNARY).
 * With neither quantiser flag this is bitlinear_w1a8 (or w158a8). Codes are
 * decided in fp64 in the order of the formula. ws: bl_workspace_bytes(
 * BL_OP_W1A8_EX, M, N, K) bytes for the per-tensor forms (else BL_OP_W1A8).
 * xq_out [M x K], gamma_out [M] (the shared gamma, repeated) and acc_out
 * [M x N] may be NULL.
 */
#define BL_W1A8_TERNARY 1u
#define BL_W1A8_PER_TENSOR 2u
#define BL_W1A8_NONNEG 4u
int bitlinear_w1a8_ex(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                      int64_t M, int64_t N, int64_t K, unsigned flags, void* ws, size_t ws_bytes,
                      int8_t* xq_out, double* gamma_out, int32_t* acc_out, void* stream);

/*
 * bin_xnor_gemm -- W1A1: products of two +-1 matrices ("BitNet-Transformers"
 * page: 1-bit operands reduce the product to XNOR / popcount arithmetic):
 *   dot[m][n] = sum_k a_mk * b_nk = K - 2 * popcount(a_m XOR b_n)   (exact int32)
 * a [M x K/32] and b [N x K/32] uint32 in the packed sign layout (bit set =
 * +1); e.g. both from bin_pack(..., BL_PACK_FBI), whose alpha output is then
 * ignored. dot [M x N] int32. Device pointers; K a multiple of 128.
 */
int bin_xnor_gemm(const uint32_t* a, const uint32_t* b, int32_t* dot, int64_t M, int64_t N, int64_t K,
                  void* stream);

/*
 * bl_device_error -- synchronise `stream`, then return the first in-kernel
 * fault recorded on the current device since the last clear (BL_OK if none;
 * BL_ERR_TIMEOUT when a bounded wait ran out). If `clear` is non-zero the
 * word is reset. `where_out` (host pointer, may be NULL) receives a code
 * naming the kernel and wait that gave up.
 */
int bl_device_error(void* stream, int clear, int* where_out);

/*
 * bitlinear_w1a8_noalloc -- bitlinear_w1a8 for callers that cannot allocate.
 *
 * The pages have no counterpart to this call: it exists for users of the
 * library, not for the method. Some callers cannot hand the layer a
 * workspace: an operator plugged into a host framework that passes it only
 * its input and output buffers, or an inference loop whose device memory is
 * planned once up front and which may not call cudaMalloc while it runs
 * (cudaMalloc can synchronise the device and stall other work). This entry
 * point runs the same kernels as bitlinear_w1a8 but keeps the int8 codes and
 * per-token gamma in a fixed scratch array that lives inside the library
 * (BL_W1A8_NOALLOC_SCRATCH_BYTES per device, held by every GPU that loads
 * the library until the process exits). It calls no allocator.
 *
 * Limit: bl_workspace_bytes(BL_OP_W1A8, M, N, K) must not exceed
 * BL_W1A8_NOALLOC_SCRATCH_BYTES (about M*K + 8*M bytes; e.g. 512 tokens of
 * K = 5632 fit), else BL_ERR_SCRATCH_LIMIT is returned and nothing runs.
 * Arguments and results are otherwise those of bitlinear_w1a8.
 *
 * The first call on a device looks up the scratch array's device address
 * (once per device, with that device current); make that first call before
 * any stream capture. All calls on a device share the one array and it keeps
 * the last call's contents; nothing in it needs to start at zero (each call
 * overwrites every byte it later reads), but calls whose kernels overlap on
 * the GPU (different streams, no ordering between them) race on it.
 */
#define BL_W1A8_NOALLOC_SCRATCH_BYTES (4u << 20)
int bitlinear_w1a8_noalloc(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                           int64_t M, int64_t N, int64_t K, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */

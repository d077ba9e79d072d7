/*
 * Oracle for the binarized linear layers -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU statement of what the layers compute,
 * in fp64 (floating point) and int64 (integer). It exists to check the CUDA
 * library against; nothing in the product links it. Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it. It shares no
 * code, header, table or helper with the CUDA sources.
 *
 * Sources (web pages, cited by title and section/equation):
 *   [FBI]    "FBI-LLM: Fully Binarized Large Language Model ... using
 *            autoregressive distillation for 1-bit weight binarization of
 *            LLMs from scratch" (cloudsagepro.com rewrite of a MarkTechPost
 *            article), the paragraph that defines FBI-linear, and the
 *            experiments paragraph (W1A16).
 *   [BitNet] "BitNet b1.58: 1bit LLM 时代" (coreui.cn), section 一 (BitNet):
 *            Eq.(1)-(3) weight binarisation, Eq.(4)-(5) absmax activation
 *            quantisation, Eq.(7)-(8) the BitLinear forward, LN and beta.
 *   [BitNet-Transformers] (dongaigc.com), the remark that 1-bit weights
 *            allow XNOR-style arithmetic (used only for the W1A1 identity).
 *
 * Readings taken where the pages are silent or ambiguous (each also listed
 * in the design notes):
 *   R1  FBI scale: one fp32 scale per output channel j, initialised as the
 *       mean of |W_jk| over that channel's K inputs ("column averages" of the
 *       weight viewed as K x N). The forward takes any alpha vector, since the
 *       page says the scales are only initialised this way.
 *   R2  FBI sign: the same Sign as BitNet Eq.(2): +1 if W > 0, else -1
 *       (so 0 maps to -1). No shift is subtracted for FBI.
 *   R3  BitNet alpha (Eq.3) and beta (Eq.8) are global scalars over the whole
 *       N x K matrix; beta uses the unshifted W.
 *   R4  Activation gamma (Eq.5) is taken per token (per row of x): the
 *       infinity norm of that token's LN output.
 *   R5  Eq.(4) has no rounding step and clips to +-(Q_b - eps). To obtain an
 *       int8 code the value x*Q_b/gamma is rounded to nearest, ties to even,
 *       then clamped to [-127, 127] (Q_b = 2^(8-1) = 128).
 *   R6  LN (Eq.8) has no affine part, uses the population variance, and its
 *       epsilon is a parameter (the library uses 1e-5).
 *   R7  gamma == 0 (a constant token) quantises to all zeros, so y = 0.
 *   R8  Packed layout (the pages give none; this is the library's written
 *       spec): row j of an N x K sign matrix takes ceil(K/32) uint32 words;
 *       element (j,k) is bit (k mod 32) of word [j*ceil(K/32) + k/32]; a set
 *       bit means +1, a clear bit -1; unused bits of a row's last word are 0.
 *   R9  Activations are bf16 (raw 16-bit patterns in, decoded exactly).
 *   R11 b1.58 weights ([BitNet] section 2, Eq.(9)-(11)): the epsilon of
 *       Eq.(9) is not given; it is a parameter (the library uses 1e-5).
 *   R12 "round" in Eq.(10): to nearest, ties to even (as R5), applied to
 *       W / (gamma + eps) evaluated in fp64.
 *   R13 Packed ternary layout (the library's written spec): row j takes
 *       ceil(K/128) blocks of 8 uint32 words; block b covers k in
 *       [128b, 128b + 128): its words 0-3 are the +1 plane, words 4-7 the
 *       -1 plane, element k at bit (k mod 32) of word (k mod 128)/32 of each
 *       plane. A weight is +1, -1 or 0 (neither bit set); never both.
 *   R15 Per-tensor activation scale ([BitNet] Eq.(5) literally: "of the input
 *       matrix"): gamma = max |LN(x)| over all M x K elements, shared by all
 *       tokens; codes as R5.
 *   R16 Eq.(6) (activations before a nonlinearity): eta = min over all M x K
 *       LN values, gamma = max over all of (LN - eta), so (LN - eta) * Q_b /
 *       gamma lies in [0, Q_b]; rounded to nearest (ties to even) and clamped
 *       to [0, 127] (the clip bounds eps and Q_b - eps as integers).
 *   R17 The forward then applies Eq.(7) as printed, y = acc * beta * gamma / Q_b
 *       (the pages give no term for eta). gamma == 0 gives all-zero codes.
 *   R18 FBI-linear backward ([FBI]: the straight-through estimator carries
 *       the gradient through the sign function). With y_mj = alpha_j * z_mj,
 *       z_mj = sum_k s_jk x_mk and an incoming gradient dy (M x N):
 *         dx_mk    = sum_j dy_mj * alpha_j * s_jk        (exact chain rule)
 *         dalpha_j = sum_m dy_mj * z_mj                 (exact chain rule)
 *         dW_jk    = alpha_j * sum_m dy_mj * x_mk        (STE: ds/dW taken as 1)
 *       The page names the estimator but gives no clipping window, so the
 *       plain identity form is used (no |W| <= 1 gate); dW is the gradient of
 *       the latent full-precision weight. dy is bf16 like the activations.
 *   R14 The b1.58 forward is the BitLinear forward of Eq.(7) with the
 *       ternary weights: the same LN and activation quantisation (section 2
 *       keeps BitNet's), and the rescale uses gamma of Eq.(11) as beta (Eq.(11)
 *       and the beta of Eq.(8) are the same mean of |W|).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- small plain helpers (this file's own; nothing shared) ------------- */

static int64_t row_words(int64_t K) { return (K + 31) / 32; }

/* exact decode of a bf16 bit pattern: it is the top half of an fp32 */
static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Sign(v) of [BitNet] Eq.(2): +1 when v > 0, otherwise -1 */
static int sign_pm1(double v) { return v > 0.0 ? 1 : -1; }

/* read element (j,k) of a packed sign matrix as +1/-1 (layout R8) */
static int packed_sign(const uint32_t* packed, int64_t K, int64_t j, int64_t k)
{
    uint32_t word = packed[j * row_words(K) + k / 32];
    return ((word >> (k % 32)) & 1u) ? 1 : -1;
}

/* store a +1/-1 value at (j,k) of a packed sign matrix (layout R8) */
static void packed_store(uint32_t* packed, int64_t K, int64_t j, int64_t k, int s)
{
    if (s == 1) packed[j * row_words(K) + k / 32] |= (1u << (k % 32));
}

/* ---- binarise and pack -------------------------------------------------- */

/* FBI-linear binarisation [FBI], readings R1, R2, R8:
 *   s_jk    = Sign(W_jk)
 *   alpha_j = (1/K) * sum_k |W_jk|     (summed in fp64, stored as fp32)
 * W is row-major N x K fp32 (row j = output channel j). */
void oracle_pack_fbi(const float* W, int64_t N, int64_t K, uint32_t* packed, float* alpha)
{
    memset(packed, 0, (size_t)(N * row_words(K)) * sizeof(uint32_t));
    for (int64_t j = 0; j < N; ++j) {
        double abs_sum = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double w = (double)W[j * K + k];
            packed_store(packed, K, j, k, sign_pm1(w));
            abs_sum += fabs(w);
        }
        alpha[j] = (float)(abs_sum / (double)K);
    }
}

/* BitNet weight binarisation [BitNet] Eq.(1)-(3), beta from Eq.(8), R3:
 *   alpha = (1/(N K)) * sum_jk W_jk            (global mean, fp64)
 *   s_jk  = Sign(W_jk - alpha)                 (compared in fp64)
 *   beta  = (1/(N K)) * sum_jk |W_jk|          (the unshifted W)     */
void oracle_pack_bitnet(const float* W, int64_t N, int64_t K, uint32_t* packed,
                        double* alpha_out, double* beta_out)
{
    double sum = 0.0, abs_sum = 0.0;
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k) {
            sum += (double)W[j * K + k];
            abs_sum += fabs((double)W[j * K + k]);
        }
    double count = (double)N * (double)K;
    double alpha = sum / count;
    memset(packed, 0, (size_t)(N * row_words(K)) * sizeof(uint32_t));
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k)
            packed_store(packed, K, j, k, sign_pm1((double)W[j * K + k] - alpha));
    *alpha_out = alpha;
    *beta_out = abs_sum / count;
}

/* ---- W1A16: FBI-linear forward ------------------------------------------ */

/* One output of the FBI-linear forward [FBI] (W1A16: 1-bit weights,
 * 16-bit activations):
 *   y_mj = alpha_j * sum_k s_jk * x_mk       (fp64)
 * x is row-major M x K bf16, packed is N rows (layout R8). */
static double w1a16_one(const uint16_t* x, const uint32_t* packed, const float* alpha,
                        int64_t K, int64_t m, int64_t j)
{
    double dot = 0.0;
    for (int64_t k = 0; k < K; ++k)
        dot += (double)packed_sign(packed, K, j, k) * bf16_value(x[m * K + k]);
    return (double)alpha[j] * dot;
}

/* full M x N output, row-major */
void oracle_w1a16(const uint16_t* x, const uint32_t* packed, const float* alpha,
                  int64_t M, int64_t N, int64_t K, double* y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j)
            y[m * N + j] = w1a16_one(x, packed, alpha, K, m, j);
}

/* the same definition at a list of (m, j) positions, for sampled checks of
 * problems too large to compute whole */
void oracle_w1a16_at(const uint16_t* x, const uint32_t* packed, const float* alpha,
                     int64_t K, const int64_t* ms, const int64_t* js, int64_t count, double* y)
{
    for (int64_t i = 0; i < count; ++i)
        y[i] = w1a16_one(x, packed, alpha, K, ms[i], js[i]);
}

/* ---- W1A8: BitNet BitLinear forward -------------------------------------- */

/* LN then absmax quantisation of each token [BitNet] Eq.(8), Eq.(4)-(5),
 * readings R4-R7:
 *   mu    = (1/K) sum_k x_k
 *   var   = (1/K) sum_k (x_k - mu)^2
 *   ln_k  = (x_k - mu) / sqrt(var + eps)
 *   gamma = max_k |ln_k|
 *   q_k   = clamp(round_half_even(ln_k * Q_b / gamma), -127, 127), Q_b = 128
 * Writes xq (M x K int8), gamma (M, fp64) and, when pre != NULL, the
 * unrounded ln_k * Q_b / gamma values (M x K, fp64; 0 where gamma == 0). */
void oracle_ln_absmax_quant(const uint16_t* x, int64_t M, int64_t K, double eps,
                            int8_t* xq, double* gamma_out, double* pre)
{
    const double Qb = 128.0;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * K;
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) sum += bf16_value(row[k]);
        double mu = sum / (double)K;
        double sq = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double d = bf16_value(row[k]) - mu;
            sq += d * d;
        }
        double var = sq / (double)K;
        double root = sqrt(var + eps);
        double gamma = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double ln = (bf16_value(row[k]) - mu) / root;
            if (fabs(ln) > gamma) gamma = fabs(ln);
        }
        gamma_out[m] = gamma;
        for (int64_t k = 0; k < K; ++k) {
            if (gamma == 0.0) {
                xq[m * K + k] = 0;
                if (pre) pre[m * K + k] = 0.0;
                continue;
            }
            double ln = (bf16_value(row[k]) - mu) / root;
            double v = ln * Qb / gamma;
            if (pre) pre[m * K + k] = v;
            double r = nearbyint(v); /* default rounding mode: nearest, ties to even */
            if (r > 127.0) r = 127.0;
            if (r < -127.0) r = -127.0;
            xq[m * K + k] = (int8_t)r;
        }
    }
}

/* Per-tensor variants of the activation quantisation, readings R15 and R16,
 * on the LN output of every token (LN as in oracle_ln_absmax_quant):
 *   mode 0 (Eq.(5), per tensor):  gamma = max_{m,k} |LN_mk|
 *          q_mk = clamp(rne(LN_mk * Q_b / gamma), -127, 127)
 *   mode 1 (Eq.(6)):              eta = min_{m,k} LN_mk,  gamma = max_{m,k} (LN_mk - eta)
 *          q_mk = clamp(rne((LN_mk - eta) * Q_b / gamma), 0, 127)
 * gamma_out[m] = gamma for every token (the forward's rescale reads it per
 * token); eta_out (may be NULL) receives eta (0 in mode 0); pre (may be
 * NULL) the unrounded values. */
void oracle_ln_quant_tensor(const uint16_t* x, int64_t M, int64_t K, double eps, int mode,
                            int8_t* xq, double* gamma_out, double* eta_out, double* pre)
{
    const double Qb = 128.0;
    if (eta_out) *eta_out = 0.0;
    if (M <= 0 || K <= 0) return;
    double* ln = (double*)malloc((size_t)(M * K) * sizeof(double));
    if (!ln) return;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * K;
        double sum = 0.0;
        for (int64_t k = 0; k < K; ++k) sum += bf16_value(row[k]);
        double mu = sum / (double)K;
        double sq = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double d = bf16_value(row[k]) - mu;
            sq += d * d;
        }
        double root = sqrt(sq / (double)K + eps);
        for (int64_t k = 0; k < K; ++k) ln[m * K + k] = (bf16_value(row[k]) - mu) / root;
    }
    double eta = 0.0, gamma = 0.0;
    if (mode == 1) {
        eta = INFINITY;
        for (int64_t i = 0; i < M * K; ++i)
            if (ln[i] < eta) eta = ln[i];
        for (int64_t i = 0; i < M * K; ++i)
            if (ln[i] - eta > gamma) gamma = ln[i] - eta;
    } else {
        for (int64_t i = 0; i < M * K; ++i)
            if (fabs(ln[i]) > gamma) gamma = fabs(ln[i]);
    }
    for (int64_t i = 0; i < M * K; ++i) {
        double v = 0.0, r = 0.0;
        if (gamma != 0.0) {
            v = (mode == 1 ? ln[i] - eta : ln[i]) * Qb / gamma;
            r = nearbyint(v);
        }
        if (r > 127.0) r = 127.0;
        if (r < (mode == 1 ? 0.0 : -127.0)) r = (mode == 1 ? 0.0 : -127.0);
        xq[i] = (int8_t)r;
        if (pre) pre[i] = v;
    }
    for (int64_t m = 0; m < M; ++m) gamma_out[m] = gamma;
    if (eta_out) *eta_out = eta;
    free(ln);
}

/* integer core of [BitNet] Eq.(7): acc_mj = sum_k s_jk * q_mk  (int64) */
static int64_t w1a8_acc_one(const int8_t* xq, const uint32_t* packed, int64_t K,
                            int64_t m, int64_t j)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k)
        acc += (int64_t)packed_sign(packed, K, j, k) * (int64_t)xq[m * K + k];
    return acc;
}

void oracle_w1a8_acc(const int8_t* xq, const uint32_t* packed, int64_t M, int64_t N, int64_t K,
                     int64_t* acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j)
            acc[m * N + j] = w1a8_acc_one(xq, packed, K, m, j);
}

void oracle_w1a8_acc_at(const int8_t* xq, const uint32_t* packed, int64_t K,
                        const int64_t* ms, const int64_t* js, int64_t count, int64_t* acc)
{
    for (int64_t i = 0; i < count; ++i)
        acc[i] = w1a8_acc_one(xq, packed, K, ms[i], js[i]);
}

/* rescale of [BitNet] Eq.(7): y_mj = acc_mj * beta * gamma_m / Q_b, fp64,
 * evaluated left to right */
void oracle_w1a8_rescale(const int64_t* acc, const double* gamma, double beta,
                         int64_t M, int64_t N, double* y)
{
    const double Qb = 128.0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j)
            y[m * N + j] = (double)acc[m * N + j] * beta * gamma[m] / Qb;
}

/* ---- b1.58 ternary weights ---------------------------------------------- */

static int64_t ternary_row_words(int64_t K) { return ((K + 127) / 128) * 8; }

/* read element (j,k) of a packed ternary matrix as +1 / 0 / -1 (layout R13) */
static int ternary_value(const uint32_t* packed, int64_t K, int64_t j, int64_t k)
{
    const uint32_t* blk = packed + j * ternary_row_words(K) + (k / 128) * 8;
    int64_t o = k % 128;
    uint32_t plus = (blk[o / 32] >> (o % 32)) & 1u;
    uint32_t minus = (blk[4 + o / 32] >> (o % 32)) & 1u;
    return (int)plus - (int)minus;
}

/* [BitNet] section 2, Eq.(9)-(11), readings R11-R13:
 *   gamma  = (1/(N K)) * sum_jk |W_jk|                      (fp64)
 *   W~_jk  = RoundClip(W_jk / (gamma + eps), -1, 1)
 *          = max(-1, min(1, round_half_even(W_jk / (gamma + eps))))  */
void oracle_pack_ternary(const float* W, int64_t N, int64_t K, double eps, uint32_t* packed,
                         double* gamma_out)
{
    double abs_sum = 0.0;
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k) abs_sum += fabs((double)W[j * K + k]);
    double gamma = abs_sum / ((double)N * (double)K);
    memset(packed, 0, (size_t)(N * ternary_row_words(K)) * sizeof(uint32_t));
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k) {
            double r = nearbyint((double)W[j * K + k] / (gamma + eps));
            if (r > 1.0) r = 1.0;
            if (r < -1.0) r = -1.0;
            if (r == 0.0) continue;
            uint32_t* blk = packed + j * ternary_row_words(K) + (k / 128) * 8;
            int64_t o = k % 128;
            blk[(r > 0.0 ? 0 : 4) + o / 32] |= 1u << (o % 32);
        }
    *gamma_out = gamma;
}

/* integer core of Eq.(7) with ternary weights (R14):
 *   acc_mj = sum_k W~_jk * q_mk          (int64) */
static int64_t w158a8_acc_one(const int8_t* xq, const uint32_t* packed, int64_t K,
                              int64_t m, int64_t j)
{
    int64_t acc = 0;
    for (int64_t k = 0; k < K; ++k)
        acc += (int64_t)ternary_value(packed, K, j, k) * (int64_t)xq[m * K + k];
    return acc;
}

void oracle_w158a8_acc(const int8_t* xq, const uint32_t* packed, int64_t M, int64_t N,
                       int64_t K, int64_t* acc)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j)
            acc[m * N + j] = w158a8_acc_one(xq, packed, K, m, j);
}

void oracle_w158a8_acc_at(const int8_t* xq, const uint32_t* packed, int64_t K,
                          const int64_t* ms, const int64_t* js, int64_t count, int64_t* acc)
{
    for (int64_t i = 0; i < count; ++i)
        acc[i] = w158a8_acc_one(xq, packed, K, ms[i], js[i]);
}

/* ---- FBI-linear backward with the straight-through estimator ----------- */

/* [FBI] training paragraph and reading R18. x (M x K) and dy (M x N) are
 * bf16 patterns, packed the N x K signs (R8), alpha the N scales. Outputs in
 * fp64: dx (M x K), dw (N x K), dalpha (N). Each is its definition summed in
 * the obvious order; z (the forward's unscaled products) is formed first
 * because dalpha is defined through it. */
void oracle_w1a16_backward(const uint16_t* x, const uint32_t* packed, const float* alpha,
                           const uint16_t* dy, int64_t M, int64_t N, int64_t K,
                           double* dx, double* dw, double* dalpha)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t j = 0; j < N; ++j)
                s += bf16_value(dy[m * N + j]) * (double)alpha[j] * (double)packed_sign(packed, K, j, k);
            dx[m * K + k] = s;
        }
    for (int64_t j = 0; j < N; ++j)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t m = 0; m < M; ++m)
                s += bf16_value(dy[m * N + j]) * bf16_value(x[m * K + k]);
            dw[j * K + k] = (double)alpha[j] * s;
        }
    for (int64_t j = 0; j < N; ++j) {
        double s = 0.0;
        for (int64_t m = 0; m < M; ++m) {
            double z = 0.0;
            for (int64_t k = 0; k < K; ++k)
                z += (double)packed_sign(packed, K, j, k) * bf16_value(x[m * K + k]);
            s += bf16_value(dy[m * N + j]) * z;
        }
        dalpha[j] = s;
    }
}

/* the same definitions at a list of positions, for sampled checks of
 * problems too large to compute whole: which = 0 gives dx at (m, k) =
 * (i0, i1), 1 gives dw at (j, k) = (i0, i1), 2 gives dalpha at j = i0 */
void oracle_w1a16_backward_at(const uint16_t* x, const uint32_t* packed, const float* alpha,
                              const uint16_t* dy, int64_t M, int64_t N, int64_t K, int which,
                              const int64_t* i0, const int64_t* i1, int64_t count, double* out)
{
    for (int64_t i = 0; i < count; ++i) {
        double s = 0.0;
        if (which == 0) {
            const int64_t m = i0[i], k = i1[i];
            for (int64_t j = 0; j < N; ++j)
                s += bf16_value(dy[m * N + j]) * (double)alpha[j] * (double)packed_sign(packed, K, j, k);
        } else if (which == 1) {
            const int64_t j = i0[i], k = i1[i];
            for (int64_t m = 0; m < M; ++m)
                s += bf16_value(dy[m * N + j]) * bf16_value(x[m * K + k]);
            s *= (double)alpha[j];
        } else {
            const int64_t j = i0[i];
            for (int64_t m = 0; m < M; ++m) {
                double z = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    z += (double)packed_sign(packed, K, j, k) * bf16_value(x[m * K + k]);
                s += bf16_value(dy[m * N + j]) * z;
            }
        }
        out[i] = s;
    }
}

/* ---- W1A1 (only as an identity check of the packed-sign reading) ------- */

/* dot_mj = sum_k a_mk * b_jk with both operands packed +-1 rows (R8);
 * [BitNet-Transformers] notes that such products reduce to XNOR/popcount. */
void oracle_w1a1(const uint32_t* a, const uint32_t* b, int64_t M, int64_t N, int64_t K,
                 int64_t* dot)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t j = 0; j < N; ++j) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)packed_sign(a, K, m, k) * (int64_t)packed_sign(b, K, j, k);
            dot[m * N + j] = s;
        }
}

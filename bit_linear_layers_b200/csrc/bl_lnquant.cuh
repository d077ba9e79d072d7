// LN + per-token absmax int8 quantisation, the prologue of BitLinear
// ("BitNet b1.58" page, section 1: LN of Eq.(8), then Eq.(4)-(5) with
// Q_b = 128). One CTA per token.
//
// Statistics are fp64: the sum of bf16 values is exact in fp64 whenever their
// exponents span less than ~40 binades (any realistic activation row), so
// mu = sum/K is the same correctly rounded double the CPU statement gets;
// var = sum (x - mu)^2 / K, root = sqrt(var + eps) follow in fp64.
// max_k |x_k - mu| is taken as max(x_max - mu, mu - x_min) in fp64: the
// rounded difference is monotonic in x, so this is exactly the largest
// rounded |x_k - mu|; and gamma = max|x - mu| / root equals max |(x - mu)/root|
// because rounded division by root > 0 is monotonic.
//
// The code q = clamp(rint(ln * 128 / gamma), -127, 127), whose exact value is
// (x - mu) * 128 / max|x - mu|, is decided as in fp64. Fast path, all fp32:
// d32 = (x - mu_hi) - mu_lo with mu = mu_hi + mu_lo to ~2^-48, times
// c32 = fp32(128 / max|x - mu|); each of the four roundings moves the value by
// at most 128 * 2^-24 (bf16 inputs that are not all equal differ by at least
// one bf16 ulp, which keeps |mu| / max|x - mu| below ~2^9, so neither the
// split of mu nor |x - mu_hi| > |x - mu| adds anything measurable), so v32
// lies within 3.1e-5 of the exact value, and the
// fp64 evaluation within ~1e-13 of it: whenever v32 is farther than 1e-4 from
// a half-integer both round to the same integer. Otherwise the fp64 steps are
// evaluated in the order of the formula. max|x - mu| == 0 (constant token)
// gives gamma = 0 and all-zero codes.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kLnThreads = 256;  // one CTA per token
constexpr int kLnWarps = kLnThreads / 32;
constexpr double kLnEps = 1e-5;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// bf16 bits -> the same value as a double, built with integer operations
// (the float -> double conversion unit is the slowest pipe of this kernel):
// for a normal bf16 the double's high word is the sign, the exponent
// rebiased by 1023 - 127 = 896 and the 7 mantissa bits; its low word is 0.
// Zeros, subnormals, infinities and NaNs take the conversion instruction.
__device__ __forceinline__ double bf16_to_double(uint32_t b16) {
  const uint32_t e = b16 & 0x7F80u;
  if (e == 0u || e == 0x7F80u) return static_cast<double>(__uint_as_float(b16 << 16));
  const uint32_t hi = ((b16 & 0x8000u) << 16) | (((b16 & 0x7FFFu) << 13) + (896u << 20));
  return __hiloint2double(static_cast<int>(hi), 0);
}

// exact fp64 evaluation of the code, in the order of the formula
__device__ __noinline__ int quant_code_exact(float xv, double mu, double root, double gamma) {
  const double d = static_cast<double>(xv) - mu;
  const double ln = d / root;
  const double v = ln * 128.0 / gamma;
  return static_cast<int>(fmin(fmax(rint(v), -127.0), 127.0));
}

struct LnQuantParams {
  float mu_hi, mu_lo, c32;
  double mu, root, gamma;
};

// |v32| <= 128 + 1e-3, so adding 1.5 * 2^23 rounds it to an integer (ties to
// even) in the float's low mantissa bits: the integer comes out of the bit
// pattern and v32 - rounded is the distance to it, without the (slow)
// conversion-unit instructions floor / rint / float-to-int.
__device__ __forceinline__ int quant_code(float xv, const LnQuantParams& p) {
  const float d32 = (xv - p.mu_hi) - p.mu_lo;
  const float v32 = d32 * p.c32;
  const float big = v32 + 12582912.0f;  // 1.5 * 2^23
  const float dist = v32 - (big - 12582912.0f);
  if (fabsf(dist) >= 0.5f - 1e-4f) return quant_code_exact(xv, p.mu, p.root, p.gamma);
  const int q = __float_as_int(big) - 0x4B400000;
  return min(max(q, -127), 127);
}

// CTA-wide sum (fp64) of one value per thread; every thread gets the total
__device__ __forceinline__ double ln_block_sum(double v, double* sh) {
  v = warp_sum(v);
  __syncthreads();  // sh may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = sh[0];
#pragma unroll
  for (int w = 1; w < kLnWarps; ++w) t += sh[w];
  return t;
}

// NV > 0: the token's row is loaded once into registers (at most NV 16-byte
// vectors per thread, K <= NV * 2048) and the three passes read it from
// there; NV = 0: every pass streams the row again (any K).
template <int NV>
__global__ void __launch_bounds__(kLnThreads) ln_quant_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                              int64_t K, int8_t* __restrict__ xq,
                                                              double* __restrict__ gamma_out) {
  __shared__ double sh[kLnWarps];
  __shared__ float shm[2][kLnWarps];
  const int64_t m = blockIdx.x;
  if (m >= M) return;  // uniform per CTA
  // a kernel launched after this one with programmatic serialisation (the
  // few-token GEMV) may be scheduled now; it waits for this grid's results
  grid_dependents_launch();
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  const int64_t nvec = K / 8;  // 8 bf16 per 16-byte load

  uint4 cache[NV > 0 ? NV : 1];
  if constexpr (NV > 0) {
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const int64_t i = threadIdx.x + static_cast<int64_t>(u) * kLnThreads;
      cache[u] = i < nvec ? row[i] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // f(i, v) for every 16-byte vector i of the row this thread owns
  auto for_each_vec = [&](auto&& f) {
    if constexpr (NV > 0) {
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const int64_t i = threadIdx.x + static_cast<int64_t>(u) * kLnThreads;
        if (i < nvec) f(i, cache[u]);
      }
    } else {
      for (int64_t i = threadIdx.x; i < nvec; i += kLnThreads) f(i, row[i]);
    }
  };

  // pass 1: fp64 sum (two chains), fp32 max and min
  double s0 = 0.0, s1 = 0.0;
  float xmax = -INFINITY, xmin = INFINITY;
  for_each_vec([&](int64_t, const uint4& v) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      s0 += bf16_to_double(h[j] & 0xFFFFu);
      s1 += bf16_to_double(h[j] >> 16);
      const float a = bf16_lo(h[j]), b = bf16_hi(h[j]);
      xmax = fmaxf(xmax, fmaxf(a, b));
      xmin = fminf(xmin, fminf(a, b));
    }
  });
  xmax = warp_max(xmax);
  xmin = -warp_max(-xmin);
  if ((threadIdx.x & 31) == 0) {
    shm[0][threadIdx.x >> 5] = xmax;
    shm[1][threadIdx.x >> 5] = xmin;
  }
  const double mu = ln_block_sum(s0 + s1, sh) / static_cast<double>(K);  // its barriers publish shm
  xmax = shm[0][0];
  xmin = shm[1][0];
#pragma unroll
  for (int w = 1; w < kLnWarps; ++w) {
    xmax = fmaxf(xmax, shm[0][w]);
    xmin = fminf(xmin, shm[1][w]);
  }

  // pass 2: sum of squared deviations in fp64
  double q0 = 0.0, q1 = 0.0;
  for_each_vec([&](int64_t, const uint4& v) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double d0 = bf16_to_double(h[j] & 0xFFFFu) - mu;
      const double d1 = bf16_to_double(h[j] >> 16) - mu;
      q0 = fma(d0, d0, q0);
      q1 = fma(d1, d1, q1);
    }
  });
  const double sq = ln_block_sum(q0 + q1, sh);
  const double dmax = fmax(static_cast<double>(xmax) - mu, mu - static_cast<double>(xmin));
  LnQuantParams p;
  p.mu = mu;
  p.root = sqrt(sq / static_cast<double>(K) + kLnEps);
  p.gamma = dmax / p.root;
  p.mu_hi = static_cast<float>(mu);
  p.mu_lo = static_cast<float>(mu - static_cast<double>(p.mu_hi));
  p.c32 = dmax > 0.0 ? static_cast<float>(128.0 / dmax) : 0.f;
  if (threadIdx.x == 0) gamma_out[m] = p.gamma;

  // pass 3: codes, 8 per thread per vector
  uint2* out = reinterpret_cast<uint2*>(xq + m * K);
  for_each_vec([&](int64_t i, const uint4& v) {
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t packed_codes[2] = {0u, 0u};
    if (dmax > 0.0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q0c = quant_code(bf16_lo(h[j]), p);
        const int q1c = quant_code(bf16_hi(h[j]), p);
        const uint32_t pair = (static_cast<uint32_t>(q0c) & 0xFFu) | ((static_cast<uint32_t>(q1c) & 0xFFu) << 8);
        packed_codes[j >> 1] |= pair << (16 * (j & 1));
      }
    }
    out[i] = make_uint2(packed_codes[0], packed_codes[1]);
  });
}

// ---------------------------------------------------------------------------
// Per-tensor variants ("BitNet b1.58" page, section 1): Eq.(5) with gamma
// over the whole LN output of the matrix, and Eq.(6), which shifts by the
// matrix's smallest LN value eta and scales the range max(LN - eta) onto
// [0, Q_b] (codes 0..127). Three kernels: per-token statistics, one CTA that
// folds them into gamma (and eta), then per-token quantisation. Codes are
// evaluated in fp64 in the order of the formula: ln = (x - mu) / root,
// v = (ln [- eta]) * 128 / gamma, rounded half to even and clamped.
struct LnTokenStats {
  double mu, root, ln_min, ln_max;  // ln_min / ln_max: the token's extreme LN values
};

__global__ void __launch_bounds__(kLnThreads) ln_stats_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                              int64_t K, LnTokenStats* __restrict__ stats) {
  __shared__ double sh[kLnWarps];
  __shared__ float shm[2][kLnWarps];
  const int64_t m = blockIdx.x;
  if (m >= M) return;  // uniform per CTA
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  const int64_t nvec = K / 8;
  double s0 = 0.0, s1 = 0.0;
  float xmax = -INFINITY, xmin = INFINITY;
  for (int64_t i = threadIdx.x; i < nvec; i += kLnThreads) {
    const uint4 v = row[i];
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      s0 += bf16_to_double(h[j] & 0xFFFFu);
      s1 += bf16_to_double(h[j] >> 16);
      const float a = bf16_lo(h[j]), b = bf16_hi(h[j]);
      xmax = fmaxf(xmax, fmaxf(a, b));
      xmin = fminf(xmin, fminf(a, b));
    }
  }
  xmax = warp_max(xmax);
  xmin = -warp_max(-xmin);
  if ((threadIdx.x & 31) == 0) {
    shm[0][threadIdx.x >> 5] = xmax;
    shm[1][threadIdx.x >> 5] = xmin;
  }
  const double mu = ln_block_sum(s0 + s1, sh) / static_cast<double>(K);
  xmax = shm[0][0];
  xmin = shm[1][0];
#pragma unroll
  for (int w = 1; w < kLnWarps; ++w) {
    xmax = fmaxf(xmax, shm[0][w]);
    xmin = fminf(xmin, shm[1][w]);
  }
  double q0 = 0.0, q1 = 0.0;
  for (int64_t i = threadIdx.x; i < nvec; i += kLnThreads) {
    const uint4 v = row[i];
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const double d0 = bf16_to_double(h[j] & 0xFFFFu) - mu;
      const double d1 = bf16_to_double(h[j] >> 16) - mu;
      q0 = fma(d0, d0, q0);
      q1 = fma(d1, d1, q1);
    }
  }
  const double sq = ln_block_sum(q0 + q1, sh);
  if (threadIdx.x == 0) {
    const double root = sqrt(sq / static_cast<double>(K) + kLnEps);
    // (x - mu) / root is monotonic in x: the token's extremes come from x_min and x_max
    stats[m] = LnTokenStats{mu, root, (static_cast<double>(xmin) - mu) / root,
                            (static_cast<double>(xmax) - mu) / root};
  }
}

// One CTA: gamma (and eta) over all tokens; gamma_out[m] = gamma for every m,
// scalars[0] = gamma, scalars[1] = eta (0 for Eq.(5)).
__global__ void __launch_bounds__(kLnThreads) ln_tensor_scalars_kernel(const LnTokenStats* __restrict__ stats,
                                                                       int64_t M, bool nonneg,
                                                                       double* __restrict__ gamma_out,
                                                                       double* __restrict__ scalars) {
  __shared__ double sh_a[kLnWarps], sh_b[kLnWarps];
  double amax = 0.0, lmin = INFINITY, lmax = -INFINITY;
  for (int64_t m = threadIdx.x; m < M; m += kLnThreads) {
    const LnTokenStats t = stats[m];
    amax = fmax(amax, fmax(fabs(t.ln_min), fabs(t.ln_max)));
    lmin = fmin(lmin, t.ln_min);
    lmax = fmax(lmax, t.ln_max);
  }
  amax = warp_max(amax);
  lmax = warp_max(lmax);
  lmin = -warp_max(-lmin);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sh_a[w] = nonneg ? lmax : amax;
    sh_b[w] = lmin;
  }
  __syncthreads();
  double g = sh_a[0], e = sh_b[0];
  for (int i = 1; i < kLnWarps; ++i) {
    g = fmax(g, sh_a[i]);
    e = fmin(e, sh_b[i]);
  }
  // Eq.(6): gamma = max (LN - eta) = max LN - eta (the rounded difference is monotonic)
  const double eta = nonneg ? e : 0.0;
  const double gamma = nonneg ? g - eta : g;
  for (int64_t m = threadIdx.x; m < M; m += kLnThreads) gamma_out[m] = gamma;
  if (threadIdx.x == 0) {
    scalars[0] = gamma;
    scalars[1] = eta;
  }
}

__global__ void __launch_bounds__(kLnThreads) ln_quant_tensor_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                     int64_t K, bool nonneg,
                                                                     const LnTokenStats* __restrict__ stats,
                                                                     const double* __restrict__ scalars,
                                                                     int8_t* __restrict__ xq) {
  const int64_t m = blockIdx.x;
  if (m >= M) return;
  const LnTokenStats t = stats[m];
  const double gamma = scalars[0], eta = scalars[1];
  const double lo = nonneg ? 0.0 : -127.0;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  uint2* out = reinterpret_cast<uint2*>(xq + m * K);
  for (int64_t i = threadIdx.x; i < K / 8; i += kLnThreads) {
    const uint4 v = row[i];
    const uint32_t h[4] = {v.x, v.y, v.z, v.w};
    uint32_t codes[2] = {0u, 0u};
    if (gamma != 0.0) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t b16 = (h[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
        const double ln = (bf16_to_double(b16) - t.mu) / t.root;
        const double val = (nonneg ? ln - eta : ln) * 128.0 / gamma;
        const int q = static_cast<int>(fmin(fmax(rint(val), lo), 127.0));
        codes[j >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (j & 3));
      }
    }
    out[i] = make_uint2(codes[0], codes[1]);
  }
}

// ---------------------------------------------------------------------------
// The same LN + per-token absmax quantisation of one token by one warp, for
// short rows (K <= 256 * NVW): the statistics are reduced by warp shuffles
// (a different summation order from ln_quant_kernel: gamma may differ in its
// last bits, within the same bound), the code decision is quant_code with the
// same fp64 fallback. `codes` may point to shared memory.
template <int NVW>
__device__ __forceinline__ void ln_quant_row_warp(const uint16_t* __restrict__ xrow, int K, int8_t* codes,
                                                  double* gamma_out) {
  const int lane = threadIdx.x & 31;
  const uint4* row = reinterpret_cast<const uint4*>(xrow);
  const int nvec = K / 8;
  uint4 cache[NVW];
#pragma unroll
  for (int u = 0; u < NVW; ++u) {
    const int i = lane + 32 * u;
    cache[u] = i < nvec ? row[i] : make_uint4(0u, 0u, 0u, 0u);
  }
  double s0 = 0.0, s1 = 0.0;
  float xmax = -INFINITY, xmin = INFINITY;
#pragma unroll
  for (int u = 0; u < NVW; ++u) {
    if (lane + 32 * u < nvec) {
      const uint32_t h[4] = {cache[u].x, cache[u].y, cache[u].z, cache[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s0 += bf16_to_double(h[j] & 0xFFFFu);
        s1 += bf16_to_double(h[j] >> 16);
        const float a = bf16_lo(h[j]), b = bf16_hi(h[j]);
        xmax = fmaxf(xmax, fmaxf(a, b));
        xmin = fminf(xmin, fminf(a, b));
      }
    }
  }
  xmax = warp_max(xmax);
  xmin = -warp_max(-xmin);
  const double mu = warp_sum(s0 + s1) / static_cast<double>(K);
  double q0 = 0.0, q1 = 0.0;
#pragma unroll
  for (int u = 0; u < NVW; ++u) {
    if (lane + 32 * u < nvec) {
      const uint32_t h[4] = {cache[u].x, cache[u].y, cache[u].z, cache[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double d0 = bf16_to_double(h[j] & 0xFFFFu) - mu;
        const double d1 = bf16_to_double(h[j] >> 16) - mu;
        q0 = fma(d0, d0, q0);
        q1 = fma(d1, d1, q1);
      }
    }
  }
  const double sq = warp_sum(q0 + q1);
  const double dmax = fmax(static_cast<double>(xmax) - mu, mu - static_cast<double>(xmin));
  LnQuantParams p;
  p.mu = mu;
  p.root = sqrt(sq / static_cast<double>(K) + kLnEps);
  p.gamma = dmax / p.root;
  p.mu_hi = static_cast<float>(mu);
  p.mu_lo = static_cast<float>(mu - static_cast<double>(p.mu_hi));
  p.c32 = dmax > 0.0 ? static_cast<float>(128.0 / dmax) : 0.f;
  if (lane == 0) *gamma_out = p.gamma;
  uint2* out = reinterpret_cast<uint2*>(codes);
#pragma unroll
  for (int u = 0; u < NVW; ++u) {
    const int i = lane + 32 * u;
    if (i < nvec) {
      const uint32_t h[4] = {cache[u].x, cache[u].y, cache[u].z, cache[u].w};
      uint32_t packed_codes[2] = {0u, 0u};
      if (dmax > 0.0) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int q0c = quant_code(bf16_lo(h[j]), p);
          const int q1c = quant_code(bf16_hi(h[j]), p);
          const uint32_t pair = (static_cast<uint32_t>(q0c) & 0xFFu) | ((static_cast<uint32_t>(q1c) & 0xFFu) << 8);
          packed_codes[j >> 1] |= pair << (16 * (j & 1));
        }
      }
      out[i] = make_uint2(packed_codes[0], packed_codes[1]);
    }
  }
}

}  // namespace bl

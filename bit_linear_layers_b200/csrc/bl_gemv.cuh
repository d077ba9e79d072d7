// Decode-sized kernels (a few tokens): memory-bound sweeps over the packed
// weights.
//
// W1A16 ("FBI-LLM" page, FBI-linear paragraph; W1A16 from its experiments
// paragraph): y_mj = alpha_j * sum_k s_jk x_mk. With s = 2b - 1 for the bit
// b this is alpha_j * (2 * S+_mj - Sx_m), where S+ sums the x_mk whose bit is
// set and Sx_m = sum_k x_mk, so the inner loop is one predicated fp32 add per
// (weight, token) and the +-1 expansion costs nothing.
//
// W1A8 small-M ("BitNet b1.58" page, section 1, Eq.(7)): the int8 codes are
// produced by the LN/quant kernel; each 32-bit word of signs expands to eight
// +-1 byte quadruples that feed dp4a, so the dot product is exact int32.
#pragma once

#include "bl_common.cuh"
#include "bl_lnquant.cuh"

namespace bl {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvRowsPerWarp = 4;
constexpr int kGemvRowsPerCta = kGemvWarps * kGemvRowsPerWarp;  // 32
constexpr int kGemvChunkK = 4096;  // K values staged per pass: one uint4 of bits per lane
constexpr int kGemvXsStride = 33;  // padded lane stride of the staged x tile

__host__ __device__ constexpr int gemv_smem_bytes(int mt) {
  return mt * 4 * 32 * kGemvXsStride * 4;
}

// x tile in shared memory, fp32: element k of the chunk sits where the lane
// that owns its packed word reads it with consecutive lanes on consecutive
// banks: k = (4*l + q)*32 + b  ->  xs[((m*4 + q)*32 + b)*33 + l].
template <int MT>
__global__ void __launch_bounds__(kGemvThreads) gemv_w1a16_kernel(
    const uint16_t* __restrict__ x, const uint32_t* __restrict__ packed,
    const float* __restrict__ alpha, uint16_t* __restrict__ y, int M, int64_t N, int64_t K) {
  extern __shared__ float xs[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kGemvRowsPerCta + warp * kGemvRowsPerWarp;
  const int64_t words = K / 32;
  float acc[kGemvRowsPerWarp][MT];
  float sx[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    sx[m] = 0.f;
#pragma unroll
    for (int r = 0; r < kGemvRowsPerWarp; ++r) acc[r][m] = 0.f;
  }

  for (int64_t k0 = 0; k0 < K; k0 += kGemvChunkK) {
    const int kc = static_cast<int>(K - k0 < kGemvChunkK ? K - k0 : kGemvChunkK);  // % 128 == 0
    __syncthreads();  // the previous chunk has been consumed
    // stage: each thread converts 8 consecutive bf16 (one 16-byte load)
    for (int e = threadIdx.x; e < MT * (kc / 8); e += kGemvThreads) {
      const int m = e / (kc / 8);
      const int kl = (e - m * (kc / 8)) * 8;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (m < M) raw = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k0 + kl);
      const uint32_t h[4] = {raw.x, raw.y, raw.z, raw.w};
      const int wl = kl >> 5, l = wl >> 2, q = wl & 3, b0 = kl & 31;
      float* dst = xs + ((m * 4 + q) * 32 + b0) * kGemvXsStride + l;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dst[(2 * i) * kGemvXsStride] = __uint_as_float(h[i] << 16);
        dst[(2 * i + 1) * kGemvXsStride] = __uint_as_float(h[i] & 0xFFFF0000u);
      }
    }
    __syncthreads();
    if (lane * 4 < kc / 32) {
      uint4 w[kGemvRowsPerWarp];
#pragma unroll
      for (int r = 0; r < kGemvRowsPerWarp; ++r) {
        const int64_t row = row0 + r;
        w[r] = make_uint4(0, 0, 0, 0);
        if (row < N)
          w[r] = __ldcs(reinterpret_cast<const uint4*>(packed + row * words + k0 / 32) + lane);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int b = 0; b < 32; ++b) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float xv = xs[((m * 4 + q) * 32 + b) * kGemvXsStride + lane];
            sx[m] += xv;
#pragma unroll
            for (int r = 0; r < kGemvRowsPerWarp; ++r) {
              const uint32_t word = q == 0 ? w[r].x : q == 1 ? w[r].y : q == 2 ? w[r].z : w[r].w;
              if ((word >> b) & 1u) acc[r][m] += xv;
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) sx[m] = warp_sum(sx[m]);
#pragma unroll
  for (int r = 0; r < kGemvRowsPerWarp; ++r) {
    const int64_t row = row0 + r;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float a = warp_sum(acc[r][m]);
      if (lane == 0 && row < N && m < M)
        y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits(alpha[row] * (2.f * a - sx[m]));
    }
  }
}

// ---------------------------------------------------------------------------
// W1A8, few tokens: acc_mj = sum_k s_jk q_mk (int32, exact) from the codes in
// `xq`, then y = fp32(acc * beta * gamma_m / 128) in fp64.

// four sign bits (nibble) -> four int8 lanes of +1 / -1
__device__ __forceinline__ uint32_t nibble_to_pm1_i8(uint32_t nib) {
  const uint32_t spread = (nib * 0x00204081u) & 0x01010101u;  // bit i -> byte i
  return spread * 0xFFFFFF02u + 0xFFFFFFFFu;                  // 1 -> 0x01, 0 -> 0xFF
}

// four ternary weights (a +1 nibble and a -1 nibble) -> four int8 lanes of +1 / 0 / -1
__device__ __forceinline__ uint32_t nibbles_to_ternary_i8(uint32_t plus, uint32_t minus) {
  const uint32_t p = (plus * 0x00204081u) & 0x01010101u;   // bit i -> byte i = 1
  const uint32_t m = (minus * 0x00204081u) & 0x01010101u;
  return p | (m * 0xFFu);                                   // -1 bytes: 0xFF (never both)
}

// kTernary: `packed` holds b1.58 weights, per 128-k block 4 words of the +1
// plane then 4 of the -1 plane (row stride K/16 words)
template <int MT, bool kTernary>
__device__ __forceinline__ void w1a8_rows(const int8_t* __restrict__ xq, const double* __restrict__ gamma,
                                          const uint32_t* __restrict__ packed, const float* __restrict__ beta,
                                          float* __restrict__ y, int32_t* __restrict__ acc_out, int M, int64_t N,
                                          int64_t K) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kGemvRowsPerCta + warp * kGemvRowsPerWarp;
  const int64_t words = K / 32;  // 32-k groups per row
  const int64_t stride = kTernary ? K / 16 : K / 32;
  int acc[kGemvRowsPerWarp][MT];
#pragma unroll
  for (int r = 0; r < kGemvRowsPerWarp; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0;

  for (int64_t wi = lane; wi < words; wi += 32) {
    uint32_t wr[kGemvRowsPerWarp], wm[kGemvRowsPerWarp];
    const int64_t off = kTernary ? (wi >> 2) * 8 + (wi & 3) : wi;
#pragma unroll
    for (int r = 0; r < kGemvRowsPerWarp; ++r) {
      const int64_t row = row0 + r;
      wr[r] = row < N ? __ldcs(packed + row * stride + off) : 0u;
      wm[r] = (kTernary && row < N) ? __ldcs(packed + row * stride + off + 4) : 0u;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      const uint4* xp = reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(m) * K + wi * 32);
      const uint4 x0 = xp[0], x1 = xp[1];
      const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int r = 0; r < kGemvRowsPerWarp; ++r) {
        int a = acc[r][m];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t wbytes = kTernary
                                      ? nibbles_to_ternary_i8((wr[r] >> (4 * i)) & 0xFu, (wm[r] >> (4 * i)) & 0xFu)
                                      : nibble_to_pm1_i8((wr[r] >> (4 * i)) & 0xFu);
          a = __dp4a(static_cast<int>(wbytes), static_cast<int>(xv[i]), a);
        }
        acc[r][m] = a;
      }
    }
  }
  const double bt = static_cast<double>(*beta);
#pragma unroll
  for (int r = 0; r < kGemvRowsPerWarp; ++r) {
    const int64_t row = row0 + r;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int a = warp_sum(acc[r][m]);
      if (lane == 0 && row < N && m < M) {
        const int64_t o = static_cast<int64_t>(m) * N + row;
        y[o] = static_cast<float>(static_cast<double>(a) * bt * gamma[m] / 128.0);
        if (acc_out) acc_out[o] = a;
      }
    }
  }
}


// The dp4a GEMV as a kernel of its own, after the LN + quantisation kernel.
// Launched with programmatic serialisation it is scheduled while that kernel
// runs and waits for its results here.
template <int MT, bool kTernary>
__global__ void __launch_bounds__(kGemvThreads) gemv_w1a8_kernel(
    const int8_t* __restrict__ xq, const double* __restrict__ gamma,
    const uint32_t* __restrict__ packed, const float* __restrict__ beta, float* __restrict__ y,
    int32_t* __restrict__ acc_out, int M, int64_t N, int64_t K) {
  grid_dependency_wait();
  w1a8_rows<MT, kTernary>(xq, gamma, packed, beta, y, acc_out, M, N, K);
}

// BitLinear for short problems in one launch ("BitNet b1.58" page, section
// 1, Eq.(4)-(5), (7)-(8)): every CTA quantises all M tokens itself (one warp
// per token, codes and gamma in shared memory), then runs the dp4a GEMV and
// the rescale for its 32 rows. For M <= 16, K <= kW1a8SmallMaxK and M * K <=
// kW1a8SmallMaxCodes, where repeating the LN in every CTA costs less than a
// second launch. xq_out / gamma_out (written by CTA 0) and acc_out may be null.
constexpr int kW1a8SmallMaxK = 1024;         // four 16-byte vectors per lane
constexpr int kW1a8SmallMaxCodes = 16384;    // shared-memory codes
template <int MT, bool kTernary>
__global__ void __launch_bounds__(kGemvThreads) bitlinear_small_kernel(
    const uint16_t* __restrict__ x, const uint32_t* __restrict__ packed, const float* __restrict__ beta,
    float* __restrict__ y, int8_t* __restrict__ xq_out, double* __restrict__ gamma_out,
    int32_t* __restrict__ acc_out, int M, int64_t N, int64_t K) {
  __shared__ __align__(16) int8_t codes[kW1a8SmallMaxCodes];
  __shared__ double gam[16];
  const int warp = threadIdx.x >> 5;
  for (int m = warp; m < M; m += kGemvWarps) {
    if (K <= 256)
      ln_quant_row_warp<1>(x + static_cast<int64_t>(m) * K, static_cast<int>(K), codes + m * K, &gam[m]);
    else if (K <= 512)
      ln_quant_row_warp<2>(x + static_cast<int64_t>(m) * K, static_cast<int>(K), codes + m * K, &gam[m]);
    else
      ln_quant_row_warp<4>(x + static_cast<int64_t>(m) * K, static_cast<int>(K), codes + m * K, &gam[m]);
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    if (xq_out)
      for (int64_t i = threadIdx.x; i < M * K / 16; i += kGemvThreads)
        reinterpret_cast<uint4*>(xq_out)[i] = reinterpret_cast<const uint4*>(codes)[i];
    if (gamma_out && threadIdx.x < M) gamma_out[threadIdx.x] = gam[threadIdx.x];
  }
  w1a8_rows<MT, kTernary>(codes, gam, packed, beta, y, acc_out, M, N, K);
}

}  // namespace bl

// Binarise-and-pack kernels.
//
// FBI-linear ("FBI-LLM" page, FBI-linear paragraph): bit = W > 0 and one
// scale per output channel, alpha_j = mean_k |W_jk| (fp64 sum, one rounding
// to fp32). BitNet ("BitNet b1.58" page, section 1, Eq.(1)-(3), (8)):
// bit = (W - mean W) > 0 compared in fp64, beta = mean |W|. b1.58 ("BitNet
// b1.58" page, section 2, Eq.(9)-(11)): W~ = RoundClip(W / (gamma + eps), -1, 1)
// with gamma = mean |W|, as a +1 and a -1 bit plane per 128-k block.
//
// A warp owns one row at a time and sweeps it 128 floats per step: each lane
// loads a float4, turns it into a 4-bit nibble, and an OR-reduction over each
// group of 8 lanes assembles one 32-bit word (LSB = lowest k). The row's
// fp64 sums ride along in the same pass, so W is read from HBM exactly once
// per pass.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kPackThreads = 256;

__device__ __forceinline__ uint32_t nibble_words(uint32_t nib, int lane) {
  // place this lane's nibble at bits 4*(lane%8) and OR over the 8-lane group
  uint32_t v = nib << (4 * (lane & 7));
  v |= __shfl_xor_sync(0xffffffffu, v, 1);
  v |= __shfl_xor_sync(0xffffffffu, v, 2);
  v |= __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

// kBitNet == false: FBI signs, alpha[row] written.
// kBitNet == true : signs of W - shift (shift read from device memory in fp64).
template <bool kBitNet>
__global__ void __launch_bounds__(kPackThreads) pack_rows_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, uint32_t* __restrict__ packed,
    float* __restrict__ alpha, const double* __restrict__ shift_ptr) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const double shift = kBitNet ? *shift_ptr : 0.0;
  const int64_t steps = K / 128;  // 128 floats (4 words) per warp step
  for (int64_t row = warp0; row < N; row += nwarps) {
    const float4* src = reinterpret_cast<const float4*>(W + row * K) + lane;
    uint32_t* dst = packed + row * (K / 32) + (lane >> 3);
    double abs_sum = 0.0;
    int64_t s = 0;
    for (; s + 4 <= steps; s += 4) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + (s + u) * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t nib;
        if (kBitNet) {
          nib = (static_cast<double>(v[u].x) - shift > 0.0 ? 1u : 0u) |
                (static_cast<double>(v[u].y) - shift > 0.0 ? 2u : 0u) |
                (static_cast<double>(v[u].z) - shift > 0.0 ? 4u : 0u) |
                (static_cast<double>(v[u].w) - shift > 0.0 ? 8u : 0u);
        } else {
          nib = (v[u].x > 0.f ? 1u : 0u) | (v[u].y > 0.f ? 2u : 0u) | (v[u].z > 0.f ? 4u : 0u) |
                (v[u].w > 0.f ? 8u : 0u);
          abs_sum += fabs(static_cast<double>(v[u].x)) + fabs(static_cast<double>(v[u].y)) +
                     fabs(static_cast<double>(v[u].z)) + fabs(static_cast<double>(v[u].w));
        }
        const uint32_t word = nibble_words(nib, lane);
        if ((lane & 7) == 0) dst[(s + u) * 4] = word;
      }
    }
    for (; s < steps; ++s) {
      const float4 v = __ldcs(src + s * 32);
      uint32_t nib;
      if (kBitNet) {
        nib = (static_cast<double>(v.x) - shift > 0.0 ? 1u : 0u) |
              (static_cast<double>(v.y) - shift > 0.0 ? 2u : 0u) |
              (static_cast<double>(v.z) - shift > 0.0 ? 4u : 0u) |
              (static_cast<double>(v.w) - shift > 0.0 ? 8u : 0u);
      } else {
        nib = (v.x > 0.f ? 1u : 0u) | (v.y > 0.f ? 2u : 0u) | (v.z > 0.f ? 4u : 0u) |
              (v.w > 0.f ? 8u : 0u);
        abs_sum += fabs(static_cast<double>(v.x)) + fabs(static_cast<double>(v.y)) +
                   fabs(static_cast<double>(v.z)) + fabs(static_cast<double>(v.w));
      }
      const uint32_t word = nibble_words(nib, lane);
      if ((lane & 7) == 0) dst[s * 4] = word;
    }
    if (!kBitNet) {
      abs_sum = warp_sum(abs_sum);
      if (lane == 0) alpha[row] = static_cast<float>(abs_sum / static_cast<double>(K));
    }
  }
}

// b1.58 ternary pass (after row_sums_kernel and global_scalars_kernel, whose
// scalars[1] is gamma = mean |W| in fp64). q = W / (gamma + eps) is divided in
// fp64 exactly as the formula reads; round-half-even then clip to [-1, 1] is
// +1 for q > 1/2, -1 for q < -1/2 and 0 otherwise (q = +-1/2 ties to 0).
// Row layout: per 128-k block, 4 words of the +1 plane then 4 of the -1 plane.
constexpr double kTernaryEps = 1e-5;
__global__ void __launch_bounds__(kPackThreads) pack_ternary_rows_kernel(
    const float* __restrict__ W, int64_t N, int64_t K, uint32_t* __restrict__ packed,
    const double* __restrict__ scalars) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const double d = scalars[1] + kTernaryEps;
  const int64_t steps = K / 128;  // one 128-k block per warp step
  for (int64_t row = warp0; row < N; row += nwarps) {
    const float4* src = reinterpret_cast<const float4*>(W + row * K) + lane;
    uint32_t* dst = packed + row * (K / 16) + (lane >> 3);
    for (int64_t s = 0; s < steps; ++s) {
      const float4 v = __ldcs(src + s * 32);
      const double q[4] = {static_cast<double>(v.x) / d, static_cast<double>(v.y) / d,
                           static_cast<double>(v.z) / d, static_cast<double>(v.w) / d};
      uint32_t plus = 0u, minus = 0u;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        plus |= (q[i] > 0.5 ? 1u : 0u) << i;
        minus |= (q[i] < -0.5 ? 1u : 0u) << i;
      }
      const uint32_t pw = nibble_words(plus, lane), mw = nibble_words(minus, lane);
      if ((lane & 7) == 0) {
        dst[s * 8] = pw;
        dst[s * 8 + 4] = mw;
      }
    }
  }
}

// BitNet pass 1: per-row sum W and sum |W| in fp64 -> sums[2*row + {0,1}].
__global__ void __launch_bounds__(kPackThreads) row_sums_kernel(const float* __restrict__ W,
                                                                int64_t N, int64_t K,
                                                                double* __restrict__ sums) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t steps = K / 128;
  for (int64_t row = warp0; row < N; row += nwarps) {
    const float4* src = reinterpret_cast<const float4*>(W + row * K) + lane;
    double s = 0.0, a = 0.0;
    int64_t i = 0;
    for (; i + 4 <= steps; i += 4) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + (i + u) * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        s += (static_cast<double>(v[u].x) + static_cast<double>(v[u].y)) +
             (static_cast<double>(v[u].z) + static_cast<double>(v[u].w));
        a += (fabs(static_cast<double>(v[u].x)) + fabs(static_cast<double>(v[u].y))) +
             (fabs(static_cast<double>(v[u].z)) + fabs(static_cast<double>(v[u].w)));
      }
    }
    for (; i < steps; ++i) {
      const float4 v = __ldcs(src + i * 32);
      s += (static_cast<double>(v.x) + static_cast<double>(v.y)) +
           (static_cast<double>(v.z) + static_cast<double>(v.w));
      a += (fabs(static_cast<double>(v.x)) + fabs(static_cast<double>(v.y))) +
           (fabs(static_cast<double>(v.z)) + fabs(static_cast<double>(v.w)));
    }
    s = warp_sum(s);
    a = warp_sum(a);
    if (lane == 0) {
      sums[2 * row] = s;
      sums[2 * row + 1] = a;
    }
  }
}

// BitNet pass 2: one block folds the row sums in a fixed order into the
// global mean (Eq.3) and beta (Eq.8). scalars[0] = mean (fp64, used by the
// sign pass), scalars[1] = beta (fp64); alpha_out[0] / beta_out[0] get the
// fp32 roundings.
constexpr int kReduceThreads = 1024;
__global__ void __launch_bounds__(kReduceThreads) global_scalars_kernel(
    const double* __restrict__ sums, int64_t N, int64_t K, double* __restrict__ scalars,
    float* __restrict__ alpha_out, float* __restrict__ beta_out) {
  __shared__ double sh_s[kReduceThreads / 32], sh_a[kReduceThreads / 32];
  double s = 0.0, a = 0.0;
  for (int64_t r = threadIdx.x; r < N; r += kReduceThreads) {
    s += sums[2 * r];
    a += sums[2 * r + 1];
  }
  s = warp_sum(s);
  a = warp_sum(a);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sh_s[warp] = s;
    sh_a[warp] = a;
  }
  __syncthreads();
  if (warp == 0) {
    s = sh_s[lane];
    a = sh_a[lane];
    s = warp_sum(s);
    a = warp_sum(a);
    if (lane == 0) {
      const double count = static_cast<double>(N) * static_cast<double>(K);
      const double mean = s / count;
      const double beta = a / count;
      scalars[0] = mean;
      scalars[1] = beta;
      if (alpha_out) alpha_out[0] = static_cast<float>(mean);
      beta_out[0] = static_cast<float>(beta);
    }
  }
}

}  // namespace bl

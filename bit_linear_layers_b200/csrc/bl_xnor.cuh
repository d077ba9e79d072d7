// W1A1: products of two +-1 matrices by XOR and population count
// ("BitNet-Transformers" page: with 1-bit weights and activations the matrix
// product reduces to XNOR / popcount arithmetic):
//   dot[m][n] = sum_k a_mk * b_nk = K - 2 * popcount(a_m XOR b_n)
// with a and b in the packed sign layout (bit set = +1). No tensor-core MMA
// kind takes 1-bit operands on sm_100, so this runs on the integer ALUs and
// is bounded by population-count throughput.
//
// A CTA of 16 x 16 threads computes a 64 x 64 tile; thread (tx, ty) owns rows
// m0 + ty + 16 i and columns n0 + tx + 16 j (i, j < 4). K is consumed in
// chunks of 32 words staged in shared memory with rows padded to 33 words,
// so the 16 distinct rows a warp reads from the B tile fall in 16 banks.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kXnorTile = 64;
constexpr int kXnorChunk = 32;  // words of K per stage
constexpr int kXnorPad = kXnorChunk + 1;

__global__ void __launch_bounds__(256) xnor_gemm_kernel(const uint32_t* __restrict__ a,
                                                        const uint32_t* __restrict__ b,
                                                        int32_t* __restrict__ dot, int64_t M, int64_t N,
                                                        int64_t K) {
  __shared__ uint32_t sa[kXnorTile][kXnorPad];
  __shared__ uint32_t sb[kXnorTile][kXnorPad];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kXnorTile;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kXnorTile;
  const int64_t words = K / 32;
  int cnt[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) cnt[i][j] = 0;

  for (int64_t w0 = 0; w0 < words; w0 += kXnorChunk) {
    // stage 64 rows x 32 words of each operand (rows past M / N and words past
    // the row are zero; they are never counted into a stored output)
    for (int e = threadIdx.x; e < kXnorTile * kXnorChunk; e += 256) {
      const int r = e / kXnorChunk, c = e % kXnorChunk;
      const int64_t w = w0 + c;
      sa[r][c] = (m0 + r < M && w < words) ? a[(m0 + r) * words + w] : 0u;
      sb[r][c] = (n0 + r < N && w < words) ? b[(n0 + r) * words + w] : 0u;
    }
    __syncthreads();
    const int cw = static_cast<int>(words - w0 < kXnorChunk ? words - w0 : kXnorChunk);
    for (int c = 0; c < cw; ++c) {
      uint32_t av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = sa[ty + 16 * i][c];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = sb[tx + 16 * j][c];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) cnt[i][j] += __popc(av[i] ^ bv[j]);
    }
    __syncthreads();
  }
  const int32_t k32 = static_cast<int32_t>(K);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx + 16 * j;
      if (n < N) dot[m * N + n] = k32 - 2 * cnt[i][j];
    }
  }
}

}  // namespace bl

// W1A16 for a decode batch of a few tokens (up to 16): y_mj = bf16(alpha_j *
// sum_k s_jk x_mk) ("FBI-LLM" page, FBI-linear paragraph; W1A16), a GEMV-like
// sweep over the packed signs whose products run on the tensor cores through
// the warp-level m16n8k16 bf16 MMA.
//
// Why this and not the tcgen05 GEMM: with at most 16 tokens the work per
// weight is tiny and the launch is latency-bound; the tcgen05 kernel's
// pipeline (tensor-memory allocation, mbarrier rings, split-K epilogue)
// costs ~15 us per call at 16 x 4096 x 4096, while this kernel has the
// structure of the single-token lookup kernel: a cluster of 8 CTAs splits K,
// every CTA holds its slice of x in shared memory and sweeps 64 rows, and
// the row owners (8 rows each) add the 8 partials. Small CTAs (4 warps) keep
// several resident per SM, so the rows spread evenly over the SMs.
//
// Per warp: 16 rows (g and g + 8 of the MMA's A fragment) over the CTA's K
// slice. Each 16-bit chunk b of a row's packed word becomes the lane's A
// registers with r = b | (b << 15): shifting r left by 15 - 2t puts bits 2t
// and 2t + 1 at the two bf16 sign positions, and the mask and xor with
// -1,-1 turn a set bit into +1 (t = lane % 4, so the lane gets columns 2t,
// 2t + 1 and, shifting by 7 - 2t, 2t + 8, 2t + 9). The B fragment is two
// adjacent bf16 of one token read from the staged x slice. Accumulation fp32.
#pragma once

#include "bl_gemv_lut.cuh"

namespace bl {

constexpr int kMmaThreads = 128;             // 4 warps x 16 rows
constexpr int kMmaRowsPerCluster = 64;       // rows swept by each CTA of a cluster (over its K slice)
constexpr int kMmaCluster = 8;               // K split
constexpr int kMmaMaxSliceWords = 48;        // K <= 8 * 48 * 32 = 12288

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte global -> shared copy that does not hold a register; src_bytes = 0
// fills the destination with zeros (nothing is read)
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void st_async_v2_f32(uint32_t remote_addr, float a, float b, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(
                   remote_addr),
               "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(remote_bar)
               : "memory");
}

// x slice row pitch in shared memory (bytes): the slice plus 16 bytes, so that
// the 8 tokens x 4 column pairs a warp reads per B fragment hit 32 banks
__host__ __device__ constexpr int mma_x_pitch(int slice_words) { return slice_words * 64 + 16; }
__host__ __device__ constexpr int mma_smem_bytes(int mt, int slice_words) { return mt * mma_x_pitch(slice_words); }

// MT = 8 or 16 tokens per tile (M <= MT); SWMAX = 16 (K <= 4096) or 48
// (K <= 12288) slice words held in registers.
template <int MT, int SWMAX>
__global__ void __launch_bounds__(kMmaThreads, SWMAX <= 16 ? 4 : 2) gemv_w1a16_mma_kernel(
    const uint16_t* __restrict__ x, const uint32_t* __restrict__ packed, const float* __restrict__ alpha,
    uint16_t* __restrict__ y, int M, int N, int K) {
  extern __shared__ __align__(16) uint8_t mma_smem[];
  __shared__ __align__(16) float inbox[kMmaCluster * 8 * MT];  // [source rank][owned row][token]
  __shared__ __align__(8) uint64_t inbox_bar;
  constexpr int H = MT / 8;  // n-halves of the token tile

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int words = K / 32;
  const int sw = words / kMmaCluster;  // slice words (K % 256 == 0)
  const int slice0 = static_cast<int>(rank) * sw;
  const int row_a = blockIdx.y * kMmaRowsPerCluster + warp * 16 + g;  // rows g and g + 8 of this warp
  const int row_b = row_a + 8;
  const int pitch = mma_x_pitch(sw);

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&inbox_bar), 1);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();  // waited on just before the first push

  // ---- 1. this warp's packed words (independent of x): two rows per lane ----
  uint32_t wa[SWMAX], wb[SWMAX];
#pragma unroll
  for (int w = 0; w < SWMAX; ++w) {
    wa[w] = (w < sw && row_a < N) ? __ldcs(packed + static_cast<int64_t>(row_a) * words + slice0 + w) : 0u;
    wb[w] = (w < sw && row_b < N) ? __ldcs(packed + static_cast<int64_t>(row_b) * words + slice0 + w) : 0u;
  }

  // x may be produced by the previous kernel on the stream
  grid_dependency_wait();
  grid_dependents_launch();

  // ---- 2. stage this CTA's slice of x with asynchronous 16-byte copies, all
  // issued before any is waited for (tokens past M are zero-filled) ----
  {
    const int vec_per_tok = sw * 4;  // 16-byte vectors per token: 32 bf16 per word
    for (int e = threadIdx.x; e < MT * vec_per_tok; e += kMmaThreads) {
      const int m = e / vec_per_tok, v = e - m * vec_per_tok;
      const uint16_t* src = x + static_cast<int64_t>(m < M ? m : 0) * K + slice0 * 32 + v * 8;
      cp_async_16(smem_u32(mma_smem + m * pitch + v * 16), src, m < M ? 16u : 0u);
    }
    cp_async_wait_all();
  }
  __syncthreads();

  // ---- 3. MMAs over the slice: 2 chunks of 16 k per packed word ----
  float acc[H][4];
#pragma unroll
  for (int hh = 0; hh < H; ++hh)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[hh][i] = 0.f;
  const uint32_t sh_lo = 15 - 2 * t, sh_hi = 7 - 2 * t;
  const uint8_t* xb = mma_smem + g * pitch + 4 * t;  // token g, column pair 2t
#pragma unroll
  for (int w = 0; w < SWMAX; ++w) {
    if (w < sw) {
#pragma unroll
      for (int o = 0; o < 2; ++o) {
        const uint32_t ba = (wa[w] >> (16 * o)) & 0xFFFFu, bb = (wb[w] >> (16 * o)) & 0xFFFFu;
        const uint32_t ra = ba | (ba << 15), rb = bb | (bb << 15);
        const uint32_t a[4] = {((ra << sh_lo) & 0x80008000u) ^ 0xBF80BF80u, ((rb << sh_lo) & 0x80008000u) ^ 0xBF80BF80u,
                               ((ra << sh_hi) & 0x80008000u) ^ 0xBF80BF80u, ((rb << sh_hi) & 0x80008000u) ^ 0xBF80BF80u};
        const int kb = (w * 32 + o * 16) * 2;  // byte offset of the chunk in a token row
#pragma unroll
        for (int hh = 0; hh < H; ++hh) {
          const uint8_t* p = xb + hh * 8 * pitch + kb;
          mma_bf16_16816(acc[hh], a, *reinterpret_cast<const uint32_t*>(p),
                         *reinterpret_cast<const uint32_t*>(p + 16));
        }
      }
    }
  }

  // ---- 4. push the partials to the rows' owners: warp w's rows g belong to rank
  // 2w and its rows g + 8 to rank 2w + 1 (8 rows each) ----
  if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(&inbox_bar), kMmaCluster * 8 * MT * 4);
  cluster_wait();  // every CTA's inbox barrier is initialised
  {
    const uint32_t own_a = static_cast<uint32_t>(2 * warp), own_b = own_a + 1;
    const uint32_t bar_a = map_to_rank(smem_u32(&inbox_bar), own_a);
    const uint32_t bar_b = map_to_rank(smem_u32(&inbox_bar), own_b);
    // acc[hh]: (row g, tokens 2t, 2t+1) and (row g + 8, same tokens), tokens offset by 8 hh
#pragma unroll
    for (int hh = 0; hh < H; ++hh) {
      const int tok = 8 * hh + 2 * t;
      const uint32_t slot = smem_u32(&inbox[(static_cast<int>(rank) * 8 + g) * MT + tok]);
      st_async_v2_f32(map_to_rank(slot, own_a), acc[hh][0], acc[hh][1], bar_a);
      st_async_v2_f32(map_to_rank(slot, own_b), acc[hh][2], acc[hh][3], bar_b);
    }
  }
  // ---- 5. owner: thread (token m, row r) adds the 8 partials in rank order ----
  if (threadIdx.x < 8 * MT) {
    const int r = threadIdx.x & 7, m = threadIdx.x >> 3;
    const int row = blockIdx.y * kMmaRowsPerCluster + static_cast<int>(rank) * 8 + r;
    if (mbar_wait(smem_u32(&inbox_bar), 0, kWhereMmaInbox)) {
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < kMmaCluster; ++q) s += inbox[(q * 8 + r) * MT + m];
      if (m < M && row < N) y[static_cast<int64_t>(m) * N + row] = float_to_bf16_bits(alpha[row] * s);
    }
  }
}

}  // namespace bl

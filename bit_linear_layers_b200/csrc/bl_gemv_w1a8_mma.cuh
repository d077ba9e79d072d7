// BitLinear W1A8 products for a decode batch of a few tokens (up to 16) on the
// warp-level int8 MMA ("BitNet b1.58" page, section 1, Eq.(7): acc_mj = sum_k
// W~_jk q_mk in exact integer arithmetic, then y_mj = acc_mj * beta *
// gamma_m / Q_b; section 2 for the ternary weights of b1.58).
//
// The codes q (int8, [M][K]) come from the LN + quantisation kernel launched
// just before; this kernel may be scheduled while that one runs
// (programmatic dependent launch) and reads the codes only after
// griddepcontrol.wait. Its weights do not depend on them, so every CTA starts
// copying its packed words into shared memory before the wait.
//
// Work split as in the few-token W1A16 GEMV (bl_gemv_mma.cuh): a cluster of 8
// CTAs splits K into slices of K / 8 (a whole number of 32-k words), each CTA
// sweeps 64 rows over its slice with 4 warps of 16 rows, and 8-row owners add
// the 8 slice partials. Per 32-k word a warp issues one m16n8k32 s8 MMA per 8
// tokens: lane (g, t)'s A registers are the +-1 (or +1 / 0 / -1) bytes of
// rows g and g + 8 at k = 4t .. 4t + 3 and 16 + 4t .. 16 + 4t + 3, i.e. one
// nibble of each packed word spread into four bytes; its B registers are the
// codes of token g at the same k, one 32-bit shared load each. The partials
// and their sums are int32 and exact, so the accumulators equal the
// oracle's integer products bit for bit; the rescale is the one of the dp4a
// GEMV (fp64, one rounding to fp32).
#pragma once

#include "bl_gemv.cuh"
#include "bl_gemv_mma.cuh"

namespace bl {

constexpr int kQmThreads = 128;        // 4 warps x 16 rows
constexpr int kQmRows = 64;            // rows per CTA
constexpr int kQmMaxSliceWords = 48;   // K <= 8 * 48 * 32 = 12288

// row pitch of the staged words (odd: the 8 rows a warp instruction reads
// fall in 8 banks); ternary rows hold the +1 words, then the -1 words
__host__ __device__ constexpr int qm_word_pitch(int sw, bool ternary) { return (ternary ? 2 * sw : sw) | 1; }
// token pitch of the staged codes in bytes: a multiple of 128 plus 16, so the
// B loads of a warp (8 tokens x 4 lanes x 4 bytes) hit 32 banks
__host__ __device__ constexpr int qm_code_pitch(int sw) { return (sw * 32 + 127) / 128 * 128 + 16; }
__host__ __device__ constexpr int qm_smem_bytes(int mt, int sw, bool ternary) {
  return kQmRows * qm_word_pitch(sw, ternary) * 4 + mt * qm_code_pitch(sw);
}

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// MT = 8 or 16 tokens per tile (M <= MT). K % 256 == 0, K <= 12288.
template <int MT, bool kTernary>
__global__ void __launch_bounds__(kQmThreads) gemv_w1a8_mma_kernel(
    const int8_t* __restrict__ xq, const double* __restrict__ gamma, const uint32_t* __restrict__ packed,
    const float* __restrict__ beta, float* __restrict__ y, int32_t* __restrict__ acc_out, int M, int N, int K) {
  extern __shared__ __align__(16) uint8_t qm_smem[];
  __shared__ __align__(16) int32_t inbox[kMmaCluster * 8 * MT];  // [source rank][owned row][token]
  __shared__ __align__(8) uint64_t inbox_bar;
  constexpr int H = MT / 8;  // MMAs per word: 8 tokens each
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int sw = K / 32 / kMmaCluster;  // words of this CTA's slice
  const int w0 = static_cast<int>(rank) * sw;
  const int wpitch = qm_word_pitch(sw, kTernary), cpitch = qm_code_pitch(sw);
  uint32_t* ws = reinterpret_cast<uint32_t*>(qm_smem);  // [64 rows][wpitch]
  uint8_t* cs = qm_smem + kQmRows * wpitch * 4;          // [MT tokens][cpitch]
  const int row0 = static_cast<int>(blockIdx.y) * kQmRows;
  const int64_t rstride = kTernary ? K / 16 : K / 32;    // words per packed row

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&inbox_bar), 1);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();  // waited on just before the first push

  // ---- 1. this CTA's packed words (independent of the codes): rows past N are zero ----
  for (int e = threadIdx.x; e < kQmRows * sw; e += kQmThreads) {
    const int r = e / sw, w = e - r * sw;
    const int row = row0 + r;
    uint32_t* d = ws + r * wpitch + w;
    if (row < N) {
      const int wi = w0 + w;
      const int64_t off = kTernary ? static_cast<int64_t>(wi >> 2) * 8 + (wi & 3) : wi;
      cp_async_4(smem_u32(d), packed + static_cast<int64_t>(row) * rstride + off);
      if (kTernary) cp_async_4(smem_u32(d + sw), packed + static_cast<int64_t>(row) * rstride + off + 4);
    } else {
      d[0] = 0u;
      if (kTernary) d[sw] = 0u;
    }
  }
  const double bt = static_cast<double>(*beta);

  // the codes and gamma may be produced by the previous kernel on the stream
  grid_dependency_wait();

  // ---- 2. the codes of this slice for every token (tokens past M are zero) ----
  {
    const int vec = sw * 2;  // 16-byte vectors per token: 32 codes per word
    for (int e = threadIdx.x; e < MT * vec; e += kQmThreads) {
      const int m = e / vec, v = e - m * vec;
      const int8_t* src = xq + static_cast<int64_t>(m < M ? m : 0) * K + w0 * 32 + v * 16;
      cp_async_16(smem_u32(cs + m * cpitch + v * 16), src, m < M ? 16u : 0u);
    }
    cp_async_wait_all();
  }
  __syncthreads();

  // ---- 3. one m16n8k32 MMA per word and 8 tokens ----
  int acc[H][4];
#pragma unroll
  for (int hh = 0; hh < H; ++hh)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[hh][i] = 0;
  const uint32_t* wra = ws + (warp * 16 + g) * wpitch;  // rows g and g + 8 of this warp
  const uint32_t* wrb = wra + 8 * wpitch;
  const uint8_t* cb = cs + g * cpitch + 4 * t;          // token g, k = 4t of each word
  const int s_lo = 4 * t, s_hi = 16 + 4 * t;
#pragma unroll 4
  for (int w = 0; w < sw; ++w) {
    const uint32_t pa = wra[w], pb = wrb[w];
    uint32_t a[4];
    if (kTernary) {
      const uint32_t ma = wra[sw + w], mb = wrb[sw + w];
      a[0] = nibbles_to_ternary_i8((pa >> s_lo) & 0xFu, (ma >> s_lo) & 0xFu);
      a[1] = nibbles_to_ternary_i8((pb >> s_lo) & 0xFu, (mb >> s_lo) & 0xFu);
      a[2] = nibbles_to_ternary_i8((pa >> s_hi) & 0xFu, (ma >> s_hi) & 0xFu);
      a[3] = nibbles_to_ternary_i8((pb >> s_hi) & 0xFu, (mb >> s_hi) & 0xFu);
    } else {
      a[0] = nibble_to_pm1_i8((pa >> s_lo) & 0xFu);
      a[1] = nibble_to_pm1_i8((pb >> s_lo) & 0xFu);
      a[2] = nibble_to_pm1_i8((pa >> s_hi) & 0xFu);
      a[3] = nibble_to_pm1_i8((pb >> s_hi) & 0xFu);
    }
#pragma unroll
    for (int hh = 0; hh < H; ++hh) {
      const uint8_t* p = cb + hh * 8 * cpitch + 32 * w;
      mma_s8_16832(acc[hh], a, *reinterpret_cast<const uint32_t*>(p), *reinterpret_cast<const uint32_t*>(p + 16));
    }
  }

  // ---- 4. partials to the rows' owners: warp w's rows g belong to rank 2w,
  // its rows g + 8 to rank 2w + 1 (8 rows each) ----
  if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(&inbox_bar), kMmaCluster * 8 * MT * 4);
  cluster_wait();  // every CTA's inbox barrier is initialised
  {
    const uint32_t own_a = static_cast<uint32_t>(2 * warp), own_b = own_a + 1;
    const uint32_t bar_a = map_to_rank(smem_u32(&inbox_bar), own_a);
    const uint32_t bar_b = map_to_rank(smem_u32(&inbox_bar), own_b);
#pragma unroll
    for (int hh = 0; hh < H; ++hh) {
      const int tok = 8 * hh + 2 * t;
      const uint32_t slot = smem_u32(&inbox[(static_cast<int>(rank) * 8 + g) * MT + tok]);
      st_async_v2_f32(map_to_rank(slot, own_a), __int_as_float(acc[hh][0]), __int_as_float(acc[hh][1]), bar_a);
      st_async_v2_f32(map_to_rank(slot, own_b), __int_as_float(acc[hh][2]), __int_as_float(acc[hh][3]), bar_b);
    }
  }
  // ---- 5. owner: thread (token m, row r) adds the 8 partials and rescales ----
  if (threadIdx.x < 8 * MT) {
    const int r = threadIdx.x & 7, m = threadIdx.x >> 3;
    const int row = row0 + static_cast<int>(rank) * 8 + r;
    if (mbar_wait(smem_u32(&inbox_bar), 0, kWhereMmaInbox) && m < M && row < N) {
      int a = 0;
#pragma unroll
      for (int q = 0; q < kMmaCluster; ++q) a += inbox[(q * 8 + r) * MT + m];
      const int64_t o = static_cast<int64_t>(m) * N + row;
      y[o] = static_cast<float>(static_cast<double>(a) * bt * gamma[m] / 128.0);
      if (acc_out) acc_out[o] = a;
    }
  }
}

}  // namespace bl

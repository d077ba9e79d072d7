// Single-token W1A16 decode GEMV by byte lookup table ("FBI-LLM" page,
// FBI-linear paragraph: y_j = alpha_j * sum_k sign(W_jk) x_k, W1A16).
//
// Every byte of a packed row covers 8 consecutive inputs, so the row's dot
// product is a sum over bytes of T_g[v] = sum_{i<8} (bit_i(v) ? +x : -x)_{8g+i},
// v being the byte's value. A CTA builds T for its slice of K once (256
// entries per byte position) and then pays, per 8 weights, one PRMT (which
// forms the shared-memory address v*256 + column directly from the packed
// word), one LDS and one FADD.
//
// Layout and schedule:
//   * a cluster of C CTAs splits K into C slices; each CTA builds the table
//     of its slice (64 byte positions per 64 KB page) and sweeps all R rows
//     of the cluster over that slice. Row r belongs to CTA r / (R/C); every
//     CTA pushes its partial sum of each row into the owner's inbox with
//     st.async, completing on the owner's mbarrier, and the owner adds the C
//     partials in a fixed order once its 1 KB of transactions has landed (no
//     cluster-wide barrier at the end; a split arrive/wait at the start makes
//     sure every inbox barrier is initialised before anything is pushed);
//   * table page layout T[v][col], 64 fp32 columns per v; the byte at
//     position i of slice word w lives in column i*16 + (w % 16), and the two
//     half-warps visit the four bytes of a word in orders rotated by one, so
//     each warp's 32 lookups land on 32 distinct banks;
//   * a warp handles 32 rows as 16 row pairs (half-warp = one row); each lane
//     reads one packed word per row per 16-word page (its 64 table lookups
//     are all issued before the adds, for latency overlap), prefetched into
//     registers before anything else (and before griddepcontrol.wait, so a
//     launch with programmatic serialisation streams its weights while the
//     previous kernel finishes);
//   * per-lane partial sums of the 16 row pairs are combined by a 4-stage
//     reduce-scatter, leaving one finished row slice per lane.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kLutThreads = 256;
constexpr int kLutWarps = kLutThreads / 32;
constexpr int kLutRowsPerCluster = kLutWarps * 32;  // 256: one 32-row chunk per warp
constexpr int kLutPageBytes = 256 * 64 * 4;         // 64 KB: 256 values x 64 columns
constexpr int kLutMaxPages = 3;                     // slice of at most 48 words

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
// shared::cluster address of `local` in the CTA of cluster rank `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  return remote;
}
// 4-byte store into another CTA's shared memory, counted on its mbarrier
__device__ __forceinline__ void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}

// ---- pieces shared with the multi-layer decode kernel ----

// Packed words of 16 row pairs of one warp (rows w0 + 2p + h), NP pages of
// this CTA's slice; rows past N and words past the slice read as zero.
template <int NP>
__device__ __forceinline__ void lut_load_rows(uint32_t (&wv)[16][NP], const uint32_t* __restrict__ packed,
                                              int N, int words, int w0, int slice0, int slice_words, int h,
                                              int wl) {
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const int row = w0 + 2 * p + h;
#pragma unroll
    for (int pg = 0; pg < NP; ++pg) {
      const int wi = pg * 16 + wl;
      wv[p][pg] = (row < N && wi < slice_words)
                      ? __ldcs(packed + static_cast<int64_t>(row) * words + slice0 + wi)
                      : 0u;
    }
  }
}

// Table of a slice whose first input is xs[0]. Task = (page, value quarter,
// column); column c holds byte i = c/16 of word c%16. kCoherent reads x
// through L2 only (it may have been written by other CTAs of the same launch).
template <int NP, bool kCoherent>
__device__ __forceinline__ void lut_build_table(const uint16_t* __restrict__ xs, int slice_words,
                                                uint8_t* lut_smem) {
  for (int task = threadIdx.x; task < NP * 4 * 64; task += kLutThreads) {
    const int c = task & 63, qtr = (task >> 6) & 3, pg = task >> 8;
    const int wi = pg * 16 + (c & 15);
    if (wi >= slice_words) continue;
    const int g = 4 * wi + (c >> 4);  // byte position within the slice
    const uint4* src = reinterpret_cast<const uint4*>(xs + 8 * g);
    const uint4 raw = kCoherent ? __ldcg(src) : *src;
    const float x0 = bf16_bits_to_float(raw.x & 0xFFFFu), x1 = __uint_as_float(raw.x & 0xFFFF0000u);
    const float x2 = bf16_bits_to_float(raw.y & 0xFFFFu), x3 = __uint_as_float(raw.y & 0xFFFF0000u);
    const float x4 = bf16_bits_to_float(raw.z & 0xFFFFu), x5 = __uint_as_float(raw.z & 0xFFFF0000u);
    const float x6 = bf16_bits_to_float(raw.w & 0xFFFFu), x7 = __uint_as_float(raw.w & 0xFFFF0000u);
    // signed pair sums, index = the two bits (bit 0 = lower k)
    const float p01[4] = {-x0 - x1, x0 - x1, -x0 + x1, x0 + x1};
    const float p23[4] = {-x2 - x3, x2 - x3, -x2 + x3, x2 + x3};
    const float p45[4] = {-x4 - x5, x4 - x5, -x4 + x5, x4 + x5};
    // bits 6 and 7 of this task's values are fixed by its quarter
    const float q67 = ((qtr & 1) ? x6 : -x6) + ((qtr & 2) ? x7 : -x7);
    float lo[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) lo[v] = p01[v & 3] + p23[v >> 2];
    float* page = reinterpret_cast<float*>(lut_smem + pg * kLutPageBytes);
#pragma unroll
    for (int hq = 0; hq < 4; ++hq) {
      const int hi = qtr * 4 + hq;
      const float hv = p45[hq] + q67;
#pragma unroll
      for (int v = 0; v < 16; ++v) page[(hi * 16 + v) * 64 + c] = lo[v] + hv;
    }
  }
}

// Lookups of the 16 row pairs over the slice, then a reduce-scatter over the
// 16 lanes of each half-warp: the return value is the slice's partial sum of
// row 2 * wl + h of the warp's 32 rows.
template <int NP>
__device__ __forceinline__ float lut_row_partial(const uint32_t (&wv)[16][NP], int slice_words,
                                                 const uint8_t* lut_smem, int h, int wl) {
  uint32_t sel[4], colb[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint32_t i = (s + h) & 3;
    colb[s] = (i * 16 + wl) * 4;
    sel[s] = 0x5504u | (i << 4);  // byte0 <- column byte, byte1 <- word byte i, bytes 2,3 <- 0
  }
  // all 64 lookups of a page are issued before any of them is added, so the
  // shared-memory latency overlaps (a lane whose word lies past the slice
  // reads a zero word: its lookups are discarded below)
  float acc[16];
#pragma unroll
  for (int p = 0; p < 16; ++p) acc[p] = 0.f;
#pragma unroll
  for (int pg = 0; pg < NP; ++pg) {
    const uint8_t* page = lut_smem + pg * kLutPageBytes;
    const bool live = pg * 16 + wl < slice_words;
    float t[16][4];
#pragma unroll
    for (int p = 0; p < 16; ++p)
#pragma unroll
      for (int s = 0; s < 4; ++s)
        t[p][s] = *reinterpret_cast<const float*>(page + __byte_perm(wv[p][pg], colb[s], sel[s]));
#pragma unroll
    for (int p = 0; p < 16; ++p)
      if (live) acc[p] += (t[p][0] + t[p][1]) + (t[p][2] + t[p][3]);
  }
  // reduce-scatter over the 16 lanes of each half: lane wl ends with row pair wl
#pragma unroll
  for (int d = 8, n = 16; d >= 1; d >>= 1, n >>= 1) {
    const bool upper = (wl & d) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? acc[j] : acc[j + n / 2];
      const float keep = upper ? acc[j + n / 2] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, d);
    }
  }
  return acc[0];
}

// NP = pages (16-word groups) per slice; slice_words <= 16 * NP.
// One-page slices fit two CTAs per SM (registers capped at 128), which lets
// an overlapped next launch co-reside with the one finishing.
template <int NP>
__global__ void __launch_bounds__(kLutThreads, NP == 1 ? 2 : 1) gemv_w1a16_lut_kernel(
    const uint16_t* __restrict__ x, const uint32_t* __restrict__ packed,
    const float* __restrict__ alpha, uint16_t* __restrict__ y, int N, int K, int slice_words) {
  extern __shared__ __align__(1024) uint8_t lut_smem[];
  __shared__ float inbox[kLutRowsPerCluster];  // [source rank][owned row]
  __shared__ __align__(8) uint64_t inbox_bar;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = lane >> 4;    // which row of the pair
  const int wl = lane & 15;   // word slot within a page
  const uint32_t rank = cluster_ctarank();
  const int C = gridDim.x;    // cluster spans the whole x extent of the grid
  const int row0 = blockIdx.y * kLutRowsPerCluster;
  const int words = K / 32;
  const int slice0 = static_cast<int>(rank) * slice_words;  // first word of this CTA's slice
  const int rows_per_cta = kLutRowsPerCluster / C;          // rows this CTA owns

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&inbox_bar), 1);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();  // waited on just before the first push

  // ---- 1. prefetch this warp's packed words (independent of x) ----
  uint32_t wv[16][NP];
  lut_load_rows<NP>(wv, packed, N, words, row0 + warp * 32, slice0, slice_words, h, wl);

  // x may be produced by the previous kernel on the stream
  grid_dependency_wait();
  grid_dependents_launch();

  // ---- 2. build the table of this slice ----
  lut_build_table<NP, false>(x + static_cast<int64_t>(slice0) * 32, slice_words, lut_smem);
  __syncthreads();

  // ---- 3./4. lookups and the per-row reduce-scatter ----
  const float part = lut_row_partial<NP>(wv, slice_words, lut_smem, h, wl);

  // ---- 5. push each row's partial to its owner; the owner adds the C partials ----
  if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(&inbox_bar), kLutRowsPerCluster * 4);
  cluster_wait();  // every CTA's inbox barrier is initialised
  {
    const int r = warp * 32 + 2 * wl + h;  // this lane's row within the cluster
    const uint32_t owner = static_cast<uint32_t>(r / rows_per_cta);
    const uint32_t slot = smem_u32(&inbox[static_cast<int>(rank) * rows_per_cta + r % rows_per_cta]);
    st_async_f32(map_to_rank(slot, owner), part, map_to_rank(smem_u32(&inbox_bar), owner));
  }
  if (threadIdx.x < rows_per_cta) {
    const int r = static_cast<int>(rank) * rows_per_cta + threadIdx.x;
    const int row = row0 + r;
    if (mbar_wait(smem_u32(&inbox_bar), 0, kWhereLutInbox)) {
      float s = 0.f;
      for (int q = 0; q < C; ++q) s += inbox[q * rows_per_cta + threadIdx.x];
      if (row < N) y[row] = float_to_bf16_bits(alpha[row] * s);
    }
  }
}

// Cluster size and slice for a given K (K % 128 == 0): the largest C in
// {8, 4, 2, 1} that splits the row into whole-word slices of 16..48 words;
// for short rows (fewer than 16 words) a single CTA takes the whole row.
// Returns false when no supported split exists.
inline bool lut_split(int K, int* C_out, int* slice_words_out, int* pages_out) {
  const int words = K / 32;
  int chosen = 0;
  for (int C : {8, 4, 2, 1}) {
    if (words % C == 0 && words / C >= 16 && words / C <= 16 * kLutMaxPages) {
      chosen = C;
      break;
    }
  }
  if (!chosen && words < 16) chosen = 1;
  if (!chosen) return false;
  *C_out = chosen;
  *slice_words_out = words / chosen;
  *pages_out = (*slice_words_out + 15) / 16;
  return true;
}

}  // namespace bl

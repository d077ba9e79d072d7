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
//     position i of window word w lives in column i*16 + (w % 16), and the two
//     half-warps visit the four bytes of a word in orders rotated by one, so
//     each warp's 32 lookups land on 32 distinct banks;
//   * 16 warps; a warp handles 16 rows as 8 row pairs (half-warp = one row);
//     each lane reads one packed word per row per 16-word page (its 32 table
//     lookups are all issued before the adds, for latency overlap, and the
//     adds of two row pairs go through one packed f32x2 add), prefetched into
//     registers before anything else (and before griddepcontrol.wait, so a
//     launch with programmatic serialisation streams its weights while the
//     previous kernel finishes);
//   * per-lane partial sums of the 8 row pairs are combined by a 3-stage
//     reduce-scatter and a final pairwise add, leaving each row's slice sum
//     in the two lanes of its word-slot pair.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kLutThreads = 512;
constexpr int kLutWarps = kLutThreads / 32;
constexpr int kLutPairs = 8;                        // row pairs per warp
constexpr int kLutRowsPerWarp = 2 * kLutPairs;      // 16
constexpr int kLutRowsPerCluster = kLutWarps * kLutRowsPerWarp;  // 256
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
//
// A CTA's slice of a packed row is words [s0, s0 + sw). It is visited through
// a window that starts at a0 = s0 rounded down to a multiple of 4 words (so
// that a 16-byte tensor copy can fetch it): page pg, lane slot wl covers word
// a0 + 16 pg + wl, which is live when it lies inside the slice. Lanes whose
// word is not live read (or are given) zero words and their lookups are
// discarded, so every kernel that uses these pieces adds the same numbers in
// the same order for a given slice.

struct LutWindow {
  int s0, sw, a0;  // slice start and length in words; window start
  __host__ __device__ int lo() const { return s0 - a0; }  // first live window word
  __host__ __device__ int hi() const { return s0 - a0 + sw; }
};
__host__ __device__ __forceinline__ int lut_window_pages(int s0, int sw) { return ((s0 & 3) + sw + 15) / 16; }

// Packed words of the 8 row pairs of one warp (rows w0 + 2p + h), NP pages
// of this CTA's window; rows past N and words outside the slice read as zero.
template <int NP>
__device__ __forceinline__ void lut_load_rows(uint32_t (&wv)[kLutPairs][NP], const uint32_t* __restrict__ packed,
                                              int N, int words, int w0, const LutWindow& win, int h, int wl) {
#pragma unroll
  for (int p = 0; p < kLutPairs; ++p) {
    const int row = w0 + 2 * p + h;
#pragma unroll
    for (int pg = 0; pg < NP; ++pg) {
      const int wi = pg * 16 + wl;
      wv[p][pg] = (row < N && wi >= win.lo() && wi < win.hi())
                      ? __ldcs(packed + static_cast<int64_t>(row) * words + win.a0 + wi)
                      : 0u;
    }
  }
}

// The 32 table values of one task: column c (byte position), value quarter
// qtr (bits 6, 7 of the byte value) and half (bit 5), from raw = the 8 bf16
// inputs of that byte position. Page layout T[v][c], 64 fp32 columns per v.
__device__ __forceinline__ void lut_write_task(uint4 raw, int c, int qtr, int half, uint8_t* page_smem) {
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
  float* page = reinterpret_cast<float*>(page_smem);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int hq = 2 * half + hh;   // bits 4 and 5
    const int hi = qtr * 4 + hq;
    const float hv = (half ? p45[2 + hh] : p45[hh]) + q67;  // constant indices: p45 stays in registers
#pragma unroll
    for (int v = 0; v < 16; ++v) page[(hi * 16 + v) * 64 + c] = lo[v] + hv;
  }
}

// One 64 KB table page: window words [16 pg, 16 pg + 16), inputs read from
// xw (the input element of window word 0, in global or shared memory).
// Task = (half, value quarter, column); column c holds byte i = c/16 of word
// c%16, and a task writes 32 of the column's 256 values; columns of words
// outside the slice are left untouched (never added). kCoherent reads global
// inputs through L2 only.
template <bool kCoherent>
__device__ __forceinline__ void lut_build_page(const uint16_t* __restrict__ xw, int pg, const LutWindow& win,
                                               uint8_t* page_smem, int tid, int nthreads) {
  for (int task = tid; task < 2 * 4 * 64; task += nthreads) {
    const int c = task & 63, qtr = (task >> 6) & 3, half = task >> 8;
    const int wi = pg * 16 + (c & 15);
    if (wi < win.lo() || wi >= win.hi()) continue;
    const int g = 4 * wi + (c >> 4);  // byte position within the window
    const uint4* src = reinterpret_cast<const uint4*>(xw + 8 * g);
    lut_write_task(kCoherent ? __ldcg(src) : *src, c, qtr, half, page_smem);
  }
}

// (a0, a1) + (b0, b1) with one packed f32x2 add: two IEEE fp32 additions,
// each rounded as a scalar add would be.
__device__ __forceinline__ void add_f32x2(float& a0, float& a1, float b0, float b1) {
  unsigned long long A, B, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(D));
}

// Lookups of one page for the 8 row pairs: acc[p] += the page's signed sum
// of row pair p at this lane's word, as (t0 + t1) + (t2 + t3) over the four
// bytes. All 32 lookups are issued before any of them is added, so the
// shared-memory latency overlaps.
__device__ __forceinline__ void lut_page_acc(const uint32_t (&wv)[kLutPairs], bool live, const uint8_t* page,
                                             int h, int wl, float (&acc)[kLutPairs]) {
  uint32_t sel[4], colb[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint32_t i = (s + h) & 3;
    colb[s] = (i * 16 + wl) * 4;
    sel[s] = 0x5504u | (i << 4);  // byte0 <- column byte, byte1 <- word byte i, bytes 2,3 <- 0
  }
  float t[kLutPairs][4];
#pragma unroll
  for (int p = 0; p < kLutPairs; ++p)
#pragma unroll
    for (int s = 0; s < 4; ++s)
      t[p][s] = *reinterpret_cast<const float*>(page + __byte_perm(wv[p], colb[s], sel[s]));
#pragma unroll
  for (int p = 0; p < kLutPairs; p += 2) {
    float u0 = t[p][0], u1 = t[p + 1][0], v0 = t[p][2], v1 = t[p + 1][2];
    add_f32x2(u0, u1, t[p][1], t[p + 1][1]);
    add_f32x2(v0, v1, t[p][3], t[p + 1][3]);
    add_f32x2(u0, u1, v0, v1);
    if (live) add_f32x2(acc[p], acc[p + 1], u0, u1);
  }
}

// Reduce-scatter of the 8 row pairs over the 16 lanes of each half-warp,
// then a pairwise add: the return value is the partial sum of row
// 2 * (wl / 2) + h of the warp's 16 rows (lanes wl and wl ^ 1 return the same).
__device__ __forceinline__ float lut_reduce_scatter(float (&acc)[kLutPairs], int wl) {
#pragma unroll
  for (int d = 8, n = kLutPairs; d >= 2; d >>= 1, n >>= 1) {
    const bool upper = (wl & d) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? acc[j] : acc[j + n / 2];
      const float keep = upper ? acc[j + n / 2] : acc[j];
      acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, d);
    }
  }
  // the two lanes of a pair hold the even and odd word slots' sums; add them
  // in a fixed order so both lanes get the same bits
  const float other = __shfl_xor_sync(0xffffffffu, acc[0], 1);
  return (wl & 1) ? other + acc[0] : acc[0] + other;
}

// NP = pages (16-word groups) per window.
// One-page windows fit two CTAs per SM (registers capped at 64), which lets
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
  LutWindow win;
  win.s0 = static_cast<int>(rank) * slice_words;  // first word of this CTA's slice
  win.sw = slice_words;
  win.a0 = win.s0 & ~3;
  const int rows_per_cta = kLutRowsPerCluster / C;  // rows this CTA owns

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&inbox_bar), 1);
    fence_mbar_init();
  }
  cluster_arrive_relaxed();  // waited on just before the first push

  // ---- 1. prefetch this warp's packed words (independent of x) ----
  uint32_t wv[kLutPairs][NP];
  lut_load_rows<NP>(wv, packed, N, words, row0 + warp * kLutRowsPerWarp, win, h, wl);

  // the owners' scales (not written by the previous kernel either)
  const int orow = row0 + static_cast<int>(rank) * rows_per_cta + static_cast<int>(threadIdx.x);
  const float oalpha = (threadIdx.x < rows_per_cta && orow < N) ? alpha[orow] : 0.f;
  // ask L2 for this slice of x now: a prefetch reads nothing into the CTA
  // and L2 is coherent, so it is safe even while the previous kernel is still
  // writing x; the loads after the wait then find it there
  if (threadIdx.x < (win.sw * 64 + 127) / 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(x + static_cast<int64_t>(win.s0) * 32 + threadIdx.x * 64) : "memory");

  // x may be produced by the previous kernel on the stream
  grid_dependency_wait();
  grid_dependents_launch();

  // ---- 2. build the table pages of this slice ----
#pragma unroll
  for (int pg = 0; pg < NP; ++pg)
    lut_build_page<false>(x + static_cast<int64_t>(win.a0) * 32, pg, win, lut_smem + pg * kLutPageBytes,
                          threadIdx.x, kLutThreads);
  __syncthreads();

  // ---- 3./4. lookups and the per-row reduce-scatter ----
  float acc[kLutPairs];
#pragma unroll
  for (int p = 0; p < kLutPairs; ++p) acc[p] = 0.f;
#pragma unroll
  for (int pg = 0; pg < NP; ++pg) {
    uint32_t w[kLutPairs];
#pragma unroll
    for (int p = 0; p < kLutPairs; ++p) w[p] = wv[p][pg];
    const int wi = pg * 16 + wl;
    lut_page_acc(w, wi >= win.lo() && wi < win.hi(), lut_smem + pg * kLutPageBytes, h, wl, acc);
  }
  const float part = lut_reduce_scatter(acc, wl);

  // ---- 5. push each row's partial to its owner; the owner adds the C partials ----
  if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(&inbox_bar), kLutRowsPerCluster * 4);
  cluster_wait();  // every CTA's inbox barrier is initialised
  if ((wl & 1) == 0) {
    const int r = warp * kLutRowsPerWarp + 2 * (wl >> 1) + h;  // this lane's row within the cluster
    const uint32_t owner = static_cast<uint32_t>(r / rows_per_cta);
    const uint32_t slot = smem_u32(&inbox[static_cast<int>(rank) * rows_per_cta + r % rows_per_cta]);
    st_async_f32(map_to_rank(slot, owner), part, map_to_rank(smem_u32(&inbox_bar), owner));
  }
  if (threadIdx.x < rows_per_cta) {
    if (mbar_wait(smem_u32(&inbox_bar), 0, kWhereLutInbox)) {
      float s = 0.f;
      for (int q = 0; q < C; ++q) s += inbox[q * rows_per_cta + threadIdx.x];
      if (orow < N) y[orow] = float_to_bf16_bits(oalpha * s);
    }
  }
}

// Cluster size and slice for a given K (K % 128 == 0): the largest C in
// {8, 4, 2, 1} that splits the row into whole-word slices of 16..48 words
// whose windows (slice start rounded down to 4 words) span at most
// kLutMaxPages pages; for short rows (fewer than 16 words) a single CTA takes
// the whole row. Returns false when no supported split exists.
inline bool lut_split(int K, int* C_out, int* slice_words_out, int* pages_out) {
  const int words = K / 32;
  auto pages_of = [](int C, int sw) {
    int np = 0;
    for (int r = 0; r < C; ++r) {
      const int p = lut_window_pages(r * sw, sw);
      np = p > np ? p : np;
    }
    return np;
  };
  int chosen = 0;
  for (int C : {8, 4, 2, 1}) {
    if (words % C == 0 && words / C >= 16 && words / C <= 16 * kLutMaxPages &&
        pages_of(C, words / C) <= kLutMaxPages) {
      chosen = C;
      break;
    }
  }
  if (!chosen && words < 16) chosen = 1;
  if (!chosen) return false;
  *C_out = chosen;
  *slice_words_out = words / chosen;
  *pages_out = pages_of(chosen, words / chosen);
  return true;
}

}  // namespace bl

// FBI-linear backward with the straight-through estimator ("FBI-LLM" page,
// FBI-linear paragraph and its training sentence: the estimator carries the
// gradient through the sign function). With y = alpha_j * z_mj,
// z_mj = sum_k s_jk x_mk, and the incoming gradient dy (M x N):
//
//   dx_mk    = sum_j (dy_mj alpha_j) s_jk      a binarized product: the
//              forward kernels with the transposed signs (below)
//   P_jk     = sum_m dy_mj x_mk                 a dense bf16 product (tensor cores)
//   dW_jk    = alpha_j P_jk                     straight-through: ds/dW = 1
//   dalpha_j = sum_m dy_mj z_mj = sum_k s_jk P_jk
//
// dx runs through the forward path unchanged: with g = dy * alpha split into
// two bf16 parts g = hi + lo (exact to ~2^-17 of g), dx = [hi | lo] x [S^T | S^T]
// is a W1A16 product of M tokens, 2N inputs and K outputs with unit scales;
// transpose_pack_dup_kernel writes S^T (each row twice) in the packed layout.
// P is a plain tcgen05 GEMM with both operands in shared memory (TMA,
// 128-byte swizzle), computed as D[k][j] = sum_m X^T[k][m] dY^T[j][m] so that
// each warp's stores of a column j are contiguous in P's row j. P itself is
// never stored: its epilogue writes dW = alpha_j P and, per 128-k tile, the
// signed sums sum_k s_jk P_jk, which a small kernel adds up into dalpha.
#pragma once

#include "bl_common.cuh"

namespace bl {

// ---- element-wise and layout kernels -----------------------------------------------

// g = dy * alpha_j in fp32, split into bf16 hi (round to nearest) and bf16 lo
// = the rounding of the remainder: row m of g2 is [hi_m0..hi_mN-1 | lo_m0..lo_mN-1].
// Each thread takes 8 consecutive outputs of a row (16-byte loads of dy and
// stores of g2); rows are spread over grid y. N % 8 == 0, 16-byte aligned rows.
__global__ void ste_scale_split_kernel(const uint16_t* __restrict__ dy, const float* __restrict__ alpha, int64_t M,
                                       int64_t N, uint16_t* __restrict__ g2) {
  const int64_t groups = N / 8;
  for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
    const uint4* drow = reinterpret_cast<const uint4*>(dy + m * N);
    uint4* hrow = reinterpret_cast<uint4*>(g2 + m * 2 * N);
    uint4* lrow = reinterpret_cast<uint4*>(g2 + m * 2 * N + N);
    for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < groups;
         q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const uint4 d = drow[q];
      const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
      float av[8];  // (alpha need not be 16-byte aligned)
#pragma unroll
      for (int e = 0; e < 8; ++e) av[e] = alpha[8 * q + e];
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t h2 = 0u, l2 = 0u;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float g = bf16_bits_to_float(static_cast<uint16_t>(dw[i] >> (16 * e))) * av[2 * i + e];
          const uint16_t hi = float_to_bf16_bits(g);
          const uint16_t lo = float_to_bf16_bits(g - bf16_bits_to_float(hi));
          h2 |= static_cast<uint32_t>(hi) << (16 * e);
          l2 |= static_cast<uint32_t>(lo) << (16 * e);
        }
        hw[i] = h2;
        lw[i] = l2;
      }
      hrow[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      lrow[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

// Packed signs [N][K/32] -> their transpose [K][2N/32], each row written
// twice (words 0..N/32-1 and again N/32..2N/32-1). A CTA takes 256 rows j
// (8 output words) by 256 k (8 input words): the rows' words are read into
// shared memory (32 bytes per row), each warp turns 32 x 32 bit blocks
// around in registers, and the output rows leave as 32-byte segments. The
// block transpose: lane l holds row l (bit c = column c); five exchange
// stages with the lane l ^ s (s = 16, 8, 4, 2, 1) swap the off-diagonal s x s
// sub-blocks of every 2s x 2s block, after which lane c holds column c (bit
// l = row l). N % 128 == 0 (a ragged last tile of rows reads zeros past N),
// K % 128 == 0.
constexpr int kTpRows = 256;                 // rows j per tile (8 output words)
constexpr int kTpWords = 8;                  // input words per row per tile (256 k)
constexpr int kTpInPitch = kTpWords + 1;     // words: a block's column reads hit 32 banks
constexpr int kTpOutWords = kTpRows / 32;    // 8
constexpr int kTpSmemBytes = (kTpRows * kTpInPitch + kTpWords * 32 * kTpOutWords) * 4;
__device__ __forceinline__ uint32_t transpose32_warp(uint32_t x, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const uint32_t m = s == 16 ? 0x0000FFFFu : s == 8 ? 0x00FF00FFu : s == 4 ? 0x0F0F0F0Fu : s == 2 ? 0x33333333u
                                                                                                     : 0x55555555u;
    const uint32_t t = __shfl_xor_sync(0xffffffffu, x, s);
    x = (lane & s) ? ((x & ~m) | ((t & ~m) >> s)) : ((x & m) | ((t & m) << s));
  }
  return x;
}
__global__ void __launch_bounds__(256) transpose_pack_dup_kernel(const uint32_t* __restrict__ packed, int64_t N,
                                                                 int64_t K, uint32_t* __restrict__ out) {
  extern __shared__ uint32_t tp_smem[];
  uint32_t* in_t = tp_smem;                            // [256 rows][9]
  uint32_t* out_t = tp_smem + kTpRows * kTpInPitch;   // [8 kw x 32 b][8 words]
  const int64_t nw = N / 32, kw_count = K / 32;
  const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kTpRows;
  const int64_t kw0 = static_cast<int64_t>(blockIdx.y) * kTpWords;  // K % 256 need not hold: kws may be 4
  const int kws = static_cast<int>(kw_count - kw0 < kTpWords ? kw_count - kw0 : kTpWords);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < kTpRows * kTpWords; e += 256) {
    const int r = e / kTpWords, c = e % kTpWords;
    in_t[r * kTpInPitch + c] = (c < kws && j0 + r < N) ? packed[(j0 + r) * kw_count + kw0 + c] : 0u;
  }
  __syncthreads();
  // block (jb, kw): rows 32 jb .. + 31 of the tile, word kw; warp w takes jb = w
  for (int kw = 0; kw < kws; ++kw) {
    const uint32_t col = transpose32_warp(in_t[(32 * warp + lane) * kTpInPitch + kw], lane);
    out_t[(kw * 32 + lane) * kTpOutWords + warp] = col;  // output row 32 (kw0 + kw) + lane, word j0 / 32 + warp
  }
  __syncthreads();
  // output rows 32 kw0 .. + 32 kws - 1: 8 words (two 16-byte stores) at column j0 / 32, twice
  const int64_t jw0 = j0 / 32;
  const int jws = static_cast<int>(nw - jw0 < kTpOutWords ? nw - jw0 : kTpOutWords);  // 4 or 8
  for (int e = tid; e < kws * 32 * 2; e += 256) {
    const int orow = e >> 1, half = e & 1;
    if (4 * half >= jws) continue;
    const uint32_t* src = out_t + orow * kTpOutWords + 4 * half;
    uint32_t* dst = out + (32 * kw0 + orow) * 2 * nw + jw0 + 4 * half;
    const uint4 v = make_uint4(src[0], src[1], src[2], src[3]);
    *reinterpret_cast<uint4*>(dst) = v;
    *reinterpret_cast<uint4*>(dst + nw) = v;
  }
}

// bf16 [R][C] -> [C][Rp] (Rp >= R; entries r >= R are zero): 64 x 64 tiles
// through shared memory, block (32, 8), pairs of elements per access (a
// warp reads or writes 128 contiguous bytes). C % 64 == 0, Rp % 64 == 0,
// 4-byte aligned rows.
constexpr int kTrTile = 64;
constexpr int kTrPitch = kTrTile + 2;  // halfwords: rows 4-byte aligned, pair stores conflict-free
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ in, int64_t R, int64_t C,
                                      uint16_t* __restrict__ out, int64_t Rp) {
  __shared__ __align__(4) uint16_t tile[kTrTile][kTrPitch];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTrTile, r0 = static_cast<int64_t>(blockIdx.y) * kTrTile;
  const int tx = threadIdx.x, ty = threadIdx.y;
  // rows r0 + ty + 8 i, columns c0 + 2 tx and + 1
#pragma unroll
  for (int i = 0; i < kTrTile; i += 8) {
    const int64_t r = r0 + ty + i;
    const uint32_t v = r < R ? *reinterpret_cast<const uint32_t*>(in + r * C + c0 + 2 * tx) : 0u;
    *reinterpret_cast<uint32_t*>(&tile[ty + i][2 * tx]) = v;
  }
  __syncthreads();
  // output rows c0 + ty + 8 i, elements r0 + 2 tx and + 1
#pragma unroll
  for (int i = 0; i < kTrTile; i += 8) {
    const int cc = ty + i;
    const uint32_t v = static_cast<uint32_t>(tile[2 * tx][cc]) | (static_cast<uint32_t>(tile[2 * tx + 1][cc]) << 16);
    *reinterpret_cast<uint32_t*>(out + (c0 + cc) * Rp + r0 + 2 * tx) = v;
  }
}

__global__ void fill_f32_kernel(float* __restrict__ p, int64_t n, float v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

// dalpha_j = sum over the 128-k tiles of the partials the dW GEMM wrote
// (part[t][j] = sum over tile t of s_jk P_jk), added in tile order in fp64.
__global__ void ste_dalpha_kernel(const float* __restrict__ part, int64_t tiles, int64_t N,
                                  float* __restrict__ dalpha) {
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < N;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int64_t t = 0; t < tiles; ++t) s += static_cast<double>(part[t * N + j]);
    dalpha[j] = static_cast<float>(s);
  }
}

// ---- P = dY^T X on the tensor cores ------------------------------------------------

constexpr int kSsThreads = 256;   // warp 0 TMA, warp 1 MMA, warps 4..7 epilogue
constexpr int kSsRowsA = 128;     // rows of X^T (k) per tile: the MMA's M
constexpr int kSsRowsB = 256;     // rows of dY^T (j) per tile: the MMA's N
constexpr int kSsUnit = 64;       // contraction (m) per stage: one 128-byte bf16 swizzle atom
constexpr int kSsStages = 4;
constexpr int kSsABytes = kSsRowsA * 128;
constexpr int kSsBBytes = kSsRowsB * 128;
constexpr int kSsStageBytes = kSsABytes + kSsBBytes;  // 48 KB
constexpr int kSsSmemBytes = kSsStages * kSsStageBytes + 1024;

// tm_a: X^T [Kdim][Mp] bf16, box 64 x 128; tm_b: dY^T [Ndim][Mp] bf16, box 64 x 256.
// P[j][k] = sum_m dY[m][j] X[m][k]. Writes dW[j][k] = alpha_j P[j][k] (fp32,
// row pitch Kdim) for j < Ndim, and for every 128-k tile t the signed sums
// part[t][j] = sum_{k in t} s_jk P[j][k] (fp32; `packed` holds s, [Ndim][Kdim/32]),
// which ste_dalpha_kernel adds up. Two accumulators in tensor memory, so the
// epilogue of one tile overlaps the next tile's MMAs.
__global__ void __launch_bounds__(kSsThreads, 1) gemm_ss_ste_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                                    const __grid_constant__ CUtensorMap tm_b,
                                                                    int Kdim, int Ndim, int Mp,
                                                                    const float* __restrict__ alpha,
                                                                    const uint32_t* __restrict__ packed,
                                                                    float* __restrict__ P, float* __restrict__ part) {
  extern __shared__ uint8_t ss_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ss_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t full[kSsStages], empty[kSsStages], d_full[2], d_empty[2];
  __shared__ uint32_t tmem_base_sh;
  // the epilogue's view of a tile: scales, sign words [j][k word] and the
  // four warps' signed partial sums
  __shared__ float alpha_sh[kSsRowsB];
  __shared__ uint32_t bits_sh[kSsRowsB][kSsRowsA / 32];
  __shared__ float part_sh[4][kSsRowsB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_a = Kdim / kSsRowsA;
  const int tiles_b = (Ndim + kSsRowsB - 1) / kSsRowsB;
  const int num_tiles = tiles_a * tiles_b;
  const int units = Mp / kSsUnit;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSsStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&d_full[b]), 1);
      mbar_init(smem_u32(&d_empty[b]), 4);
    }
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int k0 = (tile % tiles_a) * kSsRowsA, j0 = (tile / tiles_a) * kSsRowsB;
        for (int u = 0; u < units; ++u, ++it) {
          const uint32_t s = it % kSsStages;
          if (it >= kSsStages && !mbar_wait(smem_u32(&empty[s]), ((it / kSsStages) - 1) & 1, kWhereSsProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, kSsStageBytes);
          uint8_t* st = smem + s * kSsStageBytes;
          tma_load_2d(smem_u32(st), &tm_a, fb, u * kSsUnit, k0);
          tma_load_2d(smem_u32(st + kSsABytes), &tm_b, fb, u * kSsUnit, j0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kSsRowsA, kSsRowsB);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        const uint32_t ab = tcount & 1u;
        if (tcount >= 2 && !mbar_wait(smem_u32(&d_empty[ab]), ((tcount / 2) - 1) & 1, kWhereSsMma)) break;
        tc_fence_after_sync();
        for (int u = 0; u < units; ++u, ++it) {
          const uint32_t s = it % kSsStages;
          if (!mbar_wait(smem_u32(&full[s]), (it / kSsStages) & 1, kWhereSsMma)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          uint8_t* st = smem + s * kSsStageBytes;
          const uint64_t ad = sw128_kmajor_desc(smem_u32(st));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(st + kSsABytes));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 16 bf16 = 32 bytes of the atom per MMA
            umma_bf16(tmem + ab * kSsRowsB, ad + static_cast<uint64_t>(kk * 2), bd + static_cast<uint64_t>(kk * 2),
                      idesc, (u > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&empty[s]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&d_full[ab]));
      }
    }
  } else if (warp >= 4) {
    const int q = warp & 3, et = threadIdx.x - 128;  // epilogue thread 0..127
    const int kwords = Kdim / 32;
    auto epi_sync = [] { asm volatile("bar.sync 2, 128;" ::: "memory"); };
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const uint32_t ab = tcount & 1u;
      const int k0 = (tile % tiles_a) * kSsRowsA, j0 = (tile / tiles_a) * kSsRowsB;
      // this tile's scales and sign words (rows past Ndim: 0)
      for (int i = et; i < kSsRowsB; i += 128) alpha_sh[i] = j0 + i < Ndim ? alpha[j0 + i] : 0.f;
      for (int i = et; i < kSsRowsB * (kSsRowsA / 32); i += 128) {
        const int jj = i / (kSsRowsA / 32), w = i % (kSsRowsA / 32);
        bits_sh[jj][w] = j0 + jj < Ndim ? packed[static_cast<int64_t>(j0 + jj) * kwords + k0 / 32 + w] : 0u;
      }
      // (the barrier also publishes the staging) the four warps leave together
      // if a wait gave up
      const bool waited = mbar_wait(smem_u32(&d_full[ab]), (tcount / 2) & 1, kWhereSsEpilogue);
      uint32_t all_ok;
      asm volatile(
          "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
          "bar.red.and.pred q, 2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
          : "=r"(all_ok)
          : "r"(static_cast<uint32_t>(waited))
          : "memory");
      if (!all_ok) break;
      tc_fence_after_sync();
      const int k = k0 + q * 32 + lane;  // this thread's row of D = column of P
#pragma unroll 1
      for (int cc = 0; cc < kSsRowsB / 32; ++cc) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + ab * kSsRowsB + cc * 32 + (static_cast<uint32_t>(q * 32) << 16), r);
        tmem_wait_ld();
        const int jc = j0 + cc * 32;
        float* pp = P + static_cast<int64_t>(jc) * Kdim + k;
        float sg[32];  // s_jk P_jk of this lane's k for the chunk's 32 rows j
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float pv = __uint_as_float(r[i]);
          sg[i] = ((bits_sh[cc * 32 + i][q] >> lane) & 1u) ? pv : -pv;
          r[i] = __float_as_uint(alpha_sh[cc * 32 + i] * pv);
        }
        if (jc + 32 <= Ndim) {
#pragma unroll
          for (int i = 0; i < 32; ++i, pp += Kdim) *pp = __uint_as_float(r[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i, pp += Kdim)
            if (jc + i < Ndim) *pp = __uint_as_float(r[i]);
        }
        // reduce-scatter over the warp's 32 k: lane L ends with row jc + L
#pragma unroll
        for (int d = 16, n = 32; d >= 1; d >>= 1, n >>= 1) {
          const bool upper = (lane & d) != 0;
#pragma unroll
          for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? sg[i] : sg[i + n / 2];
            const float keep = upper ? sg[i + n / 2] : sg[i];
            sg[i] = keep + __shfl_xor_sync(0xffffffffu, send, d);
          }
        }
        part_sh[q][cc * 32 + lane] = sg[0];
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&d_empty[ab]));
      epi_sync();  // the four warps' partials are in part_sh; the tile's staging is free again
      for (int i = et; i < kSsRowsB; i += 128)
        if (j0 + i < Ndim)
          part[static_cast<int64_t>(k0 / kSsRowsA) * Ndim + j0 + i] =
              (part_sh[0][i] + part_sh[1][i]) + (part_sh[2][i] + part_sh[3][i]);
      epi_sync();  // part_sh has been read before the next tile writes it
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bl

// Prefill GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
//   W1A16 ("FBI-LLM" page, FBI-linear paragraph, W1A16 configuration):
//     Y[m][j] = bf16( alpha_j * sum_k X[m][k] * s_jk )      kind::f16, bf16 in, fp32 TMEM
//   W1A8 ("BitNet b1.58" page, section 1, Eq.(7)-(8)):
//     acc[m][j] = sum_k q[m][k] * s_jk  (exact int32)       kind::i8, int8 in, s32 TMEM
//     Y[m][j]   = fp32( acc * beta * gamma_m / 128 )        epilogue in fp64
//
// One CTA computes a 128 (tokens) x BN (output channels) tile; K advances
// 128 elements per pipeline stage. Warp roles (256 threads):
//   warp 0      one thread issues TMA loads of the activation tile (128B
//               swizzle) and of the packed sign tile (BN rows x 16 bytes);
//   warp 1      allocates TMEM; one thread issues tcgen05.mma, committing
//               each stage's completion to the stage's "empty" barrier;
//   warps 4..7  expand the sign bits of each stage into +-1 operands
//               (bf16 or int8) written straight into the 128B-swizzled
//               K-major layout the MMA reads, then run the epilogue:
//               tcgen05.ld from TMEM, scale, store.
// The signs are the MMA's B operand (N = output channels); the activations
// are A (M = tokens). Every wait is bounded; a wait that runs out records
// BL_ERR_TIMEOUT and the CTA winds down, still freeing its TMEM.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kGemmThreads = 256;
constexpr int kBM = 128;      // tokens per tile (UMMA M)
constexpr int kStageK = 128;  // K elements per stage: 4 packed words per row

template <int KIND>
struct GemmCfg;

// W1A16: bf16 operands, two 64-element swizzle atoms per stage.
template <>
struct GemmCfg<0> {
  static constexpr int BN = 128;
  static constexpr int STAGES = 3;
  static constexpr int ELEM = 2;
  static constexpr int SUBTILES = kStageK * ELEM / 128;  // 2
  static constexpr int MMA_K = 16;
};
// W1A8: int8 operands, one 128-element swizzle atom per stage.
template <>
struct GemmCfg<1> {
  static constexpr int BN = 256;
  static constexpr int STAGES = 4;
  static constexpr int ELEM = 1;
  static constexpr int SUBTILES = 1;
  static constexpr int MMA_K = 32;
};

template <int KIND>
struct GemmLayout {
  using C = GemmCfg<KIND>;
  static constexpr int A_SUB_BYTES = kBM * 128;                      // one swizzle atom column
  static constexpr int B_SUB_BYTES = C::BN * 128;
  static constexpr int A_BYTES = A_SUB_BYTES * C::SUBTILES;
  static constexpr int B_BYTES = B_SUB_BYTES * C::SUBTILES;
  static constexpr int BITS_BYTES = C::BN * 16;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + BITS_BYTES;  // multiple of 1024
  static constexpr int SMEM_BYTES = C::STAGES * STAGE_BYTES + 1024;   // + alignment slack
  static constexpr int TMEM_COLS = C::BN;
  static_assert(STAGE_BYTES % 1024 == 0, "stage must keep 1024-byte swizzle alignment");
};

// two sign bits -> a pair of bf16 +-1 (low half = lower k)
__device__ __forceinline__ uint32_t pair_to_pm1_bf16(uint32_t q2) {
  return ((q2 * 0x40008000u) & 0x80008000u) ^ 0xBF80BF80u;
}
// four sign bits -> four int8 +-1 (byte i = bit i)
__device__ __forceinline__ uint32_t nib_to_pm1_i8(uint32_t nib) {
  const uint32_t spread = (nib * 0x00204081u) & 0x01010101u;
  return spread * 0xFFFFFF02u + 0xFFFFFFFFu;
}

template <int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_bin_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_bits, int M,
    int N, int K, const float* __restrict__ alpha, const double* __restrict__ gamma,
    const float* __restrict__ beta, void* __restrict__ y, int32_t* __restrict__ acc_out) {
  using C = GemmCfg<KIND>;
  using L = GemmLayout<KIND>;
  constexpr int BN = C::BN;
  constexpr int STAGES = C::STAGES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_full[STAGES];   // TMA bytes landed
  __shared__ __align__(8) uint64_t bar_bfull[STAGES];  // expanded signs written
  __shared__ __align__(8) uint64_t bar_empty[STAGES];  // MMA done reading the stage
  __shared__ __align__(8) uint64_t bar_done;           // all MMAs done
  __shared__ uint32_t tmem_base_sh;
  __shared__ float alpha_sh[KIND == 0 ? BN : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * kBM;
  const int num_kb = K / kStageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_bfull[s]), 4);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    mbar_init(smem_u32(&bar_done), 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_bits);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (KIND == 0 && threadIdx.x >= 128) {
    for (int i = threadIdx.x - 128; i < BN; i += 128) alpha_sh[i] = n0 + i < N ? alpha[n0 + i] : 0.f;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_d = tmem_base_sh;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES;
        if (kb >= STAGES &&
            !mbar_wait(smem_u32(&bar_empty[s]), ((kb / STAGES) - 1) & 1, kWhereGemmProducer))
          break;
        uint8_t* st = smem + s * L::STAGE_BYTES;
        const uint32_t fb = smem_u32(&bar_full[s]);
        mbar_arrive_expect_tx(fb, L::A_BYTES + L::BITS_BYTES);
#pragma unroll
        for (int h = 0; h < C::SUBTILES; ++h)
          tma_load_2d(smem_u32(st + h * L::A_SUB_BYTES), &tm_a, fb, kb * kStageK + h * (128 / C::ELEM),
                      m0);
        tma_load_2d(smem_u32(st + L::A_BYTES + L::B_BYTES), &tm_bits, fb, kb * (kStageK / 32), n0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = KIND == 0 ? idesc_bf16_f32(kBM, BN) : idesc_s8_s32(kBM, BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t par = (kb / STAGES) & 1;
        if (!mbar_wait(smem_u32(&bar_full[s]), par, kWhereGemmMma)) break;
        if (!mbar_wait(smem_u32(&bar_bfull[s]), par, kWhereGemmMma)) break;
        tc_fence_after_sync();
        const uint8_t* st = smem + s * L::STAGE_BYTES;
#pragma unroll
        for (int h = 0; h < C::SUBTILES; ++h) {
          const uint32_t a_base = smem_u32(st + h * L::A_SUB_BYTES);
          const uint32_t b_base = smem_u32(st + L::A_BYTES + h * L::B_SUB_BYTES);
#pragma unroll
          for (int kk = 0; kk < 128 / (C::MMA_K * C::ELEM); ++kk) {
            const uint64_t ad = sw128_kmajor_desc(a_base + kk * 32);
            const uint64_t bd = sw128_kmajor_desc(b_base + kk * 32);
            const uint32_t accum = (kb | h | kk) != 0;
            if (KIND == 0)
              umma_bf16(tmem_d, ad, bd, idesc, accum);
            else
              umma_i8(tmem_d, ad, bd, idesc, accum);
          }
        }
        umma_commit(smem_u32(&bar_empty[s]));
      }
      umma_commit(smem_u32(&bar_done));
    }
  } else if (warp >= 4) {
    // ---------------- sign expanders, then epilogue ----------------
    const int t = threadIdx.x - 128;  // 0..127
    bool ok = true;
    for (int kb = 0; kb < num_kb; ++kb) {
      const int s = kb % STAGES;
      if (!mbar_wait(smem_u32(&bar_full[s]), (kb / STAGES) & 1, kWhereGemmExpander)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + s * L::STAGE_BYTES;
      const uint8_t* bits = st + L::A_BYTES + L::B_BYTES;
      uint8_t* bt = st + L::A_BYTES;
#pragma unroll
      for (int rr = 0; rr < BN / 128; ++rr) {
        const int r = t + rr * 128;
        const uint4 wv = *reinterpret_cast<const uint4*>(bits + r * 16);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        const int sw = r & 7;
        if (KIND == 0) {
          // word i covers k = 32i..32i+31 of the stage: subtile i/2, 16-byte chunks (i%2)*4 + byte
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint8_t* row = bt + (i >> 1) * L::B_SUB_BYTES + r * 128;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
              const uint32_t v = wd[i] >> (8 * cb);
              uint4 o;
              o.x = pair_to_pm1_bf16(v & 3u);
              o.y = pair_to_pm1_bf16((v >> 2) & 3u);
              o.z = pair_to_pm1_bf16((v >> 4) & 3u);
              o.w = pair_to_pm1_bf16((v >> 6) & 3u);
              const int c = (i & 1) * 4 + cb;
              *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = o;
            }
          }
        } else {
          // word i covers k = 32i..32i+31: chunks 2i (bits 0-15) and 2i+1 (bits 16-31)
          uint8_t* row = bt + r * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t v = wd[i] >> (16 * hh);
              uint4 o;
              o.x = nib_to_pm1_i8(v & 0xFu);
              o.y = nib_to_pm1_i8((v >> 4) & 0xFu);
              o.z = nib_to_pm1_i8((v >> 8) & 0xFu);
              o.w = nib_to_pm1_i8((v >> 12) & 0xFu);
              const int c = 2 * i + hh;
              *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = o;
            }
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_bfull[s]));
    }

    // epilogue: TMEM lane quarter (warp % 4) holds tokens m0 + 32*(warp%4) + lane
    if (ok && mbar_wait(smem_u32(&bar_done), 0, kWhereGemmEpilogue)) {
      tc_fence_after_sync();
      const int q = warp & 3;
      const int m = m0 + q * 32 + lane;
      double gscale = 0.0;
      if (KIND == 1 && m < M) gscale = static_cast<double>(*beta);
      const double gm = (KIND == 1 && m < M) ? gamma[m] : 0.0;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t r[32];
        __syncwarp();  // the TMEM load below is warp-collective
        tmem_ld_32x32b_x32(tmem_d + (static_cast<uint32_t>(q * 32) << 16) + cc * 32, r);
        tmem_wait_ld();
        const int nb = n0 + cc * 32;
        if (m >= M || nb >= N) continue;
        const bool full = nb + 32 <= N;
        if (KIND == 0) {
          uint16_t* yr = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(m) * N + nb;
          if (full && (N % 8) == 0) {
            uint32_t o[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t lo = float_to_bf16_bits(__uint_as_float(r[2 * i]) * alpha_sh[cc * 32 + 2 * i]);
              const uint32_t hi =
                  float_to_bf16_bits(__uint_as_float(r[2 * i + 1]) * alpha_sh[cc * 32 + 2 * i + 1]);
              o[i] = lo | (hi << 16);
            }
            uint4* dst = reinterpret_cast<uint4*>(yr);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (nb + i < N) yr[i] = float_to_bf16_bits(__uint_as_float(r[i]) * alpha_sh[cc * 32 + i]);
          }
        } else {
          float* yr = reinterpret_cast<float*>(y) + static_cast<int64_t>(m) * N + nb;
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            o[i] = static_cast<float>(static_cast<double>(static_cast<int32_t>(r[i])) * gscale * gm / 128.0);
          if (full && (N % 4) == 0) {
            float4* dst = reinterpret_cast<float4*>(yr);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (nb + i < N) yr[i] = o[i];
          }
          if (acc_out) {
            int32_t* ar = acc_out + static_cast<int64_t>(m) * N + nb;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (nb + i < N) ar[i] = static_cast<int32_t>(r[i]);
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_d, L::TMEM_COLS);
  }
}

}  // namespace bl

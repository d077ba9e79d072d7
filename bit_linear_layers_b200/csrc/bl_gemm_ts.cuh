// Binarized GEMMs on the 5th-generation tensor cores with the signs as the
// tensor-memory operand (tcgen05.mma with A in TMEM, B in shared memory).
//
//   W1A16 ("FBI-LLM" page, FBI-linear paragraph; W1A16 configuration):
//     y[m][j] = bf16( alpha_j * sum_k s_jk x[m][k] )          kind::f16, fp32 accumulate
//   W1A8 ("BitNet b1.58" page, section 1, Eq.(7)-(8)):
//     acc[m][j] = sum_k s_jk q[m][k]  (exact int32)            kind::i8
//     y[m][j]   = fp32( acc * beta * gamma_m / 128 )           fp64 epilogue
//
// The product is computed transposed, D[j][m] = sum_k S[j][k] X[m][k]: the
// 1-bit weights are the MMA's M side (two M = 128 blocks per tile, 256 rows),
// the tokens its N side (T per tile). Shared-memory traffic is then only the
// activation tile (TMA, 128-byte swizzle); the expanded +-1 signs never touch
// shared memory: eight expander warps read each stage's packed bits, build
// the +-1 operand in registers and write it to a ring of tensor-memory stages
// with tcgen05.st. A tile moves T*2 + 256/8 bytes per k for 2*256*T flops.
//
// Persistent kernel, one CTA per SM, 512 threads:
//   warp 0      TMA producer: activation tile + packed sign tile per stage
//   warp 1      TMEM allocation; one thread issues the MMAs and commits
//   warps 4..7  epilogue (tcgen05.ld of the accumulators, scale, store)
//   warps 8..15 sign expanders: warp 8 + 4*b + q expands block b (rows
//               128*b .. 128*b + 127) into TMEM lane quarter q = warp % 4
// Tensor memory (512 columns): two accumulators of T columns, then the ring
// of sign stages (two 128-row blocks per stage). All waits are bounded.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kTsThreads = 512;
constexpr int kTsExpanders = 8;  // warps
constexpr int kTsRows = 256;     // weight rows per tile (two UMMA M=128 blocks)
constexpr int kTsStageK = 128;   // K elements per pipeline stage

template <int KIND, int T>
struct TsCfg {
  static constexpr int ELEM = KIND == 0 ? 2 : 1;                // activation bytes
  static constexpr int XSUB = kTsStageK * ELEM / 128;           // 128 B swizzle atoms per stage
  static constexpr int X_SUB_BYTES = T * 128;
  static constexpr int X_BYTES = X_SUB_BYTES * XSUB;
  static constexpr int BITS_BYTES = kTsRows * 16;
  static constexpr int STAGE_BYTES = X_BYTES + BITS_BYTES;
  static constexpr int OUT_ELEM = KIND == 0 ? 2 : 4;             // y element bytes
  static constexpr int OUT_BYTES = kTsRows * T * OUT_ELEM;         // staged output tile [T][256]
  static constexpr int SX_FIT = (208 * 1024 - OUT_BYTES) / STAGE_BYTES;
  static constexpr int SX = SX_FIT > 8 ? 8 : SX_FIT;
  static constexpr int SMEM_BYTES = SX * STAGE_BYTES + OUT_BYTES + 1024;
  static constexpr int MMA_K = KIND == 0 ? 16 : 32;             // elements per MMA
  static constexpr int KSTEPS = kTsStageK / MMA_K;              // MMAs per block per stage
  static constexpr int A_COLS = kTsStageK * ELEM / 4;           // TMEM columns per block per stage
  static constexpr int D_COLS = 2 * T;                          // two accumulators
  static constexpr int SA_MAX = (512 - D_COLS) / (2 * A_COLS);
  static constexpr int SA = SA_MAX > 4 ? 4 : SA_MAX;            // sign stages in TMEM
  static_assert(SA >= 2, "need at least two sign stages");
  static_assert(SX >= 2, "need at least two activation stages");
  static_assert(X_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "swizzle alignment");
};

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// bulk tensor store of a shared-memory tile (no multicast), tracked by bulk groups
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// barrier among the four epilogue warps only
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// D(tmem) (+)= A(tmem) * B(smem desc)
__device__ __forceinline__ void umma_ts_bf16(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void umma_ts_i8(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// 16 sign bits (zero-extended) -> 16 bf16 +-1 packed in 8 words (low half =
// lower k). With r = x | (x << 15), shifting r left by 15 - 2i puts bit 2i
// at position 15 and bit 2i+1 at position 31, the two bf16 sign bits; the
// mask and the xor with -1,-1 turn a set bit into +1.
__device__ __forceinline__ void expand16_bf16(uint32_t bits, uint32_t* out) {
  const uint32_t r = bits | (bits << 15);
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = ((r << (15 - 2 * i)) & 0x80008000u) ^ 0xBF80BF80u;
}
// 16 sign bits -> 16 int8 +-1 packed in 4 words (byte i = bit i)
__device__ __forceinline__ void expand16_i8(uint32_t bits, uint32_t* out) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t spread = (((bits >> (4 * i)) & 0xFu) * 0x00204081u) & 0x01010101u;
    out[i] = spread * 0xFFFFFF02u + 0xFFFFFFFFu;
  }
}

template <int KIND, int T>
__global__ void __launch_bounds__(kTsThreads, 1) gemm_ts_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_bits,
    const __grid_constant__ CUtensorMap tm_y, int use_tma_store, int M, int N, int K,
    const float* __restrict__ alpha, const double* __restrict__ gamma, const float* __restrict__ beta,
    void* __restrict__ y, int32_t* __restrict__ acc_out) {
  using C = TsCfg<KIND, T>;
  constexpr int SX = C::SX, SA = C::SA;

  extern __shared__ uint8_t ts_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ts_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t x_full[SX], x_empty[SX], a_full[SA], a_empty[SA], d_full, d_empty;
  __shared__ uint32_t tmem_base_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_kb = K / kTsStageK;
  const int tiles_t = (M + T - 1) / T;
  const int tiles_w = (N + kTsRows - 1) / kTsRows;
  const int num_tiles = tiles_t * tiles_w;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(smem_u32(&x_full[s]), 1);
      mbar_init(smem_u32(&x_empty[s]), 1 + kTsExpanders);  // MMA commit + expander warps
    }
    for (int a = 0; a < SA; ++a) {
      mbar_init(smem_u32(&a_full[a]), kTsExpanders);
      mbar_init(smem_u32(&a_empty[a]), 1);
    }
    mbar_init(smem_u32(&d_full), 1);
    mbar_init(smem_u32(&d_empty), 4);
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_bits);
    if (use_tma_store) tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_sh), 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t a_base = tmem + C::D_COLS;  // sign ring starts after the two accumulators

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int t0 = (tile % tiles_t) * T, w0 = (tile / tiles_t) * kTsRows;
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % SX;
          if (it >= SX && !mbar_wait(smem_u32(&x_empty[s]), ((it / SX) - 1) & 1, kWhereGemmProducer)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::STAGE_BYTES;
          const uint32_t fb = smem_u32(&x_full[s]);
          mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
#pragma unroll
          for (int h = 0; h < C::XSUB; ++h)
            tma_load_2d(smem_u32(st + h * C::X_SUB_BYTES), &tm_x, fb, kb * kTsStageK + h * (128 / C::ELEM), t0);
          tma_load_2d(smem_u32(st + C::X_BYTES), &tm_bits, fb, kb * (kTsStageK / 32), w0);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = KIND == 0 ? idesc_bf16_f32(128, T) : idesc_s8_s32(128, T);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tcount) {
        if (tcount > 0 && !mbar_wait(smem_u32(&d_empty), (tcount - 1) & 1, kWhereGemmMma)) break;
        tc_fence_after_sync();
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const uint32_t s = it % SX, a = it % SA;
          if (!mbar_wait(smem_u32(&x_full[s]), (it / SX) & 1, kWhereGemmMma) ||
              !mbar_wait(smem_u32(&a_full[a]), (it / SA) & 1, kWhereGemmMma)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t xs = smem_u32(smem + s * C::STAGE_BYTES);
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            const uint32_t a_tm = a_base + (a * 2 + blk) * C::A_COLS;
            const uint32_t d_tm = tmem + blk * T;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              // MMA_K elements = 32 bytes of an activation row; 4 per 128-byte atom
              const uint32_t xaddr = xs + (kk / 4) * C::X_SUB_BYTES + (kk % 4) * 32;
              const uint64_t bd = sw128_kmajor_desc(xaddr);
              const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
              if (KIND == 0)
                umma_ts_bf16(d_tm, a_tm + kk * 8, bd, idesc, accum);
              else
                umma_ts_i8(d_tm, a_tm + kk * 8, bd, idesc, accum);
            }
          }
          umma_commit(smem_u32(&x_empty[s]));
          umma_commit(smem_u32(&a_empty[a]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&d_full));
      }
    }
  } else if (warp >= 8) {
    // ---------------- sign expanders ----------------
    const int q = warp & 3, blk = (warp - 8) >> 2;
    const int r = blk * 128 + q * 32 + lane;  // sign row within the tile = TMEM lane in its block
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const uint32_t s = it % SX, a = it % SA;
        if (!mbar_wait(smem_u32(&x_full[s]), (it / SX) & 1, kWhereGemmExpander) ||
            (it >= SA && !mbar_wait(smem_u32(&a_empty[a]), ((it / SA) - 1) & 1, kWhereGemmExpander))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint8_t* bits = smem + s * C::STAGE_BYTES + C::X_BYTES;
        const uint4 wv = *reinterpret_cast<const uint4*>(bits + r * 16);
        const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
        const uint32_t taddr = a_base + (a * 2 + blk) * C::A_COLS + (static_cast<uint32_t>(q * 32) << 16);
        if (KIND == 0) {
          // 128 bf16 = 64 columns, written as two halves of 32
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              expand16_bf16((wd[half * 2 + j / 2] >> (16 * (j & 1))) & 0xFFFFu, v + 8 * j);
            tmem_st_32x32b_x32(taddr + half * 32, v);
          }
        } else {
          // 128 int8 = 32 columns
          uint32_t v[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) expand16_i8((wd[j / 2] >> (16 * (j & 1))) & 0xFFFFu, v + 4 * j);
          tmem_st_32x32b_x32(taddr, v);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&a_full[a]));
          mbar_arrive(smem_u32(&x_empty[s]));
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    // Accumulators -> scaled outputs -> staging tile [T tokens][256 rows] in
    // shared memory; the accumulators are released as soon as they are read,
    // then one bulk tensor store writes the tile (rows/tokens past N/M are
    // clipped by the store). Without an aligned output (N % 8 for bf16,
    // N % 4 for fp32) the outputs are stored directly instead.
    const int q = warp & 3;
    uint8_t* stage_out = smem + SX * C::STAGE_BYTES;
    const bool leader = (warp == 4 && lane == 0);
    uint32_t tcount = 0;
    double bt = 0.0;
    if (KIND == 1) bt = static_cast<double>(*beta);
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tcount) {
      const int t0 = (tile % tiles_t) * T, w0 = (tile / tiles_t) * kTsRows;
      if (!mbar_wait(smem_u32(&d_full), tcount & 1, kWhereGemmEpilogue)) break;
      tc_fence_after_sync();
      if (use_tma_store) {
        if (leader) bulk_wait_read0();  // the previous tile's store has read the staging tile
        epilogue_bar();
      }
#pragma unroll 1
      for (int blk = 0; blk < 2; ++blk) {
        const int jl = blk * 128 + q * 32 + lane;  // row of the tile = output channel w0 + jl
        const int j = w0 + jl;
        const bool jv = j < N;
        float aj = 0.f;
        if (KIND == 0 && jv) aj = alpha[j];
#pragma unroll 1
        for (int cc = 0; cc < T / 32; ++cc) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + blk * T + cc * 32 + (static_cast<uint32_t>(q * 32) << 16), r);
          tmem_wait_ld();
          if (blk == 1 && cc == T / 32 - 1) {
            // every accumulator column of this tile has been read: free them
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&d_empty));
          }
          const int ml0 = cc * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int m = t0 + ml0 + i;
            if (KIND == 0) {
              const uint16_t v = float_to_bf16_bits(__uint_as_float(r[i]) * aj);
              if (use_tma_store)
                reinterpret_cast<uint16_t*>(stage_out)[(ml0 + i) * kTsRows + jl] = v;
              else if (jv && m < M)
                reinterpret_cast<uint16_t*>(y)[static_cast<int64_t>(m) * N + j] = v;
            } else {
              const int32_t acc = static_cast<int32_t>(r[i]);
              const double gm = m < M ? gamma[m] : 0.0;
              const float v = static_cast<float>(static_cast<double>(acc) * bt * gm / 128.0);
              if (use_tma_store)
                reinterpret_cast<float*>(stage_out)[(ml0 + i) * kTsRows + jl] = v;
              else if (jv && m < M)
                reinterpret_cast<float*>(y)[static_cast<int64_t>(m) * N + j] = v;
              if (acc_out && jv && m < M) acc_out[static_cast<int64_t>(m) * N + j] = acc;
            }
          }
        }
      }
      if (use_tma_store) {
        fence_proxy_async_smem();  // staging writes -> visible to the bulk store
        epilogue_bar();
        if (leader) {
          tma_store_2d(&tm_y, smem_u32(stage_out), w0, t0);
          bulk_commit();
        }
      }
    }
    if (use_tma_store && leader) bulk_wait0();
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

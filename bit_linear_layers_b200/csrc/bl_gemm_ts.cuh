// Binarized GEMMs on the 5th-generation tensor cores with the signs as the
// tensor-memory operand (tcgen05.mma with A in TMEM, B in shared memory).
//
//   W1A16 ("FBI-LLM" page, FBI-linear paragraph; W1A16 configuration):
//     y[m][j] = bf16( alpha_j * sum_k s_jk x[m][k] )          kind::f16, fp32 accumulate
//   W1A8 ("BitNet b1.58" page, section 1, Eq.(7)-(8)):
//     acc[m][j] = sum_k s_jk q[m][k]  (exact int32)            kind::i8
//     y[m][j]   = fp32( acc * beta * gamma_m / 128 )           per-token scale in fp64
//   W1.58A8 (same page, section 2, Eq.(9)-(11)): as W1A8 with ternary weights
//     W~_jk in {-1, 0, +1}, stored as a +1 and a -1 bit plane per 128-k block
//     (KIND 2)
//
// The product is computed transposed, D[j][m] = sum_k S[j][k] X[m][k]: the
// 1-bit weights are the MMA's M side (NB blocks of 128 rows per tile), the
// tokens its N side (T per tile). Shared-memory traffic is then only the
// activation tile (TMA, 128-byte swizzle); the expanded +-1 signs never touch
// shared memory: eight expander warps read each stage's packed bits, build
// the +-1 operand in registers and write it to a ring of tensor-memory stages
// with tcgen05.st.
//
// Each tcgen05.mma instruction costs the single issuing thread a roughly
// fixed time, so the largest problems use 128 x 256 MMAs (NB = 1, T = 256):
// enough tensor work per instruction to keep the pipe busy. Smaller problems
// use two 128-row blocks (NB = 2) and fewer tokens per tile.
//
// The pipeline unit is one 128-byte swizzle atom of every activation row
// (64 k for bf16, 128 k for int8). Activation units and 128-k sign stages
// travel in separate shared-memory rings: the expanders only need the signs
// and run ahead into a ring of tensor-memory sign units, while only the MMA
// waits for the (much larger) activation units.
//
// Persistent kernel, one CTA per SM, 512 threads:
//   warp 0      TMA producer: sign stages and activation units
//   warp 1      TMEM allocation; one thread issues the MMAs and commits
//   warps 4..7  epilogue (tcgen05.ld of the accumulators, scale, store)
//   warps 8..15 sign expanders; each writes one TMEM lane quarter (warp % 4)
//               of one block (NB = 2) or of half a unit (NB = 1)
// Tensor memory (512 columns): NB accumulators of T columns, then the ring
// of sign units (NB blocks of 32 columns per unit). All waits are bounded.
//
// Split-K mode (few tiles, e.g. decode batches): a cluster of S CTAs shares
// one tile and splits its k-blocks; each CTA pushes the partial sums of
// every row to the CTA that owns the row (rows split S ways) with 16-byte
// st.async stores counted on the owner's mbarrier, and the owner adds the S
// partials in a fixed order (exact in int32 for W1A8) before the epilogue.
#pragma once

#include "bl_common.cuh"

namespace bl {

constexpr int kTsThreads = 512;
constexpr int kTsExpanders = 8;  // warps
constexpr int kTsStageK = 128;   // K elements per pipeline stage

// KIND 0: bf16 activations, +-1 weights; 1: int8 codes, +-1 weights;
// 2: int8 codes, ternary weights (two bit planes per 128-k stage)
template <int KIND, int NB, int T, bool SPLIT>
struct TsCfg {
  static constexpr int ROWS = 128 * NB;                         // weight rows per tile
  static constexpr int ELEM = KIND == 0 ? 2 : 1;                // activation bytes
  static constexpr int PLANES = KIND == 2 ? 2 : 1;              // sign bit planes per weight
  // pipeline unit: one 128-k sign stage; its activations are ATOMS 128-byte
  // swizzle atoms of every token row (64 k each for bf16, 128 k for int8)
  static constexpr int ATOM_K = 128 / ELEM;
  static constexpr int ATOMS = kTsStageK / ATOM_K;              // 2 (bf16) or 1 (int8)
  static constexpr int ATOM_BYTES = T * 128;
  static constexpr int X_UNIT_BYTES = ATOMS * ATOM_BYTES;
  static constexpr int BITS_BYTES = ROWS * 16 * PLANES;         // one 128-k sign stage
  static constexpr int OUT_ELEM = KIND == 0 ? 2 : 4;            // y element bytes
  // int8 tiles stage the fp32 output in shared memory and write it by bulk
  // tensor stores (the whole tile at once when it fits in 64 KB, else one
  // 128-row block at a time). bf16 tiles store straight from registers (each
  // warp store is 64 contiguous bytes of a token row): the 64 KB a staging
  // tile would take holds a third activation unit instead, and the mainloop
  // waits on activation delivery (prefill 1049 -> 1217 TFLOP/s, measured)
  static constexpr int STAGE_COLS = ROWS * T * OUT_ELEM <= 64 * 1024 ? ROWS : 128;
  static constexpr bool STAGE_OUT = KIND != 0 && !SPLIT && STAGE_COLS * T * OUT_ELEM <= 64 * 1024;
  // split-K inbox rows: T partials padded by 16 bytes, so that a warp's
  // 16-byte reads of consecutive rows spread over all banks
  static constexpr int IN_STRIDE = T + 4;
  // staged output [T][STAGE_COLS], or the split-K inbox [S][ROWS/S][IN_STRIDE] of 4-byte partials
  static constexpr int OUT_BYTES = SPLIT ? ROWS * IN_STRIDE * 4 : (STAGE_OUT ? STAGE_COLS * T * OUT_ELEM : 0);
  // sign stages in shared memory. A row tile's signs come from HBM on first
  // touch, and the stages in flight must cover that latency: int8 problems
  // (one unit is only 4-8 MMAs) take 16 stages unless that would leave fewer
  // than four activation units; the bf16 configurations keep 4.
  static constexpr int SX_IF_DEEP = (220 * 1024 - OUT_BYTES - 16 * BITS_BYTES) / X_UNIT_BYTES;
  static constexpr int SB = (KIND != 0 && SX_IF_DEEP >= 4) ? 16 : 4;
  static constexpr int SX_FIT = (220 * 1024 - OUT_BYTES - SB * BITS_BYTES) / X_UNIT_BYTES;
  static constexpr int SX = SX_FIT > 8 ? 8 : SX_FIT;           // activation units in flight
  static constexpr int X_RING = SX * X_UNIT_BYTES;
  static constexpr int SMEM_BYTES = X_RING + SB * BITS_BYTES + OUT_BYTES + 1024;
  static constexpr int KSTEPS = 4 * ATOMS;                      // MMAs per block per unit (32 bytes of k each)
  static constexpr int A_COLS = 32 * ATOMS;                     // TMEM columns per block per unit
  static constexpr int CH = kTsStageK / 16;                     // 16-bit sign chunks per unit (8)
  static constexpr int COLS_PER_CH = A_COLS / CH;               // 8 (bf16) or 4 (int8)
  static constexpr int D_COLS = NB * T;                         // accumulators
  static constexpr int SA_MAX = (512 - D_COLS) / (NB * A_COLS);
  static constexpr int SA = SA_MAX > 8 ? 8 : SA_MAX;            // sign units in TMEM
  static_assert(SA >= 2, "need at least two sign units");
  static_assert(SX >= 2, "need at least two activation units");
  static_assert(ATOM_BYTES % 1024 == 0 && BITS_BYTES % 1024 == 0, "swizzle alignment");
  static_assert(NB == 1 || NB == 2, "one or two 128-row blocks per tile");
};

template <int N>
__device__ __forceinline__ void tmem_st_32x32b(uint32_t taddr, const uint32_t* r);
template <>
__device__ __forceinline__ void tmem_st_32x32b<32>(uint32_t taddr, const uint32_t* r) {
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
template <>
__device__ __forceinline__ void tmem_st_32x32b<16>(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// N consecutive 32-bit columns of this warp's lane quarter (N = 16, 32 or 64)
template <int N>
__device__ __forceinline__ void tmem_st_wide(uint32_t taddr, const uint32_t* r) {
  if constexpr (N == 64) {
    tmem_st_32x32b<32>(taddr, r);
    tmem_st_32x32b<32>(taddr + 32, r + 32);
  } else {
    tmem_st_32x32b<N>(taddr, r);
  }
}

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
// the same barrier, returning the AND of every epilogue thread's `v`
__device__ __forceinline__ bool epilogue_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

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

// W1A8 output y = acc * s, s = beta * gamma_m / 128 formed in fp64 once per
// token and carried as two floats (s = hi + lo to about 2^-48). For
// |acc| < 2^22 the product is evaluated in fp32 with an error-free product
// (the magic-number add turns acc into a float exactly, the fma recovers the
// rounding error of acc * hi), so y is the fp32 rounding of the exact value
// except within ~2^-46 of a rounding midpoint; larger |acc| take fp64.
struct TokScale {
  float hi, lo;
};
__device__ __forceinline__ TokScale w1a8_token_scale(double beta, double gamma) {
  const double sc = beta * gamma * 0.0078125;  // division by 128 = exact scaling by 2^-7
  const float hi = static_cast<float>(sc);
  return TokScale{hi, static_cast<float>(sc - static_cast<double>(hi))};
}
constexpr int32_t kW1a8FastLimit = 1 << 22;
__device__ __forceinline__ bool w1a8_fast_ok(int32_t acc) {
  return acc > -kW1a8FastLimit && acc < kW1a8FastLimit;
}
// |acc| < 2^22 only (no branch, so that unrolled loops interleave)
__device__ __forceinline__ float w1a8_output_fast(int32_t acc, TokScale s) {
  const float a = __int_as_float(0x4B400000 + acc) - 12582912.0f;  // exact: 1.5 * 2^23 + acc - 1.5 * 2^23
  const float p = a * s.hi;
  const float e = fmaf(a, s.hi, -p);  // a * hi - p, exactly
  return p + fmaf(a, s.lo, e);
}
__device__ __forceinline__ float w1a8_output_wide(int32_t acc, TokScale s) {
  return static_cast<float>(static_cast<double>(acc) * (static_cast<double>(s.hi) + static_cast<double>(s.lo)));
}
__device__ __forceinline__ float w1a8_output(int32_t acc, TokScale s) {
  return w1a8_fast_ok(acc) ? w1a8_output_fast(acc, s) : w1a8_output_wide(acc, s);
}

// 16 ternary weights (16 bits of the +1 plane, 16 of the -1 plane) -> 16
// int8 values +1 / 0 / -1 in 4 words
__device__ __forceinline__ void expand16_ternary(uint32_t plus, uint32_t minus, uint32_t* out) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t p = (((plus >> (4 * i)) & 0xFu) * 0x00204081u) & 0x01010101u;
    const uint32_t m = (((minus >> (4 * i)) & 0xFu) * 0x00204081u) & 0x01010101u;
    out[i] = p | (m * 0xFFu);
  }
}

// Shared-memory accesses by address. The epilogue's loads and stores take no
// "memory" clobber: as volatile asm they stay ordered with the barrier waits
// and fences (also volatile asm) around them, and may overlap the plain
// global stores in between.
__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t* v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3])
               : "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t* v) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(addr));
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v));
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v));
}
__device__ __forceinline__ void st_async_v4(uint32_t remote_addr, const uint32_t* v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   remote_addr),
               "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(remote_bar)
               : "memory");
}
__device__ __forceinline__ uint32_t ts_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t ts_map_rank(uint32_t local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  return remote;
}

template <int KIND, int NB, int T, bool SPLIT>
__global__ void __launch_bounds__(kTsThreads, 1) gemm_ts_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_bits,
    const __grid_constant__ CUtensorMap tm_y, int use_tma_store, int M, int N, int K,
    const float* __restrict__ alpha, const double* __restrict__ gamma, const float* __restrict__ beta,
    void* __restrict__ y, int32_t* __restrict__ acc_out) {
  using C = TsCfg<KIND, NB, T, SPLIT>;
  constexpr int SX = C::SX, SA = C::SA, ROWS = C::ROWS;

  extern __shared__ uint8_t ts_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ts_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t x_full[SX], x_empty[SX], b_full[C::SB], b_empty[C::SB];
  __shared__ __align__(8) uint64_t a_full[SA], a_empty[SA], d_full, d_empty;
  __shared__ uint32_t tmem_base_sh;
  __shared__ __align__(8) uint64_t inbox_bar;
  // epilogue scales staged once per tile: beta * gamma / 128 of the tile's tokens (W1A8),
  // alpha of the rows a split-K owner finishes (W1A16)
  __shared__ TokScale tok_scale[KIND != 0 ? T : 1];
  __shared__ float row_alpha[SPLIT && KIND == 0 ? ROWS : 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_kb = K / kTsStageK;
  const int tiles_t = (M + T - 1) / T;
  const int tiles_w = (N + ROWS - 1) / ROWS;
  const int num_tiles = tiles_t * tiles_w;
  // persistent over tiles; in split-K mode one tile per cluster and a k range per CTA
  const int tile_first = SPLIT ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
  const int tile_step = SPLIT ? static_cast<int>(gridDim.y) : static_cast<int>(gridDim.x);
  const uint32_t rank = SPLIT ? ts_cluster_rank() : 0u;
  const int S = SPLIT ? static_cast<int>(gridDim.x) : 1;
  const int kb_per = (num_kb + S - 1) / S;
  const int kb_first = SPLIT ? static_cast<int>(rank) * kb_per : 0;
  const int kb_last = SPLIT ? min(num_kb, kb_first + kb_per) : num_kb;
  // pipeline units (128-k sign stages) of this CTA within each tile
  const int u_first = kb_first, u_last = kb_last;
  uint8_t* const bits_ring = smem + C::X_RING;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(smem_u32(&x_full[s]), 1);
      mbar_init(smem_u32(&x_empty[s]), 1);  // MMA commit
    }
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(smem_u32(&b_full[s]), 1);
      mbar_init(smem_u32(&b_empty[s]), kTsExpanders);
    }
    for (int a = 0; a < SA; ++a) {
      mbar_init(smem_u32(&a_full[a]), kTsExpanders);
      mbar_init(smem_u32(&a_empty[a]), 1);
    }
    mbar_init(smem_u32(&d_full), 1);
    mbar_init(smem_u32(&d_empty), 4);
    if (SPLIT) mbar_init(smem_u32(&inbox_bar), 1);
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
  if (SPLIT) asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");  // waited before pushing
  const uint32_t tmem = tmem_base_sh;
  const uint32_t a_base = tmem + C::D_COLS;  // sign ring starts after the accumulators

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // per unit: the sign stage first (the expanders need only that), then the
    // unit's activation atoms, all counted on one barrier
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = tile_first; tile < num_tiles && ok; tile += tile_step) {
        const int t0 = (tile % tiles_t) * T, w0 = (tile / tiles_t) * ROWS;
        for (int u = u_first; u < u_last; ++u, ++it) {
          const uint32_t bs = it % C::SB;
          if (it >= C::SB && !mbar_wait(smem_u32(&b_empty[bs]), ((it / C::SB) - 1) & 1, kWhereGemmProducer)) {
            ok = false;
            break;
          }
          const uint32_t bb = smem_u32(&b_full[bs]);
          mbar_arrive_expect_tx(bb, C::BITS_BYTES);
          tma_load_2d(smem_u32(bits_ring + bs * C::BITS_BYTES), &tm_bits, bb, u * 4 * C::PLANES, w0);
          const uint32_t xs = it % SX;
          if (it >= SX && !mbar_wait(smem_u32(&x_empty[xs]), ((it / SX) - 1) & 1, kWhereGemmProducer)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&x_full[xs]);
          mbar_arrive_expect_tx(fb, C::X_UNIT_BYTES);
#pragma unroll
          for (int h = 0; h < C::ATOMS; ++h)
            tma_load_2d(smem_u32(smem + xs * C::X_UNIT_BYTES + h * C::ATOM_BYTES), &tm_x, fb,
                        u * kTsStageK + h * C::ATOM_K, t0);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // One barrier per unit: a_full completes once the signs are in tensor
    // memory and (through the expander that waited for them) the activations
    // are in shared memory. Every mbarrier test the issuing thread makes holds
    // up its next MMA by ~100 ns, so it makes exactly one per unit.
    if (lane == 0) {
      const uint32_t idesc = KIND == 0 ? idesc_bf16_f32(128, T) : idesc_s8_s32(128, T);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = tile_first; tile < num_tiles && ok; tile += tile_step, ++tcount) {
        if (tcount > 0 && !mbar_wait(smem_u32(&d_empty), (tcount - 1) & 1, kWhereGemmMma)) break;
        tc_fence_after_sync();
        for (int u = u_first; u < u_last; ++u, ++it) {
          const uint32_t xs = it % SX, a = it % SA;
          if (!mbar_wait(smem_u32(&a_full[a]), (it / SA) & 1, kWhereGemmMma)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          // descriptor of each atom's first 32-byte k slice; later slices add
          // their byte offset >> 4 to the start-address field (never carries:
          // the ring lies inside the 256 KB window of the 14-bit field)
          const uint32_t a_tm0 = a_base + (a * NB) * C::A_COLS;
#pragma unroll
          for (int h = 0; h < C::ATOMS; ++h) {
            const uint64_t bd0 = sw128_kmajor_desc(smem_u32(smem + xs * C::X_UNIT_BYTES + h * C::ATOM_BYTES));
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              const int kk = h * 4 + k4;
              const uint64_t bd = bd0 + static_cast<uint64_t>((k4 * 32) >> 4);
              const uint32_t accum = (u > u_first || kk > 0) ? 1u : 0u;
#pragma unroll
              for (int blk = 0; blk < NB; ++blk) {
                const uint32_t a_tm = a_tm0 + blk * C::A_COLS + kk * 8;
                if (KIND == 0)
                  umma_ts_bf16(tmem + blk * T, a_tm, bd, idesc, accum);
                else
                  umma_ts_i8(tmem + blk * T, a_tm, bd, idesc, accum);
              }
            }
          }
          umma_commit(smem_u32(&x_empty[xs]));
          umma_commit(smem_u32(&a_empty[a]));
        }
        if (!ok) break;
        umma_commit(smem_u32(&d_full));
      }
    }
  } else if (warp >= 8) {
    // ---------------- sign expanders ----------------
    // With two blocks, warp 8 + 4*b + q expands block b, lane quarter q, all
    // CH chunks of the unit; with one block the two warps of a lane quarter
    // take half of the chunks each. Chunk g of a unit = bits 16g..16g+15 of
    // the row's 128-bit sign stage. The expander of rank it % 8 also waits
    // for the unit's activations before it arrives, so that a_full alone
    // tells the MMA issuer the unit is ready.
    const int q = warp & 3, part = (warp - 8) >> 2;
    const int blk = NB == 2 ? part : 0;
    constexpr int MY_CH = NB == 2 ? C::CH : C::CH / 2;      // chunks this warp expands
    constexpr int COLS_PER_CH = C::COLS_PER_CH;
    const int ch0 = NB == 2 ? 0 : part * MY_CH;
    const int r = blk * 128 + q * 32 + lane;  // sign row within the tile = TMEM lane in its block
    // The expanders see only a flat sequence of units (ring slots). Software
    // pipelined: the store of unit `it` is in flight while the warp waits for
    // the inputs of unit it + 1; only then is unit `it` signalled.
    const int my_tiles = tile_first < num_tiles ? (num_tiles - tile_first + tile_step - 1) / tile_step : 0;
    const uint32_t total = static_cast<uint32_t>(my_tiles * (u_last - u_first));
    uint32_t v[MY_CH * COLS_PER_CH];
    auto inputs_ready = [&](uint32_t it) -> bool {
      const uint32_t a = it % SA, bs = it % C::SB;
      const bool ok = (it < static_cast<uint32_t>(SA) ||
                       mbar_wait(smem_u32(&a_empty[a]), ((it / SA) - 1) & 1, kWhereGemmExpander)) &&
                      mbar_wait(smem_u32(&b_full[bs]), (it / C::SB) & 1, kWhereGemmExpander);
      return __all_sync(0xffffffffu, ok);
    };
    auto expand_and_store = [&](uint32_t it) {
      tc_fence_after_sync();
      const uint32_t a = it % SA, bs = it % C::SB;
      const uint4 wv = *reinterpret_cast<const uint4*>(bits_ring + bs * C::BITS_BYTES + r * 16 * C::PLANES);
      const uint32_t wd[4] = {wv.x, wv.y, wv.z, wv.w};
      uint4 mv = make_uint4(0u, 0u, 0u, 0u);
      if (KIND == 2) mv = *reinterpret_cast<const uint4*>(bits_ring + bs * C::BITS_BYTES + r * 32 + 16);
      const uint32_t md[4] = {mv.x, mv.y, mv.z, mv.w};
      const uint32_t taddr = a_base + (a * NB + blk) * C::A_COLS + ch0 * COLS_PER_CH +
                             (static_cast<uint32_t>(q * 32) << 16);
      // this warp's chunks are words ch0/2 .. ch0/2 + MY_CH/2 - 1 of the row
#pragma unroll
      for (int j = 0; j < MY_CH; ++j) {
        const uint32_t word = NB == 2 ? wd[j >> 1] : (ch0 == 0 ? wd[j >> 1] : wd[2 + (j >> 1)]);
        const uint32_t chunk = (word >> (16 * (j & 1))) & 0xFFFFu;  // ch0 is even
        if (KIND == 0) {
          expand16_bf16(chunk, v + j * COLS_PER_CH);
        } else if (KIND == 1) {
          expand16_i8(chunk, v + j * COLS_PER_CH);
        } else {
          const uint32_t mword = NB == 2 ? md[j >> 1] : (ch0 == 0 ? md[j >> 1] : md[2 + (j >> 1)]);
          expand16_ternary(chunk, (mword >> (16 * (j & 1))) & 0xFFFFu, v + j * COLS_PER_CH);
        }
      }
      tmem_st_wide<MY_CH * COLS_PER_CH>(taddr, v);
    };
    bool ok = total > 0 && inputs_ready(0);
    if (ok) expand_and_store(0);
    for (uint32_t it = 0; ok && it < total; ++it) {
      const bool more = it + 1 < total;
      const bool next_ok = !more || inputs_ready(it + 1);
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        // the expander of rank it % 8 also waits for the unit's activations
        const bool x_waiter = (warp - 8) == static_cast<int>(it % kTsExpanders);
        if (x_waiter && !mbar_wait(smem_u32(&x_full[it % SX]), (it / SX) & 1, kWhereGemmExpander))
          ok = false;  // a_full then never completes: the MMA issuer gives up on its own bounded wait
        else
          mbar_arrive(smem_u32(&a_full[it % SA]));
        mbar_arrive(smem_u32(&b_empty[it % C::SB]));
      }
      ok = (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0) && next_ok;
      if (ok && more) expand_and_store(it + 1);
    }
  } else if (warp >= 4 && SPLIT) {
    // ---------------- split-K epilogue: push partials, owner reduces ----------------
    const int q = warp & 3, et = threadIdx.x - 128;
    const int rows_per = ROWS / S;                      // rows owned by each CTA of the cluster
    constexpr int IN_STRIDE = C::IN_STRIDE;             // 4-byte words per inbox row
    uint8_t* inbox = bits_ring + C::SB * C::BITS_BYTES;  // [S][rows_per][IN_STRIDE] 4-byte partials
    const int tile = tile_first;
    const int t0 = (tile % tiles_t) * T, w0 = (tile / tiles_t) * ROWS;
    // scales of the rows this CTA finishes / of the tile's tokens, read while the MMAs run
    if (KIND != 0) {
      const double bt = static_cast<double>(*beta);
      for (int tt = et; tt < T; tt += 128)
        tok_scale[tt] = w1a8_token_scale(bt, t0 + tt < M ? gamma[t0 + tt] : 0.0);
    } else {
      for (int rr = et; rr < rows_per; rr += 128) {
        const int j = w0 + static_cast<int>(rank) * rows_per + rr;
        row_alpha[rr] = j < N ? alpha[j] : 0.f;
      }
    }
    // partials of the rows this CTA owns go to its own inbox with plain shared
    // stores; only the other S - 1 CTAs' partials are counted on the barrier
    if (threadIdx.x == 128) mbar_arrive_expect_tx(smem_u32(&inbox_bar), (S - 1) * rows_per * T * 4);
    asm volatile("barrier.cluster.wait;" ::: "memory");  // every inbox barrier is initialised
    // warp-uniform outcome: the TMEM loads below are warp-collective
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&d_full), 0, kWhereGemmEpilogue));
    tc_fence_after_sync();
#pragma unroll 1
    for (int blk = 0; blk < NB && ok; ++blk) {
      const int jl = blk * 128 + q * 32 + lane;
      const uint32_t owner = static_cast<uint32_t>(jl / rows_per);
      const uint32_t slot0 =
          smem_u32(inbox + (static_cast<int>(rank) * rows_per + jl % rows_per) * IN_STRIDE * 4);
      const bool local = owner == rank;
      const uint32_t rslot = local ? slot0 : ts_map_rank(slot0, owner);
      const uint32_t rbar = ts_map_rank(smem_u32(&inbox_bar), owner);
#pragma unroll 1
      for (int cc = 0; cc < T / 32; ++cc) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + blk * T + cc * 32 + (static_cast<uint32_t>(q * 32) << 16), r);
        tmem_wait_ld();
        if (local) {
#pragma unroll
          for (int v = 0; v < 8; ++v) st_shared_v4(rslot + (cc * 32 + v * 4) * 4, r + v * 4);
        } else {
#pragma unroll
          for (int v = 0; v < 8; ++v) st_async_v4(rslot + (cc * 32 + v * 4) * 4, r + v * 4, rbar);
        }
      }
    }
    epilogue_bar();  // tok_scale / row_alpha and the local partials are written
    // owner: add the S partials of its rows in rank order, then scale and store.
    // A thread keeps one row (rows_per is 16, 32 or 64, so lanes are consecutive
    // rows and each output store of a warp is contiguous) and steps over groups
    // of four tokens; the padded inbox rows make the 16-byte reads conflict-free.
    if (mbar_wait(smem_u32(&inbox_bar), 0, kWhereGemmEpilogue)) {
      const int rows_shift = __ffs(rows_per) - 1;
      const int rr = et & (rows_per - 1);
      const int j = w0 + static_cast<int>(rank) * rows_per + rr;
      const float arow = (KIND == 0) ? row_alpha[rr] : 0.f;
      const uint32_t in0 = smem_u32(inbox + rr * IN_STRIDE * 4);
      constexpr int kQuads = T / 4;
      for (int tq = et >> rows_shift; j < N && tq < kQuads; tq += 128 >> rows_shift) {
        uint32_t sum[4] = {0u, 0u, 0u, 0u};
        float fsum[4] = {0.f, 0.f, 0.f, 0.f};
        for (int src = 0; src < S; ++src) {
          uint32_t w[4];
          ld_shared_v4(in0 + (src * rows_per * IN_STRIDE + 4 * tq) * 4, w);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (KIND == 0)
              fsum[i] += __uint_as_float(w[i]);
            else
              sum[i] += w[i];  // two's complement: exact int32 sum
          }
        }
        const int m0 = t0 + 4 * tq;
        if (KIND == 0) {
          uint16_t* yp = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(m0) * N + j;
#pragma unroll
          for (int i = 0; i < 4; ++i, yp += N)
            if (m0 + i < M) *yp = float_to_bf16_bits(fsum[i] * arow);
        } else {
          float out[4];
          const bool fast = w1a8_fast_ok(static_cast<int32_t>(sum[0])) && w1a8_fast_ok(static_cast<int32_t>(sum[1])) &&
                            w1a8_fast_ok(static_cast<int32_t>(sum[2])) && w1a8_fast_ok(static_cast<int32_t>(sum[3]));
          if (fast) {
#pragma unroll
            for (int i = 0; i < 4; ++i) out[i] = w1a8_output_fast(static_cast<int32_t>(sum[i]), tok_scale[4 * tq + i]);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) out[i] = w1a8_output(static_cast<int32_t>(sum[i]), tok_scale[4 * tq + i]);
          }
          float* yp = reinterpret_cast<float*>(y) + static_cast<int64_t>(m0) * N + j;
          if (m0 + 4 <= M) {
#pragma unroll
            for (int i = 0; i < 4; ++i, yp += N) *yp = out[i];
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i, yp += N)
              if (m0 + i < M) *yp = out[i];
          }
          if (acc_out) {
            int32_t* ap = acc_out + static_cast<int64_t>(m0) * N + j;
#pragma unroll
            for (int i = 0; i < 4; ++i, ap += N)
              if (m0 + i < M) *ap = static_cast<int32_t>(sum[i]);
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ---------------- epilogue ----------------
    // Accumulators -> scaled outputs -> (int8 kinds) staging tile [T tokens]
    // [STAGE_COLS] in shared memory -> one bulk tensor store per staged group
    // of rows (rows/tokens past N/M are clipped by the store), or (bf16, and
    // any unaligned output: N % 4 for fp32) stores straight to global memory,
    // the range tests made once per 32-element chunk. The accumulators are
    // released as soon as the last of them is read. The per-row alpha and per-token scale are read once
    // per tile into registers / shared memory, never per element.
    constexpr int BLK_PER_GROUP = C::STAGE_COLS / 128;
    const int q = warp & 3, et = threadIdx.x - 128;
    uint8_t* stage_out = bits_ring + C::SB * C::BITS_BYTES;
    const bool staged = C::STAGE_OUT && use_tma_store;
    const bool leader = (warp == 4 && lane == 0);
    uint32_t tcount = 0;
    double bt = 0.0;
    if (KIND != 0) bt = static_cast<double>(*beta);
    for (int tile = tile_first; tile < num_tiles; tile += tile_step, ++tcount) {
      const int t0 = (tile % tiles_t) * T, w0 = (tile / tiles_t) * ROWS;
      if (KIND != 0) {
        epilogue_bar();  // the previous tile's readers of tok_scale are done
        for (int tt = et; tt < T; tt += 128)
          tok_scale[tt] = w1a8_token_scale(bt, t0 + tt < M ? gamma[t0 + tt] : 0.0);
      }
      float aj[NB];
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const int j = w0 + blk * 128 + q * 32 + lane;
        aj[blk] = (KIND == 0 && j < N) ? alpha[j] : 0.f;
      }
      // all four warps leave together if the accumulators never arrive
      if (!epilogue_bar_and(mbar_wait(smem_u32(&d_full), tcount & 1, kWhereGemmEpilogue))) break;
      tc_fence_after_sync();
#pragma unroll 1
      for (int g = 0; g < NB / BLK_PER_GROUP; ++g) {
        if (staged && leader) bulk_wait_read0();  // the previous store has read the staging tile
        epilogue_bar();                           // (and tok_scale is written)
#pragma unroll 1
        for (int b = 0; b < BLK_PER_GROUP; ++b) {
          const int blk = g * BLK_PER_GROUP + b;
          const int jl = blk * 128 + q * 32 + lane;  // row of the tile = output channel w0 + jl
          const int js = b * 128 + q * 32 + lane;    // column in the staging tile
          const int j = w0 + jl;
          const bool jv = j < N;
          const float a = (NB == 1 || blk == 0) ? aj[0] : aj[NB - 1];
#pragma unroll 1
          for (int cc = 0; cc < T / 32; ++cc) {
            uint32_t r[32];
            __syncwarp();
            tmem_ld_32x32b_x32(tmem + blk * T + cc * 32 + (static_cast<uint32_t>(q * 32) << 16), r);
            tmem_wait_ld();
            if (blk == NB - 1 && cc == T / 32 - 1) {
              // every accumulator column of this tile has been read: free them
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&d_empty));
            }
            const int ml0 = cc * 32;
            // rows past N and tokens past M are skipped; the tests are hoisted
            // out of the element loops, which stay free of branches
            const bool chunk_full = jv && t0 + ml0 + 32 <= M;
            if (KIND == 0) {
              uint16_t v[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = float_to_bf16_bits(__uint_as_float(r[i]) * a);
              if (staged) {
                const uint32_t so = smem_u32(stage_out) + (ml0 * C::STAGE_COLS + js) * 2;
#pragma unroll
                for (int i = 0; i < 32; ++i) st_shared_u16(so + i * C::STAGE_COLS * 2, v[i]);
              } else if (chunk_full) {
                uint16_t* yp = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(t0 + ml0) * N + j;
#pragma unroll
                for (int i = 0; i < 32; ++i, yp += N) *yp = v[i];
              } else if (jv) {
                uint16_t* yp = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(t0 + ml0) * N + j;
#pragma unroll
                for (int i = 0; i < 32; ++i, yp += N)
                  if (t0 + ml0 + i < M) *yp = v[i];
              }
            } else {
              // the fp32 form covers the chunk unless some |acc| is very large
              // (K beyond ~33k); the test is made once per chunk, so the
              // element loop stays free of branches
              bool fast = true;
#pragma unroll
              for (int i = 0; i < 32; ++i) fast &= w1a8_fast_ok(static_cast<int32_t>(r[i]));
              float v[32];
              if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = w1a8_output_fast(static_cast<int32_t>(r[i]), tok_scale[ml0 + i]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = w1a8_output(static_cast<int32_t>(r[i]), tok_scale[ml0 + i]);
              }
              if (staged) {
                const uint32_t so = smem_u32(stage_out) + (ml0 * C::STAGE_COLS + js) * 4;
#pragma unroll
                for (int i = 0; i < 32; ++i) st_shared_f32(so + i * C::STAGE_COLS * 4, v[i]);
              } else if (chunk_full) {
                float* yp = reinterpret_cast<float*>(y) + static_cast<int64_t>(t0 + ml0) * N + j;
#pragma unroll
                for (int i = 0; i < 32; ++i, yp += N) *yp = v[i];
              } else if (jv) {
                float* yp = reinterpret_cast<float*>(y) + static_cast<int64_t>(t0 + ml0) * N + j;
#pragma unroll
                for (int i = 0; i < 32; ++i, yp += N)
                  if (t0 + ml0 + i < M) *yp = v[i];
              }
              if (acc_out && jv) {
                int32_t* ap = acc_out + static_cast<int64_t>(t0 + ml0) * N + j;
#pragma unroll
                for (int i = 0; i < 32; ++i, ap += N)
                  if (t0 + ml0 + i < M) *ap = static_cast<int32_t>(r[i]);
              }
            }
          }
        }
        if (staged) {
          fence_proxy_async_smem();  // staging writes -> visible to the bulk store
          epilogue_bar();
          if (leader) {
            tma_store_2d(&tm_y, smem_u32(stage_out), w0 + g * C::STAGE_COLS, t0);
            bulk_commit();
          }
        }
      }
    }
    if (staged && leader) bulk_wait0();
  }

  if (SPLIT && !(warp >= 4 && warp < 8))
    asm volatile("barrier.cluster.wait;" ::: "memory");  // matches the arrive above (lanes may diverge)
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace bl

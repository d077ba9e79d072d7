// Decode of a batch of 2..16 tokens through a stack of binarized linear
// layers in one persistent launch ("FBI-LLM" page, FBI-linear paragraph:
// y_mj = bf16(alpha_j * sum_k sign(W_jk) x_mk) for every linear, the levels
// one after another).
//
// The same machinery as the single-token stack kernel (bl_gemv_stream.cuh):
// clusters of 8 CTAs splitting K into slices, balanced runs of 16-row chunks
// cut into slabs of up to 256 rows, a producer warp streaming 16 KB weight
// slots into a ring by tensor copies, outputs published as tagged words, an
// 8-way exchange of the slice partials through the row owners' inboxes. What
// differs is the arithmetic: with up to 16 tokens the products run on the
// warp-level m16n8k16 bf16 MMA, as in the few-token GEMV (bl_gemv_mma.cuh):
// the signs of 16 rows turned into +-1 bf16 A registers in place (shift,
// mask, xor), the tokens the 8-wide N side (one or two MMAs per 16 k), fp32
// accumulation. No lookup table is built, so each level needs only its input
// slice in shared memory ([token][k - 32 s0], each 32-k word permuted so that
// an A register is one shift and one LOP3 of a packed word and a B fragment
// one 64-bit load; rows padded so those loads hit 32 banks).
//
// Work per pass: kSmWarps compute warps each take kSmTiles 16-row MMA tiles
// (sharing every B fragment) of one of the pass's one or two slabs. A row's
// partial over the CTA's slice is the MMAs of its tile in (word, half)
// order whatever the tiling, so outputs do not depend on it.
//
// Tagged buffers hold [token][N] words; the exchange carries up to 16 tokens
// per row, plus the per-pass token from every peer that keeps the
// double-buffered inbox safe (see bl_gemv_stream.cuh). Waits are bounded as
// in the single-token kernel.
#pragma once

#include "bl_gemv_mma.cuh"
#include "bl_gemv_stream.cuh"

namespace bl {

// Compute warps and 16-row MMA tiles per warp. Measured on the 7B chain (80
// levels, 16 / 8 tokens): 16 warps x 1 tile 1636 / 1190 us, 16 x 2 1664 /
// 1372, 8 x 2 1892 / 1526, 8 x 4 1965 / 1601, 4 x 4 2777 / 2120 (all
// bit-identical): a warp's MMA chain is latency-bound, so warps (17 with the
// producer, which caps registers at 96) beat tiles that share B fragments.
#ifndef BL_SM_WARPS
#define BL_SM_WARPS 16
#endif
#ifndef BL_SM_TILES
#define BL_SM_TILES 1
#endif
constexpr int kSmMaxSlice = 48;               // words of a slice (K <= 12288)
constexpr int kSmWarps = BL_SM_WARPS;         // compute warps
constexpr int kSmThreads = kSmWarps * 32;
constexpr int kSmTiles = BL_SM_TILES;         // 16-row MMA tiles per warp
constexpr int kSmPass = kSmWarps * kSmTiles * kStrChunk / kStrRows;  // slabs per pass
constexpr int kSmWarpsPerSlab = kSmWarps / kSmPass;
constexpr int kSmOwned = kStrRows / kStrCluster;  // 32 rows of a slab per owner
static_assert(kSmPass >= 1 && kSmPass <= 2 && kSmWarps * kSmTiles * kStrChunk == kSmPass * kStrRows,
              "the warps cover one or two slabs");

// bytes per token row of the staged inputs: the slice plus 32 bytes, so that
// the 64-bit B-fragment loads of a half-warp (4 tokens x 4 lanes) hit 32 banks
__host__ __device__ constexpr int sm_x_pitch(int mt) { (void)mt; return kSmMaxSlice * 64 + 32; }

// Order of the inputs within a 32-k word as staged for the MMAs. The dot
// product does not depend on the order of k, so the inputs are permuted (and
// the signs read at the matching bits) to make the A registers cheap: lane t's
// register j of 16-k chunk o takes the signs of bits b and b + 16 of the
// packed word, b = 4t + 2o + j, which one shift brings to the two bf16 sign
// positions (15 and 31). Staged position p (0..31) of a word holds input
//   k(p) = b + 16 (p & 1),  b = 4 ((p >> 2) & 3) + 2 (p >> 4) + ((p >> 1) & 1),
// so that lane t's B fragment of chunk o (the MMA's k = 2t, 2t + 1, 2t + 8,
// 2t + 9) is the 4 consecutive positions 16 o + 4 t .. + 3.
__host__ __device__ constexpr int sm_perm_k(int p) {
  return 4 * ((p >> 2) & 3) + 2 * (p >> 4) + ((p >> 1) & 1) + 16 * (p & 1);
}
template <int MT>
struct SmCfg {
  static constexpr int kSlots = (MT > 8 && kSmPass > 1) ? 6 : 8;            // ring depth (shared memory)
  static constexpr int kInboxHalf = kSmPass * kStrCluster * kSmOwned * MT;  // floats: [slab][src rank][owned row][token]
  static constexpr int kXBytes = MT * sm_x_pitch(MT);
  static constexpr int kSmemBytes = kSlots * kStrSlotBytes + kXBytes + 2 * kInboxHalf * 4;  // dynamic
  static constexpr int kOwned = kSmPass * kSmOwned * MT;                    // outputs a CTA owns per pass
  static constexpr int kOwnerItems = (kOwned + kSmThreads - 1) / kSmThreads;  // per thread
};

template <int MT>
__global__ void __launch_bounds__(kSmThreads + 32, 1) gemv_w1a16_stream_mma_kernel(const __grid_constant__ StrParams P,
                                                                                   int M) {
  using C = SmCfg<MT>;
  constexpr int H = MT / 8;  // n-halves of the token tile
  constexpr int S = C::kSlots;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;                                      // S x 16 KB
  uint8_t* xs = smem + S * kStrSlotBytes;                    // [token][slice k] bf16, padded rows
  float* inbox = reinterpret_cast<float*>(xs + C::kXBytes);  // [pass % 2][slab][src rank][owned row][token]
  __shared__ __align__(8) uint64_t inbox_full[2];
  __shared__ float tokens[2][kStrCluster];  // [pass % 2][source rank]
  __shared__ __align__(8) uint64_t full[S];
  __shared__ __align__(8) uint64_t empty[S];
  __shared__ StrLevel lvs[kStrMaxLevels];
  __shared__ StrJob jobs[kStrMaxJobs];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int G = static_cast<int>(gridDim.y), cid = static_cast<int>(blockIdx.y);
  const int pitch = sm_x_pitch(MT);

  for (int i = tid; i < P.num_levels * static_cast<int>(sizeof(StrLevel) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(lvs)[i] = reinterpret_cast<const uint4*>(P.lv)[i];
  for (int i = tid; i < P.num_jobs * static_cast<int>(sizeof(StrJob) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(jobs)[i] = reinterpret_cast<const uint4*>(P.jobs)[i];
  // tokens past M stay zero in the input slices for the whole launch
  for (int i = tid; i < C::kXBytes / 16; i += blockDim.x) reinterpret_cast<uint4*>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    mbar_init(smem_u32(&inbox_full[0]), 1);
    mbar_init(smem_u32(&inbox_full[1]), 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kSmWarps);
    }
    fence_mbar_init();
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  const int num_levels = P.num_levels;

  if (warp == kSmWarps) {
    if (lane == 0) str_produce<kSmPass, S>(P, lvs, jobs, num_levels, cid, G, rank, ring, full, empty);
    __syncwarp();
  } else {
    uint32_t q = 0, n = 0;
    bool ok = true;
    const int my_slab = warp / kSmWarpsPerSlab;    // slab of the pass this warp computes
    const int c4 = warp % kSmWarpsPerSlab;         // its rows: chunks kSmTiles c4 .. + kSmTiles - 1 of the slab
    for (int l = 0; l < num_levels; ++l) {
      const StrLevel& lv = lvs[l];
      StrRun run = str_run(jobs, lv, cid, G);
      if (run.cur >= run.end) continue;
      const LutWindow win = str_window(lv.K, rank);
      const int np = str_pages(win);

      // ---- the slice of every token's input, each 32-k word in the
      // permuted order above: xs[m][32 w + p] = x[m][32 (s0 + w) + k(p)] ----
      {
        const int e0 = win.s0 * 32, blocks = M * win.sw;  // (token, word) blocks
        for (int blk = tid; blk < blocks; blk += kSmThreads) {
          const int m = blk / win.sw, w = blk - m * win.sw;
          uint32_t v[16];  // bf16 pairs of inputs k = 2i, 2i + 1
          if (lv.xt) {
            const uint32_t* src = lv.xt + static_cast<int64_t>(m) * lv.K + e0 + 32 * w;
            uint4 tv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) tv[i] = ld_relaxed_gpu_v4(src + 4 * i);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (!((tv[i].x & tv[i].y & tv[i].z & tv[i].w) & kStrReady) && ok) {
                const uint64_t t0 = global_timer_ns();
                do {
                  tv[i] = ld_relaxed_gpu_v4(src + 4 * i);
                  if ((tv[i].x & tv[i].y & tv[i].z & tv[i].w) & kStrReady) break;
                  if (ld_relaxed_gpu_u32(P.abort) != 0u) {
                    ok = false;
                    break;
                  }
                  if (global_timer_ns() - t0 > kWaitTimeoutNs) {
                    record_error(BL_ERR_TIMEOUT, kWhereStackLevel);
                    st_relaxed_gpu_u32(P.abort, 1u);
                    ok = false;
                    break;
                  }
                } while (true);
              }
              v[2 * i] = (tv[i].x & 0xFFFFu) | (tv[i].y << 16);
              v[2 * i + 1] = (tv[i].z & 0xFFFFu) | (tv[i].w << 16);
            }
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(lv.x + static_cast<int64_t>(m) * lv.K + e0 + 32 * w);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 q4 = src[i];
              v[4 * i] = q4.x, v[4 * i + 1] = q4.y, v[4 * i + 2] = q4.z, v[4 * i + 3] = q4.w;
            }
          }
          // output pair (p, p + 1), p even: inputs k(p) and k(p) + 16
          uint32_t o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k0 = sm_perm_k(2 * i);  // even input index? take its half of the pair
            const uint32_t lo = (k0 & 1) ? (v[k0 >> 1] >> 16) : (v[k0 >> 1] & 0xFFFFu);
            const int k1 = k0 + 16;
            const uint32_t hi = (k1 & 1) ? (v[k1 >> 1] & 0xFFFF0000u) : (v[k1 >> 1] << 16);
            o[i] = lo | hi;
          }
          uint4* dst = reinterpret_cast<uint4*>(xs + m * pitch + 64 * w);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
      consumers_sync<kSmThreads>();

      while (true) {
        // the pass's slabs (constant indices only: the pair stays in registers)
        StrSlab sl[kSmPass];
        int npass = 0;
        if (str_next_slab(jobs, lv, run, sl[0])) npass = (kSmPass > 1 && str_next_slab(jobs, lv, run, sl[kSmPass - 1])) ? 2 : 1;
        if (npass == 0) break;
        auto slab = [&](int s) -> const StrSlab& { return s == 0 ? sl[0] : sl[kSmPass - 1]; };
        float* ib = inbox + (n & 1u) * C::kInboxHalf;
        // bytes this CTA receives: 8 ranks x MT tokens x 4 bytes per owned
        // live row, and one 4-byte pass token from each rank
        if (tid == 0) {
          uint32_t rows = 0;
          for (int s = 0; s < npass; ++s) {
            const int r = slab(s).nc() * kStrChunk - static_cast<int>(rank) * kSmOwned;
            rows += r <= 0 ? 0u : (r >= kSmOwned ? static_cast<uint32_t>(kSmOwned) : static_cast<uint32_t>(r));
          }
          mbar_arrive_expect_tx(smem_u32(&inbox_full[n & 1u]), (rows * MT + 1) * kStrCluster * 4);
        }
        // owners: item e of thread tid is (slab, owned row, token) index
        // tid + kSmThreads e, tokens fastest (a warp's inbox reads are
        // consecutive words); their scales are loaded now, used after the exchange
        float oalpha[C::kOwnerItems];
#pragma unroll
        for (int e = 0; e < C::kOwnerItems; ++e) {
          const int idx = tid + kSmThreads * e;
          const int s = idx / (kSmOwned * MT), orr = (idx / MT) % kSmOwned, om = idx % MT;
          const int orow_s = static_cast<int>(rank) * kSmOwned + orr;
          oalpha[e] = 0.f;
          if (idx < C::kOwned && s < npass && om < M && orow_s < slab(s).nc() * kStrChunk) {
            const StrJob& jb = jobs[slab(s).j()];
            if (slab(s).row0 + orow_s < jb.N) oalpha[e] = jb.alpha[slab(s).row0 + orow_s];
          }
        }

        // live tiles of this warp: chunks of its slab from 4 c4 on
        int ntile = 0;
        if (my_slab < npass) {
          const int r = slab(my_slab).nc() - kSmTiles * c4;
          ntile = r <= 0 ? 0 : (r >= kSmTiles ? kSmTiles : r);
        }
        float acc[kSmTiles][H][4];
#pragma unroll
        for (int tt = 0; tt < kSmTiles; ++tt)
#pragma unroll
          for (int hh = 0; hh < H; ++hh)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[tt][hh][i] = 0.f;
        // lane t's A register j of chunk o: signs of bits 4t + 2o + j and + 16
        const uint32_t sh00 = 15 - 4 * t, sh01 = 14 - 4 * t, sh10 = 13 - 4 * t, sh11 = 12 - 4 * t;
        for (int pg = 0; pg < np; ++pg) {
          // every slot of the page has landed (each warp waits for all of
          // them: it releases all of them below)
          for (int s = 0; s < npass; ++s) {
            const uint32_t k = q + static_cast<uint32_t>(s);
            if (ok && !mbar_wait(smem_u32(&full[k % S]), (k / S) & 1u, kWhereStackRing)) {
              st_relaxed_gpu_u32(P.abort, 1u);
              ok = false;
            }
          }
          if (ntile > 0) {
            const uint32_t* sw = reinterpret_cast<const uint32_t*>(ring + ((q + my_slab) % S) * kStrSlotBytes);
            const int rbase = kSmTiles * c4 * kStrChunk + g;  // row g of tile 0 of this warp in the slab
            const bool full_page = pg * 16 >= win.lo() && pg * 16 + 16 <= win.hi();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              // words 4c .. 4c + 3 of the page, rows g and g + 8 of each tile
              uint32_t wa[kSmTiles][4], wb[kSmTiles][4];
#pragma unroll
              for (int tt = 0; tt < kSmTiles; ++tt) {
                const uint4 va = *reinterpret_cast<const uint4*>(sw + (rbase + 16 * tt) * 16 + 4 * c);
                const uint4 vb = *reinterpret_cast<const uint4*>(sw + (rbase + 16 * tt + 8) * 16 + 4 * c);
                wa[tt][0] = va.x, wa[tt][1] = va.y, wa[tt][2] = va.z, wa[tt][3] = va.w;
                wb[tt][0] = vb.x, wb[tt][1] = vb.y, wb[tt][2] = vb.z, wb[tt][3] = vb.w;
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int wi = pg * 16 + 4 * c + i;
                if (!full_page && (wi < win.lo() || wi >= win.hi())) continue;  // uniform across the warp
#pragma unroll
                for (int o = 0; o < 2; ++o) {
                  const uint32_t s0 = o ? sh10 : sh00, s1 = o ? sh11 : sh01;
                  const int kb = (wi - win.lo()) * 64 + o * 32 + 8 * t;  // lane's 4 staged inputs
                  uint2 bv[H];
#pragma unroll
                  for (int hh = 0; hh < H; ++hh)
                    bv[hh] = *reinterpret_cast<const uint2*>(xs + (8 * hh + g) * pitch + kb);
#pragma unroll
                  for (int tt = 0; tt < kSmTiles; ++tt) {
                    if (tt < ntile) {  // uniform across the warp
                      // bit b -> bit 15 and bit b + 16 -> bit 31; set bit -> +1 (0x3F80)
                      const uint32_t a[4] = {((wa[tt][i] << s0) & 0x80008000u) ^ 0xBF80BF80u,
                                             ((wb[tt][i] << s0) & 0x80008000u) ^ 0xBF80BF80u,
                                             ((wa[tt][i] << s1) & 0x80008000u) ^ 0xBF80BF80u,
                                             ((wb[tt][i] << s1) & 0x80008000u) ^ 0xBF80BF80u};
#pragma unroll
                      for (int hh = 0; hh < H; ++hh) mma_bf16_16816(acc[tt][hh], a, bv[hh].x, bv[hh].y);
                    }
                  }
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0)
            for (int s = 0; s < npass; ++s) mbar_arrive(smem_u32(&empty[(q + static_cast<uint32_t>(s)) % S]));
          q += static_cast<uint32_t>(npass);
        }

        // ---- partials to the rows' owners: tile tt of warp (slab, c4) is
        // chunk kSmTiles c4 + tt of the slab, owned by rank chunk / 2 ----
#pragma unroll
        for (int tt = 0; tt < kSmTiles; ++tt) {
          if (tt < ntile) {
            const int ch = kSmTiles * c4 + tt;
            const uint32_t owner_rank = static_cast<uint32_t>(ch >> 1);
            const uint32_t bar = map_to_rank(smem_u32(&inbox_full[n & 1u]), owner_rank);
            const int r0 = 16 * (ch & 1) + g;  // owned row of row g of the tile (row g + 8: r0 + 8)
            float* dst = ib + ((my_slab * kStrCluster + static_cast<int>(rank)) * kSmOwned + r0) * MT;
#pragma unroll
            for (int hh = 0; hh < H; ++hh) {
              const int tok = 8 * hh + 2 * t;
              st_async_v2_f32(map_to_rank(smem_u32(dst + tok), owner_rank), acc[tt][hh][0], acc[tt][hh][1], bar);
              st_async_v2_f32(map_to_rank(smem_u32(dst + 8 * MT + tok), owner_rank), acc[tt][hh][2],
                              acc[tt][hh][3], bar);
            }
          }
        }
        if (warp == 0 && lane < kStrCluster) {  // this pass's token to rank `lane`
          const uint32_t dst = static_cast<uint32_t>(lane);
          st_async_f32(map_to_rank(smem_u32(&tokens[n & 1u][rank]), dst), 0.f,
                       map_to_rank(smem_u32(&inbox_full[n & 1u]), dst));
        }
        bool got = false;
        if (ok) {
          got = mbar_wait(smem_u32(&inbox_full[n & 1u]), (n >> 1) & 1u, kWhereStackInbox);
          if (!got) {
            st_relaxed_gpu_u32(P.abort, 1u);
            ok = false;
          }
        }
        if (got) {
#pragma unroll
          for (int e = 0; e < C::kOwnerItems; ++e) {
            const int idx = tid + kSmThreads * e;
            const int s = idx / (kSmOwned * MT), orr = (idx / MT) % kSmOwned, om = idx % MT;
            const int orow_s = static_cast<int>(rank) * kSmOwned + orr;
            if (idx < C::kOwned && s < npass && om < M && orow_s < slab(s).nc() * kStrChunk) {
              const StrJob& jb = jobs[slab(s).j()];
              const int orow = slab(s).row0 + orow_s;
              if (orow < jb.N) {
                const float* in = ib + (s * kStrCluster * kSmOwned + orr) * MT + om;
                float sum = 0.f;
#pragma unroll
                for (int r = 0; r < kStrCluster; ++r) sum += in[r * kSmOwned * MT];
                const uint16_t yv = float_to_bf16_bits(oalpha[e] * sum);
                const int64_t o = static_cast<int64_t>(om) * jb.N + orow;
                if (jb.tagged) st_relaxed_gpu_u32(jb.tagged + o, kStrReady | yv);  // publish first
                jb.y[o] = yv;
              }
            }
          }
        }
        // the owners have read this pass's inbox before any warp pushes the next pass
        consumers_sync<kSmThreads>();
        ++n;
      }
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
}

}  // namespace bl

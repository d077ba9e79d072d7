// Decode of a batch of 2..16 tokens through a stack of binarized linear
// layers in one persistent launch ("FBI-LLM" page, FBI-linear paragraph:
// y_mj = bf16(alpha_j * sum_k sign(W_jk) x_mk) for every linear, the levels
// one after another).
//
// The same machinery as the single-token stack kernel (bl_gemv_stream.cuh):
// clusters of 8 CTAs splitting K into slices, balanced runs of 16-row chunks
// cut into slabs, a producer warp streaming 16 KB weight slots into a ring by
// tensor copies, outputs published as tagged words, an 8-way exchange of the
// slice partials through the row owners' inboxes. What differs is the
// arithmetic: with up to 16 tokens the products run on the warp-level
// m16n8k16 bf16 MMA, as in the few-token GEMV (bl_gemv_mma.cuh): a warp's 16
// rows (g and g + 8 of the A fragment) over the CTA's K slice, the signs
// turned into +-1 bf16 A registers in place (r = b | b << 15, shift, mask,
// xor), the tokens the 8-wide N side (one or two MMAs per 16 k), fp32
// accumulation. No lookup table is built, so each level needs only its input
// slice in shared memory ([token][k - 32 s0], each 32-k word permuted so that
// an A register is one shift and one LOP3 of a packed word and a B fragment
// one 64-bit load; rows padded so those loads hit 32 banks), one slab per pass.
//
// Tagged buffers hold [token][N] words; the exchange carries up to 16 tokens
// per row, plus the per-pass token from every peer that keeps the
// double-buffered inbox safe (see bl_gemv_stream.cuh). Waits are bounded as
// in the single-token kernel.
//
// Other shapes of the work were measured on the 7B chain (80 levels, 16 / 8
// tokens, compute warps x 16-row tiles per warp, one or two 256-row slabs per
// pass, outputs bit-identical): 16 x 1 (this kernel) 1636 / 1190 us, 16 x 2
// 1664 / 1372, 8 x 2 1892 / 1526, 8 x 4 1965 / 1601, 4 x 4 2777 / 2120: a
// warp's MMA chain is latency-bound, so warps (17 with the producer, which
// caps registers at 96) beat tiles that share B fragments.
#pragma once

#include "bl_gemv_mma.cuh"
#include "bl_gemv_stream.cuh"

namespace bl {

constexpr int kSmMaxSlice = 48;                                  // words of a slice (K <= 12288)
constexpr int kSmThreads = kStrThreads;                          // 16 compute warps
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
  static constexpr int kInbox = 2 * kStrCluster * 32 * MT;        // floats: [pass % 2][src rank][owned row][token]
  static constexpr int kXBytes = MT * sm_x_pitch(MT);
  static constexpr int kSmemBytes = kStrSlots * kStrSlotBytes + kXBytes + kInbox * 4;  // dynamic
};

template <int MT>
__global__ void __launch_bounds__(kStrThreads + 32, 1) gemv_w1a16_stream_mma_kernel(const __grid_constant__ StrParams P,
                                                                                     int M) {
  using C = SmCfg<MT>;
  constexpr int H = MT / 8;  // n-halves of the token tile
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;                                          // kStrSlots x 16 KB
  uint8_t* xs = smem + kStrSlots * kStrSlotBytes;                // [token][slice k] bf16, padded rows
  float* inbox = reinterpret_cast<float*>(xs + C::kXBytes);
  __shared__ __align__(8) uint64_t inbox_full[2];
  __shared__ float tokens[2][kStrCluster];  // [pass % 2][source rank]
  __shared__ __align__(8) uint64_t full[kStrSlots];
  __shared__ __align__(8) uint64_t empty[kStrSlots];
  __shared__ StrLevel lvs[kStrMaxLevels];
  __shared__ StrJob jobs[kStrMaxJobs];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int G = static_cast<int>(gridDim.y), cid = static_cast<int>(blockIdx.y);
  constexpr int kOwned = kStrRows / kStrCluster;  // 32 rows of a slab per owner
  constexpr int kWarps = kStrThreads / 32;
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
    for (int s = 0; s < kStrSlots; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kWarps);
    }
    fence_mbar_init();
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  const int num_levels = P.num_levels;

  if (warp == kWarps) {
    if (lane == 0) str_produce<1>(P, lvs, jobs, num_levels, cid, G, rank, ring, full, empty);
    __syncwarp();
  } else {
    uint32_t q = 0, n = 0;
    bool ok = true;
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
        for (int blk = tid; blk < blocks; blk += kStrThreads) {
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
      consumers_sync();

      StrSlab sl;
      while (str_next_slab(jobs, lv, run, sl)) {
        // bytes this CTA receives: 8 ranks x MT tokens x 4 bytes per owned
        // live row, and one 4-byte pass token from each rank
        if (tid == 0) {
          const int r = sl.nc() * kStrChunk - static_cast<int>(rank) * kOwned;
          const uint32_t rows = r <= 0 ? 0u : (r >= kOwned ? static_cast<uint32_t>(kOwned) : static_cast<uint32_t>(r));
          mbar_arrive_expect_tx(smem_u32(&inbox_full[n & 1u]), (rows * MT + 1) * kStrCluster * 4);
        }
        // this pass's token to every rank: "done reading my pass n - 1 inbox"
        // (true since the barrier that ended that pass), sent first so that it
        // never holds up an inbox
        if (warp == 0 && lane < kStrCluster) {
          const uint32_t dst = static_cast<uint32_t>(lane);
          st_async_f32(map_to_rank(smem_u32(&tokens[n & 1u][rank]), dst), 0.f,
                       map_to_rank(smem_u32(&inbox_full[n & 1u]), dst));
        }
        // owners: thread (row r = tid / MT, token m = tid % MT) of the slab
        // (tokens fastest: a warp's inbox reads are consecutive words)
        const int om = tid % MT, orr = tid / MT;
        const int orow_s = static_cast<int>(rank) * kOwned + orr;  // row within the slab
        const StrJob& jb = jobs[sl.j()];
        const bool owner = om < M && orow_s < sl.nc() * kStrChunk && sl.row0 + orow_s < jb.N;
        const int orow = sl.row0 + orow_s;
        const float oalpha = owner ? jb.alpha[orow] : 0.f;

        float acc[H][4];
#pragma unroll
        for (int hh = 0; hh < H; ++hh)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[hh][i] = 0.f;
        // lane t's A register j of chunk o: signs of bits 4t + 2o + j and + 16
        const uint32_t sh00 = 15 - 4 * t, sh01 = 14 - 4 * t, sh10 = 13 - 4 * t, sh11 = 12 - 4 * t;
        for (int pg = 0; pg < np; ++pg) {
          const uint32_t slot = q % kStrSlots;
          if (ok && !mbar_wait(smem_u32(&full[slot]), (q / kStrSlots) & 1u, kWhereStackRing)) {
            st_relaxed_gpu_u32(P.abort, 1u);
            ok = false;
          }
          if (warp < sl.nc()) {
            const uint32_t* sw = reinterpret_cast<const uint32_t*>(ring + slot * kStrSlotBytes);
            const int ra = warp * kStrChunk + g;  // rows ra and ra + 8 of the slab
            // one 16-bit half (o) of window word w (bits wa of row ra, wb of
            // row ra + 8): 16 k, H MMAs
            auto chunk = [&](uint32_t wa, uint32_t wb, int w, int o) {
              const uint32_t s0 = o ? sh10 : sh00, s1 = o ? sh11 : sh01;
              // bit b -> bit 15 and bit b + 16 -> bit 31; set bit -> +1 (0x3F80)
              const uint32_t a[4] = {((wa << s0) & 0x80008000u) ^ 0xBF80BF80u, ((wb << s0) & 0x80008000u) ^ 0xBF80BF80u,
                                     ((wa << s1) & 0x80008000u) ^ 0xBF80BF80u, ((wb << s1) & 0x80008000u) ^ 0xBF80BF80u};
              const int kb = (pg * 16 + w - win.lo()) * 64 + o * 32 + 8 * t;  // lane's 4 staged inputs
#pragma unroll
              for (int hh = 0; hh < H; ++hh) {
                const uint2 bv = *reinterpret_cast<const uint2*>(xs + (8 * hh + g) * pitch + kb);
                mma_bf16_16816(acc[hh], a, bv.x, bv.y);
              }
            };
            const bool full_page = pg * 16 >= win.lo() && pg * 16 + 16 <= win.hi();
            // the page's words of both rows, four at a time
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 va = *reinterpret_cast<const uint4*>(sw + ra * 16 + 4 * c);
              const uint4 vb = *reinterpret_cast<const uint4*>(sw + (ra + 8) * 16 + 4 * c);
              const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
              if (full_page) {  // every word live: straight-line code
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  chunk(wa[i], wb[i], 4 * c + i, 0);
                  chunk(wa[i], wb[i], 4 * c + i, 1);
                }
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int wi = pg * 16 + 4 * c + i;
                  if (wi < win.lo() || wi >= win.hi()) continue;  // uniform across the warp
                  chunk(wa[i], wb[i], 4 * c + i, 0);
                  chunk(wa[i], wb[i], 4 * c + i, 1);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));
          ++q;
        }

        // ---- partials to the rows' owners: rows ra, ra + 8 of warp w belong to rank w / 2 ----
        if (warp < sl.nc()) {
          const uint32_t owner_rank = static_cast<uint32_t>(warp >> 1);
          const uint32_t bar = map_to_rank(smem_u32(&inbox_full[n & 1u]), owner_rank);
          const int r0 = (warp * kStrChunk + g) & (kOwned - 1);
          float* ib = inbox + (n & 1u) * (C::kInbox / 2);
#pragma unroll
          for (int hh = 0; hh < H; ++hh) {
            const int tok = 8 * hh + 2 * t;
            const uint32_t sa = smem_u32(&ib[(static_cast<int>(rank) * kOwned + r0) * MT + tok]);
            const uint32_t sb = smem_u32(&ib[(static_cast<int>(rank) * kOwned + r0 + 8) * MT + tok]);
            st_async_v2_f32(map_to_rank(sa, owner_rank), acc[hh][0], acc[hh][1], bar);
            st_async_v2_f32(map_to_rank(sb, owner_rank), acc[hh][2], acc[hh][3], bar);
          }
        }
        uint16_t yv = 0;
        bool got = false;
        if (tid < MT * kOwned) {
          if (ok) {
            got = mbar_wait(smem_u32(&inbox_full[n & 1u]), (n >> 1) & 1u, kWhereStackInbox);
            if (!got) {
              st_relaxed_gpu_u32(P.abort, 1u);
              ok = false;
            }
          }
          if (got && owner) {
            const float* in = inbox + (n & 1u) * (C::kInbox / 2) + orr * MT + om;
            float sum = 0.f;
#pragma unroll
            for (int r = 0; r < kStrCluster; ++r) sum += in[r * kOwned * MT];
            yv = float_to_bf16_bits(oalpha * sum);
          }
        }
        if (got && owner) {
          const int64_t o = static_cast<int64_t>(om) * jb.N + orow;
          if (jb.tagged) st_relaxed_gpu_u32(jb.tagged + o, kStrReady | yv);  // publish first
          jb.y[o] = yv;
        }
        // the owners have read this pass's inbox before any warp pushes the next pass
        consumers_sync();
        ++n;
      }
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
}

}  // namespace bl

// Single-token W1A16 decode through a stack of binarized linear layers in one
// persistent launch ("FBI-LLM" page, FBI-linear paragraph: every linear of the
// model is y_j = alpha_j * sum_k sign(W_jk) x_k; the decode step runs them one
// dependent level after another).
//
// The stack is a list of levels. A level has one input vector x (K) and one or
// more linears that read it (q, k, v of a block share one x; so do gate and
// up); a level's input may be any output of an earlier level. Each launch:
//
//   * a grid of G clusters of 8 CTAs, one CTA per SM, all co-resident; the
//     8 CTAs of a cluster split K into slices as in the single-layer lookup
//     kernel (byte tables of the slice in shared memory, one PRMT + LDS + FADD
//     per 8 weights) and sweep 256-row blocks, block b of a level going to
//     cluster b % G;
//   * the packed words of a pass (up to 4 blocks) are loaded into registers
//     before the lookups, and those of a level's first pass before the CTA
//     waits for the level's input (prefetching the next level into L2, with
//     per-line or bulk prefetches, measured no faster and is not done);
//   * levels are separated by a grid-wide completion count: every CTA adds 1
//     (release, GPU scope) once its outputs of level l are written, and a CTA
//     reads the input of level l + 1 only after the count of level l reached
//     the number of CTAs (acquire), through L2 (ld.global.cg), never from L1;
//   * within a cluster, per block, each CTA pushes its slice's partial of
//     every row to the row's owner (st.async counted on the owner's
//     mbarrier) and the owner adds the 8 partials in rank order: the same
//     arithmetic, in the same order, as the single-layer kernel with 8-way
//     slices. A cluster barrier per block (arrive after the owner has read its
//     inbox, wait just before the next push) guards the single inbox.
//
// Waits on the completion counts and on the inbox are bounded: past the
// limit the kernel records BL_ERR_TIMEOUT, stops waiting and finishes with
// undefined outputs. Every CTA of a cluster takes the same path through the
// cluster barriers whatever happens, so none of those can wait forever.
#pragma once

#include "bl_gemv_lut.cuh"

namespace bl {

constexpr int kStackCluster = 8;       // CTAs per cluster = K slices
constexpr int kStackPages = 3;         // table pages provisioned: slices of up to 48 words
constexpr int kStackMaxLevels = 128;   // per launch (longer stacks take several launches)
constexpr int kStackMaxJobs = 256;     // per launch

struct StackJob {
  const uint32_t* packed;  // [N][K/32]
  const float* alpha;      // [N]
  uint16_t* y;             // [N] bf16
  int N;
  int block0;              // first 256-row block of this linear within its level
};
struct StackLevel {
  const uint16_t* x;  // [K] bf16
  int K;              // multiple of 256, at most 12288
  int job0, njobs;    // jobs[job0 .. job0 + njobs)
  int nblocks;        // 256-row blocks of all its linears
};
struct StackParams {
  StackLevel lv[kStackMaxLevels];
  StackJob jb[kStackMaxJobs];
  uint32_t* done;  // [num_levels] completion counts, zero at launch
  int num_levels;
  int total_ctas;
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the linear of level `lv` that block b falls in
__device__ __forceinline__ const StackJob& stack_job_of(const StackParams& P, const StackLevel& lv, int b) {
  int j = lv.job0;
  while (j + 1 < lv.job0 + lv.njobs && b >= P.jb[j + 1].block0) ++j;
  return P.jb[j];
}

// Blocks of one level held in registers at once, per table page count.
template <int NP>
struct StackPass {
  static constexpr int kBlocks = NP == 1 ? 4 : (NP == 2 ? 2 : 1);
};

// One level with NP table pages. A cluster's blocks of the level go in
// passes of up to StackPass<NP>::kBlocks blocks: the packed words of a whole
// pass are loaded first (for the first pass, before waiting for the level's
// input), then the lookups of every block of the pass, then one round of
// pushes to the row owners. `n` counts the passes this cluster has finished
// (the inbox barrier's phase); `waiting` turns false after a bounded wait
// gave up.
template <int NP>
__device__ __forceinline__ void stack_level(const StackParams& P, int l, uint32_t rank, uint8_t* lut_smem,
                                            float* inbox, uint64_t* inbox_bar, uint32_t& n, bool& waiting) {
  constexpr int B = StackPass<NP>::kBlocks;
  const StackLevel& lv = P.lv[l];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = lane >> 4, wl = lane & 15;
  const int words = lv.K / 32, slice_words = words / kStackCluster;
  const int slice0 = static_cast<int>(rank) * slice_words;
  const int G = static_cast<int>(gridDim.y), cid = static_cast<int>(blockIdx.y);
  constexpr int kRowsPerCta = kLutRowsPerCluster / kStackCluster;  // 32: warp w's rows belong to rank w
  const int my_blocks = cid < lv.nblocks ? (lv.nblocks - cid + G - 1) / G : 0;

  uint32_t wv[B][16][NP];
  auto load_pass = [&](int i0) {
#pragma unroll
    for (int i = 0; i < B; ++i) {
      if (i0 + i < my_blocks) {
        const int b = cid + (i0 + i) * G;
        const StackJob& jb = stack_job_of(P, lv, b);
        lut_load_rows<NP>(wv[i], jb.packed, jb.N, words, (b - jb.block0) * kLutRowsPerCluster + warp * 32,
                          slice0, slice_words, h, wl);
      }
    }
    // keep the loads ahead of everything that follows (they are only waited
    // for where their registers are first used)
    asm volatile("" ::: "memory");
  };

  // the first pass's words do not depend on x: load them before waiting
  if (my_blocks > 0) load_pass(0);

  // the input of this level is complete once every CTA has finished level l - 1
  if (l > 0) {
    if (threadIdx.x == 0 && waiting) {
      const uint32_t* cnt = P.done + (l - 1);
      const uint32_t target = static_cast<uint32_t>(P.total_ctas);
      if (ld_acquire_gpu(cnt) < target) {
        const uint64_t t0 = global_timer_ns();
        while (ld_acquire_gpu(cnt) < target) {
          if (global_timer_ns() - t0 > kWaitTimeoutNs) {
            record_error(BL_ERR_TIMEOUT, kWhereStackLevel);
            waiting = false;
            break;
          }
        }
      }
    }
    __syncthreads();
  }
  if (my_blocks > 0) {
    lut_build_table<NP, true>(lv.x + static_cast<int64_t>(slice0) * 32, slice_words, lut_smem);
    __syncthreads();
  }

  for (int i0 = 0; i0 < my_blocks; i0 += B) {
    const int nb = my_blocks - i0 < B ? my_blocks - i0 : B;
    if (i0 > 0) load_pass(i0);
    // this pass's inbox phase expects nb blocks of partials (its pushes may
    // land before or after this; the phase cannot complete without it)
    if (threadIdx.x == 0) mbar_arrive_expect_tx(smem_u32(inbox_bar), static_cast<uint32_t>(nb) * kLutRowsPerCluster * 4);
    float part[B];
#pragma unroll
    for (int i = 0; i < B; ++i)
      if (i < nb) part[i] = lut_row_partial<NP>(wv[i], slice_words, lut_smem, h, wl);

    cluster_wait_acquire();  // every owner has read its inbox of the previous pass
    {
      const int r = warp * 32 + 2 * wl + h;  // lane's row within a block, owned by rank r / 32 = warp
      const uint32_t slot = smem_u32(&inbox[static_cast<int>(rank) * kRowsPerCta + (r & (kRowsPerCta - 1))]);
      const uint32_t rslot = map_to_rank(slot, static_cast<uint32_t>(warp));
      const uint32_t rbar = map_to_rank(smem_u32(inbox_bar), static_cast<uint32_t>(warp));
#pragma unroll
      for (int i = 0; i < B; ++i)
        if (i < nb) st_async_f32(rslot + i * kLutRowsPerCluster * 4, part[i], rbar);
    }
    // owners: thread t adds the 8 partials of row t % 32 of block t / 32
    uint16_t* yp = nullptr;
    uint16_t yv = 0;
    if (threadIdx.x < nb * kRowsPerCta) {
      const int i = static_cast<int>(threadIdx.x) / kRowsPerCta, t = static_cast<int>(threadIdx.x) % kRowsPerCta;
      const int b = cid + (i0 + i) * G;
      const StackJob& jb = stack_job_of(P, lv, b);
      const int row = (b - jb.block0) * kLutRowsPerCluster + static_cast<int>(rank) * kRowsPerCta + t;
      if (mbar_wait(smem_u32(inbox_bar), n & 1u, kWhereStackInbox)) {
        const float* in = inbox + i * kLutRowsPerCluster + t;
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < kStackCluster; ++q) s += in[q * kRowsPerCta];
        if (row < jb.N) {
          yp = jb.y + row;
          yv = float_to_bf16_bits(jb.alpha[row] * s);
        }
      }
    }
    __syncthreads();  // the inbox has been read
    cluster_arrive_release();
    if (yp) *yp = yv;  // after the arrive, so that it does not wait for these stores
    ++n;
  }

  // this CTA's outputs of level l are written: count it
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) red_release_gpu_add(P.done + l, 1u);
}

__global__ void __launch_bounds__(kLutThreads, 1) gemv_w1a16_stack_kernel(const __grid_constant__ StackParams P) {
  extern __shared__ __align__(1024) uint8_t lut_smem[];
  // [block of the pass][source rank][owned row]
  __shared__ float inbox[StackPass<1>::kBlocks * kLutRowsPerCluster];
  __shared__ __align__(8) uint64_t inbox_bar;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&inbox_bar), 1);
    fence_mbar_init();
  }
  // pairs with the wait before the first push: every inbox barrier is initialised
  cluster_arrive_release();

  uint32_t n = 0;
  bool waiting = true;
  for (int l = 0; l < P.num_levels; ++l) {
    const int slice_words = P.lv[l].K / (32 * kStackCluster);
    if (slice_words <= 16)
      stack_level<1>(P, l, rank, lut_smem, inbox, &inbox_bar, n, waiting);
    else if (slice_words <= 32)
      stack_level<2>(P, l, rank, lut_smem, inbox, &inbox_bar, n, waiting);
    else
      stack_level<3>(P, l, rank, lut_smem, inbox, &inbox_bar, n, waiting);
  }
  // pairs with the last arrive: no CTA leaves while a peer may still push to it
  cluster_wait_acquire();
}

}  // namespace bl

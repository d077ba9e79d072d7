// Single-token W1A16 decode through a stack of binarized linear layers in one
// persistent launch, with the packed weights streamed into shared memory ahead
// of the activations ("FBI-LLM" page, FBI-linear paragraph: every linear of the
// model is y_j = alpha_j * sum_k sign(W_jk) x_k; a decode step runs them one
// dependent level after another).
//
// The stack is a list of levels. A level has one input vector x (K) and one or
// more linears that read it (q, k, v of a block share one x; so do gate and
// up). Its x is either a buffer written before the launch or the output of one
// linear of an earlier level of the same launch.
//
// Work split. A grid of G clusters of 8 CTAs (one CTA per SM, all resident at
// once). The 8 CTAs of a cluster split K into slices exactly as the
// single-layer lookup-table kernel does (same windows, same table pages, same
// per-lane order of additions, same reduce-scatter, same rank-ordered owner
// sum), so every output is bit-identical to bin_linear_w1a16 wherever that
// call also splits K eight ways. A level's rows are cut into 16-row chunks
// (one per warp); cluster c takes the c-th of G equal runs of the level's
// chunks, processed as slabs of up to 16 chunks (256 rows) of one linear.
//
// Weights never wait for activations. Each CTA's sequence of 16 KB weight
// slots (for every level, slab and table page it will process, in processing
// order) is fetched by 2-D tensor copies (cp.async.bulk.tensor of 64-row
// boxes, no multicast) into a ring of kStrSlots slots, each completing on its
// own mbarrier. A producer warp issues the copies as soon as the 16 compute
// warps have released a slot (one arrival per warp on the slot's empty
// barrier), so while a level waits for its input, the weights of that level
// and of the next ones are already arriving, and the HBM stream runs ahead of
// the dependency chain.
//
// Activations carry their own ready flag. An output read by a later level of
// the same launch is also written as one 32-bit word per element, the bf16
// value in the low half and 1 in the high half, into a tagged buffer that the
// call zero-fills before the launch. A CTA that needs a slice of that vector
// polls those words (relaxed loads at GPU scope) until every high half is set;
// value and flag arrive in one single-copy-atomic store, so no fence or
// completion counter stands between a producer's store and a consumer's use.
// Levels with no blocks for a cluster are skipped by it without waiting.
// (Outputs and inputs never overlap otherwise: the call checks that every
// linear writes its own buffer and that an input read from outside the
// launch is written by none of its linears.)
//
// Table pages. One 64 KB page is resident. A level whose window spans several
// pages is processed in passes of up to kStrPass slabs; within a pass, page
// by page: build the page from the input slice held in shared memory, then
// the lookups of every slab of the pass on that page. Per-lane partial sums
// stay in registers across pages, so the additions happen in the single-layer
// kernel's order.
//
// Partial sums. After a pass, each row's slice partial goes to the row's
// owner in the cluster (st.async into inbox buffer n % 2 of pass n, counted
// on that buffer's inbox_full barrier). At the start of every pass each CTA
// also sends each peer (itself included) a 4-byte token on that barrier: it
// has read its inbox of the previous pass (a barrier of the compute warps
// ends every pass). No CTA can overwrite a buffer that is still being read:
// a CTA pushes pass n + 2 only after its own pass n + 1 inbox has filled,
// which takes every peer's pass n + 1 token, which a peer sends only once it
// has read its pass n inbox. (Without the tokens a CTA that owns no live row
// of a pass would expect no bytes and nothing would hold it back.)
//
// Waits on weight slots, on input flags and on the partial-sum inbox are
// bounded: past the limit the kernel records BL_ERR_TIMEOUT, sets the
// launch's abort word (so that waits for inputs elsewhere stop at once
// instead of each running out in turn) and carries on with undefined
// outputs; every CTA of a cluster still takes the same path through the
// cluster barriers, and before leaving, thread 0 waits (bounded) for every
// tensor copy it issued.
#pragma once

#include "bl_gemv_lut.cuh"

namespace bl {

constexpr int kStrCluster = 8;                           // CTAs per cluster = K slices
constexpr int kStrThreads = kLutThreads;                 // 16 compute warps x 16 rows = one slab
constexpr int kStrRows = kLutRowsPerCluster;             // 256 rows per slab at most
constexpr int kStrChunk = kLutRowsPerWarp;               // 16 rows: one warp's share of a slab
constexpr int kStrBoxRows = 64;                          // rows per tensor copy
constexpr int kStrSlotBytes = kStrRows * 16 * 4;         // 16 KB: 256 rows x one page of words
constexpr int kStrSlots = 8;                             // ring depth
constexpr int kStrPass = 4;                              // slabs per pass
constexpr int kStrMaxWindowWords = 64;                   // 48-word slice + offset, 4 pages
constexpr int kStrXBytes = kStrMaxWindowWords * 32 * 2;  // the slice's inputs (bf16): 4 KB
constexpr int kStrSmemBytes = kLutPageBytes + kStrSlots * kStrSlotBytes + kStrXBytes;  // 196 KB
constexpr int kStrMaxLevels = 96;                        // per launch (kernel parameter space)
constexpr int kStrMaxJobs = 144;                         // per launch
constexpr uint32_t kStrReady = 1u << 16;                 // high half of a published tagged word

struct alignas(16) StrJob {
  const float* alpha;  // [N]
  uint16_t* y;         // [N] bf16
  uint32_t* tagged;    // [N] tagged copy when a later level of the launch reads y, else null
  int N;
  int chunk0;          // first 16-row chunk of this linear within its level
};
struct alignas(16) StrLevel {
  const uint16_t* x;   // input written before the launch (bf16), or null
  const uint32_t* xt;  // tagged copy of an earlier linear's output, or null
  int K;               // multiple of 256, at most 12288
  int job0, njobs;     // jobs[job0 .. job0 + njobs)
  int nchunks;         // 16-row chunks of all its linears
};
struct StrParams {
  CUtensorMap maps[kStrMaxJobs];  // packed [N][K/32] uint32, box 16 words x 64 rows
  StrJob jobs[kStrMaxJobs];
  StrLevel lv[kStrMaxLevels];
  uint32_t* abort;                // zero at launch; set once any wait of the launch gave up
  int num_levels;
  int num_jobs;
};
static_assert(sizeof(StrJob) % 16 == 0 && sizeof(StrLevel) % 16 == 0, "copied to shared memory in 16-byte words");

__device__ __forceinline__ uint4 ld_relaxed_gpu_v4(const uint32_t* p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_gpu_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
template <int NTHREADS = kStrThreads>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NTHREADS) : "memory");
}

// this CTA's slice window of a level with K inputs
__device__ __forceinline__ LutWindow str_window(int K, uint32_t rank) {
  LutWindow w;
  w.sw = K / (32 * kStrCluster);
  w.s0 = static_cast<int>(rank) * w.sw;
  w.a0 = w.s0 & ~3;
  return w;
}
__device__ __forceinline__ int str_pages(const LutWindow& w) { return lut_window_pages(w.s0, w.sw); }

// A slab: up to 16 chunks of one linear, rows [row0, row0 + 16 nc); the
// linear's index and the chunk count share one word (registers are scarce).
struct StrSlab {
  int row0;
  int jnc;  // j << 8 | nc
  __device__ __forceinline__ int j() const { return jnc >> 8; }
  __device__ __forceinline__ int nc() const { return jnc & 0xFF; }
};
// Chunks [cur, end) of a level still to be cut into slabs; the linear that
// holds chunk cur is j, whose chunks are [jbeg, jend) (kept in registers so
// that cutting a slab costs no dependent shared-memory reads).
struct StrRun {
  int cur, end, j, jbeg, jend, jlast;
};
// the linear holding chunk run.cur, from linear run.j on
__device__ __forceinline__ void str_seek(const StrJob* jobs, const StrLevel& lv, StrRun& r) {
  while (r.cur >= r.jend && r.j < r.jlast) {
    ++r.j;
    r.jbeg = r.jend;
    r.jend = r.j < r.jlast ? jobs[r.j + 1].chunk0 : lv.nchunks;
  }
}
// cluster cid's run of chunks of level lv (empty when the level has fewer chunks than clusters)
__device__ __forceinline__ StrRun str_run(const StrJob* jobs, const StrLevel& lv, int cid, int G) {
  StrRun r;
  // nchunks < 2^27 and G <= 32: the products fit 32 bits
  r.cur = static_cast<int>((static_cast<uint32_t>(lv.nchunks) * static_cast<uint32_t>(cid)) / static_cast<uint32_t>(G));
  r.end = static_cast<int>((static_cast<uint32_t>(lv.nchunks) * static_cast<uint32_t>(cid + 1)) / static_cast<uint32_t>(G));
  r.j = lv.job0;
  r.jlast = lv.job0 + lv.njobs - 1;
  r.jbeg = 0;
  r.jend = r.j < r.jlast ? jobs[r.j + 1].chunk0 : lv.nchunks;
  if (r.cur < r.end) str_seek(jobs, lv, r);
  return r;
}
__device__ __forceinline__ bool str_next_slab(const StrJob* jobs, const StrLevel& lv, StrRun& run, StrSlab& sl) {
  if (run.cur >= run.end) return false;
  int e = run.cur + kStrRows / kStrChunk;
  e = e < run.end ? e : run.end;
  e = e < run.jend ? e : run.jend;
  sl.row0 = (run.cur - run.jbeg) * kStrChunk;
  sl.jnc = (run.j << 8) | (e - run.cur);
  run.cur = e;
  if (run.cur < run.end) str_seek(jobs, lv, run);
  return true;
}

// The weight stream of one CTA (run by one thread): for every level, pass of
// up to PASS slabs, table page and slab of the pass, in that order (the order
// the compute warps consume them), one slot of tensor copies into the ring,
// each slot reused once the compute warps have released it. Afterwards it
// waits (bounded) for the last use of every slot, so that no copy is in
// flight when the CTA exits.
template <int PASS, int SLOTS = kStrSlots>
__device__ __forceinline__ void str_produce(const StrParams& P, const StrLevel* lvs, const StrJob* jobs,
                                            int num_levels, int cid, int G, uint32_t rank, uint8_t* ring,
                                            uint64_t* full, uint64_t* empty) {
  uint32_t issued = 0;
  bool live = true;
  for (int l = 0; l < num_levels; ++l) {
    const StrLevel& lv = lvs[l];
    StrRun run = str_run(jobs, lv, cid, G);
    if (run.cur >= run.end) continue;
    const LutWindow win = str_window(lv.K, rank);
    const int np = str_pages(win);
    while (true) {
      StrSlab sl[PASS];
      int npass = 0;
      while (npass < PASS && str_next_slab(jobs, lv, run, sl[npass])) ++npass;
      if (npass == 0) break;
      for (int pg = 0; pg < np; ++pg) {
        for (int i = 0; i < npass; ++i) {
          const uint32_t slot = issued % SLOTS;
          if (issued >= static_cast<uint32_t>(SLOTS) && live &&
              !mbar_wait(smem_u32(&empty[slot]), ((issued / SLOTS) - 1) & 1u, kWhereStackRing)) {
            st_relaxed_gpu_u32(P.abort, 1u);
            live = false;  // stop waiting; the outputs are undefined from here on
          }
          const uint32_t bar = smem_u32(&full[slot]);
          const int boxes = (sl[i].nc() * kStrChunk + kStrBoxRows - 1) / kStrBoxRows;
          mbar_arrive_expect_tx(bar, static_cast<uint32_t>(boxes) * kStrBoxRows * 16 * 4);
          // x: window word (a multiple of 4 words = 16 bytes); y: row
          for (int bx = 0; bx < boxes; ++bx)
            tma_load_2d(smem_u32(ring + slot * kStrSlotBytes + bx * kStrBoxRows * 16 * 4), &P.maps[sl[i].j()], bar,
                        win.a0 + 16 * pg, sl[i].row0 + bx * kStrBoxRows);
          ++issued;
        }
      }
    }
  }
  const uint32_t first = issued > static_cast<uint32_t>(SLOTS) ? issued - SLOTS : 0u;
  for (uint32_t k = first; k < issued; ++k)
    if (!mbar_wait(smem_u32(&full[k % SLOTS]), (k / SLOTS) & 1u, kWhereStackRing)) break;
}

// Warps 0..15 compute (kStrThreads threads); warp 16 streams the weights.
// (17 warps: one SM sub-partition hosts 5 of them, which caps registers at 96.)
__global__ void __launch_bounds__(kStrThreads + 32, 1) gemv_w1a16_stream_kernel(const __grid_constant__ StrParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* table = smem;                                // one 64 KB page
  uint8_t* ring = smem + kLutPageBytes;                 // kStrSlots x 16 KB
  uint16_t* xs = reinterpret_cast<uint16_t*>(ring + kStrSlots * kStrSlotBytes);  // window inputs
  __shared__ float inbox[2][kStrPass * kStrRows];       // [pass % 2][slab of the pass][source rank][owned row]
  static_assert(kStrThreads >= kStrPass * kStrRows / kStrCluster, "one owner thread per owned row of a pass");
  __shared__ __align__(8) uint64_t inbox_full[2];       // a pass's partials and tokens have all landed (bytes)
  __shared__ float tokens[2][kStrCluster];              // [pass % 2][source rank]
  __shared__ __align__(8) uint64_t full[kStrSlots];     // a slot's tensor copies have landed
  __shared__ __align__(8) uint64_t empty[kStrSlots];    // every compute warp is done with a slot
  // the level and linear descriptors, read many times: kept in shared memory
  // (dynamically indexed kernel parameters go through the small constant cache)
  __shared__ StrLevel lvs[kStrMaxLevels];
  __shared__ StrJob jobs[kStrMaxJobs];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = lane >> 4, wl = lane & 15;
  const uint32_t rank = cluster_ctarank();
  const int G = static_cast<int>(gridDim.y), cid = static_cast<int>(blockIdx.y);
  constexpr int kOwned = kStrRows / kStrCluster;  // 32 rows of a slab per owner (two warps' chunks)
  constexpr int kWarps = kStrThreads / 32;

  for (int i = tid; i < P.num_levels * static_cast<int>(sizeof(StrLevel) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(lvs)[i] = reinterpret_cast<const uint4*>(P.lv)[i];
  for (int i = tid; i < P.num_jobs * static_cast<int>(sizeof(StrJob) / 16); i += blockDim.x)
    reinterpret_cast<uint4*>(jobs)[i] = reinterpret_cast<const uint4*>(P.jobs)[i];
  if (tid == 0) {
    mbar_init(smem_u32(&inbox_full[0]), 1);
    mbar_init(smem_u32(&inbox_full[1]), 1);
    for (int s = 0; s < kStrSlots; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), kWarps);
    }
    fence_mbar_init();
  }
  // every barrier of the cluster is initialised (and the descriptors copied)
  // before anyone uses one
  cluster_arrive_release();
  cluster_wait_acquire();
  const int num_levels = P.num_levels;

  if (warp == kWarps) {
    // ---- the weight stream (one thread): slots in processing order ----
    if (lane == 0) str_produce<kStrPass>(P, lvs, jobs, num_levels, cid, G, rank, ring, full, empty);
    __syncwarp();
  } else {
    uint32_t q = 0;  // slots consumed
    uint32_t n = 0;  // passes finished (inbox phase)
    bool ok = true;  // false once a bounded wait gave up
    for (int l = 0; l < num_levels; ++l) {
      const StrLevel& lv = lvs[l];
      StrRun run = str_run(jobs, lv, cid, G);
      if (run.cur >= run.end) continue;
      const LutWindow win = str_window(lv.K, rank);
      const int np = str_pages(win);

      // ---- this slice's inputs into shared memory (xs[k - 32 a0]) ----
      // (the barrier that ended the previous level's last pass also ended its
      // table builds, the last readers of xs)
      {
        const int e0 = win.s0 * 32, ne = win.sw * 32;   // elements of the slice
        uint16_t* dst = xs + (win.s0 - win.a0) * 32;
        if (lv.xt) {
          for (int v = tid; v < ne / 4; v += kStrThreads) {
            const uint32_t* src = lv.xt + e0 + 4 * v;
            uint4 t = ld_relaxed_gpu_v4(src);
            if (!((t.x & t.y & t.z & t.w) & kStrReady) && ok) {
              const uint64_t t0 = global_timer_ns();
              do {
                t = ld_relaxed_gpu_v4(src);
                if ((t.x & t.y & t.z & t.w) & kStrReady) break;
                // a wait elsewhere gave up: this input may never come
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
            uint2 packed2;
            packed2.x = (t.x & 0xFFFFu) | (t.y << 16);
            packed2.y = (t.z & 0xFFFFu) | (t.w << 16);
            *reinterpret_cast<uint2*>(dst + 4 * v) = packed2;
          }
        } else {
          for (int v = tid; v < ne / 8; v += kStrThreads)
            *reinterpret_cast<uint4*>(dst + 8 * v) = *reinterpret_cast<const uint4*>(lv.x + e0 + 8 * v);
        }
      }
      consumers_sync();

      bool first_pass = true;
      while (true) {
        StrSlab sl[kStrPass];
        int npass = 0;
#pragma unroll
        for (int i = 0; i < kStrPass; ++i)
          if (npass == i && str_next_slab(jobs, lv, run, sl[i])) ++npass;
        if (npass == 0) break;
        // bytes this CTA will receive: 8 ranks x 4 bytes per owned live row,
        // and one 4-byte token from each rank
        if (tid == 0) {
          uint32_t rows = 0;
          for (int i = 0; i < npass; ++i) {
            const int r = sl[i].nc() * kStrChunk - static_cast<int>(rank) * kOwned;
            rows += r <= 0 ? 0u : (r >= kOwned ? static_cast<uint32_t>(kOwned) : static_cast<uint32_t>(r));
          }
          mbar_arrive_expect_tx(smem_u32(&inbox_full[n & 1u]), (rows + 1) * kStrCluster * 4);
        }
        // this pass's token to every rank: "done reading my pass n - 1 inbox"
        // (true since the barrier that ended that pass), sent first so that it
        // never holds up an inbox
        if (warp == 0 && lane < kStrCluster) {
          const uint32_t dst = static_cast<uint32_t>(lane);
          st_async_f32(map_to_rank(smem_u32(&tokens[n & 1u][rank]), dst), 0.f,
                       map_to_rank(smem_u32(&inbox_full[n & 1u]), dst));
        }
        // owners: thread t will add the 8 partials of row t % 32 of slab t / 32;
        // its scale is read now, off the critical path
        const StrJob* ojb = nullptr;
        int orow = 0;
        float oalpha = 0.f;
        if (tid < npass * kOwned) {
          int i = tid / kOwned;
          StrSlab o = sl[0];
#pragma unroll
          for (int k = 1; k < kStrPass; ++k)
            if (i == k) o = sl[k];
          const int r = static_cast<int>(rank) * kOwned + tid % kOwned;  // row within the slab
          if (r < o.nc() * kStrChunk) {
            ojb = &jobs[o.j()];
            orow = o.row0 + r;
            if (orow < ojb->N) oalpha = ojb->alpha[orow];
          }
        }
        float acc[kStrPass][kLutPairs];
#pragma unroll
        for (int i = 0; i < kStrPass; ++i)
#pragma unroll
          for (int p = 0; p < kLutPairs; ++p) acc[i][p] = 0.f;

        for (int pg = 0; pg < np; ++pg) {
          // a one-page window keeps its table for every pass of the level
          if (np > 1 || first_pass) {
            if (pg > 0 || !first_pass) consumers_sync();  // every warp is done with the previous page
            lut_build_page<false>(xs, pg, win, table, tid, kStrThreads);
            consumers_sync();
          }
          // every slot of this page phase has landed (then the lookups of all
          // slabs can be scheduled together)
#pragma unroll
          for (int i = 0; i < kStrPass; ++i) {
            if (i < npass) {
              const uint32_t qq = q + static_cast<uint32_t>(i);
              if (ok && !mbar_wait(smem_u32(&full[qq % kStrSlots]), (qq / kStrSlots) & 1u, kWhereStackRing)) {
                st_relaxed_gpu_u32(P.abort, 1u);
                ok = false;
              }
            }
          }
          const int wi = pg * 16 + wl;
          const bool live = wi >= win.lo() && wi < win.hi();
#pragma unroll
          for (int i = 0; i < kStrPass; ++i) {
            if (i < npass && warp < sl[i].nc()) {  // warps past the slab's chunks have nothing to add
              const uint32_t slot = (q + static_cast<uint32_t>(i)) % kStrSlots;
              const uint32_t* sw = reinterpret_cast<const uint32_t*>(ring + slot * kStrSlotBytes);
              uint32_t wv[kLutPairs];
#pragma unroll
              for (int p = 0; p < kLutPairs; ++p) wv[p] = sw[(warp * kStrChunk + 2 * p + h) * 16 + wl];
              lut_page_acc(wv, live, table, h, wl, acc[i]);
            }
          }
          // this warp is done with the phase's slots
          __syncwarp();
          if (lane == 0)
            for (int i = 0; i < npass; ++i) mbar_arrive(smem_u32(&empty[(q + static_cast<uint32_t>(i)) % kStrSlots]));
          q += static_cast<uint32_t>(npass);
        }
        first_pass = false;

        // (unused slabs reduce zeros: no branch keeps the four chains apart)
        float part[kStrPass];
#pragma unroll
        for (int i = 0; i < kStrPass; ++i) part[i] = lut_reduce_scatter(acc[i], wl);

        if ((wl & 1) == 0) {
          // lane's row within a slab, owned by rank r / 32 = warp / 2
          const int r = warp * kStrChunk + 2 * (wl >> 1) + h;
          const uint32_t owner = static_cast<uint32_t>(warp >> 1);
          const uint32_t slot = smem_u32(&inbox[n & 1u][static_cast<int>(rank) * kOwned + (r & (kOwned - 1))]);
          const uint32_t rslot = map_to_rank(slot, owner);
          const uint32_t rbar = map_to_rank(smem_u32(&inbox_full[n & 1u]), owner);
#pragma unroll
          for (int i = 0; i < kStrPass; ++i)
            if (i < npass && warp < sl[i].nc()) st_async_f32(rslot + i * kStrRows * 4, part[i], rbar);
        }
        uint16_t* yp = nullptr;
        uint32_t* tp = nullptr;
        uint16_t yv = 0;
        if (tid < npass * kOwned) {
          bool got = false;
          if (ok) {
            got = mbar_wait(smem_u32(&inbox_full[n & 1u]), (n >> 1) & 1u, kWhereStackInbox);
            if (!got) {
              st_relaxed_gpu_u32(P.abort, 1u);
              ok = false;
            }
          }
          if (got && ojb) {
            const float* in = inbox[n & 1u] + (tid / kOwned) * kStrRows + tid % kOwned;
            float sum = 0.f;
#pragma unroll
            for (int r = 0; r < kStrCluster; ++r) sum += in[r * kOwned];
            if (orow < ojb->N) {
              yp = ojb->y + orow;
              yv = float_to_bf16_bits(oalpha * sum);
              if (ojb->tagged) tp = ojb->tagged + orow;
            }
          }
        }
        if (tp) st_relaxed_gpu_u32(tp, kStrReady | yv);  // publish first: a later level may wait for it
        if (yp) *yp = yv;
        // the owners have read this pass's inbox before any warp pushes the next pass
        consumers_sync();
        ++n;
      }
    }
  }
  // no CTA leaves while a peer may still push to it or arrive on its barriers
  cluster_arrive_release();
  cluster_wait_acquire();
}

}  // namespace bl

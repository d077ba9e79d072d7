// libbitlinear.so: the C ABI declared in include/bitlinear.h.
//
// Host side only: argument validation, per-device one-time set-up, TMA
// descriptor encoding and kernel dispatch. All kernels live in the headers
// included below, so the library is one translation unit (no relocatable
// device code). Nothing here allocates memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "bitlinear.h"
#include "bl_backward.cuh"
#include "bl_common.cuh"
#include "bl_gemm_ts.cuh"
#include "bl_gemv.cuh"
#include "bl_gemv_lut.cuh"
#include "bl_gemv_mma.cuh"
#include "bl_gemv_stream.cuh"
#include "bl_gemv_stream_mma.cuh"
#include "bl_gemv_w1a8_mma.cuh"
#include "bl_lnquant.cuh"
#include "bl_pack.cuh"
#include "bl_xnor.cuh"

namespace bl {
namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxProduct = int64_t(1) << 40;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- per-device set-up ------------------------------------------------------
struct DeviceState {
  std::once_flag once;
  int status = BL_ERR_NO_DEVICE;
  int num_sms = 0;
  // how many clusters of 2 / 4 / 8 tensor-core GEMM CTAs (one CTA per SM)
  // can be resident at once: clusters must fit inside a GPC, so this is
  // below num_sms / S (on B200: 74 / 33 / 15)
  int cluster_cap[9] = {};
  // clusters of 8 layer-stack decode CTAs that can be resident at once
  // (single token; 8 and 16 token tiles)
  int stack_clusters = 0;
  int stack_mma_clusters[2] = {0, 0};
};
DeviceState g_devices[kMaxDevices];

template <typename Kernel>
bool set_smem(Kernel k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// every tensor-core GEMM configuration the dispatch below can launch
template <int KIND, int T>
bool set_ts_smem_t() {
  return set_smem(gemm_ts_kernel<KIND, 1, T, false>, TsCfg<KIND, 1, T, false>::SMEM_BYTES) &&
         set_smem(gemm_ts_kernel<KIND, 1, T, true>, TsCfg<KIND, 1, T, true>::SMEM_BYTES);
}
template <int KIND>
bool set_ts_smem() {
  return set_smem(gemm_ts_kernel<KIND, 1, 256, false>, TsCfg<KIND, 1, 256, false>::SMEM_BYTES) &&
         set_ts_smem_t<KIND, 128>() && set_ts_smem_t<KIND, 64>() && set_ts_smem_t<KIND, 32>();
}

int device_setup(int* num_sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return BL_ERR_NO_DEVICE;
  }
  DeviceState& st = g_devices[dev];
  std::call_once(st.once, [&st, dev] {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) {
      cudaGetLastError();
      st.status = BL_ERR_NO_DEVICE;
      return;
    }
    st.num_sms = prop.multiProcessorCount;
    bool ok = set_smem(gemv_w1a16_kernel<1>, gemv_smem_bytes(1)) &&
              set_smem(gemv_w1a16_kernel<2>, gemv_smem_bytes(2)) &&
              set_smem(gemv_w1a16_kernel<4>, gemv_smem_bytes(4)) &&
              set_smem(gemv_w1a16_lut_kernel<1>, 1 * kLutPageBytes) &&
              set_smem(gemv_w1a16_lut_kernel<2>, 2 * kLutPageBytes) &&
              set_smem(gemv_w1a16_lut_kernel<3>, 3 * kLutPageBytes) &&
              set_ts_smem<0>() && set_ts_smem<1>() && set_ts_smem<2>() &&
              set_smem(gemv_w1a16_stream_kernel, kStrSmemBytes) &&
              set_smem(gemv_w1a16_stream_mma_kernel<8>, SmCfg<8>::kSmemBytes) &&
              set_smem(gemv_w1a16_stream_mma_kernel<16>, SmCfg<16>::kSmemBytes) &&
              set_smem(gemm_ss_ste_kernel, kSsSmemBytes) &&
              set_smem(transpose_pack_dup_kernel, kTpSmemBytes) &&
              set_smem(gemv_w1a8_mma_kernel<8, false>, qm_smem_bytes(8, kQmMaxSliceWords, false)) &&
              set_smem(gemv_w1a8_mma_kernel<16, false>, qm_smem_bytes(16, kQmMaxSliceWords, false)) &&
              set_smem(gemv_w1a8_mma_kernel<8, true>, qm_smem_bytes(8, kQmMaxSliceWords, true)) &&
              set_smem(gemv_w1a8_mma_kernel<16, true>, qm_smem_bytes(16, kQmMaxSliceWords, true)) &&
              set_smem(gemv_w1a16_mma_kernel<8, 16>, mma_smem_bytes(8, 16)) &&
              set_smem(gemv_w1a16_mma_kernel<16, 16>, mma_smem_bytes(16, 16)) &&
              set_smem(gemv_w1a16_mma_kernel<8, kMmaMaxSliceWords>, mma_smem_bytes(8, kMmaMaxSliceWords)) &&
              set_smem(gemv_w1a16_mma_kernel<16, kMmaMaxSliceWords>, mma_smem_bytes(16, kMmaMaxSliceWords));
    if (!ok) cudaGetLastError();
    {
      // how many clusters of 8 of a stack kernel can be resident at once
      auto stack_capacity = [](auto kernel, int threads, int smem) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kStrCluster, 1, 1);
        cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kStrCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
          cudaGetLastError();
          n = 0;  // the stacked decode then reports BL_ERR_CUDA
        }
        return n;
      };
      st.stack_clusters = stack_capacity(gemv_w1a16_stream_kernel, kStrThreads + 32, kStrSmemBytes);
      st.stack_mma_clusters[0] = stack_capacity(gemv_w1a16_stream_mma_kernel<8>, kSmThreads + 32, SmCfg<8>::kSmemBytes);
      st.stack_mma_clusters[1] = stack_capacity(gemv_w1a16_stream_mma_kernel<16>, kSmThreads + 32, SmCfg<16>::kSmemBytes);
    }
    for (int S : {2, 4, 8}) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(S), 1, 1);
      cfg.blockDim = dim3(kTsThreads, 1, 1);
      cfg.dynamicSmemBytes = TsCfg<0, 1, 128, true>::SMEM_BYTES;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(S);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, gemm_ts_kernel<0, 1, 128, true>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = st.num_sms / (2 * S);  // conservative: half of the SMs
      }
      st.cluster_cap[S] = n;
    }
    st.status = ok ? BL_OK : BL_ERR_CUDA;
  });
  if (num_sms) *num_sms = st.num_sms;
  return st.status;
}

// resident clusters of the stack kernel for M tokens (1, <= 8, <= 16)
int stack_cluster_capacity(int64_t M = 1) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  const DeviceState& st = g_devices[dev];
  return M <= 1 ? st.stack_clusters : st.stack_mma_clusters[M <= 8 ? 0 : 1];
}

// co-resident cluster capacity of the current device for clusters of S GEMM CTAs
int cluster_capacity(int S) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 0;
  }
  return g_devices[dev].cluster_cap[S];
}

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

// ---- TMA descriptors ----------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `dtype`, box [box_rows][box_cols].
bool make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                 uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                 CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (K % 128 != 0) return BL_ERR_UNSUPPORTED;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return BL_ERR_UNSUPPORTED;
  if (M * K >= kMaxProduct || N * K >= kMaxProduct || M * N >= kMaxProduct) return BL_ERR_UNSUPPORTED;
  return BL_OK;
}

// ---- few-token warp-MMA GEMV (2 <= M <= 16, K % 256 == 0, K <= 12288) ---------------
template <int MT, int SWMAX>
cudaError_t launch_mma_t(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y, int M,
                         int N, int K, bool overlap, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kMmaCluster, static_cast<unsigned>(cdiv(N, kMmaRowsPerCluster)), 1);
  cfg.blockDim = dim3(kMmaThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(mma_smem_bytes(MT, K / 256));
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = kMmaCluster;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = overlap ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemv_w1a16_mma_kernel<MT, SWMAX>, x, packed, alpha, y, M, N, K);
}
cudaError_t launch_mma(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y, int M, int N,
                       int K, bool overlap, cudaStream_t s) {
  const bool small_k = K / 256 <= 16;
  if (M <= 8)
    return small_k ? launch_mma_t<8, 16>(x, packed, alpha, y, M, N, K, overlap, s)
                   : launch_mma_t<8, kMmaMaxSliceWords>(x, packed, alpha, y, M, N, K, overlap, s);
  return small_k ? launch_mma_t<16, 16>(x, packed, alpha, y, M, N, K, overlap, s)
                 : launch_mma_t<16, kMmaMaxSliceWords>(x, packed, alpha, y, M, N, K, overlap, s);
}

// ---- single-token lookup-table GEMV ------------------------------------------------
template <int NP>
cudaError_t launch_lut(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y,
                       int N, int K, int C, int slice_words, bool overlap, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(C), static_cast<unsigned>(cdiv(N, kLutRowsPerCluster)), 1);
  cfg.blockDim = dim3(kLutThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(NP) * kLutPageBytes;
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = static_cast<unsigned>(C);
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = overlap ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemv_w1a16_lut_kernel<NP>, x, packed, alpha, y, N, K, slice_words);
}

// ---- tensor-core GEMM with the signs in tensor memory ------------------------------
// activations [M][K] (bf16 for KIND 0, int8 codes for KIND 1) x packed signs [N][K/32]
// Split factor for a problem of `tiles` output tiles and `num_kb` k-blocks:
// the largest S in {8, 4, 2} (S divides the 128 rows of a tile) whose
// `tiles` clusters of S CTAs are all resident at once (one wave) and that
// leaves every CTA at least one k-block. Returns 1 when the persistent
// (unsplit) kernel should be used.
int split_factor(int64_t tiles, int num_kb, int num_sms) {
  for (int S : {8, 4, 2}) {
    if (tiles * S > num_sms || tiles > cluster_capacity(S) || S > num_kb) continue;
    if (((num_kb + S - 1) / S) * (S - 1) >= num_kb) continue;
    return S;
  }
  return 1;
}

template <int KIND, int NB, int T, bool SPLIT>
int launch_ts_cfg(const CUtensorMap& tm_x, const CUtensorMap& tm_bits, int64_t M, int64_t N, int64_t K,
                  int S, const float* alpha, const double* gamma, const float* beta, void* y,
                  int32_t* acc_out, int num_sms, cudaStream_t s) {
  using C = TsCfg<KIND, NB, T, SPLIT>;
  const int64_t tiles = cdiv(M, T) * cdiv(N, C::ROWS);
  CUtensorMap tm_y;
  std::memset(&tm_y, 0, sizeof tm_y);
  if (SPLIT) {
    // a cluster of S CTAs per tile, each with a slice of the k-blocks
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(S), static_cast<unsigned>(tiles), 1);
    cfg.blockDim = dim3(kTsThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_ts_kernel<KIND, NB, T, SPLIT>, tm_x, tm_bits, tm_y, 0,
                                             int(M), int(N), int(K), alpha, gamma, beta, y, acc_out);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return launch_status();
  }
  // persistent: output tile written by bulk tensor stores when the row pitch allows it
  const int use_tma_store =
      C::STAGE_OUT && (N * C::OUT_ELEM) % 16 == 0 &&
      make_map_2d(&tm_y, y, KIND == 0 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  C::OUT_ELEM, uint64_t(N), uint64_t(M), C::STAGE_COLS, T, CU_TENSOR_MAP_SWIZZLE_NONE);
  const unsigned grid = static_cast<unsigned>(tiles < num_sms ? tiles : num_sms);
  gemm_ts_kernel<KIND, NB, T, SPLIT><<<grid, kTsThreads, C::SMEM_BYTES, s>>>(
      tm_x, tm_bits, tm_y, use_tma_store, int(M), int(N), int(K), alpha, gamma, beta, y, acc_out);
  return launch_status();
}

// activations [M][K] (bf16 for KIND 0, int8 codes for KIND 1) x packed signs [N][K/32].
// Tiles of 128 weight rows. Problems with M >= 256 whose 128-row x 256-token
// tiles occupy at least half of the SMs use those (one 128x256 MMA per
// k-step, the most tensor work per instruction). Otherwise tiles of 32, 64 or 128 tokens
// (the smallest that covers M, up to 128), split over a cluster along K when
// the tiles alone would leave SMs idle. (Chosen from timings of every
// configuration on the decode-batch, 1.3B and 7B shapes: 128-row tiles beat
// 256-row ones, and split-K pays whenever it raises the CTA count.)
template <int KIND, int T>
int launch_ts_t(const CUtensorMap& tm_x, const CUtensorMap& tm_bits, int64_t M, int64_t N, int64_t K,
                const float* alpha, const double* gamma, const float* beta, void* y, int32_t* acc_out,
                int num_sms, cudaStream_t s) {
  const int64_t tiles = cdiv(M, T) * cdiv(N, 128);
  const int S = split_factor(tiles, int(K / kTsStageK), num_sms);
  return S > 1 ? launch_ts_cfg<KIND, 1, T, true>(tm_x, tm_bits, M, N, K, S, alpha, gamma, beta, y, acc_out, num_sms, s)
               : launch_ts_cfg<KIND, 1, T, false>(tm_x, tm_bits, M, N, K, 1, alpha, gamma, beta, y, acc_out, num_sms, s);
}

template <int KIND>
int launch_ts(const void* act, const uint32_t* packed, int64_t M, int64_t N, int64_t K,
              const float* alpha, const double* gamma, const float* beta, void* y, int32_t* acc_out,
              int num_sms, cudaStream_t s) {
  const int elem = KIND == 0 ? 2 : 1;
  const CUtensorMapDataType xt = KIND == 0 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int64_t big_tiles = cdiv(M, 256) * cdiv(N, 128);
  const int T = (M >= 256 && 2 * big_tiles >= int64_t(num_sms)) ? 256 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
  CUtensorMap tm_x, tm_bits;
  if (!make_map_2d(&tm_x, act, xt, elem, uint64_t(K), uint64_t(M), 128 / elem, uint32_t(T), CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tm_bits, packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(K / 32) * TsCfg<KIND, 1, 32, false>::PLANES,
                   uint64_t(N), 4 * TsCfg<KIND, 1, 32, false>::PLANES, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return BL_ERR_CUDA;
  switch (T) {
    case 256:
      return launch_ts_cfg<KIND, 1, 256, false>(tm_x, tm_bits, M, N, K, 1, alpha, gamma, beta, y, acc_out, num_sms, s);
    case 128:
      return launch_ts_t<KIND, 128>(tm_x, tm_bits, M, N, K, alpha, gamma, beta, y, acc_out, num_sms, s);
    case 64:
      return launch_ts_t<KIND, 64>(tm_x, tm_bits, M, N, K, alpha, gamma, beta, y, acc_out, num_sms, s);
    default:
      return launch_ts_t<KIND, 32>(tm_x, tm_bits, M, N, K, alpha, gamma, beta, y, acc_out, num_sms, s);
  }
}

// ---- W1A8 shared body -----------------------------------------------------------
// `ternary`: packed holds b1.58 weights (two planes, K/16 words per row).
// `quant`: 0 per-token gamma; BL_W1A8_PER_TENSOR: Eq.(5) over the matrix;
// BL_W1A8_NONNEG: Eq.(6) (per tensor). The per-tensor forms need the larger
// workspace of BL_OP_W1A8_EX.
int w1a8_impl(const uint16_t* x, const uint32_t* packed, const float* beta, float* y, int64_t M,
              int64_t N, int64_t K, void* ws, size_t ws_bytes, int8_t* xq_out, double* gamma_out,
              int32_t* acc_out, const int8_t* xq_in, const double* gamma_in, bool ternary, void* stream,
              unsigned quant = 0u) {
  int rc = check_shape(M, N, K);
  if (rc != BL_OK) return rc;
  if (M == 0) return BL_OK;
  if (!packed || !beta || !y || !aligned16(packed) || !aligned16(y)) return BL_ERR_INVALID_ARG;
  if (xq_in) {
    if (!gamma_in || !aligned16(xq_in)) return BL_ERR_INVALID_ARG;
  } else {
    if (!x || !aligned16(x)) return BL_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws) ||
        ws_bytes < bl_workspace_bytes(quant ? BL_OP_W1A8_EX : BL_OP_W1A8, M, N, K))
      return BL_ERR_INVALID_ARG;
  }
  rc = device_setup(nullptr);
  if (rc != BL_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // short problems: LN, quantisation, products and rescale in one launch
  if (!quant && !xq_in && M <= 16 && K <= kW1a8SmallMaxK && M * K <= kW1a8SmallMaxCodes &&
      (!xq_out || aligned16(xq_out))) {
    const unsigned grid = static_cast<unsigned>(cdiv(N, kGemvRowsPerCta));
    const int m = int(M);
    if (ternary) {
      if (M <= 4)
        bitlinear_small_kernel<4, true><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
      else if (M <= 8)
        bitlinear_small_kernel<8, true><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
      else
        bitlinear_small_kernel<16, true><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
    } else {
      if (M <= 4)
        bitlinear_small_kernel<4, false><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
      else if (M <= 8)
        bitlinear_small_kernel<8, false><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
      else
        bitlinear_small_kernel<16, false><<<grid, kGemvThreads, 0, s>>>(x, packed, beta, y, xq_out, gamma_out, acc_out, m, N, K);
    }
    return launch_status();
  }

  const int8_t* codes = xq_in;
  const double* gam = gamma_in;
  if (!xq_in) {
    int8_t* xq_ws = static_cast<int8_t*>(ws);
    double* g_ws = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + align256(size_t(M * K)));
    if (!quant) {
      const int64_t nv = cdiv(K / 8, kLnThreads);  // 16-byte vectors per thread
      if (nv <= 1)
        ln_quant_kernel<1><<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, xq_ws, g_ws);
      else if (nv <= 2)
        ln_quant_kernel<2><<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, xq_ws, g_ws);
      else if (nv <= 4)
        ln_quant_kernel<4><<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, xq_ws, g_ws);
      else
        ln_quant_kernel<0><<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, xq_ws, g_ws);
      if ((rc = launch_status()) != BL_OK) return rc;
    } else {
      const bool nonneg = (quant & BL_W1A8_NONNEG) != 0;
      auto* stats = reinterpret_cast<LnTokenStats*>(reinterpret_cast<uint8_t*>(g_ws) +
                                                    align256(size_t(M) * sizeof(double)));
      auto* scalars = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(stats) +
                                                align256(size_t(M) * sizeof(LnTokenStats)));
      ln_stats_kernel<<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, stats);
      if ((rc = launch_status()) != BL_OK) return rc;
      ln_tensor_scalars_kernel<<<1, kLnThreads, 0, s>>>(stats, M, nonneg, g_ws, scalars);
      if ((rc = launch_status()) != BL_OK) return rc;
      ln_quant_tensor_kernel<<<static_cast<unsigned>(M), kLnThreads, 0, s>>>(x, M, K, nonneg, stats, scalars, xq_ws);
      if ((rc = launch_status()) != BL_OK) return rc;
    }
    codes = xq_ws;
    gam = g_ws;
  }
  if (xq_out && cudaMemcpyAsync(xq_out, codes, size_t(M * K), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return BL_ERR_CUDA;
  if (gamma_out &&
      cudaMemcpyAsync(gamma_out, gam, size_t(M) * sizeof(double), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return BL_ERR_CUDA;

  if (M <= 16 && K % 256 == 0 && K / 256 <= kQmMaxSliceWords) {
    // warp-level int8 MMA GEMV, a cluster of 8 CTAs per 64 rows; launched with
    // programmatic serialisation (its weight copies start while the LN kernel
    // runs; it waits for the codes before reading them)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMmaCluster, static_cast<unsigned>(cdiv(N, kQmRows)), 1);
    cfg.blockDim = dim3(kQmThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(qm_smem_bytes(M <= 8 ? 8 : 16, int(K / 256), ternary));
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kMmaCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const int m = int(M), n = int(N), k = int(K);
    cudaError_t e;
    if (ternary)
      e = M <= 8 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_mma_kernel<8, true>, codes, gam, packed, beta, y, acc_out, m, n, k)
                 : cudaLaunchKernelEx(&cfg, gemv_w1a8_mma_kernel<16, true>, codes, gam, packed, beta, y, acc_out, m, n, k);
    else
      e = M <= 8 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_mma_kernel<8, false>, codes, gam, packed, beta, y, acc_out, m, n, k)
                 : cudaLaunchKernelEx(&cfg, gemv_w1a8_mma_kernel<16, false>, codes, gam, packed, beta, y, acc_out, m, n, k);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return launch_status();
  }
  if (M <= 16) {
    // dp4a GEMV (K outside the MMA kernel's range), launched with programmatic
    // serialisation: scheduled while the LN kernel runs, it waits for that
    // kernel's codes before reading them
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cdiv(N, kGemvRowsPerCta)), 1, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int m = int(M);
    cudaError_t e;
    if (ternary)
      e = M <= 4 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<4, true>, codes, gam, packed, beta, y, acc_out, m, N, K)
        : M <= 8 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<8, true>, codes, gam, packed, beta, y, acc_out, m, N, K)
                 : cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<16, true>, codes, gam, packed, beta, y, acc_out, m, N, K);
    else
      e = M <= 4 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<4, false>, codes, gam, packed, beta, y, acc_out, m, N, K)
        : M <= 8 ? cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<8, false>, codes, gam, packed, beta, y, acc_out, m, N, K)
                 : cudaLaunchKernelEx(&cfg, gemv_w1a8_kernel<16, false>, codes, gam, packed, beta, y, acc_out, m, N, K);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return launch_status();
  }
  int sms = 0;
  device_setup(&sms);
  return ternary ? launch_ts<2>(codes, packed, M, N, K, nullptr, gam, beta, y, acc_out, sms, s)
                 : launch_ts<1>(codes, packed, M, N, K, nullptr, gam, beta, y, acc_out, sms, s);
}

}  // namespace
}  // namespace bl

using namespace bl;

extern "C" {

int bl_abi_version(void) { return 1; }

const char* bl_status_string(int status) {
  switch (status) {
    case BL_OK: return "ok";
    case BL_ERR_INVALID_ARG: return "invalid argument (null, negative size, misaligned or short workspace)";
    case BL_ERR_UNSUPPORTED: return "unsupported shape (K must be a positive multiple of 128; sizes below 2^31, products below 2^40)";
    case BL_ERR_CUDA: return "CUDA runtime or launch error";
    case BL_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case BL_ERR_NO_DEVICE: return "no usable sm_100 device is current";
    case BL_ERR_SCRATCH_LIMIT:
      return "problem exceeds the fixed scratch of bitlinear_w1a8_noalloc "
             "(bl_workspace_bytes(BL_OP_W1A8, M, N, K) must be at most 4 MiB)";
    default: return "unknown status";
  }
}

size_t bl_workspace_bytes(int op, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  switch (op) {
    case BL_OP_PACK_BITNET:
    case BL_OP_PACK_TERNARY: return align256(size_t(N) * 2 * sizeof(double)) + 256;
    case BL_OP_W1A8:
    case BL_OP_W158A8: return align256(size_t(M * K)) + align256(size_t(M) * sizeof(double));
    case BL_OP_W1A8_EX:
      return align256(size_t(M * K)) + align256(size_t(M) * sizeof(double)) +
             align256(size_t(M) * sizeof(LnTokenStats)) + 256;
    case BL_OP_W1A16_STACK: return 256 + align256(size_t(M > 1 ? M : 1) * size_t(N) * sizeof(uint32_t));
    case BL_OP_W1A16_BACKWARD: {
      const size_t Mp = size_t(cdiv(M, kSsUnit) * kSsUnit);
      return align256(size_t(M) * size_t(N) * 4) + align256(size_t(K) * size_t(N) / 4) +
             align256(size_t(K) * 4) + align256(size_t(K) * Mp * 2) + align256(size_t(N) * Mp * 2) +
             align256(size_t(K / kSsRowsA) * size_t(N) * 4);
    }
    default: return 0;
  }
}

int bin_pack(const float* W, int64_t N, int64_t K, int mode, uint32_t* packed, float* alpha,
             float* beta, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_shape(0, N, K);
  if (rc != BL_OK) return rc;
  if (mode != BL_PACK_FBI && mode != BL_PACK_BITNET && mode != BL_PACK_TERNARY) return BL_ERR_INVALID_ARG;
  if (!W || !packed || !aligned16(W) || !aligned16(packed)) return BL_ERR_INVALID_ARG;
  if (mode != BL_PACK_TERNARY && !alpha) return BL_ERR_INVALID_ARG;
  if (mode != BL_PACK_FBI &&
      (!beta || !ws || !aligned16(ws) || ws_bytes < bl_workspace_bytes(BL_OP_PACK_BITNET, 0, N, K)))
    return BL_ERR_INVALID_ARG;
  int sms = 0;
  rc = device_setup(&sms);
  if (rc != BL_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t warps_per_block = kPackThreads / 32;
  const unsigned grid = static_cast<unsigned>(
      cdiv(N, warps_per_block) < int64_t(sms) * 16 ? cdiv(N, warps_per_block) : int64_t(sms) * 16);
  if (mode == BL_PACK_FBI) {
    pack_rows_kernel<false><<<grid, kPackThreads, 0, s>>>(W, N, K, packed, alpha, nullptr);
    return launch_status();
  }
  double* sums = static_cast<double*>(ws);
  double* scalars = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + align256(size_t(N) * 2 * sizeof(double)));
  row_sums_kernel<<<grid, kPackThreads, 0, s>>>(W, N, K, sums);
  if ((rc = launch_status()) != BL_OK) return rc;
  global_scalars_kernel<<<1, kReduceThreads, 0, s>>>(sums, N, K, scalars,
                                                      mode == BL_PACK_TERNARY ? nullptr : alpha, beta);
  if ((rc = launch_status()) != BL_OK) return rc;
  if (mode == BL_PACK_TERNARY)
    pack_ternary_rows_kernel<<<grid, kPackThreads, 0, s>>>(W, N, K, packed, scalars);
  else
    pack_rows_kernel<true><<<grid, kPackThreads, 0, s>>>(W, N, K, packed, nullptr, scalars);
  return launch_status();
}

int bin_linear_w1a16(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y,
                     int64_t M, int64_t N, int64_t K, void* stream) {
  return bin_linear_w1a16_ex(x, packed, alpha, y, M, N, K, 0u, stream);
}

int bin_linear_w1a16_ex(const uint16_t* x, const uint32_t* packed, const float* alpha, uint16_t* y,
                        int64_t M, int64_t N, int64_t K, unsigned flags, void* stream) {
  int rc = check_shape(M, N, K);
  if (rc != BL_OK) return rc;
  if (flags & ~BL_FLAG_OVERLAP_PREVIOUS) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!x || !packed || !alpha || !y || !aligned16(x) || !aligned16(packed) || !aligned16(y))
    return BL_ERR_INVALID_ARG;
  rc = device_setup(nullptr);
  if (rc != BL_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int C = 0, slice_words = 0, pages = 0;
  if (M == 1 && lut_split(int(K), &C, &slice_words, &pages)) {
    const bool overlap = (flags & BL_FLAG_OVERLAP_PREVIOUS) != 0;
    cudaError_t e;
    if (pages == 1)
      e = launch_lut<1>(x, packed, alpha, y, int(N), int(K), C, slice_words, overlap, s);
    else if (pages == 2)
      e = launch_lut<2>(x, packed, alpha, y, int(N), int(K), C, slice_words, overlap, s);
    else
      e = launch_lut<3>(x, packed, alpha, y, int(N), int(K), C, slice_words, overlap, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return launch_status();
  }
  if (M > 1 && M <= 16 && K % 256 == 0 && K / 256 <= kMmaMaxSliceWords) {  // measured faster than tcgen05 here
    const cudaError_t e = launch_mma(x, packed, alpha, y, int(M), int(N), int(K),
                                     (flags & BL_FLAG_OVERLAP_PREVIOUS) != 0, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return launch_status();
  }
  if (M > 4) {
    int sms = 0;
    device_setup(&sms);
    return launch_ts<0>(x, packed, M, N, K, alpha, nullptr, nullptr, y, nullptr, sms, s);
  }
  const unsigned grid = static_cast<unsigned>(cdiv(N, kGemvRowsPerCta));
  if (M == 1)
    gemv_w1a16_kernel<1><<<grid, kGemvThreads, gemv_smem_bytes(1), s>>>(x, packed, alpha, y, int(M), N, K);
  else if (M == 2)
    gemv_w1a16_kernel<2><<<grid, kGemvThreads, gemv_smem_bytes(2), s>>>(x, packed, alpha, y, int(M), N, K);
  else
    gemv_w1a16_kernel<4><<<grid, kGemvThreads, gemv_smem_bytes(4), s>>>(x, packed, alpha, y, int(M), N, K);
  return launch_status();
}

int bitlinear_w1a8(const uint16_t* x, const uint32_t* packed, const float* beta, float* y, int64_t M,
                   int64_t N, int64_t K, void* ws, size_t ws_bytes, void* stream) {
  return w1a8_impl(x, packed, beta, y, M, N, K, ws, ws_bytes, nullptr, nullptr, nullptr, nullptr,
                   nullptr, false, stream);
}

int bitlinear_w158a8(const uint16_t* x, const uint32_t* packed, const float* beta, float* y, int64_t M,
                     int64_t N, int64_t K, void* ws, size_t ws_bytes, void* stream) {
  return w1a8_impl(x, packed, beta, y, M, N, K, ws, ws_bytes, nullptr, nullptr, nullptr, nullptr,
                   nullptr, true, stream);
}

int bitlinear_w1a8_ex(const uint16_t* x, const uint32_t* packed, const float* beta, float* y, int64_t M,
                      int64_t N, int64_t K, unsigned flags, void* ws, size_t ws_bytes, int8_t* xq_out,
                      double* gamma_out, int32_t* acc_out, void* stream) {
  if (flags & ~(BL_W1A8_TERNARY | BL_W1A8_PER_TENSOR | BL_W1A8_NONNEG)) return BL_ERR_INVALID_ARG;
  const unsigned quant = flags & (BL_W1A8_PER_TENSOR | BL_W1A8_NONNEG);
  return w1a8_impl(x, packed, beta, y, M, N, K, ws, ws_bytes, xq_out, gamma_out, acc_out, nullptr, nullptr,
                   (flags & BL_W1A8_TERNARY) != 0, stream, quant);
}

int bin_linear_w1a16_stack(const bl_stack_level* levels, int num_levels, const bl_stack_job* jobs,
                           int num_jobs, void* ws, size_t ws_bytes, void* stream) {
  return bin_linear_w1a16_stack_batch(levels, num_levels, jobs, num_jobs, 1, ws, ws_bytes, stream);
}

int bin_linear_w1a16_stack_batch(const bl_stack_level* levels, int num_levels, const bl_stack_job* jobs,
                                 int num_jobs, int64_t M, void* ws, size_t ws_bytes, void* stream) {
  if (num_levels < 0 || num_jobs < 0 || M < 1 || M > 16) return BL_ERR_INVALID_ARG;
  if (num_levels == 0) return BL_OK;
  if (!levels || !jobs || !ws || !aligned16(ws)) return BL_ERR_INVALID_ARG;
  // level of every linear; the linears' outputs as byte ranges
  std::vector<int> level_of(static_cast<size_t>(num_jobs), -1);
  std::vector<std::pair<uintptr_t, int>> outs;  // (start, linear), sorted below
  for (int i = 0; i < num_levels; ++i) {
    const bl_stack_level& lv = levels[i];
    if (!lv.x || !aligned16(lv.x) || lv.num_jobs < 1 || lv.first_job < 0 ||
        int64_t(lv.first_job) + lv.num_jobs > num_jobs || lv.num_jobs > kStrMaxJobs)
      return BL_ERR_INVALID_ARG;
    if (lv.K < 256 || lv.K > 32 * kStrCluster * 48 || lv.K % 256 != 0) return BL_ERR_UNSUPPORTED;
    for (int j = lv.first_job; j < lv.first_job + lv.num_jobs; ++j) {
      const bl_stack_job& jb = jobs[j];
      if (level_of[size_t(j)] != -1) return BL_ERR_INVALID_ARG;  // a linear listed by two levels
      if (!jb.packed || !jb.alpha || !jb.y || jb.N < 1 || !aligned16(jb.packed)) return BL_ERR_INVALID_ARG;
      if (jb.N > kMaxDim || jb.N * lv.K >= kMaxProduct) return BL_ERR_UNSUPPORTED;
      level_of[size_t(j)] = i;
      outs.emplace_back(reinterpret_cast<uintptr_t>(jb.y), j);
    }
  }
  // every linear writes its own buffer
  std::sort(outs.begin(), outs.end());
  const uintptr_t m2 = 2 * uintptr_t(M);  // bytes per element of a row, over the M tokens
  for (size_t t = 1; t < outs.size(); ++t)
    if (outs[t].first < outs[t - 1].first + m2 * uintptr_t(jobs[outs[t - 1].second].N)) return BL_ERR_INVALID_ARG;
  // the input of each level: a buffer written by no linear of the call, or
  // exactly the output of one linear of an earlier level
  std::vector<int> src(static_cast<size_t>(num_levels), -1);
  int64_t total_n = 0;
  for (int i = 0; i < num_levels; ++i) {
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(levels[i].x), x1 = x0 + m2 * uintptr_t(levels[i].K);
    auto it = std::upper_bound(outs.begin(), outs.end(), std::make_pair(x1, -1));
    if (it != outs.begin()) {
      const auto& o = *(it - 1);  // the last output starting before x ends
      const uintptr_t o1 = o.first + m2 * uintptr_t(jobs[o.second].N);
      if (o1 > x0) {  // overlaps
        if (o.first != x0 || jobs[o.second].N != levels[i].K || level_of[size_t(o.second)] >= i)
          return BL_ERR_INVALID_ARG;
        src[size_t(i)] = o.second;
      }
    }
  }
  for (int j = 0; j < num_jobs; ++j) total_n += level_of[size_t(j)] >= 0 ? jobs[j].N : 0;
  if (ws_bytes < bl_workspace_bytes(BL_OP_W1A16_STACK, M, total_n, 0)) return BL_ERR_INVALID_ARG;
  int sms = 0;
  int rc = device_setup(&sms);
  if (rc != BL_OK) return rc;
  const int G = stack_cluster_capacity(M);
  if (G < 1) return BL_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // Launches of at most kStrMaxLevels levels and kStrMaxJobs linears. An
  // output read by a later level of the same launch gets a tagged copy in
  // the workspace; the copies are zero-filled once, before the first launch.
  std::vector<int> launch_of(static_cast<size_t>(num_levels));
  {
    int li = 0, nl = 0, nj = 0;
    for (int i = 0; i < num_levels; ++i) {
      if (nl == kStrMaxLevels || nj + levels[i].num_jobs > kStrMaxJobs) {
        ++li;
        nl = nj = 0;
      }
      launch_of[size_t(i)] = li;
      ++nl;
      nj += levels[i].num_jobs;
    }
  }
  std::vector<int64_t> tag_off(static_cast<size_t>(num_jobs), -1);
  int64_t tagged_words = 0;
  for (int i = 0; i < num_levels; ++i) {
    const int j = src[size_t(i)];
    if (j >= 0 && launch_of[size_t(level_of[size_t(j)])] == launch_of[size_t(i)] && tag_off[size_t(j)] < 0) {
      tag_off[size_t(j)] = tagged_words;
      tagged_words += M * jobs[j].N;
    }
  }
  // ws: the abort word (first 256 bytes), then the tagged outputs; only
  // launches with tagged outputs wait on anything outside their clusters
  uint32_t* abort_word = static_cast<uint32_t*>(ws);
  uint32_t* tags = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + 256);
  if (tagged_words > 0 && cudaMemsetAsync(ws, 0, 256 + size_t(tagged_words) * 4, s) != cudaSuccess) {
    cudaGetLastError();
    return BL_ERR_CUDA;
  }
  static thread_local StrParams P;  // ~29 KB: too large for the stack of every caller
  int i = 0;
  while (i < num_levels) {
    std::memset(&P, 0, sizeof P);
    const int li = launch_of[size_t(i)];
    int nl = 0, nj = 0;
    int64_t max_chunks = 0;
    for (; i < num_levels && launch_of[size_t(i)] == li; ++i) {
      const bl_stack_level& lv = levels[i];
      StrLevel& d = P.lv[nl++];
      const int j_src = src[size_t(i)];
      if (j_src >= 0 && tag_off[size_t(j_src)] >= 0)
        d.xt = tags + tag_off[size_t(j_src)];
      else
        d.x = lv.x;
      d.K = int(lv.K);
      d.job0 = nj;
      d.njobs = lv.num_jobs;
      int64_t chunks = 0;
      for (int j = lv.first_job; j < lv.first_job + lv.num_jobs; ++j) {
        StrJob& e = P.jobs[nj];
        if (!make_map_2d(&P.maps[nj], jobs[j].packed, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, uint64_t(lv.K / 32),
                         uint64_t(jobs[j].N), 16, kStrBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE))
          return BL_ERR_CUDA;
        ++nj;
        e.alpha = jobs[j].alpha;
        e.y = jobs[j].y;
        e.tagged = tag_off[size_t(j)] >= 0 ? tags + tag_off[size_t(j)] : nullptr;
        e.N = int(jobs[j].N);
        e.chunk0 = int(chunks);
        chunks += cdiv(jobs[j].N, kStrChunk);
      }
      if (chunks > kMaxDim / kStrChunk) return BL_ERR_UNSUPPORTED;
      d.nchunks = int(chunks);
      if (chunks > max_chunks) max_chunks = chunks;
    }
    P.num_levels = nl;
    P.num_jobs = nj;
    P.abort = abort_word;
    const int clusters = int(max_chunks < G ? max_chunks : G);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kStrCluster, static_cast<unsigned>(clusters), 1);
    cfg.blockDim = dim3(M == 1 ? kStrThreads + 32 : kSmThreads + 32, 1, 1);
    cfg.dynamicSmemBytes = M == 1 ? kStrSmemBytes : (M <= 8 ? SmCfg<8>::kSmemBytes : SmCfg<16>::kSmemBytes);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kStrCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int m = int(M);
    const cudaError_t e = M == 1  ? cudaLaunchKernelEx(&cfg, gemv_w1a16_stream_kernel, P)
                          : M <= 8 ? cudaLaunchKernelEx(&cfg, gemv_w1a16_stream_mma_kernel<8>, P, m)
                                   : cudaLaunchKernelEx(&cfg, gemv_w1a16_stream_mma_kernel<16>, P, m);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    if ((rc = launch_status()) != BL_OK) return rc;
  }
  return BL_OK;
}

int bin_linear_w1a16_backward(const uint16_t* x, const uint32_t* packed, const float* alpha, const uint16_t* dy,
                              uint16_t* dx, float* dw, float* dalpha, int64_t M, int64_t N, int64_t K, void* ws,
                              size_t ws_bytes, void* stream) {
  int rc = check_shape(M, N, K);
  if (rc != BL_OK) return rc;
  if (N % 128 != 0) return BL_ERR_UNSUPPORTED;
  if ((dw == nullptr) != (dalpha == nullptr)) return BL_ERR_INVALID_ARG;
  if (!packed || !alpha || !aligned16(packed) || (dw && !aligned16(dw)) || (dx && !aligned16(dx)))
    return BL_ERR_INVALID_ARG;
  const int64_t Mp = cdiv(M, kSsUnit) * kSsUnit;
  if (cdiv(Mp, 32) > 65535 || cdiv(N, 32) > 65535 || cdiv(K, 32) > 65535) return BL_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M == 0) {  // an empty batch: zero weight and scale gradients, no dx
    if (dw && (cudaMemsetAsync(dw, 0, size_t(N) * size_t(K) * 4, s) != cudaSuccess ||
               cudaMemsetAsync(dalpha, 0, size_t(N) * 4, s) != cudaSuccess)) {
      cudaGetLastError();
      return BL_ERR_CUDA;
    }
    return BL_OK;
  }
  if (!x || !dy || !aligned16(x) || !aligned16(dy)) return BL_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws) || ws_bytes < bl_workspace_bytes(BL_OP_W1A16_BACKWARD, M, N, K))
    return BL_ERR_INVALID_ARG;
  int sms = 0;
  rc = device_setup(&sms);
  if (rc != BL_OK) return rc;
  uint8_t* w = static_cast<uint8_t*>(ws);
  auto* g2 = reinterpret_cast<uint16_t*>(w);
  w += align256(size_t(M) * size_t(N) * 4);
  auto* packed_t2 = reinterpret_cast<uint32_t*>(w);
  w += align256(size_t(K) * size_t(N) / 4);
  auto* ones = reinterpret_cast<float*>(w);
  w += align256(size_t(K) * 4);
  auto* xt = reinterpret_cast<uint16_t*>(w);
  w += align256(size_t(K) * size_t(Mp) * 2);
  auto* dyt = reinterpret_cast<uint16_t*>(w);
  w += align256(size_t(N) * size_t(Mp) * 2);
  auto* part = reinterpret_cast<float*>(w);  // [K / 128][N] signed partial sums for dalpha
  if (dx) {
    // dx = [hi | lo] x [S^T | S^T] through the forward path (unit scales)
    ste_scale_split_kernel<<<dim3(static_cast<unsigned>(cdiv(N / 8, 256)), static_cast<unsigned>(M < 8192 ? M : 8192)),
                             256, 0, s>>>(dy, alpha, M, N, g2);
    if ((rc = launch_status()) != BL_OK) return rc;
    transpose_pack_dup_kernel<<<dim3(static_cast<unsigned>(cdiv(N, kTpRows)), static_cast<unsigned>(cdiv(K / 32, kTpWords))),
                                256, kTpSmemBytes, s>>>(packed, N, K, packed_t2);
    if ((rc = launch_status()) != BL_OK) return rc;
    fill_f32_kernel<<<static_cast<unsigned>(cdiv(K, 256) < sms ? cdiv(K, 256) : sms), 256, 0, s>>>(ones, K, 1.0f);
    if ((rc = launch_status()) != BL_OK) return rc;
    rc = bin_linear_w1a16_ex(g2, packed_t2, ones, dx, M, K, 2 * N, 0u, stream);
    if (rc != BL_OK) return rc;
  }
  if (dw) {
    // P = dY^T X on the tensor cores, then dW = alpha P and dalpha = sum_k s P in place
    const dim3 tb(32, 8);
    transpose_bf16_kernel<<<dim3(unsigned(K / kTrTile), unsigned(Mp / kTrTile)), tb, 0, s>>>(x, M, K, xt, Mp);
    if ((rc = launch_status()) != BL_OK) return rc;
    transpose_bf16_kernel<<<dim3(unsigned(N / kTrTile), unsigned(Mp / kTrTile)), tb, 0, s>>>(dy, M, N, dyt, Mp);
    if ((rc = launch_status()) != BL_OK) return rc;
    CUtensorMap tm_a, tm_b;
    if (!make_map_2d(&tm_a, xt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(Mp), uint64_t(K), kSsUnit, kSsRowsA,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tm_b, dyt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(Mp), uint64_t(N), kSsUnit, kSsRowsB,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return BL_ERR_CUDA;
    const int64_t tiles = (K / kSsRowsA) * cdiv(N, kSsRowsB);
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    // dW = alpha P and the per-tile signed sums for dalpha come out of the GEMM's epilogue
    gemm_ss_ste_kernel<<<grid, kSsThreads, kSsSmemBytes, s>>>(tm_a, tm_b, int(K), int(N), int(Mp), alpha, packed,
                                                               dw, part);
    if ((rc = launch_status()) != BL_OK) return rc;
    const int64_t dblocks = cdiv(N, 256) < int64_t(sms) * 4 ? cdiv(N, 256) : int64_t(sms) * 4;
    ste_dalpha_kernel<<<static_cast<unsigned>(dblocks), 256, 0, s>>>(part, K / kSsRowsA, N, dalpha);
    if ((rc = launch_status()) != BL_OK) return rc;
  }
  return BL_OK;
}

int bitlinear_w158a8_debug(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                           int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes, int8_t* xq_out,
                           double* gamma_out, int32_t* acc_out, const int8_t* xq_in,
                           const double* gamma_in, void* stream) {
  return w1a8_impl(x, packed, beta, y, M, N, K, ws, ws_bytes, xq_out, gamma_out, acc_out, xq_in,
                   gamma_in, true, stream);
}

int bitlinear_w1a8_debug(const uint16_t* x, const uint32_t* packed, const float* beta, float* y,
                         int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes, int8_t* xq_out,
                         double* gamma_out, int32_t* acc_out, const int8_t* xq_in,
                         const double* gamma_in, void* stream) {
  return w1a8_impl(x, packed, beta, y, M, N, K, ws, ws_bytes, xq_out, gamma_out, acc_out, xq_in,
                   gamma_in, false, stream);
}

int bin_xnor_gemm(const uint32_t* a, const uint32_t* b, int32_t* dot, int64_t M, int64_t N, int64_t K,
                  void* stream) {
  int rc = check_shape(M, N, K);
  if (rc != BL_OK) return rc;
  if (M == 0) return BL_OK;
  if (K > (int64_t(1) << 30)) return BL_ERR_UNSUPPORTED;  // dot must fit int32
  if (!a || !b || !dot) return BL_ERR_INVALID_ARG;
  rc = device_setup(nullptr);
  if (rc != BL_OK) return rc;
  if (cdiv(M, kXnorTile) > 65535) return BL_ERR_UNSUPPORTED;  // grid y limit
  const dim3 grid(static_cast<unsigned>(cdiv(N, kXnorTile)), static_cast<unsigned>(cdiv(M, kXnorTile)), 1);
  xnor_gemm_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(a, b, dot, M, N, K);
  return launch_status();
}

int bl_device_error(void* stream, int clear, int* where_out) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BL_ERR_CUDA;
  DeviceError e{0, 0};
  if (cudaMemcpyFromSymbol(&e, g_device_error, sizeof e) != cudaSuccess) return BL_ERR_CUDA;
  if (clear) {
    const DeviceError z{0, 0};
    if (cudaMemcpyToSymbol(g_device_error, &z, sizeof z) != cudaSuccess) return BL_ERR_CUDA;
  }
  if (where_out) *where_out = e.where;
  return e.code;
}

}  // extern "C"

// ---- allocation-free BitLinear ------------------------------------------------
// bitlinear_w1a8_noalloc serves callers that cannot allocate device memory:
// operators embedded in a host framework that only hands them their inputs
// and outputs, and loops with a fixed up-front memory plan that must not call
// cudaMalloc while running. It runs the same LN/quant and GEMM kernels as
// bitlinear_w1a8, with the codes and gamma kept in the array below instead
// of a caller workspace.
namespace bl {
namespace {

// Lives on every device that loads this library, until the process exits.
static __device__ __align__(256) uint8_t g_w1a8_noalloc_scratch[BL_W1A8_NOALLOC_SCRATCH_BYTES];

struct NoallocScratch {
  std::once_flag once;
  void* ptr = nullptr;
  int status = BL_ERR_NO_DEVICE;
};
NoallocScratch g_noalloc[kMaxDevices];

// Device address of the scratch array on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return BL_ERR_NO_DEVICE;
  }
  NoallocScratch& st = g_noalloc[dev];
  std::call_once(st.once, [&st] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_w1a8_noalloc_scratch) == cudaSuccess && p != nullptr) {
      st.ptr = p;
      st.status = BL_OK;
    } else {
      cudaGetLastError();
      st.status = BL_ERR_CUDA;
    }
  });
  *out = st.ptr;
  return st.status;
}

}  // namespace
}  // namespace bl

extern "C" int bitlinear_w1a8_noalloc(const uint16_t* x, const uint32_t* packed, const float* beta,
                                      float* y, int64_t M, int64_t N, int64_t K, void* stream) {
  int rc = check_shape(M, N, K);
  if (rc != BL_OK) return rc;
  if (M == 0) return BL_OK;
  if (bl_workspace_bytes(BL_OP_W1A8, M, N, K) > BL_W1A8_NOALLOC_SCRATCH_BYTES) return BL_ERR_SCRATCH_LIMIT;
  if (!x || !packed || !beta || !y) return BL_ERR_INVALID_ARG;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != BL_OK) return rc;
  return w1a8_impl(x, packed, beta, y, M, N, K, scratch, BL_W1A8_NOALLOC_SCRATCH_BYTES, nullptr,
                   nullptr, nullptr, nullptr, nullptr, false, stream);
}

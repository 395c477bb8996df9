// mxq.cu - the C ABI (include/mxq.h): argument checks, dispatch, launches.
//
// One translation unit holds every kernel (quant.cuh, gemm.cuh) so that they
// share the device error word.  Built with nvcc for sm_100a only, without
// fast-math (the quantisers must round exactly like the definition).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/mxq.h"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "quant.cuh"
#include "attention.cuh"
#include "gemv.cuh"

namespace {

constexpr int kMaxDevices = 64;
thread_local int t_last_cuda_error = 0;

inline int64_t pad_to(int64_t n, int64_t m) { return (n + m - 1) / m * m; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

mxq_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return MXQ_ERR_CUDA;
}

// ------------------------------------------------------- device properties
struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 supported, 2 unsupported
  int sms = 0;
  std::atomic<uint32_t> smem_attr_set{0};  // bit per GEMM instantiation
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

mxq_status current_device(int* dev_out, int* sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    t_last_cuda_error = static_cast<int>(e);
    cudaGetLastError();
    return MXQ_ERR_ARCH;
  }
  if (dev < 0 || dev >= kMaxDevices) return MXQ_ERR_ARCH;
  DeviceInfo& d = g_dev[dev];
  int st = d.state.load(std::memory_order_acquire);
  if (st == 0) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    st = d.state.load(std::memory_order_relaxed);
    if (st == 0) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return MXQ_ERR_ARCH;
      }
      d.sms = sms;
      st = (major == 10 && minor == 0) ? 1 : 2;  // sm_100a code runs on compute capability 10.0
      d.state.store(st, std::memory_order_release);
    }
  }
  if (st != 1) return MXQ_ERR_ARCH;
  *dev_out = dev;
  if (sms_out) *sms_out = d.sms;
  return MXQ_OK;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

mxq_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    } else {
      cudaGetLastError();
    }
  });
  return g_encode ? MXQ_OK : MXQ_ERR_CUDA;
}

// 2-D row-major tensor [outer][inner] with a row stride in bytes.
mxq_status tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
                   uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                   uint32_t box_outer, CUtensorMapSwizzle swz) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return MXQ_ERR_CUDA;
  }
  return MXQ_OK;
}

// Grid of the two-pass kernels, which deal row chunks of `chunk_elems`
// elements to warps: a warp per chunk up to 8 blocks per SM and at most
// kMaxAmaxPartials blocks (the partial-amax array size).
int quant_grid(int64_t rows, int64_t k, int64_t chunk_elems, int sms) {
  const int64_t warps_per_block = mxq::kQuantThreads / 32;
  const int64_t chunks = rows * ((k + chunk_elems - 1) / chunk_elems);
  int64_t g = (chunks + warps_per_block - 1) / warps_per_block;
  int64_t cap = static_cast<int64_t>(sms) * 8;
  if (cap > mxq::kMaxAmaxPartials) cap = mxq::kMaxAmaxPartials;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

mxq_status check_bf16_matrix(const void* x, int64_t rows, int64_t k, int64_t ld) {
  if (rows < 0 || k < 0) return MXQ_ERR_INVALID_ARG;
  if (rows > 0 && k > 0 && x == nullptr) return MXQ_ERR_INVALID_ARG;
  if (ld < k || ld < 1) return MXQ_ERR_INVALID_ARG;
  if (ld % 8 != 0) return MXQ_ERR_ALIGNMENT;
  if (!aligned16(x)) return MXQ_ERR_ALIGNMENT;
  if (rows > INT32_MAX || k > INT32_MAX) return MXQ_ERR_UNSUPPORTED_SHAPE;
  return MXQ_OK;
}

// ----------------------------------------------------------------- launches
// Every kernel is launched with programmatic stream serialization: it may
// start while the previous kernel of the stream finishes, and waits
// (griddepcontrol.wait) before reading anything that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// amax into one fp32 (zeroed first, then atomicMax of every block's maximum).
mxq_status launch_amax(const void* x, int64_t rows, int64_t k, int64_t ld, float* amax,
                       cudaStream_t s, int sms) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), s);
  if (e != cudaSuccess) return cuda_fail(e);
  if (rows == 0 || k == 0) return MXQ_OK;
  e = launch_pdl(mxq::amax_kernel, dim3(quant_grid(rows, k, mxq::kAmaxChunk, sms)), dim3(mxq::kQuantThreads), 0, s,
                 static_cast<const __nv_bfloat16*>(x), static_cast<int>(rows), static_cast<int>(k), ld,
                 static_cast<float*>(nullptr), amax);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

// amax as per-block partial maxima (no zeroing needed); returns their count.
mxq_status launch_amax_partials(const void* x, int64_t rows, int64_t k, int64_t ld, float* partials,
                                int* n_partials, cudaStream_t s, int sms) {
  const int grid = quant_grid(rows, k, mxq::kAmaxChunk, sms);
  cudaError_t e = launch_pdl(mxq::amax_kernel, dim3(grid), dim3(mxq::kQuantThreads), 0, s,
                             static_cast<const __nv_bfloat16*>(x), static_cast<int>(rows),
                             static_cast<int>(k), ld, partials, static_cast<float*>(nullptr));
  *n_partials = grid;
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

mxq_status launch_quant_nvfp4(const void* x, int64_t rows, int64_t k, int64_t ld,
                              const float* amax_vals, int n_amax, uint8_t* codes, uint8_t* sf,
                              float* g, float* amax_out, cudaStream_t s, int sms) {
  cudaError_t e = launch_pdl(mxq::quantize_nvfp4_kernel, dim3(quant_grid(rows, k, mxq::kNvfp4Chunk, sms)),
                             dim3(mxq::kQuantThreads), 0, s, static_cast<const __nv_bfloat16*>(x),
                             static_cast<int>(rows), static_cast<int>(k), ld, amax_vals, n_amax, codes,
                             sf, g, amax_out);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

// ---- single-pass NVFP4 quantisation (rows held in shared memory)
constexpr int kFusedMaxGrid = 256;          // tag capacity in the workspace header
constexpr size_t kFusedSmemLimit = 227 * 1024 - 1024;  // dynamic bytes, static ones kept aside

struct FusedPlan {
  int grid = 0, rows_per_cta = 0;
  size_t smem = 0;
};

// One CTA per SM, each holding ceil(rows / SMs) rows and one mbarrier per row.
FusedPlan plan_fused(int64_t rows, int64_t k, int sms) {
  FusedPlan p;
  if (rows <= 0 || k <= 0 || sms <= 0) return p;
  const int64_t rpc = (rows + sms - 1) / sms;
  const size_t smem = static_cast<size_t>(rpc) * static_cast<size_t>(k) * 2 + 8 * static_cast<size_t>(rpc);
  const int64_t grid = (rows + rpc - 1) / rpc;
  if (smem > kFusedSmemLimit || grid > kFusedMaxGrid) return p;
  p.grid = static_cast<int>(grid);
  p.rows_per_cta = static_cast<int>(rpc);
  p.smem = smem;
  return p;
}

// Cooperative launch (the grid barrier needs every CTA resident), with
// programmatic stream serialization when the CUDA driver accepts both.
template <typename... KArgs, typename... Args>
cudaError_t launch_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                        Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e == cudaSuccess) return e;
  cudaGetLastError();
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

mxq_status launch_quant_nvfp4_fused(const void* x, int64_t rows, int64_t k, int64_t ld,
                                    const FusedPlan& p, mxq::FusedSync* sync, uint8_t* codes,
                                    uint8_t* sf, float* g, float* amax_out, cudaStream_t s,
                                    int dev) {
  constexpr uint32_t bit = 1u << 20;  // GEMM instantiations use the low bits
  if (!(g_dev[dev].smem_attr_set.load(std::memory_order_acquire) & bit)) {
    cudaError_t e = cudaFuncSetAttribute(mxq::quantize_nvfp4_fused_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kFusedSmemLimit));
    if (e != cudaSuccess) return cuda_fail(e);
    g_dev[dev].smem_attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  cudaError_t e = launch_coop(mxq::quantize_nvfp4_fused_kernel, dim3(p.grid), dim3(mxq::kFusedThreads),
                              p.smem, s, static_cast<const __nv_bfloat16*>(x), static_cast<int>(rows),
                              static_cast<int>(k), ld, p.rows_per_cta, sync, codes, sf, g, amax_out);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

mxq_status launch_quant_mxfp8(const void* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                              uint8_t* sf, cudaStream_t s, int sms, int rceil = 0) {
  // one thread per 32-element block, up to 8 CTAs per SM, grid-stride beyond
  const int64_t nblk = rows * (k >> 5);
  int64_t grid = (nblk + mxq::kMxThreads - 1) / mxq::kMxThreads;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  if (grid < 1) grid = 1;
  cudaError_t e = launch_pdl(mxq::quantize_mxfp8_kernel, dim3(static_cast<unsigned>(grid)),
                             dim3(mxq::kMxThreads), 0, s, static_cast<const __nv_bfloat16*>(x),
                             static_cast<int>(rows), static_cast<int>(k), ld, codes, sf, rceil);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

// Epilogue options of the pair kernel's producer variant (mxq_linear_opts).
struct Epilogue {
  int act = 0;             // MXQ_ACT_*
  float* y_amax = nullptr; // receives max |y| (atomicMax on the bits; zeroed by the caller)
};

template <mxq::Fmt F, int BN>
mxq_status launch_gemm_bn(int dev, int sms, int slot, int64_t M, int64_t N, int64_t K,
                          const void* a, const uint8_t* a_sf, const float* a_g, const void* b,
                          const uint8_t* b_sf, const float* b_g, const void* bias, void* y,
                          int64_t ldy, cudaStream_t s) {
  using C = mxq::GemmCfg<F, BN>;
  auto kern = mxq::gemm_kernel<F, BN>;
  const uint32_t bit = 1u << slot;
  if (!(g_dev[dev].smem_attr_set.load(std::memory_order_acquire) & bit)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    g_dev[dev].smem_attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap ta, tb, ty;
  mxq_status st;
  if (F == mxq::Fmt::BF16) {
    st = tmap_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, C::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == MXQ_OK)
      st = tmap_2d(&tb, b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, N, K * 2, 64, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    const int64_t row_bytes = F == mxq::Fmt::NVFP4 ? K / 2 : K;
    st = tmap_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes, M, row_bytes, 128, C::BM,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == MXQ_OK)
      st = tmap_2d(&tb, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes, N, row_bytes, 128, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (st == MXQ_OK)
    st = tmap_2d(&ty, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, ldy * 2, 32, 32,
                 CU_TENSOR_MAP_SWIZZLE_64B);
  if (st != MXQ_OK) return st;
  mxq::GemmArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.a_sf = a_sf;
  args.b_sf = b_sf;
  args.a_g = a_g;
  args.b_g = b_g;
  args.bias = static_cast<const __nv_bfloat16*>(bias);
  const int64_t tiles = ((M + C::BM - 1) / C::BM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  cudaError_t e = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, ta, tb, ty, args);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

template <mxq::Fmt F, int BN, int EPI>
mxq_status launch_gemm_pair(int dev, int sms, int slot, int64_t M, int64_t N, int64_t K,
                            const void* a, const uint8_t* a_sf, const float* a_g, const void* b,
                            const uint8_t* b_sf, const float* b_g, const void* bias, void* y,
                            int64_t ldy, const Epilogue& ep, cudaStream_t s) {
  using C = mxq::PairCfg<F, BN>;
  auto kern = mxq::gemm_pair_kernel<F, BN, EPI>;
  const uint32_t bit = 1u << slot;
  if (!(g_dev[dev].smem_attr_set.load(std::memory_order_acquire) & bit)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    g_dev[dev].smem_attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap ta, tb, tsa, tsb, ty;
  mxq_status st;
  if (F == mxq::Fmt::BF16) {
    st = tmap_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, C::BM_CTA,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == MXQ_OK)
      st = tmap_2d(&tb, b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, N, K * 2, 64, C::BN_CTA,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    tsa = ta;
    tsb = tb;
  } else {
    const int64_t row_bytes = F == mxq::Fmt::NVFP4 ? K / 2 : K;
    const mxq_format f = F == mxq::Fmt::NVFP4 ? MXQ_NVFP4 : MXQ_MXFP8;
    st = tmap_2d(&ta, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes, M, row_bytes, 128, C::BM_CTA,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == MXQ_OK)
      st = tmap_2d(&tb, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes, N, row_bytes, 128, C::BN_CTA,
                   CU_TENSOR_MAP_SWIZZLE_128B);
    // scale arrays viewed as rows of 256 bytes (a 512-byte chunk is two rows)
    if (st == MXQ_OK)
      st = tmap_2d(&tsa, a_sf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, mxq_sf_bytes(M, K, f) / 256, 256,
                   256, C::SF_BOX_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st == MXQ_OK)
      st = tmap_2d(&tsb, b_sf, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, mxq_sf_bytes(N, K, f) / 256, 256,
                   256, C::SF_BOX_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (st == MXQ_OK)
    st = tmap_2d(&ty, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, ldy * 2, C::EPI_SUB, 32,
                 C::EPI_ROW == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : (C::EPI_ROW == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B));
  if (st != MXQ_OK) return st;
  mxq::PairArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.a_g = a_g;
  args.b_g = b_g;
  args.bias = static_cast<const __nv_bfloat16*>(bias);
  args.act = ep.act;
  args.y_amax = reinterpret_cast<unsigned int*>(ep.y_amax);
  const int64_t tiles = ((M + C::BM - 1) / C::BM) * ((N + BN - 1) / BN);
  const int64_t pairs = sms / 2;
  const int grid = 2 * static_cast<int>(tiles < pairs ? tiles : pairs);
  cudaError_t e = launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, ta, tb, tsa, tsb, ty,
                             args);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

template <int EPI>
mxq_status launch_gemm_pairs(mxq_format f, int dev, int sms, int64_t M, int64_t N, int64_t K,
                             const void* a, const uint8_t* a_sf, const float* a_g, const void* b,
                             const uint8_t* b_sf, const float* b_g, const void* bias, void* y,
                             int64_t ldy, const Epilogue& ep, cudaStream_t s) {
  // slots 6-11: plain epilogue; 12-17: producer epilogue
  const int base = EPI ? 12 : 6;
  // 256-column tiles, unless they would leave more than half of the CTA pairs
  // without a tile (e.g. M = 512, N = 3072: 24 tiles for 74 pairs); 128-column
  // tiles double the count
  const int64_t tiles256 = ((M + 255) / 256) * ((N + 255) / 256);
  const bool wide = N > 128 && tiles256 > (sms / 2) / 2;
  switch (f) {
    case MXQ_NVFP4:
      if (wide)
        return launch_gemm_pair<mxq::Fmt::NVFP4, 256, EPI>(dev, sms, base, M, N, K, a, a_sf, a_g, b,
                                                           b_sf, b_g, bias, y, ldy, ep, s);
      return launch_gemm_pair<mxq::Fmt::NVFP4, 128, EPI>(dev, sms, base + 1, M, N, K, a, a_sf, a_g, b,
                                                         b_sf, b_g, bias, y, ldy, ep, s);
    case MXQ_MXFP8:
      if (wide)
        return launch_gemm_pair<mxq::Fmt::MXFP8, 256, EPI>(dev, sms, base + 2, M, N, K, a, a_sf, a_g, b,
                                                           b_sf, b_g, bias, y, ldy, ep, s);
      return launch_gemm_pair<mxq::Fmt::MXFP8, 128, EPI>(dev, sms, base + 3, M, N, K, a, a_sf, a_g, b,
                                                         b_sf, b_g, bias, y, ldy, ep, s);
    case MXQ_BF16:
      if (wide)
        return launch_gemm_pair<mxq::Fmt::BF16, 256, EPI>(dev, sms, base + 4, M, N, K, a, a_sf, a_g, b,
                                                          b_sf, b_g, bias, y, ldy, ep, s);
      return launch_gemm_pair<mxq::Fmt::BF16, 128, EPI>(dev, sms, base + 5, M, N, K, a, a_sf, a_g, b,
                                                        b_sf, b_g, bias, y, ldy, ep, s);
  }
  return MXQ_ERR_INVALID_ARG;
}

// bf16 layers with M <= 8: CUDA-core weight stream over all SMs (gemv.cuh).
mxq_status launch_gemv(int sms, int64_t M, int64_t N, int64_t K, const void* x, const void* w,
                       const void* bias, void* y, int64_t ldy, cudaStream_t s) {
  const int rw = M <= 2 ? mxq::gemv_rows<2>() : mxq::gemv_rows<8>();
  const int64_t tasks = (N + rw - 1) / rw;  // one warp each
  int64_t grid = (tasks + mxq::kGemvThreads / 32 - 1) / (mxq::kGemvThreads / 32);
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  if (grid < 1) grid = 1;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  const auto* bb = static_cast<const __nv_bfloat16*>(bias);
  auto* yb = static_cast<__nv_bfloat16*>(y);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  cudaError_t e;
  const dim3 g(static_cast<unsigned>(grid)), b(mxq::kGemvThreads);
  if (M == 1) e = launch_pdl(mxq::gemv_bf16_kernel<1>, g, b, 0, s, xb, m, k, wb, n, bb, yb, ldy);
  else if (M == 2) e = launch_pdl(mxq::gemv_bf16_kernel<2>, g, b, 0, s, xb, m, k, wb, n, bb, yb, ldy);
  else if (M <= 4) e = launch_pdl(mxq::gemv_bf16_kernel<4>, g, b, 0, s, xb, m, k, wb, n, bb, yb, ldy);
  else e = launch_pdl(mxq::gemv_bf16_kernel<8>, g, b, 0, s, xb, m, k, wb, n, bb, yb, ldy);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

mxq_status launch_gemm(mxq_format f, int dev, int sms, int64_t M, int64_t N, int64_t K,
                       const void* a, const uint8_t* a_sf, const float* a_g, const void* b,
                       const uint8_t* b_sf, const float* b_g, const void* bias, void* y,
                       int64_t ldy, cudaStream_t s, const Epilogue& ep = Epilogue{}) {
  const bool producer = ep.act != 0 || ep.y_amax != nullptr;
  if (M > 128) {
    // CTA-pair kernel (M = 256 MMAs)
    if (producer)
      return launch_gemm_pairs<1>(f, dev, sms, M, N, K, a, a_sf, a_g, b, b_sf, b_g, bias, y, ldy, ep, s);
    return launch_gemm_pairs<0>(f, dev, sms, M, N, K, a, a_sf, a_g, b, b_sf, b_g, bias, y, ldy, ep, s);
  }
  if (producer) return MXQ_ERR_UNSUPPORTED_SHAPE;  // the single-CTA kernel has the plain epilogue only
  switch (f) {
    case MXQ_NVFP4:
      if (N % 192 == 0)
        return launch_gemm_bn<mxq::Fmt::NVFP4, 192>(dev, sms, 0, M, N, K, a, a_sf, a_g, b, b_sf,
                                                     b_g, bias, y, ldy, s);
      return launch_gemm_bn<mxq::Fmt::NVFP4, 128>(dev, sms, 1, M, N, K, a, a_sf, a_g, b, b_sf,
                                                   b_g, bias, y, ldy, s);
    case MXQ_MXFP8:
      if (N % 192 == 0)
        return launch_gemm_bn<mxq::Fmt::MXFP8, 192>(dev, sms, 2, M, N, K, a, a_sf, a_g, b, b_sf,
                                                     b_g, bias, y, ldy, s);
      return launch_gemm_bn<mxq::Fmt::MXFP8, 128>(dev, sms, 3, M, N, K, a, a_sf, a_g, b, b_sf,
                                                   b_g, bias, y, ldy, s);
    case MXQ_BF16:
      if (M <= mxq::kGemvMaxM) return launch_gemv(sms, M, N, K, a, b, bias, y, ldy, s);
      if (N % 256 == 0)
        return launch_gemm_bn<mxq::Fmt::BF16, 256>(dev, sms, 4, M, N, K, a, a_sf, a_g, b, b_sf,
                                                    b_g, bias, y, ldy, s);
      return launch_gemm_bn<mxq::Fmt::BF16, 128>(dev, sms, 5, M, N, K, a, a_sf, a_g, b, b_sf,
                                                  b_g, bias, y, ldy, s);
  }
  return MXQ_ERR_INVALID_ARG;
}

bool valid_format(int f) { return f == MXQ_NVFP4 || f == MXQ_MXFP8 || f == MXQ_BF16; }

// Byte layout of the weight storage and of the activation workspace:
// [0,4) amax, [4,8) g, then (workspace only) the per-block amax partials at
// [256, 256 + 4 * kMaxAmaxPartials), the single-pass quantiser's barrier
// state (mxq::FusedSync, 256 bytes, then two 128-byte lines per CTA) from 4352, then
// the codes and the scales, each 256-byte aligned.
constexpr size_t kPartialsOff = 256;
constexpr size_t kSyncOff = 4352;
constexpr size_t kWorkspaceHeader = 4352 + 256 + 2 * 128 * 256 + 256;  // 70 KB
static_assert(kPartialsOff + 4 * mxq::kMaxAmaxPartials <= kSyncOff, "workspace header");
static_assert(kSyncOff + sizeof(mxq::FusedSync) + 2 * 8 * mxq::kSyncLine * kFusedMaxGrid <= kWorkspaceHeader,
              "workspace header");
struct QuantLayout {
  size_t codes_off, sf_off, total;
};
QuantLayout quant_layout(int64_t rows, int64_t k, mxq_format f, size_t header = 256) {
  QuantLayout l;
  l.codes_off = header;
  l.sf_off = l.codes_off + static_cast<size_t>(pad_to(mxq_codes_bytes(rows, k, f), 256));
  l.total = l.sf_off + static_cast<size_t>(pad_to(mxq_sf_bytes(rows, k, f), 256));
  return l;
}

// Byte layout of the attention workspace: MXFP8 codes and scales of Q and K
// (rows heads * tokens, 128 channels) and of V^T (rows heads * 128, tokens),
// each part 256-byte aligned.
struct AttLayout {
  size_t q_codes, q_sf, k_codes, k_sf, v_codes, v_sf, total;
};
AttLayout att_layout(int64_t heads, int64_t tokens) {
  AttLayout l;
  const int64_t rows = heads * tokens, vrows = heads * mxq::kAttD;
  size_t off = 0;
  auto take = [&](size_t n) { const size_t o = off; off += static_cast<size_t>(pad_to(static_cast<int64_t>(n), 256)); return o; };
  l.q_codes = take(static_cast<size_t>(rows) * mxq::kAttD);
  l.q_sf = take(mxq_sf_bytes(rows, mxq::kAttD, MXQ_MXFP8));
  l.k_codes = take(static_cast<size_t>(rows) * mxq::kAttD);
  l.k_sf = take(mxq_sf_bytes(rows, mxq::kAttD, MXQ_MXFP8));
  l.v_codes = take(static_cast<size_t>(vrows) * tokens);
  l.v_sf = take(mxq_sf_bytes(vrows, tokens, MXQ_MXFP8));
  l.total = off;
  return l;
}

}  // namespace

// =====================================================================  ABI
extern "C" {

const char* mxq_status_string(mxq_status s) {
  switch (s) {
    case MXQ_OK: return "ok";
    case MXQ_ERR_INVALID_ARG: return "invalid argument";
    case MXQ_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case MXQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MXQ_ERR_WORKSPACE: return "workspace or storage too small";
    case MXQ_ERR_ARCH: return "no sm_100 CUDA device";
    case MXQ_ERR_CUDA: return "CUDA error";
    case MXQ_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int mxq_version(void) { return (1 << 16) | 1; }

int mxq_last_cuda_error(void) { return t_last_cuda_error; }

size_t mxq_sf_bytes(int64_t rows, int64_t k, mxq_format f) {
  if (rows < 0 || k < 0) return 0;
  if (f == MXQ_NVFP4) return static_cast<size_t>(pad_to(rows, 128) * pad_to(k / 16, 4));
  if (f == MXQ_MXFP8) return static_cast<size_t>(pad_to(rows, 128) * pad_to(k / 32, 4));
  return 0;
}

size_t mxq_codes_bytes(int64_t rows, int64_t k, mxq_format f) {
  if (rows < 0 || k < 0) return 0;
  if (f == MXQ_NVFP4) return static_cast<size_t>(rows * k / 2);
  if (f == MXQ_MXFP8) return static_cast<size_t>(rows * k);
  if (f == MXQ_BF16) return static_cast<size_t>(rows * k * 2);
  return 0;
}

mxq_status mxq_amax(const void* x_bf16, int64_t rows, int64_t k, int64_t ld, float* amax_dev,
                    mxq_stream_t stream) {
  if (amax_dev == nullptr) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_bf16_matrix(x_bf16, rows, k, ld);
  if (st != MXQ_OK) return st;
  if (k % 8 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (reinterpret_cast<uintptr_t>(amax_dev) & 3u) return MXQ_ERR_ALIGNMENT;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  return launch_amax(x_bf16, rows, k, ld, amax_dev, reinterpret_cast<cudaStream_t>(stream), sms);
}

mxq_status mxq_quantize_nvfp4(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                              const float* amax_dev, uint8_t* codes, uint8_t* sf_swz,
                              float* g_dev, mxq_stream_t stream) {
  mxq_status st = check_bf16_matrix(x_bf16, rows, k, ld);
  if (st != MXQ_OK) return st;
  if (g_dev == nullptr) return MXQ_ERR_INVALID_ARG;
  if (rows > 0 && k > 0 && (codes == nullptr || sf_swz == nullptr)) return MXQ_ERR_INVALID_ARG;
  if (k % 64 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(codes) || !aligned16(sf_swz)) return MXQ_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(amax_dev) & 3u) || (reinterpret_cast<uintptr_t>(g_dev) & 3u))
    return MXQ_ERR_ALIGNMENT;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  if (rows == 0 || k == 0) return MXQ_OK;
  // no amax: the kernel reduces zero values to amax 0, whose scale is g = 1
  return launch_quant_nvfp4(x_bf16, rows, k, ld, amax_dev, amax_dev != nullptr ? 1 : 0, codes,
                            sf_swz, g_dev, nullptr, reinterpret_cast<cudaStream_t>(stream), sms);
}

mxq_status mxq_quantize_mxfp8(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                              uint8_t* codes, uint8_t* sf_swz, mxq_stream_t stream) {
  return mxq_quantize_mxfp8_rule(x_bf16, rows, k, ld, MXQ_SCALE_FLOOR, codes, sf_swz, stream);
}

mxq_status mxq_quantize_mxfp8_rule(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                                   int scale_rule, uint8_t* codes, uint8_t* sf_swz,
                                   mxq_stream_t stream) {
  if (scale_rule != MXQ_SCALE_FLOOR && scale_rule != MXQ_SCALE_RCEIL) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_bf16_matrix(x_bf16, rows, k, ld);
  if (st != MXQ_OK) return st;
  if (rows > 0 && k > 0 && (codes == nullptr || sf_swz == nullptr)) return MXQ_ERR_INVALID_ARG;
  if (k % 128 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(codes) || !aligned16(sf_swz)) return MXQ_ERR_ALIGNMENT;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  if (rows == 0 || k == 0) return MXQ_OK;
  return launch_quant_mxfp8(x_bf16, rows, k, ld, codes, sf_swz,
                            reinterpret_cast<cudaStream_t>(stream), sms,
                            scale_rule == MXQ_SCALE_RCEIL ? 1 : 0);
}

}  // extern "C"

namespace {

// mxq_gemm_blockscaled with an epilogue (the producer variant for mxq_linear).
mxq_status gemm_checked(mxq_format f, int64_t M, int64_t N, int64_t K, const void* a_codes,
                        const uint8_t* a_sf, const float* a_g_dev, const void* b_codes,
                        const uint8_t* b_sf, const float* b_g_dev, const void* bias_bf16,
                        void* y_bf16, int64_t ldy, mxq_stream_t stream, const Epilogue& ep) {
  if (!valid_format(f)) return MXQ_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K < 0) return MXQ_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (K == 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (f == MXQ_NVFP4 && K % 64 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (f == MXQ_MXFP8 && K % 128 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (f == MXQ_BF16 && K % 8 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (ldy < N || ldy < 1) return MXQ_ERR_INVALID_ARG;
  if (ldy % 8 != 0) return MXQ_ERR_ALIGNMENT;
  const bool nonempty = M > 0 && N > 0;
  if (nonempty) {
    if (a_codes == nullptr || b_codes == nullptr || y_bf16 == nullptr) return MXQ_ERR_INVALID_ARG;
    if (f != MXQ_BF16 && (a_sf == nullptr || b_sf == nullptr)) return MXQ_ERR_INVALID_ARG;
    if (f == MXQ_NVFP4 && (a_g_dev == nullptr || b_g_dev == nullptr)) return MXQ_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(y_bf16)) return MXQ_ERR_ALIGNMENT;
    if (f != MXQ_BF16 && (!aligned16(a_sf) || !aligned16(b_sf))) return MXQ_ERR_ALIGNMENT;
    if (bias_bf16 != nullptr && (reinterpret_cast<uintptr_t>(bias_bf16) & 1u)) return MXQ_ERR_ALIGNMENT;
  }
  int dev, sms;
  mxq_status st;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  if (!nonempty) return MXQ_OK;
  if ((st = get_encoder()) != MXQ_OK) return st;
  return launch_gemm(f, dev, sms, M, N, K, a_codes, a_sf, a_g_dev, b_codes, b_sf, b_g_dev,
                     bias_bf16, y_bf16, ldy, reinterpret_cast<cudaStream_t>(stream), ep);
}

}  // namespace

extern "C" {

mxq_status mxq_gemm_blockscaled(mxq_format f, int64_t M, int64_t N, int64_t K,
                                const void* a_codes, const uint8_t* a_sf, const float* a_g_dev,
                                const void* b_codes, const uint8_t* b_sf, const float* b_g_dev,
                                const void* bias_bf16, void* y_bf16, int64_t ldy,
                                mxq_stream_t stream) {
  return gemm_checked(f, M, N, K, a_codes, a_sf, a_g_dev, b_codes, b_sf, b_g_dev, bias_bf16, y_bf16,
                      ldy, stream, Epilogue{});
}

size_t mxq_weight_storage_bytes(int64_t N, int64_t K, mxq_format f) {
  if (f != MXQ_NVFP4 && f != MXQ_MXFP8) return 0;
  if (N < 0 || K < 0) return 0;
  return quant_layout(N, K, f).total;
}

mxq_status mxq_weight_prepare(mxq_format f, const void* w_bf16, int64_t N, int64_t K,
                              const void* bias_bf16, int flags, void* storage,
                              size_t storage_bytes, mxq_weight* out, mxq_stream_t stream) {
  if (out == nullptr || !valid_format(f)) return MXQ_ERR_INVALID_ARG;
  if (flags & ~(MXQ_WEIGHT_KEEP_BF16 | MXQ_WEIGHT_NO_TENSOR_SCALE | MXQ_WEIGHT_MXFP8_RCEIL))
    return MXQ_ERR_INVALID_ARG;
  const bool keep_bf16 = (flags & MXQ_WEIGHT_KEEP_BF16) != 0;
  const bool no_tensor_scale = (flags & MXQ_WEIGHT_NO_TENSOR_SCALE) != 0;
  const int rceil = (flags & MXQ_WEIGHT_MXFP8_RCEIL) ? 1 : 0;
  if (no_tensor_scale && f != MXQ_NVFP4) return MXQ_ERR_INVALID_ARG;
  if (rceil && f != MXQ_MXFP8) return MXQ_ERR_INVALID_ARG;
  mxq_status st = check_bf16_matrix(w_bf16, N, K, K);
  if (st != MXQ_OK) return st;
  if (bias_bf16 != nullptr && (reinterpret_cast<uintptr_t>(bias_bf16) & 1u)) return MXQ_ERR_ALIGNMENT;
  mxq_weight w;
  std::memset(&w, 0, sizeof(w));
  w.format = f;
  w.flags = flags;
  w.N = N;
  w.K = K;
  w.w_bf16 = w_bf16;
  w.bias_bf16 = bias_bf16;
  const bool quantize = (f != MXQ_BF16) && !keep_bf16;
  if (quantize) {
    if (f == MXQ_NVFP4 && K % 64 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
    if (f == MXQ_MXFP8 && K % 128 != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
    const QuantLayout l = quant_layout(N, K, f);
    if (storage == nullptr) return MXQ_ERR_INVALID_ARG;
    if (!aligned256(storage)) return MXQ_ERR_ALIGNMENT;
    if (storage_bytes < l.total) return MXQ_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(storage);
    float* amax = reinterpret_cast<float*>(base);
    float* g = reinterpret_cast<float*>(base + 4);
    uint8_t* codes = base + l.codes_off;
    uint8_t* sf = base + l.sf_off;
    int dev, sms;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (f == MXQ_NVFP4 && no_tensor_scale) {
      // g_W = 1: the quantiser reduces no amax values (amax 0 -> g = 1) and
      // writes 0 to the amax slot
      if (N > 0 && K > 0 &&
          (st = launch_quant_nvfp4(w_bf16, N, K, K, nullptr, 0, codes, sf, g, amax, s, sms)) != MXQ_OK)
        return st;
      w.g_dev = g;
      w.amax_dev = amax;
    } else if (f == MXQ_NVFP4) {
      if ((st = launch_amax(w_bf16, N, K, K, amax, s, sms)) != MXQ_OK) return st;
      if (N > 0 && K > 0 &&
          (st = launch_quant_nvfp4(w_bf16, N, K, K, amax, 1, codes, sf, g, nullptr, s, sms)) != MXQ_OK)
        return st;
      w.g_dev = g;
      w.amax_dev = amax;
    } else {
      if (N > 0 && K > 0 && (st = launch_quant_mxfp8(w_bf16, N, K, K, codes, sf, s, sms, rceil)) != MXQ_OK)
        return st;
    }
    w.codes = codes;
    w.sf = sf;
  }
  *out = w;
  return MXQ_OK;
}

int mxq_linear_path(const mxq_weight* w, int64_t M, const mxq_linear_opts* opts) {
  if (w == nullptr) return 0;
  const int64_t min_dim = (opts != nullptr && opts->min_dim > 0) ? opts->min_dim : 1024;
  if ((w->flags & MXQ_WEIGHT_KEEP_BF16) || w->format == MXQ_BF16) return MXQ_BF16;
  int64_t m = M < w->K ? M : w->K;
  m = m < w->N ? m : w->N;
  if (m < min_dim) return MXQ_BF16;
  return w->format;
}

size_t mxq_linear_workspace_bytes(int64_t M, int64_t K, mxq_format f) {
  if (f != MXQ_NVFP4 && f != MXQ_MXFP8) return 0;
  if (M < 0 || K < 0) return 0;
  return quant_layout(M, K, f, kWorkspaceHeader).total;
}

mxq_status mxq_linear(const mxq_weight* w, const void* x_bf16, int64_t M, void* y_bf16, void* ws,
                      size_t ws_bytes, const mxq_linear_opts* opts, mxq_stream_t stream) {
  if (w == nullptr || !valid_format(w->format)) return MXQ_ERR_INVALID_ARG;
  const int64_t N = w->N, K = w->K;
  mxq_status st = check_bf16_matrix(x_bf16, M, K, K);
  if (st != MXQ_OK) return st;
  if (M > 0 && N > 0 && y_bf16 == nullptr) return MXQ_ERR_INVALID_ARG;
  if (!aligned16(y_bf16)) return MXQ_ERR_ALIGNMENT;
  if (N % 8 != 0) return MXQ_ERR_ALIGNMENT;  // y rows are N elements apart
  const int path = mxq_linear_path(w, M, opts);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaEvent_t ev0 = nullptr, ev1 = nullptr;
  Epilogue ep;
  const float* x_amax = nullptr;
  if (opts != nullptr) {
    if ((opts->gemm_event_start == nullptr) != (opts->gemm_event_end == nullptr))
      return MXQ_ERR_INVALID_ARG;
    ev0 = static_cast<cudaEvent_t>(opts->gemm_event_start);
    ev1 = static_cast<cudaEvent_t>(opts->gemm_event_end);
    if (opts->activation != MXQ_ACT_NONE && opts->activation != MXQ_ACT_GELU) return MXQ_ERR_INVALID_ARG;
    ep.act = opts->activation;
    ep.y_amax = opts->y_amax_dev;
    x_amax = opts->x_amax_dev;
    if ((reinterpret_cast<uintptr_t>(ep.y_amax) & 3u) || (reinterpret_cast<uintptr_t>(x_amax) & 3u))
      return MXQ_ERR_ALIGNMENT;
    if (ep.y_amax != nullptr && static_cast<const float*>(ep.y_amax) == x_amax) return MXQ_ERR_INVALID_ARG;
  }
  const bool producer = ep.act != MXQ_ACT_NONE || ep.y_amax != nullptr;
  // the producer epilogue lives in the CTA-pair kernel (M > 128) only
  if (producer && M > 0 && M <= 128 && N > 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  // max |y| is folded in with atomicMax: it starts from 0 (also the value for
  // an empty y), set on the stream once every check has passed
  auto zero_y_amax = [&]() -> mxq_status {
    if (ep.y_amax == nullptr) return MXQ_OK;
    const cudaError_t e = cudaMemsetAsync(ep.y_amax, 0, sizeof(float), s);
    return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
  };
  if (path == MXQ_BF16) {
    if (M > 0 && N > 0 && w->w_bf16 == nullptr) return MXQ_ERR_INVALID_ARG;
    if (!aligned16(w->w_bf16)) return MXQ_ERR_ALIGNMENT;
    if (w->bias_bf16 != nullptr && (reinterpret_cast<uintptr_t>(w->bias_bf16) & 1u)) return MXQ_ERR_ALIGNMENT;
    if (K == 0) return MXQ_ERR_UNSUPPORTED_SHAPE;  // as mxq_gemm_blockscaled
    int dev, sms;
    if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
    if ((st = zero_y_amax()) != MXQ_OK) return st;
    cudaError_t e;
    if (ev0 != nullptr && (e = cudaEventRecord(ev0, s)) != cudaSuccess) return cuda_fail(e);
    st = gemm_checked(MXQ_BF16, M, N, K, x_bf16, nullptr, nullptr, w->w_bf16, nullptr, nullptr,
                      w->bias_bf16, y_bf16, N, stream, ep);
    if (st == MXQ_OK && ev1 != nullptr && (e = cudaEventRecord(ev1, s)) != cudaSuccess)
      return cuda_fail(e);
    return st;
  }
  const mxq_format f = static_cast<mxq_format>(path);
  if (w->codes == nullptr || w->sf == nullptr) return MXQ_ERR_INVALID_ARG;
  if (f == MXQ_NVFP4 && w->g_dev == nullptr) return MXQ_ERR_INVALID_ARG;
  const QuantLayout l = quant_layout(M, K, f, kWorkspaceHeader);
  if (ws == nullptr) return MXQ_ERR_INVALID_ARG;
  if (!aligned256(ws)) return MXQ_ERR_ALIGNMENT;
  if (ws_bytes < l.total) return MXQ_ERR_WORKSPACE;
  int dev, sms;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  if ((st = zero_y_amax()) != MXQ_OK) return st;
  if (M == 0 || N == 0) return MXQ_OK;
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* amax = reinterpret_cast<float*>(base);
  float* g = reinterpret_cast<float*>(base + 4);
  uint8_t* codes = base + l.codes_off;
  uint8_t* sf = base + l.sf_off;
  if (f == MXQ_NVFP4 && (w->flags & MXQ_WEIGHT_NO_TENSOR_SCALE)) {
    // no per-tensor scale: one pass, g = 1 (no amax values to reduce)
    if ((st = launch_quant_nvfp4(x_bf16, M, K, K, nullptr, 0, codes, sf, g, amax, s, sms)) != MXQ_OK)
      return st;
  } else if (f == MXQ_NVFP4 && x_amax != nullptr) {
    // the input's amax is known (e.g. from the producing layer's epilogue): one pass
    if ((st = launch_quant_nvfp4(x_bf16, M, K, K, x_amax, 1, codes, sf, g, amax, s, sms)) != MXQ_OK)
      return st;
  } else if (f == MXQ_NVFP4) {
    float* partials = reinterpret_cast<float*>(base + kPartialsOff);
    const FusedPlan plan = plan_fused(M, K, sms);
    if (plan.grid > 0) {
      // the activation fits in shared memory: one pass over HBM
      st = launch_quant_nvfp4_fused(x_bf16, M, K, K, plan,
                                    reinterpret_cast<mxq::FusedSync*>(base + kSyncOff), codes, sf,
                                    g, amax, s, dev);
      if (st != MXQ_OK) return st;
    } else {
      int n_partials = 0;
      if ((st = launch_amax_partials(x_bf16, M, K, K, partials, &n_partials, s, sms)) != MXQ_OK)
        return st;
      if ((st = launch_quant_nvfp4(x_bf16, M, K, K, partials, n_partials, codes, sf, g, amax, s,
                                   sms)) != MXQ_OK)
        return st;
    }
  } else {
    const int rceil = (w->flags & MXQ_WEIGHT_MXFP8_RCEIL) ? 1 : 0;
    if ((st = launch_quant_mxfp8(x_bf16, M, K, K, codes, sf, s, sms, rceil)) != MXQ_OK) return st;
  }
  if ((st = get_encoder()) != MXQ_OK) return st;
  cudaError_t e;
  if (ev0 != nullptr && (e = cudaEventRecord(ev0, s)) != cudaSuccess) return cuda_fail(e);
  st = launch_gemm(f, dev, sms, M, N, K, codes, sf, g, w->codes, w->sf, w->g_dev, w->bias_bf16,
                   y_bf16, N, s, ep);
  if (st == MXQ_OK && ev1 != nullptr && (e = cudaEventRecord(ev1, s)) != cudaSuccess)
    return cuda_fail(e);
  return st;
}

int mxq_linear_kernel_count(const mxq_weight* w, int64_t M, const mxq_linear_opts* opts) {
  if (w == nullptr || M <= 0 || w->N <= 0) return 0;
  const int path = mxq_linear_path(w, M, opts);
  if (path == MXQ_BF16) return 1;
  if (path == MXQ_MXFP8 || (w->flags & MXQ_WEIGHT_NO_TENSOR_SCALE)) return 2;
  if (opts != nullptr && opts->x_amax_dev != nullptr) return 2;
  int dev, sms;
  if (current_device(&dev, &sms) != MXQ_OK) return -1;
  return plan_fused(M, w->K, sms).grid > 0 ? 2 : 3;
}

size_t mxq_attention_workspace_bytes(int64_t heads, int64_t tokens, int64_t d) {
  if (heads <= 0 || tokens <= 0 || d != mxq::kAttD) return 0;
  return att_layout(heads, tokens).total;
}

mxq_status mxq_attention_mxfp8(const void* q, const void* k, const void* v, int64_t heads,
                               int64_t tokens, int64_t d, float tau, void* out, void* ws,
                               size_t ws_bytes, mxq_stream_t stream) {
  if (heads < 0 || tokens < 0) return MXQ_ERR_INVALID_ARG;
  if (d != mxq::kAttD) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (heads == 0 || tokens == 0) return MXQ_OK;
  if (tokens % mxq::kAttTile != 0) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (heads * tokens > INT32_MAX / 2 || heads * tokens * d > (int64_t(1) << 40)) return MXQ_ERR_UNSUPPORTED_SHAPE;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || ws == nullptr) return MXQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MXQ_ERR_ALIGNMENT;
  if (!aligned256(ws)) return MXQ_ERR_ALIGNMENT;
  const AttLayout l = att_layout(heads, tokens);
  if (ws_bytes < l.total) return MXQ_ERR_WORKSPACE;
  if (!(tau > 0.0f) || !(tau < INFINITY)) tau = 1.0f / sqrtf(static_cast<float>(d));
  int dev, sms;
  mxq_status st;
  if ((st = current_device(&dev, &sms)) != MXQ_OK) return st;
  if ((st = get_encoder()) != MXQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int64_t rows = heads * tokens;
  // per-token MXFP8 of Q and K (rows of 128 channels), V^T along tokens
  if ((st = launch_quant_mxfp8(q, rows, d, d, base + l.q_codes, base + l.q_sf, s, sms)) != MXQ_OK) return st;
  if ((st = launch_quant_mxfp8(k, rows, d, d, base + l.k_codes, base + l.k_sf, s, sms)) != MXQ_OK) return st;
  const int grid = static_cast<int>(heads * (tokens / mxq::kAttTile));
  cudaError_t e = launch_pdl(mxq::quantize_mxfp8_vt_kernel, dim3(grid), dim3(mxq::kVtThreads), 0, s,
                             static_cast<const __nv_bfloat16*>(v), static_cast<int>(heads),
                             static_cast<int>(tokens), base + l.v_codes, base + l.v_sf);
  if (e != cudaSuccess) return cuda_fail(e);
  constexpr uint32_t bit = 1u << 21;  // GEMM instantiations and the fused quantiser use lower bits
  if (!(g_dev[dev].smem_attr_set.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(mxq::attention_mxfp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             mxq::AttCfg::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_fail(e);
    g_dev[dev].smem_attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  CUtensorMap tq, tk, tv;
  if ((st = tmap_2d(&tq, base + l.q_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, d, rows, d, 128, mxq::kAttTile,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != MXQ_OK)
    return st;
  if ((st = tmap_2d(&tk, base + l.k_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, d, rows, d, 128, mxq::kAttTile,
                    CU_TENSOR_MAP_SWIZZLE_128B)) != MXQ_OK)
    return st;
  if ((st = tmap_2d(&tv, base + l.v_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, tokens, heads * d, tokens, 128,
                    mxq::kAttD, CU_TENSOR_MAP_SWIZZLE_128B)) != MXQ_OK)
    return st;
  mxq::AttArgs args;
  args.heads = static_cast<int>(heads);
  args.tokens = static_cast<int>(tokens);
  args.c = tau * 1.4426950408889634f;  // tau * log2(e): the weights are powers of two
  args.q_sf = base + l.q_sf;
  args.k_sf = base + l.k_sf;
  args.v_sf = base + l.v_sf;
  args.out = static_cast<__nv_bfloat16*>(out);
  e = launch_pdl(mxq::attention_mxfp8_kernel, dim3(grid), dim3(mxq::AttCfg::THREADS), mxq::AttCfg::SMEM_BYTES, s,
                 tq, tk, tv, args);
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

mxq_status mxq_get_device_error(mxq_stream_t stream) {
  int dev, sms;
  mxq_status st = current_device(&dev, &sms);
  if (st != MXQ_OK) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, mxq::g_device_error, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e);
  if (v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(mxq::g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
    return MXQ_ERR_TIMEOUT;
  }
  return MXQ_OK;
}

mxq_status mxq_convert_f32(const float* in, int64_t n, int code_fmt, uint8_t* out,
                           mxq_stream_t stream) {
  if (n < 0 || (code_fmt != 1 && code_fmt != 2)) return MXQ_ERR_INVALID_ARG;
  if (n > 0 && (in == nullptr || out == nullptr)) return MXQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(in) & 3u) return MXQ_ERR_ALIGNMENT;
  int dev, sms;
  mxq_status st = current_device(&dev, &sms);
  if (st != MXQ_OK) return st;
  if (n == 0) return MXQ_OK;
  int64_t blocks = (n + 255) / 256;
  if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
  mxq::convert_kernel<<<static_cast<int>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      in, n, code_fmt, out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MXQ_OK : cuda_fail(e);
}

}  // extern "C"

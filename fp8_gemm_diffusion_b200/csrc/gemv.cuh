// gemv.cuh - the selective rule's bf16 layer at a handful of rows.
//
// Y = bf16(X W^T + bias) for M <= 8 rows of X (the modulation layers of a
// FLUX-shaped DiT run at M = batch).  The layer is a stream of W (N x K bf16)
// with M multiply-adds per weight: far below the tensor cores' rate, and a
// 128-row MMA tile would be at least 120 rows of padding.  So it runs on the
// CUDA cores, every SM streaming its own rows of W:
//   one warp per RW = 4 (M <= 2) or 2 consecutive rows of W at a time, each
//   lane taking 8-element chunks k = 8 (lane + 32 i) of those rows (16-byte loads,
//   a warp reading 512 contiguous bytes of a row per step, two steps in
//   flight), X's matching chunks from L1 (all warps read the same X), fp32
//   multiply-adds, a butterfly reduction across the warp, then bias and the
//   bf16 rounding; lane r * MB + m writes Y[m][n0 + r].
// Accumulation order differs from the tensor-core path; both are fp32.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace mxq {

constexpr int kGemvThreads = 256;
// rows of W per warp task: 4 for one or two rows of X, 2 beyond (fewer
// accumulators, so that more warps stay resident to keep loads in flight)
template <int MB>
__host__ __device__ constexpr int gemv_rows() { return MB <= 2 ? 4 : 2; }
constexpr int kGemvMaxM = 8;

// 8 bf16 in a 16-byte vector -> fp32 (element 2i of a word in its low half).
__device__ __forceinline__ void gemv_unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int MB>
__global__ void __launch_bounds__(kGemvThreads)
    gemv_bf16_kernel(const __nv_bfloat16* __restrict__ x, int M, int K, const __nv_bfloat16* __restrict__ w,
                     int N, const __nv_bfloat16* __restrict__ bias, __nv_bfloat16* __restrict__ y,
                     int64_t ldy) {
  grid_dep_wait();  // X may be the previous kernel's output
  grid_dep_launch();
  constexpr int RW = gemv_rows<MB>();
  const int lane = threadIdx.x & 31;
  const int64_t warp_g = (static_cast<int64_t>(blockIdx.x) * kGemvThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kGemvThreads / 32);
  const int kc = K >> 3;  // 8-element chunks per row
  for (int64_t n0 = warp_g * RW; n0 < N; n0 += nwarps * RW) {
    float acc[RW][MB];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[r][m] = 0.0f;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int c0 = lane; c0 < kc; c0 += 64) {
      // two steps of the four rows in flight, then X's chunks
      uint4 wv[2][RW];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int c = c0 + 32 * s;
#pragma unroll
        for (int r = 0; r < RW; ++r)
          wv[s][r] = (c < kc && n0 + r < N) ? ldg_nc_v4(w + (n0 + r) * static_cast<int64_t>(K) + 8 * c) : zero;
      }
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int c = c0 + 32 * s;
        if (c >= kc) break;  // the loads above are guarded the same way
        float wf[RW][8];  // the rows' chunks, unpacked once for all rows of X
#pragma unroll
        for (int r = 0; r < RW; ++r) gemv_unpack8(wv[s][r], wf[r]);
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          if (m >= M) break;
          float xf[8];
          gemv_unpack8(ldg_nc_v4_l1(x + static_cast<int64_t>(m) * K + 8 * c), xf);
#pragma unroll
          for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r][m] = fmaf(wf[r][e], xf[e], acc[r][m]);
        }
      }
    }
    // butterfly: every lane ends with every sum
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int m = 0; m < MB; ++m)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], o);
#pragma unroll
    for (int r = 0; r < RW; ++r) {
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        if (lane == r * MB + m && m < M && n0 + r < N) {
          float v = acc[r][m];
          if (bias != nullptr) v += __bfloat162float(bias[n0 + r]);
          y[static_cast<int64_t>(m) * ldy + n0 + r] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

}  // namespace mxq

// quant.cuh - dynamic activation quantisation kernels (HBM-bound).
//
//   amax_kernel           max |x| of a bf16 matrix -> one fp32 (atomicMax on
//                         the bit pattern, valid because |x| >= 0)
//   quantize_nvfp4_kernel per 16-element block: E4M3 scale, E2M1 codes
//   quantize_mxfp8_kernel per 32-element block: E8M0 scale, E4M3 codes
//
// Source: B200 MXFP8/NVFP4 diffusion article, Glossary "Microscaling
// Formats" (16-32 element blocks share a scale), "MXFP8" (OCP MX 8-bit),
// "NVFP4" (Blackwell 4-bit float); the TorchAO listing in "Detailed by
// section" (use_dynamic_per_tensor_scale: per-tensor fp32 scale from amax,
// recomputed on every call).  Arithmetic (fp32, round-to-nearest-even,
// subnormals kept; no fast-math anywhere in this library):
//   NVFP4: g = amax/2688 (1 if amax == 0); sf = E4M3(bamax/(6g));
//          s = value(sf)*g; code = E2M1(x * (1/s)), 0 when s == 0.
//   MXFP8: X = clamp(floor(log2 bamax) - 8, -127, 127) (-127 for a zero
//          block); sf = X + 127; code = E4M3(x * 2^-X).
// Conversions use the hardware cvt.rn.satfinite instructions (RNE, finite
// overflow saturates to the largest magnitude, sign kept).
//
// Memory layout: each thread owns one 16-byte vector (8 bf16) of a row; the
// 2 (NVFP4) or 4 (MXFP8) lanes of a block combine their maxima with warp
// shuffles; a warp reads 512 contiguous bytes per vector load.  Scale bytes
// go straight to the tensor-core block-scaling layout (see sf_offset).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace mxq {

// Byte offset of scale (row r, scale column c) in the block-scaling layout:
// 512-byte tiles of 128 rows x 4 columns, tile = (r/128)*(C4) + c/4 where C4
// is the number of 4-column groups; inside: (r%32)*16 + ((r/32)%4)*4 + c%4.
__device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t c4) {
  const int64_t tile = (r >> 7) * c4 + (c >> 2);
  return tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// --------------------------------------------------------------- converts
// Two fp32 -> two E4M3 bytes; `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Eight fp32 -> eight E2M1 nibbles packed into 32 bits; v[0] in bits 0-3.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// One fp32 -> one E2M1 code in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1(float x) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.u32.u8 %0, b0;\n\t}"
      : "=r"(r)
      : "f"(x), "f"(0.0f));
  return r & 0xFu;
}

// Value of a non-negative E4M3 code (0x00..0x7E), exactly: e == 0 gives the
// subnormal m * 2^-9, otherwise (1 + m/8) * 2^(e-7).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xFu;
  const uint32_t m = code & 0x7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));     // bias 127 - 7
}

// floor(log2(a)) of a positive finite fp32, exactly, from its bits.
__device__ __forceinline__ int floor_log2_f32(float a) {
  const uint32_t b = __float_as_uint(a);
  const uint32_t ex = (b >> 23) & 0xFFu;
  if (ex != 0) return static_cast<int>(ex) - 127;
  return -118 - static_cast<int>(__clz(b & 0x7FFFFFu));  // subnormal: mant * 2^-149
}

// 2^p as fp32 for p in [-127, 127], exactly (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int p) {
  if (p >= -126) return __uint_as_float(static_cast<uint32_t>(p + 127) << 23);
  return __uint_as_float(0x00400000u);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float absmax8(const float (&v)[8]) {
  float m = fabsf(v[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ------------------------------------------------------------------- amax
// Work split: one warp per row (rows strided over all warps of the grid); a
// lane owns every 32nd 16-byte vector of the row, four loads in flight.  No
// integer division anywhere on the path.
constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;
constexpr int kMaxAmaxPartials = 1024;

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// Block-wide max of `m` (every thread gets it).
__device__ __forceinline__ float block_max(float m) {
  __shared__ float s_max[kQuantThreads / 32];
  m = warp_max(m);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
  __syncthreads();
  float b = s_max[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) b = fmaxf(b, s_max[i]);
  return b;
}

// max |x| of the rows this block's warps own, written to partial[blockIdx.x]
// (or folded into *amax_atomic with atomicMax when partial is null).
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                             int rows, int k, int64_t ld,
                                                             float* __restrict__ partial,
                                                             float* __restrict__ amax_atomic) {
  grid_dep_wait();  // x may be the previous kernel's output
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kQuantThreads / 32);
  const int vpr = k >> 3;  // 16-byte vectors per row
  float m = 0.0f;
  for (int r = blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const __nv_bfloat16* row = x + static_cast<int64_t>(r) * ld;
    for (int v0 = lane; v0 < vpr; v0 += 32 * kQuantUnroll) {
      uint4 u[kQuantUnroll];
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int v = v0 + 32 * j;
        u[j] = v < vpr ? ldg_nc_v4(row + v * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        float f[8];
        bf16x8_to_f32(u[j], f);
        m = fmaxf(m, absmax8(f));
      }
    }
  }
  m = block_max(m);
  if (threadIdx.x == 0) {
    if (partial != nullptr) {
      partial[blockIdx.x] = m;
    } else {
      // non-negative floats order like their bit patterns
      atomicMax(reinterpret_cast<unsigned int*>(amax_atomic), __float_as_uint(m));
    }
  }
}

// -------------------------------------------------------------- NVFP4
__device__ __forceinline__ float nvfp4_global_scale(float amax) {
  return amax == 0.0f ? 1.0f : amax / 2688.0f;  // IEEE division (no fast-math)
}

// Zero the scale bytes of padding rows [rows, pad128(rows)).
__device__ __forceinline__ void zero_sf_padding(uint8_t* __restrict__ sf, int rows, int c) {
  const int rp = (rows + 127) / 128 * 128;
  const int total = (rp - rows) * c;
  const int c4 = c >> 2;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
    const int r = rows + t / c, cc = t - (t / c) * c;
    sf[sf_offset(r, cc, c4)] = 0;
  }
}

// amax_in: n_amax values whose max is the tensor's amax (1 value, or the
// per-block partials of amax_kernel).
__global__ void __launch_bounds__(kQuantThreads)
    quantize_nvfp4_kernel(const __nv_bfloat16* __restrict__ x, int rows, int k, int64_t ld,
                          const float* __restrict__ amax_in, int n_amax, uint8_t* __restrict__ codes,
                          uint8_t* __restrict__ sf, float* __restrict__ g_out,
                          float* __restrict__ amax_out) {
  grid_dep_wait();  // the amax (partials) comes from the previous kernel
  grid_dep_launch();
  float a = 0.0f;
  for (int i = threadIdx.x; i < n_amax; i += kQuantThreads) a = fmaxf(a, amax_in[i]);
  a = block_max(a);
  const float g = nvfp4_global_scale(a);
  const float six_g = 6.0f * g;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *g_out = g;
    if (amax_out != nullptr) *amax_out = a;
  }
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kQuantThreads / 32);
  const int vpr = k >> 3;  // even: k is a multiple of 16
  const int c4 = k >> 6;   // 4-column scale groups per row
  for (int r = blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const __nv_bfloat16* row = x + static_cast<int64_t>(r) * ld;
    uint32_t* crow = reinterpret_cast<uint32_t*>(codes + static_cast<int64_t>(r) * (k >> 1));
    for (int v0 = lane; v0 - lane < vpr; v0 += 32 * kQuantUnroll) {
      uint4 u[kQuantUnroll];
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int v = v0 + 32 * j;
        u[j] = v < vpr ? ldg_nc_v4(row + v * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int v = v0 + 32 * j;
        if (v - lane >= vpr) break;  // warp-uniform
        float f[8];
        bf16x8_to_f32(u[j], f);
        float bmax = absmax8(f);
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));  // 16-element block
        const uint32_t sfc = cvt_e4m3x2(bmax / six_g, 0.0f) & 0xFFu;
        const float s = e4m3_value(sfc) * g;
        const float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = f[i] * inv;
        const uint32_t packed = cvt_e2m1x8(f);
        if (v < vpr) {
          crow[v] = packed;
          if ((v & 1) == 0) sf[sf_offset(r, v >> 1, c4)] = static_cast<uint8_t>(sfc);
        }
      }
    }
  }
  zero_sf_padding(sf, rows, k >> 4);
}

// -------------------------------------------------------------- MXFP8
__global__ void __launch_bounds__(kQuantThreads)
    quantize_mxfp8_kernel(const __nv_bfloat16* __restrict__ x, int rows, int k, int64_t ld,
                          uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kQuantThreads / 32);
  const int vpr = k >> 3;  // multiple of 16: k is a multiple of 128
  const int c4 = k >> 7;
  for (int r = blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const __nv_bfloat16* row = x + static_cast<int64_t>(r) * ld;
    uint2* crow = reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * k);
    for (int v0 = lane; v0 - lane < vpr; v0 += 32 * kQuantUnroll) {
      uint4 u[kQuantUnroll];
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int v = v0 + 32 * j;
        u[j] = v < vpr ? ldg_nc_v4(row + v * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int v = v0 + 32 * j;
        if (v - lane >= vpr) break;  // warp-uniform
        float f[8];
        bf16x8_to_f32(u[j], f);
        float bmax = absmax8(f);
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
        bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 2));  // 32-element block
        int X = -127;
        if (bmax > 0.0f) X = min(max(floor_log2_f32(bmax) - 8, -127), 127);
        const float mult = exp2_int(-X);
        uint2 out;
        out.x = cvt_e4m3x2(f[0] * mult, f[1] * mult) | (cvt_e4m3x2(f[2] * mult, f[3] * mult) << 16);
        out.y = cvt_e4m3x2(f[4] * mult, f[5] * mult) | (cvt_e4m3x2(f[6] * mult, f[7] * mult) << 16);
        if (v < vpr) {
          crow[v] = out;
          if ((v & 3) == 0) sf[sf_offset(r, v >> 2, c4)] = static_cast<uint8_t>(X + 127);
        }
      }
    }
  }
  zero_sf_padding(sf, rows, k >> 5);
}

// ----------------------------------------------- conversion check kernel
__global__ void convert_kernel(const float* __restrict__ in, int64_t n, int fmt,
                               uint8_t* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = in[i];
    out[i] = static_cast<uint8_t>(fmt == 1 ? cvt_e2m1(v) : (cvt_e4m3x2(v, 0.0f) & 0xFFu));
  }
}

}  // namespace mxq

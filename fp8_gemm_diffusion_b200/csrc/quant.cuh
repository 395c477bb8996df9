// quant.cuh - dynamic activation quantisation kernels (HBM-bound).
//
//   amax_kernel           max |x| of a bf16 matrix -> one fp32 (atomicMax on
//                         the bit pattern, valid because |x| >= 0)
//   quantize_nvfp4_kernel per 16-element block: E4M3 scale, E2M1 codes
//   quantize_nvfp4_fused_kernel  both of the above in one pass, for an
//                         activation that fits in the grid's shared memory
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
// Work split: the amax and NVFP4 passes deal fixed-size row chunks to warps
// (ChunkWalk); NVFP4 encodes one 16-element block per lane (two 16-byte
// loads), so the block's scale arithmetic runs once per block.  MXFP8: one
// thread per 32-element block, consecutive threads on consecutive blocks.
// Scale bytes go straight to the tensor-core block-scaling layout (see
// sf_offset).
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

// Same, allocating in L1: for a lane that reads both 16-byte halves of a
// 32-byte sector with two loads, the second is served by L1.
__device__ __forceinline__ uint4 ldg_nc_v4_l1(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 16 bf16 (two 16-byte vectors) -> fp32, element 2i of a word in its low half.
__device__ __forceinline__ void bf16x16_to_f32(const uint4& u0, const uint4& u1, float (&f)[16]) {
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ------------------------------------------------------------------- amax
// A warp's chunk is 32 x kQuantUnroll consecutive 16-byte vectors of a row:
// lane l loads vectors l, l + 32, ..., four loads in flight.
constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;
constexpr int kAmaxChunk = 32 * kQuantUnroll * 8;    // elements per chunk of the amax pass
constexpr int kNvfp4Chunk = 32 * kQuantUnroll * 16;  // elements per chunk of the NVFP4 pass
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

// Work split of the two-pass kernels: each row is cut into chunks of a fixed
// number of vectors (32 lanes x kQuantUnroll), and the chunks of all rows are
// dealt to the warps in turn, so every warp gets the same share to within one
// chunk.  (With whole rows per warp, 16896 rows on 8192 warps left a third
// round of rows to 512 warps, which could not keep HBM busy: ~12 us of the
// amax pass's 73 us.)  The walk advances (row, chunk) by the grid's warp count
// without a division per step.
// (Rows are below 2^31 and a step adds at most the grid's warp count, 8192,
// to the row, so the unsigned row never wraps before it passes the last row.)
struct ChunkWalk {
  unsigned int r;    // row
  unsigned int c;    // chunk within the row
  unsigned int dr;   // rows per step
  unsigned int dc;   // chunks per step beyond whole rows
  unsigned int cpr;  // chunks per row
  __device__ __forceinline__ ChunkWalk(unsigned int first, unsigned int step, unsigned int chunks_per_row)
      : r(first / chunks_per_row), c(first % chunks_per_row), dr(step / chunks_per_row),
        dc(step % chunks_per_row), cpr(chunks_per_row) {}
  __device__ __forceinline__ void next() {
    r += dr;
    c += dc;
    if (c >= cpr) {
      c -= cpr;
      ++r;
    }
  }
};

// max |x| of the chunks this block's warps own, written to partial[blockIdx.x]
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
  const int cpr = (vpr + 32 * kQuantUnroll - 1) / (32 * kQuantUnroll);  // chunks per row
  float m = 0.0f;
  if (cpr > 0) {
    for (ChunkWalk w(blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5), warps, cpr);
         w.r < static_cast<unsigned int>(rows); w.next()) {
      const __nv_bfloat16* row = x + static_cast<int64_t>(w.r) * ld;
      const int v0 = static_cast<int>(w.c) * (32 * kQuantUnroll) + lane;
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

// One 16-element block held by one lane (so the block-level steps -- the
// division, the E4M3 scale, the reciprocal -- run once per block).  Returns
// the 16 E2M1 codes (element 2i in the low nibble of byte i); sfc receives
// the block's E4M3 scale code.
__device__ __forceinline__ uint2 nvfp4_block16(float (&f)[16], float g, float six_g,
                                               uint32_t& sfc) {
  float bmax = fabsf(f[0]);
#pragma unroll
  for (int i = 1; i < 16; ++i) bmax = fmaxf(bmax, fabsf(f[i]));
  sfc = cvt_e4m3x2(bmax / six_g, 0.0f) & 0xFFu;
  const float s = e4m3_value(sfc) * g;
  const float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = f[i] * inv;
    hi[i] = f[8 + i] * inv;
  }
  return make_uint2(cvt_e2m1x8(lo), cvt_e2m1x8(hi));
}

constexpr unsigned long long kKeyMask = 0xFFFFFFFF00000000ull;

// amax_in: n_amax values whose max is the tensor's amax (1 value, or the
// per-block partials of amax_kernel).
__global__ void __launch_bounds__(kQuantThreads, 4)
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
  const int bpr = k >> 4;  // 16-element blocks per row, one per lane per step
  const int cpr = (bpr + 32 * kQuantUnroll - 1) / (32 * kQuantUnroll);  // chunks per row
  const uint32_t c4 = static_cast<uint32_t>(k >> 6);  // 4-column scale groups per row
  // rows last to first: the amax pass just before read them first to last,
  // so the tail of the activation is still in L2 when this pass starts, and
  // the rows this pass writes last (the first ones) are where the GEMM begins
  if (cpr > 0) {
    for (ChunkWalk w(blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5), warps, cpr);
         w.r < static_cast<unsigned int>(rows); w.next()) {
      const int r = rows - 1 - static_cast<int>(w.r);
      const __nv_bfloat16* row = x + static_cast<int64_t>(r) * ld;
      uint2* crow = reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * (k >> 1));
      // this row's scale bytes: 512-byte tile (r / 128, c / 4), byte (r % 32) * 16 + (r / 32 % 4) * 4 + c % 4
      uint8_t* sf_row = sf + static_cast<int64_t>(r >> 7) * c4 * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
      const int c0 = static_cast<int>(w.c) * (32 * kQuantUnroll) + lane;
      uint4 u[kQuantUnroll][2];
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int c = c0 + 32 * j;
        if (c < bpr) {
          u[j][0] = ldg_nc_v4_l1(row + 16 * c);
          u[j][1] = ldg_nc_v4_l1(row + 16 * c + 8);
        } else {
          u[j][0] = u[j][1] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int j = 0; j < kQuantUnroll; ++j) {
        const int c = c0 + 32 * j;
        if (c >= bpr) break;
        float f[16];
        bf16x16_to_f32(u[j][0], u[j][1], f);
        uint32_t sfc;
        crow[c] = nvfp4_block16(f, g, six_g, sfc);
        sf_row[(c >> 2) * 512 + (c & 3)] = static_cast<uint8_t>(sfc);
      }
    }
  }
  zero_sf_padding(sf, rows, k >> 4);
}

// ------------------------------------------------ NVFP4 in a single pass
// For an activation that fits in the grid's shared memory.  Each CTA copies
// its rows into shared memory once (bulk copies, one mbarrier per row), takes
// their maximum, the CTAs exchange maxima through a grid-wide barrier, and
// each CTA quantises its rows from shared memory: the activation crosses HBM
// once instead of twice, and one launch replaces two.
//
// Grid barrier, state in caller memory with any initial contents
// (FusedSync below, then tags[grid], then done[grid], one 128-byte line per
// word, so that no line is polled by more than one CTA).  Every exchanged
// word is 64 bits, written and read whole (single-copy atomic), so no fences
// are needed:
//   key     (epoch & 0xffff) << 48 | (~epoch & 0xffff) << 32, where epoch is
//           read by every CTA at entry and advanced by CTA 0 once all CTAs
//           have arrived (so no CTA reads the advanced value in the same
//           launch).  Zeroed or byte-filled memory never matches a key (its
//           two halves are not complements);
//   tags[b] key | bits(maximum of CTA b), its arrival;
//   done[b] key | bits(amax), CTA b's copy of the result: CTA 0 waits for
//           every tag, writes every CTA's copy and clears the tags; CTA b
//           waits on its own copy and clears it once read.  (With every CTA
//           on one shared word, and the tags packed into a few lines, the
//           polling itself slowed the exchange to several microseconds.)
// The launch is cooperative (all CTAs resident together) and every wait is
// bounded: on timeout the CTA records kErrTimeout and leaves its rows
// unquantised (CTA 0 still advances the epoch, so a later launch never
// matches a word of this one).
constexpr int kFusedThreads = 1024;
constexpr int kFusedWarps = kFusedThreads / 32;

constexpr int kSyncLine = 16;      // 64-bit words per 128-byte line

struct FusedSync {                 // 256 bytes, then tags[grid] and done[grid], a line each
  unsigned int epoch;
  unsigned int pad0;
  unsigned long long done;
  unsigned int pad1[60];
};
static_assert(sizeof(FusedSync) == 256, "FusedSync layout");

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Relaxed loads: independent, so a lane keeps several in flight at once.
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned int ld_relaxed_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

// Bounded spin until the word's upper half equals `key`; its lower half out.
__device__ __forceinline__ bool spin_for_key(const unsigned long long* p, unsigned long long key,
                                             uint32_t& value) {
  const uint64_t t0 = globaltimer_ns();
  unsigned long long w;
  while (((w = ld_relaxed_u64(p)) & kKeyMask) != key) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  value = static_cast<uint32_t>(w);
  return true;
}

// Dynamic shared memory: rows_per_cta rows of k bf16, then one mbarrier per row.
__global__ void __launch_bounds__(kFusedThreads, 1)
    quantize_nvfp4_fused_kernel(const __nv_bfloat16* __restrict__ x, int rows, int k, int64_t ld,
                                int rows_per_cta, FusedSync* sync, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
                                float* __restrict__ g_out, float* __restrict__ amax_out) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_red[kFusedWarps];
  __shared__ float s_amax;
  __shared__ unsigned int s_epoch;
  __shared__ int s_ok;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t row_bytes = static_cast<uint32_t>(k) * 2u;
  const uint32_t rows_s = smem_u32(smem);
  const uint32_t bar0 = rows_s + static_cast<uint32_t>(rows_per_cta) * row_bytes;
  const int r0 = blockIdx.x * rows_per_cta;
  const int nr = min(rows_per_cta, rows - r0);
  const int vpr = k >> 3;  // 16-byte vectors per row
  unsigned long long* const tags = reinterpret_cast<unsigned long long*>(sync + 1);
  unsigned long long* const done = tags + static_cast<size_t>(gridDim.x) * kSyncLine;

  grid_dep_wait();  // x is the previous kernel's output
  if (threadIdx.x == 0) {
    s_epoch = ld_relaxed_u32(&sync->epoch);
    for (int i = 0; i < nr; ++i) mbar_init(bar0 + 8u * i, 1);
    fence_barrier_init();
    for (int i = 0; i < nr; ++i) {
      mbar_arrive_expect_tx(bar0 + 8u * i, row_bytes);
      bulk_load(rows_s + static_cast<uint32_t>(i) * row_bytes, x + static_cast<int64_t>(r0 + i) * ld,
                row_bytes, bar0 + 8u * i);
    }
  }
  __syncthreads();
  grid_dep_launch();

  // ---- this CTA's maximum, row by row as the rows land
  float m = 0.0f;
  for (int i = warp; i < nr; i += kFusedWarps) {
    mbar_wait_bounded(bar0 + 8u * i, 0);
    const uint32_t row = rows_s + static_cast<uint32_t>(i) * row_bytes;
    for (int v = lane; v < vpr; v += 32) {
      float f[8];
      bf16x8_to_f32(lds_v4(row + 16u * v), f);
      m = fmaxf(m, absmax8(f));
    }
  }
  m = warp_max(m);
  if (lane == 0) s_red[warp] = m;
  __syncthreads();

  // ---- grid barrier: arrive, CTA 0 gathers and publishes, everyone reads
  const uint32_t e16 = s_epoch & 0xFFFFu;
  const unsigned long long key =
      (static_cast<unsigned long long>(e16) << 48) | (static_cast<unsigned long long>(~e16 & 0xFFFFu) << 32);
  if (warp == 0) {
    float b = lane < kFusedWarps ? s_red[lane] : 0.0f;
    b = warp_max(b);
    if (lane == 0) st_relaxed_u64(tags + blockIdx.x * kSyncLine, key | __float_as_uint(b));
    __syncwarp();
    bool ok = true;
    if (blockIdx.x == 0) {
      const int nb = gridDim.x;
      const uint64_t t0 = globaltimer_ns();
      float a = 0.0f;
      while (true) {
        bool mine = true;
        a = 0.0f;
        for (int c = lane; c < nb; c += 32) {
          const unsigned long long w = ld_relaxed_u64(tags + c * kSyncLine);
          mine &= (w & kKeyMask) == key;
          a = fmaxf(a, __uint_as_float(static_cast<uint32_t>(w)));
        }
        if (__all_sync(0xffffffffu, mine)) break;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
      a = warp_max(a);
      for (int c = lane; c < nb; c += 32) {
        if (ok) st_relaxed_u64(done + c * kSyncLine, key | __float_as_uint(a));
        st_relaxed_u64(tags + c * kSyncLine, 0ull);
      }
      if (lane == 0) sync->epoch = s_epoch + 1u;  // every CTA read the epoch before its tag
    }
    if (lane == 0) {
      uint32_t bits = 0;
      ok = ok && spin_for_key(done + blockIdx.x * kSyncLine, key, bits);
      if (ok) {
        s_amax = __uint_as_float(bits);
        st_relaxed_u64(done + blockIdx.x * kSyncLine, 0ull);  // read: cleared for later launches
      } else {
        record_error(kErrTimeout);
      }
      s_ok = ok ? 1 : 0;
    }
  }
  __syncthreads();
  if (!s_ok) return;
  const float a = s_amax;
  const float g = nvfp4_global_scale(a);
  const float six_g = 6.0f * g;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *g_out = g;
    if (amax_out != nullptr) *amax_out = a;
  }

  // ---- quantise this CTA's rows from shared memory: one lane per 16-element block
  const int bpr = k >> 4;       // blocks per row
  const uint32_t c4 = static_cast<uint32_t>(k >> 6);
  for (int i = warp; i < nr; i += kFusedWarps) {
    const int r = r0 + i;
    const uint32_t row = rows_s + static_cast<uint32_t>(i) * row_bytes;
    uint2* crow = reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * (k >> 1));
    // this row's scale bytes: 512-byte tile (r / 128, c / 4), byte (r % 32) * 16 + (r / 32 % 4) * 4 + c % 4
    uint8_t* sf_row = sf + static_cast<int64_t>(r >> 7) * c4 * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
    for (int c = lane; c < bpr; c += 32) {
      float f[16];
      bf16x16_to_f32(lds_v4(row + 32u * c), lds_v4(row + 32u * c + 16u), f);
      uint32_t sfc;
      crow[c] = nvfp4_block16(f, g, six_g, sfc);
      sf_row[(c >> 2) * 512 + (c & 3)] = static_cast<uint8_t>(sfc);
    }
  }
  zero_sf_padding(sf, rows, k >> 4);
}

// -------------------------------------------------------------- MXFP8
// bmax > 1.75 * 2^floor(log2 bmax), exactly, for a positive finite fp32 (the
// ceiling rule's "one more" decision: 448 * 2^(e - 8) = 1.75 * 2^e).  A
// normal value compares its fraction bits with 0.75 (0x600000); a subnormal
// m * 2^-149 compares m with 1.75 * 2^floor(log2 m) in integers.
__device__ __forceinline__ bool above_1p75(float bmax) {
  const uint32_t b = __float_as_uint(bmax);
  if (b >= 0x00800000u) return (b & 0x7FFFFFu) > 0x600000u;
  const uint32_t m = b & 0x7FFFFFu;
  const int fl = 31 - __clz(m);
  return 4u * m > (7u << fl);
}

// One thread per 32-element block: 64 bytes in (four 16-byte loads), 32
// bytes of codes out (two 16-byte stores) and the block's scale byte;
// consecutive threads take consecutive blocks of a row, then the next row,
// so a warp reads and writes contiguous memory for any k.
constexpr int kMxThreads = 256;
__global__ void __launch_bounds__(kMxThreads)
    quantize_mxfp8_kernel(const __nv_bfloat16* __restrict__ x, int rows, int k, int64_t ld,
                          uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, int rceil) {
  grid_dep_wait();
  grid_dep_launch();
  const int bpr = k >> 5;  // blocks per row
  const int c4 = k >> 7;
  const int64_t nblk = static_cast<int64_t>(rows) * bpr;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kMxThreads + threadIdx.x; t < nblk;
       t += static_cast<int64_t>(gridDim.x) * kMxThreads) {
    const int r = static_cast<int>(t / bpr), c = static_cast<int>(t - static_cast<int64_t>(r) * bpr);
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(r) * ld + 32 * c);
    // each 16-byte load covers half of a 32-byte sector per lane; loads that
    // allocate in L1 serve the other half from there instead of L2
    uint4 u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = ldg_nc_v4_l1(src + i);
    float f[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) bf16x8_to_f32(u[i], *reinterpret_cast<float(*)[8]>(f + 8 * i));
    float bmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) bmax = fmaxf(bmax, fabsf(f[i]));
    int X = -127;
    if (bmax > 0.0f) {
      // floor rule (OCP): X = floor(log2 bmax) - 8; ceiling rule: the smallest
      // X with bmax <= 448 * 2^X, one more when bmax > 1.75 * 2^floor(log2 bmax)
      const int e = floor_log2_f32(bmax) - 8 + ((rceil && above_1p75(bmax)) ? 1 : 0);
      X = min(max(e, -127), 127);
    }
    const float mult = exp2_int(-X);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = cvt_e4m3x2(f[4 * i] * mult, f[4 * i + 1] * mult) | (cvt_e4m3x2(f[4 * i + 2] * mult, f[4 * i + 3] * mult) << 16);
    uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<int64_t>(r) * k + 32 * c);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    sf[sf_offset(r, c, c4)] = static_cast<uint8_t>(X + 127);
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

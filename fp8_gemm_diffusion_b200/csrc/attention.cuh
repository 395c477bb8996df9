// attention.cuh - 8-bit (MXFP8) attention with per-token scales on the
// 5th-generation tensor cores (sm_100a).
//
// Source: the devin.kr page on Blackwell FLUX image generation ("엔비디아
// 블랙웰 기반 플럭스 3 이미지 생성 4.45배 가속"), section "연산 효율화와 가속
// 기술": attention through a dedicated 8-bit floating-point path that corrects
// the quantisation error token by token.  Per head (T tokens, d = 128):
//
//   Qq = MXFP8(Q), Kq = MXFP8(K)       scales per token and per 32 channels
//   Vq = MXFP8(V^T)                    scales per channel and per 32 tokens
//   S  = deq(Qq) deq(Kq)^T             block-scaled MMAs, fp32 in tensor memory
//   m  = rowmax(S)                     first pass over the key blocks
//   E  = 2^((S - m) * tau * log2 e)    second pass, fp32, in [0, 1]
//   Eq = MXFP8(E) along keys, ceiling scale rule (no saturation)
//   O  = deq(Eq) deq(Vq)^T / rowsum(E) block-scaled MMAs, fp32; bf16 out
//
// Two passes over the keys keep the softmax exact without rescaling the
// output accumulator: the first finds each row's maximum (no exponentials),
// the second weights every key against the final maximum.
//
// One CTA per (head, 128-query tile), 6 warps:
//   warp 0      TMA producer: the Q tile and its scales once, then a ring of
//               K blocks (first pass) and K + V^T blocks (second pass), each
//               with its 512-byte scale chunks;
//   warp 1      tensor memory; one lane issues the scale copies (tcgen05.cp)
//               and the MMAs: S = Q K^T into one of two S buffers, and
//               O += Eq V^T behind the softmax of the same block;
//   warps 2-5   softmax, one query row per thread (tensor-memory sub-partition
//               warp % 4): row maxima, then weights, row sums, MXFP8 codes of
//               E into shared memory (the MMA's A operand) and their scales
//               into tensor memory; at the end O / rowsum -> bf16.
// Every wait is bounded (ptx.cuh).
#pragma once

#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "gemm.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace mxq {

constexpr int kAttD = 128;       // head dimension
constexpr int kAttTile = 128;    // query rows per CTA = keys per block
constexpr int kAttStages = 4;

struct AttCfg {
  static constexpr int TILE_BYTES = kAttTile * 128;                 // 128 rows x 128 bytes (E4M3)
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + 1024;         // K, V^T, their scale chunks
  static constexpr int OFF_QSF = TILE_BYTES;                        // Q scale chunk (512 B)
  static constexpr int OFF_STAGE = TILE_BYTES + 1024;
  static constexpr int OFF_P = OFF_STAGE + kAttStages * STAGE_BYTES;  // two E-code buffers
  static constexpr int OFF_BAR = OFF_P + 2 * TILE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
  // tensor memory columns: two S buffers, O, then scale sets of 4 columns
  static constexpr uint32_t T_S = 0, T_O = 256, T_QSF = 384, T_KSF = 388, T_VSF = 392, T_PSF = 396;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 192;
  static constexpr int SOFT_WARP0 = 2;
};

struct AttArgs {
  int heads, tokens;
  float c;                          // tau * log2(e)
  const uint8_t* q_sf;              // swizzled scales of Qq (rows heads*tokens)
  const uint8_t* k_sf;              // of Kq
  const uint8_t* v_sf;              // of V^T (rows heads*128, tokens/32 scale columns)
  __nv_bfloat16* out;               // [heads][tokens][128]
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// MXFP8 shared exponent by the ceiling rule: the smallest X with
// bmax <= 448 * 2^X (bmax > 0), clamped to [-127, 127].
__device__ __forceinline__ int mx_ceil_exponent(float bmax) {
  if (!(bmax > 0.0f)) return -127;
  const int e = floor_log2_f32(bmax);
  int X = e - 8;
  if (static_cast<double>(bmax) > ldexp(1.75, e)) X += 1;  // bmax > 448 * 2^(e - 8)
  return min(max(X, -127), 127);
}

__global__ void __launch_bounds__(AttCfg::THREADS, 1)
    attention_mxfp8_kernel(const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v, const AttArgs args) {
  using C = AttCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t bar = base + C::OFF_BAR;
  // barriers: q_full, kv_full[4], kv_empty[4], s_full[2], s_free[2], p_full[2], p_free[2], o_full
  const uint32_t q_full = bar;
  auto kv_full = [&](int s) { return bar + 8u + 8u * s; };
  auto kv_empty = [&](int s) { return bar + 8u + 8u * (kAttStages + s); };
  auto s_full = [&](int b) { return bar + 8u + 8u * (2 * kAttStages + b); };
  auto s_free = [&](int b) { return bar + 8u + 8u * (2 * kAttStages + 2 + b); };
  auto p_full = [&](int b) { return bar + 8u + 8u * (2 * kAttStages + 4 + b); };
  auto p_free = [&](int b) { return bar + 8u + 8u * (2 * kAttStages + 6 + b); };
  const uint32_t o_full = bar + 8u + 8u * (2 * kAttStages + 8);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + 8 * (2 * kAttStages + 10));
  static_assert(8 * (2 * kAttStages + 10) + 4 <= C::BAR_BYTES, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = args.tokens;
  const int nkb = T / kAttTile;
  const int h = blockIdx.x / nkb, q0 = (blockIdx.x % nkb) * kAttTile;
  const int qrow0 = h * T + q0;  // first row of this tile in the [heads * tokens] arrays

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kAttStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 4);
      mbar_init(p_full(b), 4);
      mbar_init(p_free(b), 1);
    }
    mbar_init(o_full, 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();  // Q, K, V^T and their scales come from the quantisers just before
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::TILE_BYTES + 512);
      tma_load_2d(base, &tmap_q, q_full, 0, qrow0);
      bulk_load(base + C::OFF_QSF, args.q_sf + static_cast<int64_t>(qrow0 / 128) * 512, 512, q_full);
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int g = 0; g < 2 * nkb; ++g) {
        const bool pv = g >= nkb;
        const int kb = pv ? g - nkb : g;
        if (!mbar_wait_bounded(kv_empty(s), ph ^ 1u)) { ok = false; break; }
        const uint32_t st = base + C::OFF_STAGE + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(kv_full(s), (C::TILE_BYTES + 512) * (pv ? 2u : 1u));
        const int krow = h * T + kb * kAttTile;
        tma_load_2d(st, &tmap_k, kv_full(s), 0, krow);
        bulk_load(st + 2 * C::TILE_BYTES, args.k_sf + static_cast<int64_t>(krow / 128) * 512, 512, kv_full(s));
        if (pv) {
          tma_load_2d(st + C::TILE_BYTES, &tmap_v, kv_full(s), kb * kAttTile, h * kAttD);
          bulk_load(st + 2 * C::TILE_BYTES + 512, args.v_sf + (static_cast<int64_t>(h) * nkb + kb) * 512, 512,
                    kv_full(s));
        }
        ++issued;
        if (++s == kAttStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        // let the loads already issued land before the CTA can exit
        for (int i = 0; i < kAttStages && i < issued; ++i) {
          if (--s < 0) { s = kAttStages - 1; ph ^= 1u; }
          mbar_wait_bounded(kv_full(s), ph);
        }
      }
      mbar_wait_bounded(q_full, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait_bounded(q_full, 0);
      tc_fence_after();
      if (ok) tc_cp_32x128b_warpx4(tmem + C::T_QSF, desc_sf_chunk(base + C::OFF_QSF));
      const uint64_t qdesc = desc_kmajor_sw128(base);
      int s = 0, s_prev = 0;
      uint32_t ph = 0;
      // S[b] = Q K^T of the block in stage s (its scale chunk copied first;
      // the copy follows the previous block's MMAs in this thread's order)
      auto qk = [&](int g, int st_idx) {
        const uint32_t st = base + C::OFF_STAGE + st_idx * C::STAGE_BYTES;
        const int b = g & 1;
        tc_cp_32x128b_warpx4(tmem + C::T_KSF, desc_sf_chunk(st + 2 * C::TILE_BYTES));
        const uint64_t kdesc = desc_kmajor_sw128(st);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t koff = static_cast<uint64_t>(2 * j);  // 32 bytes of d per MMA
          mma_mxfp8(tmem + C::T_S + b * kAttTile, qdesc + koff, kdesc + koff, make_idesc<Fmt::MXFP8>(kAttTile, j),
                    (tmem + C::T_QSF) | (static_cast<uint32_t>(j) << 30),
                    (tmem + C::T_KSF) | (static_cast<uint32_t>(j) << 30), j > 0 ? 1u : 0u);
        }
        tc_commit(s_full(b));
      };
      // O += Eq V^T of key block kb (stage st_idx), once its weights are in place
      auto pv_mma = [&](int kb, int st_idx) -> bool {
        const int b = kb & 1;
        if (!mbar_wait_bounded(p_full(b), (kb >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t st = base + C::OFF_STAGE + st_idx * C::STAGE_BYTES;
        tc_cp_32x128b_warpx4(tmem + C::T_VSF, desc_sf_chunk(st + 2 * C::TILE_BYTES + 512));
        const uint64_t pdesc = desc_kmajor_sw128(base + C::OFF_P + b * C::TILE_BYTES);
        const uint64_t vdesc = desc_kmajor_sw128(st + C::TILE_BYTES);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t koff = static_cast<uint64_t>(2 * j);  // 32 keys per MMA
          mma_mxfp8(tmem + C::T_O, pdesc + koff, vdesc + koff, make_idesc<Fmt::MXFP8>(kAttD, j),
                    (tmem + C::T_PSF + 4 * b) | (static_cast<uint32_t>(j) << 30),
                    (tmem + C::T_VSF) | (static_cast<uint32_t>(j) << 30), (kb > 0 || j > 0) ? 1u : 0u);
        }
        tc_commit(p_free(b));
        tc_commit(kv_empty(st_idx));
        return true;
      };
      for (int g = 0; g < 2 * nkb && ok; ++g) {
        const bool pv = g >= nkb;
        const int kb = pv ? g - nkb : g;
        if (!mbar_wait_bounded(kv_full(s), ph)) { ok = false; break; }
        // S buffer g & 1 was read by the softmax of block g - 2
        if (!mbar_wait_bounded(s_free(g & 1), ((g >> 1) & 1) ^ 1u)) { ok = false; break; }
        tc_fence_after();
        qk(g, s);
        if (!pv) {
          tc_commit(kv_empty(s));  // first pass: K only
        } else if (kb > 0) {
          if (!(ok = pv_mma(kb - 1, s_prev))) break;
        }
        s_prev = s;
        if (++s == kAttStages) { s = 0; ph ^= 1u; }
      }
      if (ok) ok = pv_mma(nkb - 1, s_prev);
      tc_commit(o_full);
      // every MMA / copy issued above must finish before tensor memory is freed
      mbar_wait_bounded(o_full, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;            // tensor-memory sub-partition
    const int r = q * 32 + lane;       // query row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const float c = args.c;
    uint32_t u[kAttTile];  // one row of S (fp32 bits), then of E, then of O
    bool ok = true;
    float m = -INFINITY;
    auto load_s = [&](int g) -> bool {
      if (!mbar_wait_bounded(s_full(g & 1), (g >> 1) & 1)) return false;
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < kAttTile / 32; ++i)
        tmem_ld_32x32b_x32_nowait(trow + C::T_S + (g & 1) * kAttTile + 32 * i, u + 32 * i);
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < kAttTile / 32; ++i) reg_fence32(u + 32 * i);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free(g & 1));  // S buffer read
      return true;
    };
    // first pass: row maxima
    for (int g = 0; g < nkb && ok; ++g) {
      if (!(ok = load_s(g))) break;
#pragma unroll
      for (int i = 0; i < kAttTile; ++i) m = fmaxf(m, __uint_as_float(u[i]));
    }
    // second pass: weights against the final maximum, row sums, MXFP8 codes
    const float mc = m * c;
    float l = 0.0f;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      if (!(ok = load_s(nkb + kb))) break;
#pragma unroll
      for (int i = 0; i < kAttTile; ++i) {
        const float e = ex2_approx(fmaf(__uint_as_float(u[i]), c, -mc));
        u[i] = __float_as_uint(e);
        l += e;
      }
      uint32_t codes[kAttTile / 4];
      uint32_t sfw = 0;
#pragma unroll
      for (int blk = 0; blk < kAttTile / 32; ++blk) {
        float bmax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) bmax = fmaxf(bmax, __uint_as_float(u[32 * blk + i]));
        const int X = mx_ceil_exponent(bmax);
        const float mult = exp2_int(-X);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int k0 = 32 * blk + 4 * i;
          codes[8 * blk + i] = cvt_e4m3x2(__uint_as_float(u[k0]) * mult, __uint_as_float(u[k0 + 1]) * mult) |
                               (cvt_e4m3x2(__uint_as_float(u[k0 + 2]) * mult, __uint_as_float(u[k0 + 3]) * mult) << 16);
        }
        sfw |= static_cast<uint32_t>(X + 127) << (8 * blk);
      }
      const int b = kb & 1;
      // the MMA of key block kb - 2 has read this buffer and its scales
      if (!(ok = mbar_wait_bounded(p_free(b), ((kb >> 1) & 1) ^ 1u))) break;
      tc_fence_after();
      // row r of the A operand: 128 bytes, 128-byte swizzle (chunk c at c ^ (r % 8))
      const uint32_t prow = base + C::OFF_P + b * C::TILE_BYTES + r * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t addr = prow + ((ch ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(codes[4 * ch]),
                     "r"(codes[4 * ch + 1]), "r"(codes[4 * ch + 2]), "r"(codes[4 * ch + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      // the row's four block scales, on the sub-partition's diagonal column
      tmem_st_32x32b_x1(trow + C::T_PSF + 4 * b + q, sfw);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(b));
    }
    // epilogue: O / rowsum -> bf16
    if (ok && mbar_wait_bounded(o_full, 0)) {
      tc_fence_after();
#pragma unroll
      for (int i = 0; i < kAttD / 32; ++i) tmem_ld_32x32b_x32_nowait(trow + C::T_O + 32 * i, u + 32 * i);
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < kAttD / 32; ++i) reg_fence32(u + 32 * i);
      const float inv_l = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>(args.out + (static_cast<int64_t>(qrow0) + r) * kAttD);
#pragma unroll
      for (int i = 0; i < kAttD / 8; ++i) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(__uint_as_float(u[8 * i + 2 * e]) * inv_l,
                                                          __uint_as_float(u[8 * i + 2 * e + 1]) * inv_l);
          pk[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        dst[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// V [heads][tokens][128] bf16 -> V^T MXFP8 codes [heads * 128][tokens] and
// scales (rows heads * 128, tokens / 32 scale columns, swizzled), quantised
// along tokens.  One CTA per (head, 128-token block); thread (c, blk)
// quantises channel c over tokens [32 blk, 32 blk + 32) of the block.
__global__ void __launch_bounds__(512) quantize_mxfp8_vt_kernel(const __nv_bfloat16* __restrict__ v, int heads,
                                                              int tokens, uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ sf) {
  __shared__ __align__(16) __nv_bfloat16 tile[kAttTile][kAttD];
  grid_dep_wait();
  grid_dep_launch();
  const int nkb = tokens / kAttTile;
  const int h = blockIdx.x / nkb, t0 = (blockIdx.x % nkb) * kAttTile;
  const uint4* src = reinterpret_cast<const uint4*>(v + (static_cast<int64_t>(h) * tokens + t0) * kAttD);
  uint4* stile = reinterpret_cast<uint4*>(&tile[0][0]);
  for (int i = threadIdx.x; i < kAttTile * kAttD / 8; i += blockDim.x) stile[i] = ldg_nc_v4(src + i);
  __syncthreads();
  const int c = threadIdx.x & (kAttD - 1), blk = threadIdx.x >> 7;
  float f[32];
  float bmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    f[i] = __bfloat162float(tile[32 * blk + i][c]);
    bmax = fmaxf(bmax, fabsf(f[i]));
  }
  int X = -127;
  if (bmax > 0.0f) X = min(max(floor_log2_f32(bmax) - 8, -127), 127);  // OCP floor rule
  const float mult = exp2_int(-X);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = cvt_e4m3x2(f[4 * i] * mult, f[4 * i + 1] * mult) | (cvt_e4m3x2(f[4 * i + 2] * mult, f[4 * i + 3] * mult) << 16);
  const int64_t row = static_cast<int64_t>(h) * kAttD + c;
  uint4* dst = reinterpret_cast<uint4*>(codes + row * tokens + t0 + 32 * blk);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  sf[sf_offset(row, (t0 >> 5) + blk, tokens >> 7)] = static_cast<uint8_t>(X + 127);
  // rows heads * 128 are a multiple of 128: no scale padding to clear
}

}  // namespace mxq

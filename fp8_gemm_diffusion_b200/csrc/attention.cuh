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
//   t  = S * tau * log2 e
//   E  = 2^(t - m), m an integer       fp32
//   Eq = MXFP8(E) along keys, ceiling scale rule (no saturation)
//   O  = deq(Eq) deq(Vq)^T / rowsum(deq(Eq))   block-scaled MMAs, fp32; bf16 out
//
// One pass over the keys.  Softmax is the same for every m; with m an
// integer the MXFP8 codes are the same for every m too (2^k times a block
// moves its shared exponent by k and leaves the codes), so m can be a
// running maximum: the first key block sets m = ceil(max t), and a later
// block whose maximum exceeds m by more than 8 raises it, after the output
// accumulator and the row sum are multiplied by 2^(m_old - m_new), exactly.
// Weights up to 2^8 stay far inside fp32, and the result is the one the
// final maximum would have given.  The row sums of the quantised weights
// come out of the second product: V^T carries 16 extra rows (a row of ones,
// then zeros) with unit scales, so O has a 129th column = sum_j deq(Eq)_j,
// rescaled with O and divided out at the end.
//
// One CTA per (head, 128-query tile), 12 warps:
//   warp 0      TMA producer of the Q tile and of K (and scales) per block;
//   warp 2      TMA producer of V^T (and scales) per block;
//   warp 1      tensor memory; one lane issues S = Q K^T of block j into S
//               buffer j % 2 (with the scale copies, tcgen05.cp);
//   warp 3      one lane issues O += Eq V^T of block j once its weights are
//               in place;
//   warps 4-7   softmax of the even key blocks, warps 8-11 of the odd ones
//               (tensor-memory sub-partition warp % 4, one query row per
//               thread): the two warpgroups work on consecutive blocks at
//               the same time (two warps per sub-partition keep the
//               exponential unit busy).  Per block:
//               block maxima, the normaliser (taken over from the other
//               warpgroup's previous block through shared memory and raised
//               if needed), weights, MXFP8 codes of E and their scales
//               into tensor memory (the second product's A operand); at
//               the end O / rowsum -> bf16.
// Every wait is bounded (ptx.cuh).  The softmax warps never leave their
// loop early: after a timeout they skip the work but keep the hand-over
// order, so no warp waits on a named barrier that is never signalled.
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
constexpr float kAttRescale = 8.0f;  // raise m when a block's maximum exceeds it by more

struct AttCfg {
  static constexpr int TILE_BYTES = kAttTile * 128;                 // 128 rows x 128 bytes (E4M3)
  static constexpr int EXT_BYTES = 16 * 128;                        // V^T rows 128..143: ones, then zeros
  // a stage: K, V^T and its 16-row extension (one B operand of 144 rows), K scales, V^T scales
  static constexpr int ST_EXT = 2 * TILE_BYTES, ST_KSF = ST_EXT + EXT_BYTES, ST_VSF = ST_KSF + 512;
  static constexpr int STAGE_BYTES = ST_VSF + 512;                  // 35 KB (multiple of 1024)
  static constexpr int OFF_QSF = TILE_BYTES;                        // Q scale chunk (512 B)
  static constexpr int OFF_ONESF = TILE_BYTES + 512;                // unit scales of the extension rows
  static constexpr int OFF_STAGE = TILE_BYTES + 1024;
  static constexpr int OFF_XCH = OFF_STAGE + kAttStages * STAGE_BYTES;  // [128 rows] normaliser, [4] flags
  static constexpr int XCH_BYTES = 128 * 4 + 64;
  static constexpr int OFF_BAR = OFF_XCH + XCH_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + OFF_BAR + BAR_BYTES;
  // the second product has N = 144: d = 128 output columns, column 128 the
  // row sum of the quantised weights (times the extension's row of ones),
  // 15 zero columns
  static constexpr int PV_N = kAttD + 16;
  // tensor memory columns: two S buffers, O (144), scale columns of Q, K,
  // V^T (two 128-row groups: the tile's and the extension's), of the
  // weights (one 4-column group per S buffer), then the weights' E4M3 codes
  // themselves, the second product's A operand (32 columns per S buffer:
  // four codes per column, the row in the lane)
  static constexpr uint32_t T_S = 0, T_O = 256, T_QSF = 400, T_KSF = 404, T_VSF = 408, T_PSF = 416,
                            T_P = 424;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static constexpr int SOFT_WARP0 = 4;
  // registers: launched with 65536 / 384 = 168 per thread; the control
  // warpgroup gives up registers so that a softmax thread holds its row of S
  static constexpr int REGS_CTRL = 56, REGS_SOFT = 224;
};
static_assert(AttCfg::STAGE_BYTES % 1024 == 0, "stage alignment (128-byte swizzle atoms)");
static_assert(AttCfg::T_P + 64 <= AttCfg::TMEM_COLS && AttCfg::T_PSF + 8 <= AttCfg::T_P &&
                  AttCfg::T_O + AttCfg::PV_N <= AttCfg::T_QSF, "tensor memory");
static_assert(128 * AttCfg::REGS_CTRL + 256 * AttCfg::REGS_SOFT <= 384 * 168, "register split");

struct AttArgs {
  int heads, tokens;
  float c;                          // tau * log2(e)
  const uint8_t* q_sf;              // swizzled scales of Qq (rows heads*tokens)
  const uint8_t* k_sf;              // of Kq
  const uint8_t* v_sf;              // of V^T (rows heads*128, tokens/32 scale columns)
  __nv_bfloat16* out;               // [heads][tokens][128]
};

// MXFP8 shared exponent by the ceiling rule for a block maximum that is 0
// or a normal fp32: the smallest X with bmax <= 448 * 2^X, clamped to
// [-127, 127].  With bmax = (1 + f) 2^e, 448 * 2^(e - 8) = 1.75 * 2^e, so X is
// e - 8, plus one when the fraction f exceeds 0.75 (bits above 0x600000).
__device__ __forceinline__ int mx_ceil_exponent_normal(float bmax) {
  const uint32_t b = __float_as_uint(bmax);
  if (b == 0u) return -127;
  const int X = static_cast<int>(b >> 23) - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return min(max(X, -127), 127);
}

// 2^x on the FMA pipe, for x <= 9: x = j + f with j the nearest integer
// (rounding by adding 1.5 * 2^23) and |f| <= 1/2, 2^f by a degree-5
// polynomial (coefficients fitted here by least squares on Chebyshev nodes
// of [-1/2, 1/2], relative error 2.2e-7 evaluated in fp32, on a par with the
// special-function unit's 2^x), j added to the exponent field.  Below -20 the
// result is clamped at 2^-20: every weight that small rounds to the E4M3
// code 0 once divided by its block's scale (the block maximum is at least
// 224 times the scale), as 2^x itself would.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -20.0f);
  const float y = x + 12582912.0f;                // 1.5 * 2^23: x rounded to an integer in the low bits
  const int j = __float_as_int(y) - 0x4B400000;    // bits of 1.5 * 2^23
  const float f = x - (y - 12582912.0f);
  float p = 0.0013266970636323094f;
  p = fmaf(p, f, 0.009675459936261177f);
  p = fmaf(p, f, 0.05550742521882057f);
  p = fmaf(p, f, 0.24022121727466583f);
  p = fmaf(p, f, 0.6931469440460205f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (j << 23));
}

// Four fp32 -> four E4M3 bytes packed into 32 bits, a in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// Instruction descriptor of an M = 128 kind::mxf8f6f4 MMA (E4M3 x E4M3,
// UE8M0 scales) with separate scale-byte selectors for A and B.
__device__ __forceinline__ uint32_t idesc_mxfp8_m128(int n, uint32_t a_id, uint32_t b_id) {
  return (b_id << 4) | ((static_cast<uint32_t>(n) >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) | (a_id << 29);
}

__device__ __forceinline__ float max32(const uint32_t* u) {
  float a = fmaxf(__uint_as_float(u[0]), __uint_as_float(u[1]));
  float b = fmaxf(__uint_as_float(u[2]), __uint_as_float(u[3]));
  float c = fmaxf(__uint_as_float(u[4]), __uint_as_float(u[5]));
  float d = fmaxf(__uint_as_float(u[6]), __uint_as_float(u[7]));
#pragma unroll
  for (int i = 8; i < 32; i += 4) {
    a = fmaxf(a, __uint_as_float(u[i]));
    b = fmaxf(b, __uint_as_float(u[i + 1]));
    c = fmaxf(c, __uint_as_float(u[i + 2]));
    d = fmaxf(d, __uint_as_float(u[i + 3]));
  }
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
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
  // barriers: q_full, k_full[4], k_empty[4], v_full[4], v_empty[4], s_full[2], s_free[2],
  // p_full[2], p_free[2], o_full, qk_drain.  K and V^T of a stage have their own
  // barriers: K is free once S of its block is computed, long before V^T
  // is, so the K ring runs ahead of the V^T ring.
  const uint32_t q_full = bar;
  auto k_full = [&](int s) { return bar + 8u + 8u * s; };
  auto k_empty = [&](int s) { return bar + 8u + 8u * (kAttStages + s); };
  auto v_full = [&](int s) { return bar + 8u + 8u * (2 * kAttStages + s); };
  auto v_empty = [&](int s) { return bar + 8u + 8u * (3 * kAttStages + s); };
  auto s_full = [&](int b) { return bar + 8u + 8u * (4 * kAttStages + b); };
  auto s_free = [&](int b) { return bar + 8u + 8u * (4 * kAttStages + 2 + b); };
  auto p_full = [&](int b) { return bar + 8u + 8u * (4 * kAttStages + 4 + b); };
  auto p_free = [&](int b) { return bar + 8u + 8u * (4 * kAttStages + 6 + b); };
  const uint32_t o_full = bar + 8u + 8u * (4 * kAttStages + 8);
  const uint32_t qk_drain = bar + 8u + 8u * (4 * kAttStages + 9);  // the S thread's last MMAs done
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::OFF_BAR + 8 * (4 * kAttStages + 11));
  static_assert(8 * (4 * kAttStages + 11) + 4 <= C::BAR_BYTES, "barrier area");
  constexpr int NSOFT = 4;  // warps of one softmax warpgroup (the one that owns S / P buffer b)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = args.tokens;
  const int nkb = T / kAttTile;
  const int h = blockIdx.x / nkb, q0 = (blockIdx.x % nkb) * kAttTile;
  const int qrow0 = h * T + q0;  // first row of this tile in the [heads * tokens] arrays

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kAttStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), NSOFT);
      mbar_init(p_full(b), NSOFT);
      mbar_init(p_free(b), 1);
    }
    mbar_init(o_full, 1);
    mbar_init(qk_drain, 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  // constant operand bytes, read by the MMAs through the async proxy: each
  // stage's V^T extension (row 128 = E4M3 1.0 = 0x38 in every key, rows
  // 129..143 zero; a row of equal bytes needs no swizzle) and a 512-byte
  // chunk of unit scales (E8M0 127)
  for (int i = threadIdx.x; i < kAttStages * C::EXT_BYTES / 16; i += C::THREADS) {
    const int st = i / (C::EXT_BYTES / 16), o = i % (C::EXT_BYTES / 16);
    const uint32_t v = o < 8 ? 0x38383838u : 0u;
    *reinterpret_cast<uint4*>(base_ptr + C::OFF_STAGE + st * C::STAGE_BYTES + C::ST_EXT + 16 * o) = make_uint4(v, v, v, v);
  }
  for (int i = threadIdx.x; i < 512 / 16; i += C::THREADS)
    *reinterpret_cast<uint4*>(base_ptr + C::OFF_ONESF + 16 * i) = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_wait();  // Q, K, V^T and their scales come from the quantisers just before
  grid_dep_launch();

  if (warp < C::SOFT_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_CTRL));
  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0: the Q tile, then K and its scales per key block; warp 2: V^T
    // and its scales per key block, each into its part of the stage ring
    if (lane == 0) {
      const bool is_k = warp == 0;
      if (is_k) {
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES + 512);
        tma_load_2d(base, &tmap_q, q_full, 0, qrow0);
        bulk_load(base + C::OFF_QSF, args.q_sf + static_cast<int64_t>(qrow0 / 128) * 512, 512, q_full);
      }
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_bounded(is_k ? k_empty(s) : v_empty(s), ph ^ 1u)) { ok = false; break; }
        const uint32_t st = base + C::OFF_STAGE + s * C::STAGE_BYTES;
        if (is_k) {
          mbar_arrive_expect_tx(k_full(s), C::TILE_BYTES + 512);
          const int krow = h * T + kb * kAttTile;
          tma_load_2d(st, &tmap_k, k_full(s), 0, krow);
          bulk_load(st + C::ST_KSF, args.k_sf + static_cast<int64_t>(krow / 128) * 512, 512, k_full(s));
        } else {
          mbar_arrive_expect_tx(v_full(s), C::TILE_BYTES + 512);
          tma_load_2d(st + C::TILE_BYTES, &tmap_v, v_full(s), kb * kAttTile, h * kAttD);
          bulk_load(st + C::ST_VSF, args.v_sf + (static_cast<int64_t>(h) * nkb + kb) * 512, 512, v_full(s));
        }
        ++issued;
        if (++s == kAttStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        // let the loads already issued land before the CTA can exit
        for (int i = 0; i < kAttStages && i < issued; ++i) {
          if (--s < 0) { s = kAttStages - 1; ph ^= 1u; }
          mbar_wait_bounded(is_k ? k_full(s) : v_full(s), ph);
        }
      }
      if (is_k) mbar_wait_bounded(q_full, 0);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads: warp 1 issues S = Q K^T (into the S buffers), warp 3 the
    // second product O += Eq V^T (into O).  They write disjoint tensor memory
    // and each product's inputs arrive through mbarriers, so the two need no
    // order between them; each thread's own MMAs (one accumulator each) stay
    // in issue order.  An MMA takes about a hundred cycles to issue, so one
    // thread for both products became the limit.
    if (lane == 0) {
      bool ok = mbar_wait_bounded(q_full, 0);
      tc_fence_after();
      if (warp == 1) {
        if (ok) tc_cp_32x128b_warpx4(tmem + C::T_QSF, desc_sf_chunk(base + C::OFF_QSF));
        const uint64_t qdesc = desc_kmajor_sw128(base);
        for (int j = 0; j < nkb && ok; ++j) {
          const int st_idx = j % kAttStages;
          // K of block j has landed; the softmax has read S of block j - 2
          if (!(ok = mbar_wait_bounded(k_full(st_idx), (j / kAttStages) & 1))) break;
          if (!(ok = mbar_wait_bounded(s_free(j & 1), ((j >> 1) & 1) ^ 1u))) break;
          tc_fence_after();
          const uint32_t st = base + C::OFF_STAGE + st_idx * C::STAGE_BYTES;
          tc_cp_32x128b_warpx4(tmem + C::T_KSF, desc_sf_chunk(st + C::ST_KSF));
          const uint64_t kdesc = desc_kmajor_sw128(st);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t koff = static_cast<uint64_t>(2 * k);  // 32 bytes of d per MMA
            mma_mxfp8(tmem + C::T_S + (j & 1) * kAttTile, qdesc + koff, kdesc + koff,
                      idesc_mxfp8_m128(kAttTile, k, k), (tmem + C::T_QSF) | (static_cast<uint32_t>(k) << 30),
                      (tmem + C::T_KSF) | (static_cast<uint32_t>(k) << 30), k > 0 ? 1u : 0u);
          }
          tc_commit(s_full(j & 1));
          tc_commit(k_empty(st_idx));
        }
        // every MMA / copy this thread issued must finish before tensor memory is freed
        tc_commit(qk_drain);
        mbar_wait_bounded(qk_drain, 0);
      } else {
        // unit scales of the V^T extension rows (128-row group 1 of the B scales), once
        tc_cp_32x128b_warpx4(tmem + C::T_VSF + 4, desc_sf_chunk(base + C::OFF_ONESF));
        for (int j = 0; j < nkb && ok; ++j) {
          const int b = j & 1, st_idx = j % kAttStages;
          // the weights of block j are in place and its V^T has landed
          if (!(ok = mbar_wait_bounded(p_full(b), (j >> 1) & 1))) break;
          if (!(ok = mbar_wait_bounded(v_full(st_idx), (j / kAttStages) & 1))) break;
          tc_fence_after();
          const uint32_t st = base + C::OFF_STAGE + st_idx * C::STAGE_BYTES;
          tc_cp_32x128b_warpx4(tmem + C::T_VSF, desc_sf_chunk(st + C::ST_VSF));
          const uint64_t vdesc = desc_kmajor_sw128(st + C::TILE_BYTES);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // MMA k covers keys [32 k, 32 k + 32), scale byte k of the row's word
            const uint64_t koff = static_cast<uint64_t>(2 * k);
            mma_mxfp8_ta(tmem + C::T_O, tmem + C::T_P + 32 * b + 8 * k, vdesc + koff, idesc_mxfp8_m128(C::PV_N, k, k),
                      (tmem + C::T_PSF + 4 * b) | (static_cast<uint32_t>(k) << 30),
                      (tmem + C::T_VSF) | (static_cast<uint32_t>(k) << 30), (j > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(p_free(b));
          tc_commit(v_empty(st_idx));
        }
        tc_commit(o_full);
        // every MMA / copy this thread issued must finish before tensor memory is freed
        mbar_wait_bounded(o_full, 0);
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_SOFT));
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;                        // tensor-memory sub-partition
    const int G = (warp - C::SOFT_WARP0) >> 2;     // 0: even key blocks, 1: odd
    const int r = q * 32 + lane;                   // query row of the tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    // named barriers of sub-partition q: normaliser hand-over even -> odd
    // (2 + q) and odd -> even (6 + q), final row sums (10 + q); 64 threads
    const uint32_t bar_to_other = (G == 0 ? 2u : 6u) + static_cast<uint32_t>(q);
    const uint32_t bar_from_other = (G == 0 ? 6u : 2u) + static_cast<uint32_t>(q);
    float* const xm = reinterpret_cast<float*>(base_ptr + C::OFF_XCH);               // [128] normaliser
    volatile int* const xok = reinterpret_cast<volatile int*>(xm + 128);             // [4] sub-partition flags
    const float c = args.c;
    uint32_t u[kAttTile];  // the row of S (fp32 bits) of the current block, then of O
    bool ok = true;
    float m = -INFINITY;   // normaliser in effect (an integer once set)
    for (int j = G; j < nkb; j += 2) {
      const int b = j & 1;  // == G
      const bool got = __all_sync(0xffffffffu, ok && mbar_wait_bounded(s_full(b), (j >> 1) & 1));
      if (got) {
        tc_fence_after();
#pragma unroll
        for (int i = 0; i < kAttTile / 32; ++i) tmem_ld_32x32b_x32_nowait(trow + C::T_S + b * kAttTile + 32 * i, u + 32 * i);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < kAttTile / 32; ++i) reg_fence32(u + 32 * i);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(b));  // S buffer read
      }
      ok = got;
      float bm[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) bm[k] = max32(u + 32 * k);
      const float tmax = fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3])) * c;
      // the normaliser after block j - 1, from the other warpgroup
      if (j >= 1) {
        named_bar_sync(bar_from_other, 64);
        m = xm[r];
        ok = ok && xok[q] != 0;
      }
      const bool raise = tmax > m + kAttRescale;
      const float m_new = raise ? ceilf(tmax) : m;
      // hand the normaliser on at once: the other warpgroup's block j + 1
      // runs its exponentials alongside these (two warps per sub-partition
      // keep the exponential unit busy)
      if (j + 1 < nkb) {
        xm[r] = m_new;
        __syncwarp();
        if (lane == 0) xok[q] = ok ? 1 : 0;
        named_bar_arrive(bar_to_other, 64);
      }
      // rows that raise the normaliser rescale O and its row-sum column by
      // 2^(m - m_new) (the others by 1) once the product of block j - 1 is
      // complete; the product of block j is issued only after this warp's
      // p_full arrival below
      if (j >= 1 && __any_sync(0xffffffffu, raise)) {
        const int dm = raise ? static_cast<int>(m - m_new) : 0;  // <= -9 where raised
        const float f = dm < -127 ? 0.0f : exp2_int(dm);
        ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(p_free((j - 1) & 1), ((j - 1) >> 1) & 1));
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < kAttD / 32; ++g) {
            uint32_t o[32];
            tmem_ld_32x32b_x32_nowait(trow + C::T_O + 32 * g, o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            uint32_t w[16];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
              for (int k = 0; k < 16; ++k) w[k] = o[16 * h2 + k];
              tmem_st_32x32b_x16(trow + C::T_O + 32 * g + 16 * h2, w);
            }
          }
          uint32_t lsum = tmem_ld_32x32b_x1_nowait(trow + C::T_O + kAttD);
          tc_wait_ld();
          asm volatile("" : "+r"(lsum)::"memory");
          tmem_st_32x32b_x1(trow + C::T_O + kAttD, __float_as_uint(__uint_as_float(lsum) * f));
          tc_wait_st();
        }
      }
      m = m_new;
      // weights of the four 32-key blocks, their MXFP8 codes and scales (the
      // row sum of the quantised weights comes out of the second product):
      // the block exponents first, then all 128 exponentials in place
      // (independent, back to back on the exponential unit), then the codes
      float mx[4];
      uint32_t sfw = 0;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const float emax = ex2_approx(fmaf(bm[blk], c, -m));
        const int X = mx_ceil_exponent_normal(emax);
        mx[blk] = m + static_cast<float>(X);  // E / 2^X = 2^(t - m - X)
        sfw |= static_cast<uint32_t>(X + 127) << (8 * blk);
      }
#pragma unroll
      for (int i = 0; i < kAttTile; ++i) {
        // every fourth weight on the FMA pipe, the rest on the special-function unit
        const float a = fmaf(__uint_as_float(u[i]), c, -mx[i >> 5]);
        u[i] = __float_as_uint((i & 3) == 3 ? exp2_poly(a) : ex2_approx(a));
      }
      uint32_t codes[kAttTile / 4];
#pragma unroll
      for (int i = 0; i < kAttTile / 4; ++i)
        codes[i] = cvt_e4m3x4(__uint_as_float(u[4 * i]), __uint_as_float(u[4 * i + 1]), __uint_as_float(u[4 * i + 2]),
                              __uint_as_float(u[4 * i + 3]));
      // the product of block j - 2 (this warpgroup's previous block) has read
      // this buffer and its scales
      ok = __all_sync(0xffffffffu, ok && mbar_wait_bounded(p_free(b), ((j >> 1) & 1) ^ 1u));
      if (ok) {
        tc_fence_after();
        // the row's codes into tensor memory (the second product's A operand)
        // and its four block scales, on the sub-partition's diagonal column
        tmem_st_32x32b_x32(trow + C::T_P + 32 * b, codes);
        tmem_st_32x32b_x1(trow + C::T_PSF + 4 * b + q, sfw);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(b));
      }
    }
    // epilogue: O / (row sum of the quantised weights, O's column 128) ->
    // bf16; warpgroup G writes columns [64 G, 64 G + 64)
    if (__all_sync(0xffffffffu, ok && mbar_wait_bounded(o_full, 0))) {
      tc_fence_after();
      tmem_ld_32x32b_x32_nowait(trow + C::T_O + 64 * G, u);
      tmem_ld_32x32b_x32_nowait(trow + C::T_O + 64 * G + 32, u + 32);
      uint32_t lsum = tmem_ld_32x32b_x1_nowait(trow + C::T_O + kAttD);
      tc_wait_ld();
      reg_fence32(u);
      reg_fence32(u + 32);
      asm volatile("" : "+r"(lsum)::"memory");
      const float inv_l = 1.0f / __uint_as_float(lsum);
      uint4* dst = reinterpret_cast<uint4*>(args.out + (static_cast<int64_t>(qrow0) + r) * kAttD + 64 * G);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
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
// along tokens.  One CTA per (head, 128-token block), 256 threads: thread
// (p = tid % 64, blk = tid / 64) quantises channels 2p and 2p + 1 over tokens
// [32 blk, 32 blk + 32) of the block, reading the staged tile as bf16 pairs
// (a warp reads 128 contiguous bytes of a token row).
constexpr int kVtThreads = 256;
__global__ void __launch_bounds__(kVtThreads) quantize_mxfp8_vt_kernel(const __nv_bfloat16* __restrict__ v, int heads,
                                                                     int tokens, uint8_t* __restrict__ codes,
                                                                     uint8_t* __restrict__ sf) {
  __shared__ __align__(16) __nv_bfloat16 tile[kAttTile][kAttD];
  grid_dep_wait();
  grid_dep_launch();
  const int nkb = tokens / kAttTile;
  const int h = blockIdx.x / nkb, t0 = (blockIdx.x % nkb) * kAttTile;
  const uint4* src = reinterpret_cast<const uint4*>(v + (static_cast<int64_t>(h) * tokens + t0) * kAttD);
  uint4* stile = reinterpret_cast<uint4*>(&tile[0][0]);
#pragma unroll
  for (int i = 0; i < kAttTile * kAttD / 8 / kVtThreads; ++i)
    stile[threadIdx.x + i * kVtThreads] = ldg_nc_v4(src + threadIdx.x + i * kVtThreads);
  __syncthreads();
  const int p = threadIdx.x & 63, blk = threadIdx.x >> 6;
  // the two channels' 32 values stay packed as bf16 pairs (32 registers)
  uint32_t pr[32];
  float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    pr[i] = *reinterpret_cast<const uint32_t*>(&tile[32 * blk + i][2 * p]);
    m0 = fmaxf(m0, fabsf(__uint_as_float(pr[i] << 16)));
    m1 = fmaxf(m1, fabsf(__uint_as_float(pr[i] & 0xFFFF0000u)));
  }
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    const float bmax = ch == 0 ? m0 : m1;
    int X = -127;
    if (bmax > 0.0f) X = min(max(floor_log2_f32(bmax) - 8, -127), 127);  // OCP floor rule
    const float mult = exp2_int(-X);
    auto val = [&](int i) { return __uint_as_float(ch == 0 ? pr[i] << 16 : pr[i] & 0xFFFF0000u) * mult; };
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = cvt_e4m3x2(val(4 * i), val(4 * i + 1)) | (cvt_e4m3x2(val(4 * i + 2), val(4 * i + 3)) << 16);
    const int64_t row = static_cast<int64_t>(h) * kAttD + 2 * p + ch;
    uint4* dst = reinterpret_cast<uint4*>(codes + row * tokens + t0 + 32 * blk);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    sf[sf_offset(row, (t0 >> 5) + blk, tokens >> 7)] = static_cast<uint8_t>(X + 127);
  }
  // rows heads * 128 are a multiple of 128: no scale padding to clear
}

}  // namespace mxq

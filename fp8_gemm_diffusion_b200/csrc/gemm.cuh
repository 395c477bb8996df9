// gemm.cuh - block-scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
//   Y[M,N] = bf16_rne( alpha * sum_k deq(A)[m,k] * deq(B)[n,k] + bias[n] )
//
// A [M,K] and B [N,K] are K-major codes (NVFP4 E2M1 packed two per byte,
// MXFP8 E4M3, or plain bf16), with block scales in the tensor-core
// block-scaling layout.  alpha = g_A * g_B (NVFP4 per-tensor scales, read on
// the device) or 1.
//
// Source: the quantised linear layer of the B200 MXFP8/NVFP4 diffusion
// article (its "Benchmark Results" speed-ups come from running these GEMMs on
// Blackwell's FP4/FP8 tensor cores); the Blackwell features the WaveSpeedAI x
// DataCrunch B200 article lists ("NVIDIA's Blackwell GPU architecture: B200":
// tensor memory, CTA pairs, 5th-generation FP8/FP4 tensor cores) are what this
// kernel is built on.
//
// Design (one CTA per SM, persistent over output tiles of 128 x BN):
//   warp 0      TMA producer: A tile (128 rows x 128 B), B tile (BN rows x
//               128 B), 128-byte swizzled, plus the scale-factor chunks (bulk
//               copies), into a STAGES-deep shared-memory ring guarded by
//               full/empty mbarriers.
//   warp 1      allocates tensor memory; one lane issues, per stage,
//               tcgen05.cp of the scale factors into tensor memory and four
//               tcgen05.mma (kind::mxf4nvf4 block16 / kind::mxf8f6f4 /
//               kind::f16), accumulating in fp32 in tensor memory; commits
//               free the smem stage and, per tile, signal the epilogue.
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time (each warp owns one
//               32-lane sub-partition = 32 rows), alpha/bias/bf16 in
//               registers, 64-byte-swizzled staging in shared memory, TMA
//               store.  Accumulators are double-buffered in tensor memory so
//               the epilogue of tile i overlaps the main loop of tile i+1.
// Every mbarrier wait is bounded (ptx.cuh); on a timeout each role stops,
// drains what it has in flight, and the CTA frees its tensor memory.
#pragma once

#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "ptx.cuh"

namespace mxq {

enum class Fmt : int { NVFP4 = 0, MXFP8 = 1, BF16 = 2 };

template <Fmt F, int BN_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "BN");
  static constexpr int ROW_BYTES = 128;  // K bytes per smem row and stage (one swizzle atom)
  static constexpr int K_STAGE = F == Fmt::NVFP4 ? 256 : (F == Fmt::MXFP8 ? 128 : 64);
  static constexpr int MMA_K = F == Fmt::NVFP4 ? 64 : (F == Fmt::MXFP8 ? 32 : 16);
  static constexpr int MMAS = K_STAGE / MMA_K;  // 4
  static constexpr bool SCALED = F != Fmt::BF16;
  // 128-row scale blocks a B tile can touch (a 192-wide tile may start mid-block)
  static constexpr int NRB = (BN + 127) / 128;
  // scale chunks (512 B = 128 rows x 4 scales) per stage
  static constexpr int SFA_CHUNKS = F == Fmt::NVFP4 ? MMAS : (F == Fmt::MXFP8 ? 1 : 0);
  static constexpr int SFB_CHUNKS = SFA_CHUNKS * NRB;
  static constexpr int A_BYTES = BM * ROW_BYTES;
  static constexpr int B_BYTES = BN * ROW_BYTES;
  static constexpr int SFA_BYTES = SFA_CHUNKS * 512;
  static constexpr int SFB_BYTES = SFB_CHUNKS * 512;
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES + 1023) / 1024 * 1024;
  // tensor memory: accumulators, then two sets of scale columns
  static constexpr int SF_SET_COLS = (SFA_CHUNKS + SFB_CHUNKS) * 4;
  static constexpr int ACC_BUFS = (2 * BN + 2 * SF_SET_COLS <= 512) ? 2 : 1;
  static constexpr int TMEM_USED = ACC_BUFS * BN + 2 * SF_SET_COLS;
  static_assert(TMEM_USED <= 512, "tensor memory");
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int SFA_COL = ACC_BUFS * BN;  // first scale set
  static constexpr int SFB_COL = SFA_COL + SFA_CHUNKS * 4;
  static constexpr int EPI_WARPS = 4;
  static constexpr int EPI_BUFS = 2;
  static constexpr int EPI_BUF_BYTES = 32 * 64;  // 32 rows x 32 bf16
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_BUFS * EPI_BUF_BYTES;
  static constexpr int STAGES_FIT = (232448 - 1024 - 512 - EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static_assert(STAGES >= 2, "shared memory");
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
};

// Instruction descriptors (32-bit), fields per the tcgen05 MMA instruction
// descriptor: [4,6) B scale id / D format, [7,10) A type, [10,13) B type,
// [15]/[16] A/B major (0 = K-major), [17,23) N>>3, [23] scale type
// (block-scaled kinds: 0 = UE4M3, 1 = UE8M0), [24,29) M>>4, [29,31) A scale id.
template <Fmt F>
__device__ __forceinline__ uint32_t make_idesc(int n, uint32_t sf_id) {
  const uint32_t m_field = (128u >> 4) << 24;
  const uint32_t n_field = (static_cast<uint32_t>(n) >> 3) << 17;
  if constexpr (F == Fmt::NVFP4) {
    // A, B = E2M1 (kind::mxf4nvf4 encoding 1), scales UE4M3
    return (sf_id << 4) | (1u << 7) | (1u << 10) | n_field | (0u << 23) | m_field | (sf_id << 29);
  } else if constexpr (F == Fmt::MXFP8) {
    // A, B = E4M3 (kind::mxf8f6f4 encoding 0), scales UE8M0
    return (sf_id << 4) | (0u << 7) | (0u << 10) | n_field | (1u << 23) | m_field | (sf_id << 29);
  } else {
    // D = F32 (1 in [4,6)), A, B = BF16 (1)
    return (1u << 4) | (1u << 7) | (1u << 10) | n_field | m_field;
  }
}

struct GemmArgs {
  int M, N, K;
  const uint8_t* a_sf;  // swizzled scales of A (NVFP4 / MXFP8)
  const uint8_t* b_sf;
  const float* a_g;     // NVFP4 per-tensor scales (device)
  const float* b_g;
  const __nv_bfloat16* bias;  // [N] or nullptr
};

template <Fmt F, int BN>
__global__ void __launch_bounds__(GemmCfg<F, BN>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  using C = GemmCfg<F, BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t epi_base = base + C::STAGES * C::STAGE_BYTES;
  const uint32_t bar_base = epi_base + C::EPI_BYTES;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * C::STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * C::STAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * C::STAGES + 4);
  uint32_t* const tmem_slot =
      reinterpret_cast<uint32_t*>(base_ptr + (bar_base - base) + 8u * (2 * C::STAGES + 5));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int M = args.M, N = args.N, K = args.K;
  const int m_tiles = (M + C::BM - 1) / C::BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (K + C::K_STAGE - 1) / C::K_STAGE;
  const int sf_rb_b = (N + 127) / 128;  // 128-row scale blocks of B
  // 512-byte scale chunks (4 scale columns) per 128-row block
  const int sf_c4 = F == Fmt::NVFP4 ? K / 64 : (F == Fmt::MXFP8 ? K / 128 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), C::EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_y);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above overlaps the previous kernel's tail; A, its scales and
  // the per-tensor scales are that kernel's output
  grid_dep_wait();
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mt = tile % m_tiles, nt = tile / m_tiles;
        const int m0 = mt * C::BM, n0 = nt * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u)) { ok = false; break; }
          const uint32_t sa = base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          uint32_t bytes = C::A_BYTES + C::B_BYTES;
          int nchunk = C::SFA_CHUNKS;
          if constexpr (F == Fmt::NVFP4) {
            const int left = K / 64 - kb * C::MMAS;
            nchunk = left < C::MMAS ? left : C::MMAS;
          }
          int nrb_b = 0;
          if constexpr (C::SCALED) {
            const int rb0 = n0 / 128;
            nrb_b = sf_rb_b - rb0 < C::NRB ? sf_rb_b - rb0 : C::NRB;
            bytes += 512u * nchunk * (1 + nrb_b);
          }
          mbar_arrive_expect_tx(full_bar(stage), bytes);
          tma_load_2d(sa, &tmap_a, full_bar(stage), kb * C::ROW_BYTES / (F == Fmt::BF16 ? 2 : 1), m0);
          tma_load_2d(sb, &tmap_b, full_bar(stage), kb * C::ROW_BYTES / (F == Fmt::BF16 ? 2 : 1), n0);
          if constexpr (C::SCALED) {
            // chunk index of (row block rb, 4-column group kc): rb * sf_c4 + kc
            const int kc0 = kb * C::SFA_CHUNKS;
            const uint32_t ssfa = sb + C::B_BYTES;
            const uint32_t ssfb = ssfa + C::SFA_BYTES;
            bulk_load(ssfa, args.a_sf + (static_cast<int64_t>(m0 / 128) * sf_c4 + kc0) * 512,
                      512u * nchunk, full_bar(stage));
            for (int c = 0; c < nrb_b; ++c) {
              bulk_load(ssfb + c * C::SFA_CHUNKS * 512,
                        args.b_sf + (static_cast<int64_t>(n0 / 128 + c) * sf_c4 + kc0) * 512,
                        512u * nchunk, full_bar(stage));
            }
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA can exit
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < C::STAGES && i < issued; ++i) {
          if (--s < 0) { s = C::STAGES - 1; ph ^= 1u; }
          mbar_wait_bounded(full_bar(s), ph);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int nt = tile / m_tiles;
        const int n0 = nt * BN;
        const uint32_t sfb_shift = (n0 & 127) >> 5;  // tile starts mid scale block
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * C::STAGE_BYTES;
          const uint32_t sb = sa + C::A_BYTES;
          int nmma = C::MMAS;
          if constexpr (F == Fmt::NVFP4) {
            const int left = K / 64 - kb * C::MMAS;
            nmma = left < C::MMAS ? left : C::MMAS;
          }
          const uint32_t set_col = (iter & 1u) * C::SF_SET_COLS;
          if constexpr (C::SCALED) {
            const uint32_t ssfa = sb + C::B_BYTES;
            const uint32_t ssfb = ssfa + C::SFA_BYTES;
            const int nchunk = F == Fmt::NVFP4 ? nmma : 1;
            for (int j = 0; j < nchunk; ++j) {
              tc_cp_32x128b_warpx4(tmem_base + C::SFA_COL + set_col + 4 * j, desc_sf_chunk(ssfa + 512 * j));
            }
            const int rb0 = n0 / 128;
            const int nrb_b = sf_rb_b - rb0 < C::NRB ? sf_rb_b - rb0 : C::NRB;
            for (int c = 0; c < nrb_b; ++c) {
              for (int j = 0; j < nchunk; ++j) {
                // scale set of MMA j holds NRB consecutive 4-column chunks
                tc_cp_32x128b_warpx4(tmem_base + C::SFB_COL + set_col + (j * C::NRB + c) * 4,
                                     desc_sf_chunk(ssfb + (c * C::SFA_CHUNKS + j) * 512));
              }
            }
          }
          const uint64_t adesc = desc_kmajor_sw128(sa);
          const uint64_t bdesc = desc_kmajor_sw128(sb);
          for (int j = 0; j < nmma; ++j) {
            const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
            // every MMA consumes 32 bytes of each row: advance the start address
            const uint64_t koff = static_cast<uint64_t>(2 * j);  // (32 * j) >> 4
            if constexpr (F == Fmt::NVFP4) {
              const uint32_t sfa = tmem_base + C::SFA_COL + set_col + 4 * j;
              const uint32_t sfb = tmem_base + C::SFB_COL + set_col + j * C::NRB * 4 + sfb_shift;
              mma_nvfp4(d_tmem, adesc + koff, bdesc + koff, make_idesc<F>(BN, 0), sfa, sfb, accum);
            } else if constexpr (F == Fmt::MXFP8) {
              const uint32_t sfa = (tmem_base + C::SFA_COL + set_col) | (static_cast<uint32_t>(j) << 30);
              const uint32_t sfb = (tmem_base + C::SFB_COL + set_col + sfb_shift) | (static_cast<uint32_t>(j) << 30);
              mma_mxfp8(d_tmem, adesc + koff, bdesc + koff, make_idesc<F>(BN, j), sfa, sfb, accum);
            } else {
              mma_bf16(d_tmem, adesc + koff, bdesc + koff, make_idesc<F>(BN, 0), accum);
            }
          }
          tc_commit(empty_bar(stage));  // smem stage free once these MMAs are done
          ++iter;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));  // accumulator ready for the epilogue
        if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
      }
      // every MMA / copy issued above must finish before tensor memory is freed
      tc_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory sub-partition this warp may access
    const uint32_t stage_buf0 = epi_base + (warp - 2) * C::EPI_BUFS * C::EPI_BUF_BYTES;
    float alpha = 1.0f;
    if constexpr (F == Fmt::NVFP4) alpha = (*args.a_g) * (*args.b_g);
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t chunk_count = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mt = tile % m_tiles, nt = tile / m_tiles;
      const int m0 = mt * C::BM, n0 = nt * BN;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tfull_bar(acc), acc_phase))) break;  // tcgen05.ld is warp-collective
      tc_fence_after();
      const int row0 = m0 + q * 32;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = n0 + c * 32;
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        tc_wait_ld();
        if (c == BN / 32 - 1) {
          // accumulator fully read: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        if (row0 >= M || col0 >= N) continue;
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float v0 = __uint_as_float(r[2 * i]), v1 = __uint_as_float(r[2 * i + 1]);
          if constexpr (F == Fmt::NVFP4) { v0 *= alpha; v1 *= alpha; }
          if (args.bias != nullptr) {
            const int n = col0 + 2 * i;
            if (n < N) v0 += __bfloat162float(args.bias[n]);
            if (n + 1 < N) v1 += __bfloat162float(args.bias[n + 1]);
          }
          const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
          packed[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        const uint32_t buf = stage_buf0 + (chunk_count % C::EPI_BUFS) * C::EPI_BUF_BYTES;
        if (lane == 0) bulk_wait_group_read<C::EPI_BUFS - 1>();
        __syncwarp();
        // row `lane`: 64 bytes = 4 chunks of 16 B, 64-byte swizzle (chunk ^= (row>>1)&3)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t addr = buf + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[4 * j]),
                       "r"(packed[4 * j + 1]), "r"(packed[4 * j + 2]), "r"(packed[4 * j + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmap_y, buf, col0, row0);
          bulk_commit_group();
        }
        ++chunk_count;
      }
      if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace mxq

// gemm_pair.cuh - block-scaled GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same result as gemm.cuh, Y = bf16(alpha * A.B^T + bias), computed with
// 256 x BN output tiles on a pair of CTAs in one cluster (the "CTA pair" of
// the WaveSpeedAI x DataCrunch B200 article, section "NVIDIA's Blackwell GPU
// architecture: B200"): each CTA loads its own 128 rows of A and BN/2 rows of
// B, and the even CTA of the pair issues M=256 MMAs that read A and B from
// both CTAs' shared memory and leave each CTA's 128 rows of D in that CTA's
// tensor memory.  Per CTA this halves the operand traffic of a 128 x BN tile
// and the pair MMA runs the tensor cores at a higher rate than M=128 MMAs.
//
// Roles (both CTAs; 16 warps, registers rebalanced per warpgroup):
//   warp 0      A/B producer: each stage's 128 rows of A and BN/2 rows of B
//               into this CTA's ring; completions land on the even CTA's full
//               barrier (cta_group::2 loads, no multicast).
//   warp 1      tensor memory (cta_group::2 allocation); on the even CTA the
//               converged warp runs the MMA loop and one elected lane issues
//               each MMA and commit (descriptors and addresses stay
//               warp-uniform).  Commits go to both CTAs' barriers (multicast
//               commit): stage free (its A/B slot, and the scale set it used),
//               right after the stage's MMAs, and accumulator full.  This
//               warp never waits on a shared-memory barrier between MMAs: a
//               shared-memory access right after a batch of MMAs stalls the
//               issuing warp for a few hundred cycles, which left the tensor
//               pipe idle once per stage.
//   warp 3      stage waiter (even CTA): waits on the accumulator-empty and
//               full barriers and hands each stage to warp 1 through a named
//               barrier that also carries the "no timeout" flag.
//   warp 2      scale loader: the scale chunks of each stage (A's 128 rows and
//               all BN columns of B: each CTA's tensor memory needs B's) into
//               a separate ring that runs ahead of the A/B ring.
//   warps 4-7   scale writers, one per tensor-memory sub-partition: chunk rows
//               from shared memory into a set of tensor-memory columns with
//               tcgen05.st, so no tcgen05.cp sits between MMAs; they arrive on
//               the even CTA's full barrier of the stage, which thus completes
//               when A, B and all scales are in place.  The scale sets form
//               their own ring (NSF <= STAGES sets, as many as tensor memory
//               holds beside the accumulator), so the A/B ring can be deeper
//               than the number of scale sets.
//   warps 8-15  epilogue, sub-partition warp % 4, column half (warp / 4) % 2:
//               the warp's accumulator columns into registers, release of the
//               accumulator, then alpha, bias, bf16, swizzled staging (two
//               buffers per warp) and TMA stores of 32 x EPI_SUB sub-tiles.
// Tiles are visited along the smaller operand first (pair_tile_coords).
// Every wait is bounded (ptx.cuh); a timed-out role stops, loads and MMAs in
// flight are drained, and both CTAs free tensor memory together.
#pragma once

#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <cstdint>

#include "gemm.cuh"
#include "ptx.cuh"

namespace mxq {

template <Fmt F, int BN_>
struct PairCfg {
  static constexpr int BM = 256;      // rows of a pair tile
  static constexpr int BM_CTA = 128;  // rows per CTA
  static constexpr int BN = BN_;
  static constexpr int BN_CTA = BN / 2;
  static_assert(BN == 128 || BN == 256, "BN: the epilogue drains 128-column batches");
  static constexpr int ROW_BYTES = 128;
  static constexpr int K_STAGE = F == Fmt::NVFP4 ? 256 : (F == Fmt::MXFP8 ? 128 : 64);
  static constexpr int MMA_K = F == Fmt::NVFP4 ? 64 : (F == Fmt::MXFP8 ? 32 : 16);
  static constexpr int MMAS = K_STAGE / MMA_K;
  static constexpr bool SCALED = F != Fmt::BF16;
  static constexpr int NRB = (BN + 127) / 128;  // 128-row scale blocks of the pair's B tile
  static constexpr int SF_CHUNKS = F == Fmt::NVFP4 ? MMAS : (F == Fmt::MXFP8 ? 1 : 0);  // per 128 rows
  static constexpr int SF_BOX_ROWS = SF_CHUNKS * 2;  // scales are loaded as [rows][256 B]
  static constexpr int A_BYTES = BM_CTA * ROW_BYTES;
  static constexpr int B_BYTES = BN_CTA * ROW_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // multiple of 1024
  static constexpr uint32_t AB_PAIR_TX = 2u * STAGE_BYTES;  // A/B of both CTAs
  static constexpr int SFA_BYTES = SF_CHUNKS * 512;
  static constexpr int SFB_BYTES = NRB * SF_CHUNKS * 512;
  static constexpr uint32_t SF_TX = SFA_BYTES + SFB_BYTES;  // this CTA's scales
  static constexpr int SF_SLOT_BYTES = SCALED ? (SFA_BYTES + SFB_BYTES + 1023) / 1024 * 1024 : 0;
  static constexpr int SF_SLOTS = SCALED ? (F == Fmt::NVFP4 ? 4 : 8) : 0;
  // tensor memory: the accumulator (BN columns), then the ring of scale sets
  // (A chunks, then B chunks in MMA-major order, 4 columns each)
  static constexpr int SF_SET_COLS = (SF_CHUNKS + NRB * SF_CHUNKS) * 4;
  static constexpr int SF_COL = BN;
  static constexpr int SFB_OFF = SF_CHUNKS * 4;
  static constexpr int TMEM_COLS = 512;
  static constexpr int NSF_FIT = SCALED ? (TMEM_COLS - BN) / SF_SET_COLS : 1;
  // warp roles, one warpgroup each for (producer, MMA, scale loader, spare),
  // the scale writers and the two halves of the epilogue
  static constexpr int SF_WARP0 = 4;   // warps 4-7, one per tensor-memory sub-partition
  static constexpr int SF_WARPS = 4;
  static constexpr int EPI_WARP0 = 8;  // warps 8-15: sub-partition warp % 4, column half (warp / 4) % 2
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_COLS = BN / 2;   // accumulator columns per epilogue warp
  static constexpr int EPI_SUB = 16;        // staging sub-tile: 32 rows x EPI_SUB columns
  static constexpr int EPI_ROW = EPI_SUB * 2;  // its row bytes, swizzled over the whole row (TMA swizzle mode)
  static constexpr int EPI_BUFS = 1;        // per warp (a second buffer measured no faster and costs a stage)
  static constexpr int EPI_BYTES = EPI_WARPS * EPI_BUFS * 32 * EPI_SUB * 2;
  // registers: launched with 65536 / 512 = 128 per thread, then rebalanced so
  // that an epilogue thread holds its 128 accumulator columns at once
  static constexpr int REGS_CTRL = 56, REGS_SFW = 80, REGS_EPI = 184;
  static constexpr int BAR_BYTES = 512;
  static constexpr int STAGES_FIT =
      (232448 - 1024 - BAR_BYTES - EPI_BYTES - SF_SLOTS * SF_SLOT_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  // scale sets: as many as fit, at most one per A/B stage (a writer's wait for
  // its set then also covers the stage's previous full-barrier phase)
  static constexpr int NSF = SCALED ? (NSF_FIT < STAGES ? NSF_FIT : STAGES) : 1;
  // arrivals that complete a stage's full barrier besides the A/B bytes: the
  // producer's expect-tx and the scale writers of both CTAs
  static constexpr int FULL_ARRIVALS = 1 + (SCALED ? 2 * SF_WARPS : 0);
  static_assert(STAGES >= 2 && (!SCALED || NSF >= 2), "shared / tensor memory");
  static_assert(4 * STAGES + 4 * SF_SLOTS + 32 <= BAR_BYTES / 4, "barrier area");
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + SF_SLOTS * SF_SLOT_BYTES + EPI_BYTES + BAR_BYTES;
  static constexpr int THREADS = 512;
  static_assert(128 * (REGS_CTRL + REGS_SFW) + 256 * REGS_EPI <= 65536, "register split");
};

// Instruction descriptor of an M=256 (pair) MMA; fields as in make_idesc.
template <Fmt F>
__device__ __forceinline__ uint32_t make_idesc_pair(int n, uint32_t sf_id) {
  const uint32_t m_field = (256u >> 4) << 24;
  const uint32_t n_field = (static_cast<uint32_t>(n) >> 3) << 17;
  if constexpr (F == Fmt::NVFP4) {
    return (sf_id << 4) | (1u << 7) | (1u << 10) | n_field | m_field | (sf_id << 29);
  } else if constexpr (F == Fmt::MXFP8) {
    return (sf_id << 4) | n_field | (1u << 23) | m_field | (sf_id << 29);
  } else {
    return (1u << 4) | (1u << 7) | (1u << 10) | n_field | m_field;
  }
}

// Tile order: tiles run along the dimension of the smaller operand first, so
// the pairs working at the same time share all of that operand (it stays in
// L2) and only a few strips of the larger one, which HBM then delivers once.
__device__ __forceinline__ void pair_tile_coords(int tile, int m_tiles, int n_tiles, bool n_fast,
                                                 int& mt, int& nt) {
  if (n_fast) {
    mt = tile / n_tiles;
    nt = tile - mt * n_tiles;
  } else {
    nt = tile / m_tiles;
    mt = tile - nt * m_tiles;
  }
}

// Named barrier between the MMA warp and the stage waiter (id 0 is __syncthreads).
constexpr uint32_t kStageBar = 1;
// MMA-issue order inside a stage: the next stage's handover goes before MMA
// kHandoverBefore of the current one; with kLateCommit a stage's commit goes
// behind the next stage's first MMA instead of right after its own MMAs.
constexpr int kHandoverBefore = 3;
constexpr bool kLateCommit = false;

struct PairArgs {
  int M, N, K;
  const float* a_g;
  const float* b_g;
  const __nv_bfloat16* bias;
  int act;                // EPI != 0 only: 1 = GELU on alpha * acc + bias before the bf16 rounding
  unsigned int* y_amax;   // EPI != 0 only: max |y| over the bf16 outputs, folded in with atomicMax
};

// GELU, x * Phi(x), Phi(x) = (1 + erf(x / sqrt 2)) / 2, in fp32, with erf by
// formula 7.1.26 of Abramowitz and Stegun's Handbook of Mathematical
// Functions: for z >= 0, 1 - erf(z) = t (a1 + t (a2 + t (a3 + t (a4 + t a5))))
// e^(-z^2), t = 1 / (1 + p z), absolute error at most 1.5e-7.  With
// z = |x| / sqrt 2 and q = 1 - erf(z): GELU(x) = x - x q / 2 for x >= 0 and
// x q / 2 for x < 0 (no cancellation on the negative side).  Two
// special-function operations (the reciprocal and 2^x) and a dozen FMAs: the
// epilogue of a whole tile then stays within the tile's MMA time.
__device__ __forceinline__ float gelu_erf(float x) {
  const float t = rcp_approx(fmaf(0.3275911f * 0.70710678118654752f, fabsf(x), 1.0f));
  float p = 1.061405429f;
  p = fmaf(p, t, -1.453152027f);
  p = fmaf(p, t, 1.421413741f);
  p = fmaf(p, t, -0.284496736f);
  p = fmaf(p, t, 0.254829592f);
  const float e = ex2_approx(-0.72134752044448170f * x * x);  // e^(-x^2 / 2)
  const float hq = 0.5f * x * (p * t) * e;                      // x q / 2
  return x >= 0.0f ? x - hq : hq;
}

// EPI = 0: the plain epilogue.  EPI = 1: the producer epilogue of a layer
// whose output feeds the next layer's quantiser: optional GELU, and the
// output's max |y| folded into one device word, so that the next layer's
// NVFP4 quantisation needs no amax pass over its input.
template <Fmt F, int BN, int EPI = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<F, BN>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa,
                     const __grid_constant__ CUtensorMap tmap_sfb,
                     const __grid_constant__ CUtensorMap tmap_y, const PairArgs args) {
  using C = PairCfg<F, BN>;
  constexpr int S = C::STAGES, R = C::SF_SLOTS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw_addr);
  const uint32_t sf_base = base + S * C::STAGE_BYTES;
  const uint32_t epi_base = sf_base + R * C::SF_SLOT_BYTES;
  const uint32_t bar_base = epi_base + C::EPI_BYTES;
  // barriers: [full S][empty S][sf_full R][sf_empty R][tfull][tempty][drain]
  auto full_bar = [&](int s) { return bar_base + 8u * s; };  // even CTA: A/B landed, scales written
  auto empty_bar = [&](int s) { return bar_base + 8u * (S + s); };          // both: A/B stage free
  auto sf_full_bar = [&](int r) { return bar_base + 8u * (2 * S + r); };    // both: own scales landed
  auto sf_empty_bar = [&](int r) { return bar_base + 8u * (2 * S + R + r); };  // both: slot read
  const uint32_t tfull_bar = bar_base + 8u * (2 * S + 2 * R);
  const uint32_t tempty_bar = tfull_bar + 8u;
  const uint32_t drain_bar = tfull_bar + 16u;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + (tfull_bar + 24u - base));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs of the pair

  const int M = args.M, N = args.N, K = args.K;
  const int m_tiles = (M + C::BM - 1) / C::BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const bool n_fast = N < M;  // B is the smaller operand
  const int num_kb = (K + C::K_STAGE - 1) / C::K_STAGE;
  const int sf_c4 = F == Fmt::NVFP4 ? K / 64 : (F == Fmt::MXFP8 ? K / 128 : 0);
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / num_pairs + 1 : 0;
  const int total_kb = my_tiles * num_kb;  // stages this pair runs

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), C::FULL_ARRIVALS);
      mbar_init(empty_bar(s), 1);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(sf_full_bar(r), 1);
      mbar_init(sf_empty_bar(r), C::SF_WARPS);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(tempty_bar, 2 * C::EPI_WARPS);
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_y);
    if constexpr (C::SCALED) {
      prefetch_tmap(&tmap_sfa);
      prefetch_tmap(&tmap_sfb);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // B (the weight) is not the previous kernel's output: the B halves of the
  // first stages are requested before the dependency wait, so that their
  // latency overlaps that kernel's tail.  The producer below then issues only
  // A for those stages.
  const int a_row_off = static_cast<int>(rank) * C::BM_CTA;
  const int b_row_off = static_cast<int>(rank) * C::BN_CTA;
  constexpr int KX = C::ROW_BYTES / (F == Fmt::BF16 ? 2 : 1);  // K coordinate step per stage
  const int n_pre = total_kb < S ? total_kb : S;                // stages with B requested early
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < n_pre; ++g) {
      const int tile = pair + (g / num_kb) * num_pairs, kb = g % num_kb;
      int mt, nt;
      pair_tile_coords(tile, m_tiles, n_tiles, n_fast, mt, nt);
      if (rank == 0) mbar_arrive_expect_tx(full_bar(g), C::AB_PAIR_TX);
      tma_load_2d_pair(base + g * C::STAGE_BYTES + C::A_BYTES, &tmap_b, map_to_cta(full_bar(g), 0),
                       kb * KX, nt * BN + b_row_off);
    }
  }
  // everything above overlaps the previous kernel's tail; A, its scales and
  // the per-tensor scales are that kernel's output
  grid_dep_wait();
  grid_dep_launch();

  // Registers move from the control and scale-writer warpgroups to the
  // epilogue: each warpgroup's setmaxnreg opens its role's code.
  if (warp < C::SF_WARP0) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_CTRL));
  if (warp == 0) {
    // ------------------------------------------------------------ A/B producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        pair_tile_coords(tile, m_tiles, n_tiles, n_fast, mt, nt);
        const int a_row = mt * C::BM + a_row_off, b_row = nt * BN + b_row_off;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u)) { ok = false; break; }
          const uint32_t leader_full = map_to_cta(full_bar(s), 0);
          const uint32_t sa = base + s * C::STAGE_BYTES;
          if (issued >= n_pre) {
            if (rank == 0) mbar_arrive_expect_tx(full_bar(s), C::AB_PAIR_TX);
            tma_load_2d_pair(sa + C::A_BYTES, &tmap_b, leader_full, kb * KX, b_row);
          }
          tma_load_2d_pair(sa, &tmap_a, leader_full, kb * KX, a_row);
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        // let every armed stage land before the pair can exit
        for (int i = 0; i < S && i < issued; ++i) {
          if (--s < 0) { s = S - 1; ph ^= 1u; }
          if (!mbar_wait_bounded(full_bar(s), ph)) break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The converged warp runs the loop (descriptors and addresses are
    // warp-uniform); one elected lane issues each MMA and commit.  Stages
    // arrive through the named barrier shared with the stage waiter (warp 3).
    if (rank == 0) {
      int s = 0, n = 0, pend = -1;  // A/B stage, scale set; pend: stage whose commit is deferred
      bool ok = true;
      const uint64_t adesc0 = desc_kmajor_sw128(base);
      const uint64_t bdesc0 = desc_kmajor_sw128(base + C::A_BYTES);
      constexpr uint64_t DSTEP = C::STAGE_BYTES >> 4;  // descriptor start-address step per stage
      const uint32_t idesc = make_idesc_pair<F>(BN, 0);
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        pair_tile_coords(tile, m_tiles, n_tiles, n_fast, mt, nt);
        const uint32_t sfb_shift = ((nt * BN) & 127) >> 5;
        // the tile's first stage has landed and the accumulator is free
        // (unless the waiter's bounded waits ran out)
        if (!(ok = named_bar_and(kStageBar, 64, true))) break;
        for (int kb = 0; kb < num_kb; ++kb) {
          tc_fence_after();
          const uint64_t adesc = adesc0 + DSTEP * s, bdesc = bdesc0 + DSTEP * s;
          const uint32_t sf = tmem_base + C::SF_COL + n * C::SF_SET_COLS;
          int nmma = C::MMAS;
          if constexpr (F == Fmt::NVFP4) {
            if (kb == num_kb - 1) nmma = K / 64 - kb * C::MMAS;  // K % 256 != 0: partial last stage
          }
          const bool next = kb + 1 < num_kb;  // then nmma == MMAS
#pragma unroll
          for (int j = 0; j < C::MMAS; ++j) {
            // The next stage's handover goes before this stage's last MMA: the
            // handover stalls this warp until the MMAs issued so far are under
            // way, and the last MMA still queued keeps the pipe busy meanwhile.
            if (j == kHandoverBefore && next) ok = named_bar_and(kStageBar, 64, true);
            if (j < nmma) {
              const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
              const uint64_t koff = static_cast<uint64_t>(2 * j);  // 32 bytes of K per MMA
              if constexpr (F == Fmt::NVFP4) {
                mma_pair_nvfp4_elect(tmem_base, adesc + koff, bdesc + koff, idesc, sf + 4 * j,
                                     sf + C::SFB_OFF + j * C::NRB * 4 + sfb_shift, accum);
              } else if constexpr (F == Fmt::MXFP8) {
                const uint32_t id = static_cast<uint32_t>(j) << 30;
                mma_pair_mxfp8_elect(tmem_base, adesc + koff, bdesc + koff,
                                     idesc | (static_cast<uint32_t>(j) << 4) | (static_cast<uint32_t>(j) << 29),
                                     sf | id, (sf + C::SFB_OFF + sfb_shift) | id, accum);
              } else {
                mma_pair_bf16_elect(tmem_base, adesc + koff, bdesc + koff, idesc, accum);
              }
            }
            // a deferred commit of the previous stage, behind this stage's first MMA
            if (kLateCommit && j == 0 && pend >= 0) {
              tc_commit_pair_elect(empty_bar(pend));
              pend = -1;
            }
          }
          if (kLateCommit) pend = s;                 // committed behind the next stage's first MMA
          else tc_commit_pair_elect(empty_bar(s));   // A/B slot s and scale set n free once these complete
          if (++s == S) s = 0;
          if (++n == C::NSF) n = 0;
          if (!ok) break;
        }
        if (pend >= 0) tc_commit_pair_elect(empty_bar(pend));
        pend = -1;
        if (!ok) break;
        tc_commit_pair_elect(tfull_bar);
      }
      tc_commit_pair_elect(drain_bar);
      mbar_wait_bounded(drain_bar, 0);
    } else if (lane == 0) {
      // odd CTA: the pair's MMAs read this CTA's memory; wait for the last one
      mbar_wait_bounded(drain_bar, 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale loader
    if constexpr (C::SCALED) if (lane == 0) {
      int r = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        pair_tile_coords(tile, m_tiles, n_tiles, n_fast, mt, nt);
        // 512-byte chunk (row block rb, 4-column group kc) is 256-byte row 2*(rb*sf_c4+kc)
        const int ya = 2 * (mt * 2 + static_cast<int>(rank)) * sf_c4;
        const int yb = 2 * (nt * BN / 128) * sf_c4;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(sf_empty_bar(r), ph ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(sf_full_bar(r), C::SF_TX);
          const uint32_t slot = sf_base + r * C::SF_SLOT_BYTES;
          const int kc2 = 2 * kb * C::SF_CHUNKS;
          tma_load_2d(slot, &tmap_sfa, sf_full_bar(r), 0, ya + kc2);
#pragma unroll
          for (int c = 0; c < C::NRB; ++c)
            tma_load_2d(slot + C::SFA_BYTES + c * C::SFA_BYTES, &tmap_sfb, sf_full_bar(r), 0,
                        yb + 2 * c * sf_c4 + kc2);
          ++issued;
          if (++r == R) { r = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        for (int i = 0; i < R && i < issued; ++i) {
          if (--r < 0) { r = R - 1; ph ^= 1u; }
          mbar_wait_bounded(sf_full_bar(r), ph);
        }
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ stage waiter
    // Waits, for the MMA warp, on the accumulator (once per tile) and on each
    // stage's full barrier, then meets the MMA warp at the named barrier.  On
    // a timeout it hands over "not ok" and both stop at the same handover.
    if (rank == 0) {
      int s = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        // the accumulator is single-buffered: the epilogue must have read the last tile
        ok = mbar_wait_bounded(tempty_bar, acc_ph ^ 1u);
        acc_ph ^= 1u;
        for (int kb = 0; kb < num_kb; ++kb) {
          ok = ok && mbar_wait_bounded(full_bar(s), ph);
          tc_fence_before();
          named_bar_and(kStageBar, 64, ok);
          if (!ok) break;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
    }
  }
  } else if (warp < C::EPI_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_SFW));
    // ------------------------------------------------ scale factors -> TMEM
    // Each warp writes the 32 lanes of its sub-partition q.  A 512-byte chunk
    // row l holds four 4-byte words, word m = the scales of row l + 32 m.
    // B's chunks go to every sub-partition whole (4 columns: every lane of D
    // needs every column's scales).  A's chunks need only their diagonal:
    // sub-partition q reads row 32 q + l's scales from column 4 j + q of A's
    // chunk j, so warp q stores word q there and nothing else (checked by the
    // GEMM parity tests: with any of these words missing the results differ).
    if constexpr (C::SCALED) {
      const uint32_t q = static_cast<uint32_t>(warp & 3);
      const uint32_t leader_full0 = map_to_cta(full_bar(0), 0);
      constexpr int NA = C::SF_CHUNKS;            // A chunks per stage
      constexpr int NB = C::SF_CHUNKS * C::NRB;   // B chunks per stage
      int r = 0, n = 0, s = 0;  // scale slot, scale set, A/B stage of g
      int sp = 0;               // A/B stage of g - NSF (the last user of set n)
      uint32_t rph = 0, spph = 0;
      for (int g = 0; g < total_kb; ++g) {
        // the tcgen05.st below is warp-collective: the warp leaves as a whole
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(sf_full_bar(r), rph))) break;
        const uint32_t slot = sf_base + r * C::SF_SLOT_BYTES;
        uint32_t va[NA], vb[NB * 4];
#pragma unroll
        for (int i = 0; i < NA; ++i)
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(va[i]) : "r"(slot + i * 512 + lane * 16 + q * 4));
#pragma unroll
        for (int i = 0; i < NB; ++i) {
          // TMEM order is MMA-major (j, c); the slot holds B as (c, j)
          const int jb = i / C::NRB, cb = i % C::NRB;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(vb[4 * i]), "=r"(vb[4 * i + 1]), "=r"(vb[4 * i + 2]), "=r"(vb[4 * i + 3])
                       : "r"(slot + C::SFA_BYTES + (cb * C::SF_CHUNKS + jb) * 512 + lane * 16));
        }
        // set n is free once the MMAs of stage g - NSF (A/B stage sp) have
        // completed.  NSF <= STAGES, so the full barrier of stage g - STAGES
        // has completed too, and the arrival below counts towards stage g.
        if (g >= C::NSF) {
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(empty_bar(sp), spph))) break;
          if (++sp == S) { sp = 0; spph ^= 1u; }
        }
        tc_fence_after();
        const uint32_t t = tmem_base + (q * 32u << 16) + C::SF_COL + n * C::SF_SET_COLS;
#pragma unroll
        for (int i = 0; i < NA; ++i) tmem_st_32x32b_x1(t + 4 * i + q, va[i]);
        if constexpr (NB * 4 % 16 == 0) {
#pragma unroll
          for (int i = 0; i < NB * 4 / 16; ++i) {
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) w[k] = vb[16 * i + k];
            tmem_st_32x32b_x16(t + C::SFB_OFF + 16 * i, w);
          }
        } else {
#pragma unroll
          for (int i = 0; i < NB; ++i)
            tmem_st_32x32b_x4(t + C::SFB_OFF + 4 * i, vb[4 * i], vb[4 * i + 1], vb[4 * i + 2], vb[4 * i + 3]);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        // The slot goes back to the loader only now that the stores have
        // consumed every value read from it.  Released right after the
        // ld.shared instructions, the refill (the stage R later) could land
        // before the warp's last loads had read the slot: a few lanes then
        // stored that stage's B scales for the last MMA of the stage.
        if (lane == 0) {
          mbar_arrive_remote(leader_full0 + 8u * s);
          mbar_arrive(sf_empty_bar(r));
        }
        if (++r == R) { r = 0; rph ^= 1u; }
        if (++n == C::NSF) n = 0;
        if (++s == S) s = 0;
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_EPI));
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // tensor-memory sub-partition = 32-row slice
    const int h = (warp >> 2) & 1;   // column half of the tile
    const uint32_t stage_buf0 = epi_base + (warp - C::EPI_WARP0) * (C::EPI_BUFS * 32 * C::EPI_SUB * 2);
    const uint32_t leader_tempty = map_to_cta(tempty_bar, 0);
    float alpha = 1.0f;
    if constexpr (F == Fmt::NVFP4) alpha = (*args.a_g) * (*args.b_g);
    const bool bias_vec = args.bias != nullptr && (reinterpret_cast<uintptr_t>(args.bias) & 15u) == 0;
    float ymax = 0.0f;  // EPI != 0: max |y| of this thread's outputs
    for (int i_tile = 0; i_tile < my_tiles; ++i_tile) {
      const int tile = pair + i_tile * num_pairs;
      int mt, nt;
      pair_tile_coords(tile, m_tiles, n_tiles, n_fast, mt, nt);
      const int row0 = mt * C::BM + static_cast<int>(rank) * C::BM_CTA + q * 32;
      // the tile's bias, prefetched before the accumulator is ready: lane l holds
      // columns [8l, 8l + 8) of the tile as four packed bf16 pairs
      uint32_t bias_l[4] = {0u, 0u, 0u, 0u};
      if (args.bias != nullptr && lane * 8 < BN) {
        const int c0 = nt * BN + lane * 8;
        if (bias_vec && c0 + 8 <= N) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(args.bias + c0));
          bias_l[0] = u.x; bias_l[1] = u.y; bias_l[2] = u.z; bias_l[3] = u.w;
        } else {
          const uint16_t* bs = reinterpret_cast<const uint16_t*>(args.bias);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t lo = (c0 + 2 * e < N) ? bs[c0 + 2 * e] : 0u;
            const uint32_t hi = (c0 + 2 * e + 1 < N) ? bs[c0 + 2 * e + 1] : 0u;
            bias_l[e] = lo | (hi << 16);
          }
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(tfull_bar, i_tile & 1))) break;  // tcgen05.ld is warp-collective
      tc_fence_after();
      // all of this warp's accumulator columns into registers, then release the accumulator
      uint32_t r[C::EPI_COLS];
      const uint32_t t_cols = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + h * C::EPI_COLS;
#pragma unroll
      for (int g = 0; g < C::EPI_COLS / 32; ++g) tmem_ld_32x32b_x32_nowait(t_cols + g * 32, r + 32 * g);
      tc_wait_ld();
#pragma unroll
      for (int g = 0; g < C::EPI_COLS / 32; ++g) reg_fence32(r + 32 * g);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_tempty);  // accumulator may be overwritten
      const int col_w = nt * BN + h * C::EPI_COLS;  // first column of this warp
#pragma unroll
      for (int sub = 0; sub < C::EPI_COLS / C::EPI_SUB; ++sub) {
        const uint32_t stage_buf = stage_buf0 + (sub % C::EPI_BUFS) * (32 * C::EPI_SUB * 2);
        // this buffer's previous store (two sub-tiles ago) has read it
        if (lane == 0) bulk_wait_group_read<C::EPI_BUFS - 1>();
        __syncwarp();
        // groups of 8 columns: alpha * acc + bias, bf16, one 16-byte store each
        // into the 32 x EPI_SUB staging sub-tile (EPI_ROW-byte rows, swizzled
        // like the TMA's EPI_ROW-byte mode: 16-byte chunk c of row l sits at
        // chunk c ^ ((l * EPI_ROW / 128) % (EPI_ROW / 16)))
#pragma unroll
        for (int j = 0; j < C::EPI_SUB / 8; ++j) {
          const int grp = h * (C::EPI_COLS / 8) + sub * (C::EPI_SUB / 8) + j;  // 8-column group in the tile
          uint32_t bw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) bw[e] = __shfl_sync(0xffffffffu, bias_l[e], grp);
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = sub * C::EPI_SUB + j * 8 + 2 * e;
            float v0 = __uint_as_float(r[c]), v1 = __uint_as_float(r[c + 1]);
            if constexpr (F == Fmt::NVFP4) { v0 *= alpha; v1 *= alpha; }
            v0 += __uint_as_float(bw[e] << 16);
            v1 += __uint_as_float(bw[e] & 0xFFFF0000u);
            if constexpr (EPI != 0) {
              if (args.act == 1) {
                v0 = gelu_erf(v0);
                v1 = gelu_erf(v1);
              }
            }
            const __nv_bfloat162 hv = __floats2bfloat162_rn(v0, v1);
            if constexpr (EPI != 0) {
              // rows and columns past the edge hold no output: leave them out
              const int cc = col_w + c;
              if (row0 + lane < M && cc < N) ymax = fmaxf(ymax, fabsf(__low2float(hv)));
              if (row0 + lane < M && cc + 1 < N) ymax = fmaxf(ymax, fabsf(__high2float(hv)));
            }
            pk[e] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          static_assert(C::EPI_ROW == 32 || C::EPI_ROW == 64 || C::EPI_ROW == 128, "staging swizzle");
          const uint32_t sw = (static_cast<uint32_t>(lane) * C::EPI_ROW / 128) & (C::EPI_ROW / 16 - 1);
          const uint32_t addr = stage_buf + lane * C::EPI_ROW + ((j ^ sw) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[0]), "r"(pk[1]),
                       "r"(pk[2]), "r"(pk[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int x = col_w + sub * C::EPI_SUB;
        if (lane == 0 && row0 < M && x < N) {
          tma_store_2d(&tmap_y, stage_buf, x, row0);
          bulk_commit_group();
        }
      }
    }
    if constexpr (EPI != 0) {
      // non-negative floats order like their bit patterns
      const unsigned int m = __reduce_max_sync(0xffffffffu, __float_as_uint(ymax));
      if (lane == 0 && args.y_amax != nullptr) atomicMax(args.y_amax, m);
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace mxq

// Medusa heads at large batch (bf16, B > 32): the compute-bound regime.
//
// Source: Medusa paper digest ("論文解説: Medusa"), section
// "Medusa Headのアーキテクチャ": H_k(h) = Linear(SiLU(Linear(h)) + h),
//   stage 1:  u_k[b]      = SiLU(W1_k h[b] + b1_k) + h[b]      (d -> d)
//   stage 2:  logits_k[b] = W2_k u_k[b]                       (d -> V)
// and the per-head top-s of section "ツリーアテンションによる並列検証".
//
// With B in the hundreds every weight byte feeds hundreds of multiply-adds,
// above the B200 ridge point, so both stages are tensor-core GEMMs with
// the weights as the A operand (M = 128 rows per tile, K-major, TMA
// 128-byte swizzle) and the activations as B with N = 256 columns per unit:
// 256 sequences in stage 1, 128 sequences x (hi, lo) in stage 2 (u is the
// bf16 pair hi + lo, ~16 significant bits, as in the small-batch kernel).
// A unit is (head, 128-row tile, 256-column chunk[, K-split]); one
// persistent CTA per SM takes units in turn:
//   warp 0     TMA producer, 3-stage ring of (16 KB of W, 32 KB of X)
//   warp 1     tcgen05.mma issuer (M 128, N 256, K 16), fp32 accumulators
//              in TMEM, double-buffered (2 x 256 columns)
//   warps 2-5  epilogue, one TMEM lane (output row) per thread
// Stage 1's epilogue writes each K-split's fp32 partial sums; a separate
// kernel adds the splits, b1, SiLU and the residual and writes u as the
// (hi, lo) pair.  Stage 2's epilogue stages the tile's 128 x 128 logits
// (hi + lo columns summed) transposed in shared memory, then each thread
// takes one sequence and keeps that column's top-s in registers (a new
// key enters only above the current s-th), writing one candidate list per
// (sequence, head, tile); the top-s kernel merges the lists.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kThreads = 192;
constexpr int BM = 128;       // output rows per tile
constexpr int BK = 64;        // K elements per stage
constexpr int NB = 256;       // accumulator columns per unit
constexpr int kStages = 3;
constexpr uint32_t A_BYTES = BM * BK * 2;   // 16 KB
constexpr uint32_t B_BYTES = NB * BK * 2;   // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int LGS = BM + 1;   // row stride (floats) of the staged logits: conflict-free columns
constexpr size_t LG_BYTES = (size_t)(NB / 2) * LGS * sizeof(float);
constexpr size_t SMEM = 1024 + (size_t)kStages * STAGE_BYTES + 512 + LG_BYTES;
static_assert(SMEM <= 227 * 1024, "shared memory of the large-batch heads kernel");
constexpr int kSmax = MEDUSA_MAX_S;

struct BigParams {
  int stage;    // 1 or 2
  int K, rows, mtiles, kchunks, splits, nchunks, units;
  int B, d;
  int bcols;    // sequences per column chunk: 256 (stage 1) or 128 (stage 2)
  float* part;  // stage 1: [splits][K][B][d]
  float* logits;     // stage 2: [B][K][V] or null
  uint64_t* cand;    // stage 2: [B*K][mtiles][s] or null
  int s;
};

__device__ __forceinline__ void big_coords(const BigParams& p, int unit, int& kh, int& mt, int& nc,
                                           int& sp, int& k0, int& k1) {
  sp = unit % p.splits;
  int t = unit / p.splits;
  nc = t % p.nchunks;
  t /= p.nchunks;
  mt = t % p.mtiles;
  kh = t / p.mtiles;
  k0 = (int)((long long)sp * p.kchunks / p.splits);
  k1 = (int)((long long)(sp + 1) * p.kchunks / p.splits);
}

__global__ void __launch_bounds__(kThreads, 1)
    heads_big_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, const BigParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)kStages * A_BYTES;
  uint64_t* full = (uint64_t*)(sB + (size_t)kStages * B_BYTES);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* lg = (float*)((uint8_t*)full + 512);  // [128 sequences][LGS] staged logits

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, 2 * NB);
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();  // TMEM taken: the next kernel may be scheduled
  griddep_wait();               // the activation operand comes from the kernel ahead

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // a weight tile is read by the units of every column chunk (adjacent
      // unit numbers, so mostly from L2 after the first): normal eviction
      const uint64_t pol_w = p.nchunks > 1 ? policy_evict_normal() : policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x) {
        int kh, mt, nc, sp, k0, k1;
        big_coords(p, unit, kh, mt, nc, sp, k0, k1);
        const int row0 = kh * p.rows + mt * BM;
        const int col0 = nc * NB;  // first activation row of the chunk
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
          tma_load_2d(sA + (size_t)st * A_BYTES, &tmA, &full[st], kc * BK, row0, pol_w);
          if (p.stage == 1)
            tma_load_2d(sB + (size_t)st * B_BYTES, &tmB, &full[st], kc * BK, col0, pol_x);
          else
            tma_load_3d(sB + (size_t)st * B_BYTES, &tmB, &full[st], kc * BK, col0, kh, pol_x);
        }
      }
      if (!ok) {
        // aborted: let every load already issued land before the CTA exits
        const uint32_t n = it < (uint32_t)kStages ? it : (uint32_t)kStages;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t last = it - 1 - j;
          mbar_wait(&full[last % kStages], (last / kStages) & 1u, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(BM, NB);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++local) {
        int kh, mt, nc, sp, k0, k1;
        big_coords(p, unit, kh, mt, nc, sp, k0, k1);
        const uint32_t acc = local & 1u;
        if (!mbar_wait(&tempty[acc], ((local >> 1) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + acc * NB;
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % kStages);
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&full[st], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128_kmajor(smem_u32(sA + (size_t)st * A_BYTES));
          const uint64_t bd = umma_desc_sw128_kmajor(smem_u32(sB + (size_t)st * B_BYTES));
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            umma_bf16(tmem_d, ad + 2u * j, bd + 2u * j, idesc, (kc > k0 || j > 0) ? 1u : 0u);
          umma_commit(&empty[st]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;
    const int et = (int)threadIdx.x - 64;  // 0..127
    uint32_t local = 0;
    for (int unit = blockIdx.x; unit < p.units; unit += gridDim.x, ++local) {
      int kh, mt, nc, sp, k0, k1;
      big_coords(p, unit, kh, mt, nc, sp, k0, k1);
      const uint32_t acc = local & 1u;
      const bool good = mbar_wait(&tfull[acc], (local >> 1) & 1u, abort_flag);
      // the four warps take one decision (OR of every thread's view), so none
      // is left waiting at a later barrier
      if (bar_red_or(1, 128, !good || *abort_flag)) break;
      tc_fence_after();
      const int m = mt * BM + r;  // output row within the head
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * NB;
      if (p.stage == 1) {
        // this K-split's partial sums, [split][head][b][d] (coalesced over m)
        float* dst = p.part + (((size_t)sp * p.K + kh) * p.B) * p.d + m;
#pragma unroll 1
        for (int c0 = 0; c0 < NB; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + (uint32_t)c0, v);
          if (m < p.rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int b = nc * p.bcols + c0 + j;
              if (b < p.B) dst[(size_t)b * p.d] = v[j];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        continue;
      }
      // stage 2: logits of 128 sequences (hi + lo columns) for this row
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += 32) {
        float v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int bl = c0 / 2 + j;  // sequence within the chunk
          const float x = v[2 * j] + v[2 * j + 1];
          lg[bl * LGS + r] = x;
          const int b = nc * p.bcols + bl;
          if (p.logits && m < p.rows && b < p.B) p.logits[((size_t)b * p.K + kh) * p.rows + m] = x;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);  // accumulator free for the next unit
      if (p.cand) {
        named_bar_sync(1, 128);  // every row of the tile is staged
        const int b = nc * p.bcols + et;
        if (b < p.B) {
          uint64_t keys[kSmax];
#pragma unroll
          for (int i = 0; i < kSmax; ++i) keys[i] = 0ull;
          uint64_t kth = 0ull;
          const int nrows = min(BM, p.rows - mt * BM);
          for (int i = 0; i < nrows; ++i) {
            const uint64_t key = make_key(lg[et * LGS + i], (uint32_t)(mt * BM + i));
            if (key > kth) topk_insert<kSmax>(keys, p.s, key, kth);
          }
          uint64_t* dst = p.cand + (((size_t)b * p.K + kh) * (size_t)p.mtiles + mt) * p.s;
#pragma unroll
          for (int i = 0; i < kSmax; ++i)
            if (i < p.s) dst[i] = keys[i];
        }
      }
      named_bar_sync(1, 128);  // the staged rows are read before the next unit writes
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * NB);
  }
}

// ---------------------------------------------------------------------------
// The same GEMMs on CTA pairs (tcgen05 cta_group::2): a cluster of two CTAs
// on a pair of SMs takes 256 weight rows (128 per CTA, A and D in each
// CTA's own smem / TMEM) and the 256 activation columns of a chunk, HALF of
// them staged in each CTA (the MMA exchanges the halves), so every SM reads
// half the activation bytes per multiply-add of the one-CTA kernel.  Rank 0
// issues M = 256 MMAs; both CTAs' loads count on rank 0's barriers
// (cta_group::2 TMA), its commits arrive on both CTAs' barriers, and each
// CTA runs the epilogue of its own 128 rows (the peer's release of an
// accumulator reaches rank 0 by a remote arrive).
constexpr int kStages2 = 4;
constexpr uint32_t B2_BYTES = (NB / 2) * BK * 2;         // this CTA's 128 activation rows
constexpr uint32_t STAGE2_BYTES = A_BYTES + B2_BYTES;    // 32 KB a CTA, 64 KB a pair
constexpr size_t SMEM2 = 1024 + (size_t)kStages2 * STAGE2_BYTES + 512 + LG_BYTES;
static_assert(SMEM2 <= 227 * 1024, "shared memory of the CTA-pair heads kernel");

__device__ __forceinline__ void big2_coords(const BigParams& p, int unit, int& kh, int& mt2,
                                            int& nc, int& sp, int& k0, int& k1) {
  sp = unit % p.splits;
  int t = unit / p.splits;
  nc = t % p.nchunks;
  t /= p.nchunks;
  const int mtiles2 = (p.mtiles + 1) / 2;
  mt2 = t % mtiles2;
  kh = t / mtiles2;
  k0 = (int)((long long)sp * p.kchunks / p.splits);
  k1 = (int)((long long)(sp + 1) * p.kchunks / p.splits);
}

__global__ void __launch_bounds__(kThreads, 1)
    heads_big2_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const BigParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)kStages2 * A_BYTES;
  uint64_t* full = (uint64_t*)(sB + (size_t)kStages2 * B2_BYTES);  // rank 0: both CTAs' bytes
  uint64_t* empty = full + kStages2;                               // both (multicast commit)
  uint64_t* tfull = empty + kStages2;                              // both (multicast commit)
  uint64_t* tempty = tfull + 2;                                    // rank 0: both epilogues
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* lg = (float*)((uint8_t*)full + 512);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const bool leader = crank == 0u;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int mtiles2 = (p.mtiles + 1) / 2;
  (void)mtiles2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or load
  if (warp == 0) {
    __syncwarp();
    tmem_alloc_cg2(tmem_slot, 2 * NB);
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_launch_dependents();  // TMEM taken: the next kernel may be scheduled
  griddep_wait();               // the activation operand comes from the kernel ahead

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      const uint64_t pol_w = p.nchunks > 1 ? policy_evict_normal() : policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      uint32_t it = 0;
      bool ok = true;
      for (int unit = pair; unit < p.units && ok; unit += npairs) {
        int kh, mt2, nc, sp, k0, k1;
        big2_coords(p, unit, kh, mt2, nc, sp, k0, k1);
        const int row0 = kh * p.rows + (2 * mt2 + (int)crank) * BM;
        const int col0 = nc * NB + (int)crank * (NB / 2);
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % kStages2);
          const uint32_t ph = (it / kStages2) & 1u;
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[st], 2 * STAGE2_BYTES);
          const uint32_t fb = mapa_shared(&full[st], 0);
          tma_load_2d_cg2(sA + (size_t)st * A_BYTES, &tmA, fb, kc * BK, row0, pol_w);
          if (p.stage == 1)
            tma_load_2d_cg2(sB + (size_t)st * B2_BYTES, &tmB, fb, kc * BK, col0, pol_x);
          else
            tma_load_3d_cg2(sB + (size_t)st * B2_BYTES, &tmB, fb, kc * BK, col0, kh, pol_x);
        }
      }
      if (!ok && leader) {
        // aborted: let every load already issued land before the pair exits
        const uint32_t n = it < (uint32_t)kStages2 ? it : (uint32_t)kStages2;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t last = it - 1 - j;
          mbar_wait(&full[last % kStages2], (last / kStages2) & 1u, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && leader) {
      const uint32_t idesc = umma_idesc_bf16_f32(2 * BM, NB);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int unit = pair; unit < p.units && ok; unit += npairs, ++local) {
        int kh, mt2, nc, sp, k0, k1;
        big2_coords(p, unit, kh, mt2, nc, sp, k0, k1);
        const uint32_t acc = local & 1u;
        if (!mbar_wait_cl(&tempty[acc], ((local >> 1) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + acc * NB;
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % kStages2);
          const uint32_t ph = (it / kStages2) & 1u;
          if (!mbar_wait_cl(&full[st], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128_kmajor(smem_u32(sA + (size_t)st * A_BYTES));
          const uint64_t bd = umma_desc_sw128_kmajor(smem_u32(sB + (size_t)st * B2_BYTES));
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            umma_bf16_cg2(tmem_d, ad + 2u * j, bd + 2u * j, idesc, (kc > k0 || j > 0) ? 1u : 0u);
          umma_commit_cg2(&empty[st], 0x3);
        }
        if (ok) umma_commit_cg2(&tfull[acc], 0x3);
      }
      umma_commit_cg2(mma_done, 0x1);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int et = (int)threadIdx.x - 64;
    uint32_t local = 0;
    for (int unit = pair; unit < p.units; unit += npairs, ++local) {
      int kh, mt2, nc, sp, k0, k1;
      big2_coords(p, unit, kh, mt2, nc, sp, k0, k1);
      const uint32_t acc = local & 1u;
      const bool good = mbar_wait(&tfull[acc], (local >> 1) & 1u, abort_flag);
      if (bar_red_or(1, 128, !good || *abort_flag)) break;
      tc_fence_after();
      const int mt = 2 * mt2 + (int)crank;  // this CTA's 128-row tile
      const int m = mt * BM + r;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + acc * NB;
      if (p.stage == 1) {
        float* dst = p.part + (((size_t)sp * p.K + kh) * p.B) * p.d + m;
#pragma unroll 1
        for (int c0 = 0; c0 < NB; c0 += 32) {
          float v[32];
          tmem_ld32(tbase + (uint32_t)c0, v);
          if (m < p.rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int b = nc * p.bcols + c0 + j;
              if (b < p.B) dst[(size_t)b * p.d] = v[j];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));
        continue;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < NB; c0 += 32) {
        float v[32];
        tmem_ld32(tbase + (uint32_t)c0, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int bl = c0 / 2 + j;
          const float x = v[2 * j] + v[2 * j + 1];
          lg[bl * LGS + r] = x;
          const int b = nc * p.bcols + bl;
          if (p.logits && m < p.rows && b < p.B) p.logits[((size_t)b * p.K + kh) * p.rows + m] = x;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[acc], 0));
      if (p.cand && mt < p.mtiles) {  // uniform over the CTA
        named_bar_sync(1, 128);
        const int b = nc * p.bcols + et;
        if (b < p.B) {
          uint64_t keys[kSmax];
#pragma unroll
          for (int i = 0; i < kSmax; ++i) keys[i] = 0ull;
          uint64_t kth = 0ull;
          const int nrows = min(BM, p.rows - mt * BM);
          for (int i = 0; i < nrows; ++i) {
            const uint64_t key = make_key(lg[et * LGS + i], (uint32_t)(mt * BM + i));
            if (key > kth) topk_insert<kSmax>(keys, p.s, key, kth);
          }
          uint64_t* dst = p.cand + (((size_t)b * p.K + kh) * (size_t)p.mtiles + mt) * p.s;
#pragma unroll
          for (int i = 0; i < kSmax; ++i)
            if (i < p.s) dst[i] = keys[i];
        }
      }
      named_bar_sync(1, 128);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the pair's MMAs, loads or arrives may touch it
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, 2 * NB);
  }
}

// u[k][b] = SiLU(sum of the K-split partials + b1[k]) + h[b], written as the
// bf16 pair (hi, lo = u - hi) in rows 2b, 2b + 1 of stage 2's B operand.
// One thread per (head, sequence, feature), coalesced over the feature.
__global__ void heads_big_silu_kernel(const float* __restrict__ part, int S, int K, int B, int d,
                                      const __nv_bfloat16* __restrict__ b1,
                                      const __nv_bfloat16* __restrict__ h,
                                      __nv_bfloat16* __restrict__ u) {
  griddep_launch_dependents();  // stage 2 may take its TMEM and wait
  griddep_wait();
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t n = (size_t)K * B * d;
  if (i >= n) return;
  const int m = (int)(i % d);
  const size_t kb = i / d;
  const int b = (int)(kb % B), kh = (int)(kb / B);
  float a = b1 ? __bfloat162float(b1[(size_t)kh * d + m]) : 0.f;
  for (int s2 = 0; s2 < S; ++s2) a += part[(((size_t)s2 * K + kh) * B + b) * d + m];
  const float uu = a / (1.f + expf(-a)) + __bfloat162float(h[(size_t)b * d + m]);
  const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
  const __nv_bfloat16 lo = __float2bfloat16_rn(uu - __bfloat162float(hi));
  __nv_bfloat16* urow = u + ((size_t)kh * 2 * B + 2 * b) * d + m;
  urow[0] = hi;
  urow[d] = lo;
}

struct BigPlan {
  int mt1, mt2, kch, nc1, nc2, S1;
  size_t off_u, off_p1, off_cand, total;
};

BigPlan make_big_plan(int B, int d, int V, int K, int s) {
  BigPlan P;
  const int sms = num_sms();
  P.mt1 = (d + BM - 1) / BM;
  P.mt2 = (V + BM - 1) / BM;
  P.kch = (d + BK - 1) / BK;
  P.nc1 = (B + NB - 1) / NB;
  P.nc2 = (2 * B + NB - 1) / NB;
  // K-splits of stage 1 until its units fill >= 90% of the last wave (each
  // split keeps at least 8 K chunks)
  P.S1 = 1;
  for (int S = 1; S <= 8 && (S == 1 || P.kch / S >= 8); ++S) {
    const long long units = (long long)K * P.mt1 * P.nc1 * S;
    const long long waves = (units + sms - 1) / sms;
    P.S1 = S;
    if ((double)units / (double)(waves * sms) >= 0.9) break;
  }
  WsCarver w;
  P.off_u = w.take<__nv_bfloat16>((size_t)K * 2 * B * d);
  P.off_p1 = w.take<float>((size_t)P.S1 * K * B * d);
  P.off_cand = w.take<uint64_t>((size_t)B * K * P.mt2 * s);
  P.total = w.total();
  return P;
}

std::atomic<bool> g_big_attr[64];
std::atomic<bool> g_big2_attr[64];

// Clusters of two heads_big2_kernel CTAs resident at once on the current
// device (0 when the query fails: the one-CTA kernel is used), cached.
int big2_slots() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  const int v = cache[dev].load(std::memory_order_relaxed);
  if (v) return v - 1;
  if (ensure_max_smem(heads_big2_kernel, (int)SMEM2, g_big2_attr,
                      "cudaFuncSetAttribute(heads_big2_kernel)"))
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM2;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)heads_big2_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cache[dev].store(n + 1, std::memory_order_relaxed);
  return n;
}

// Units of the CTA-pair kernel: (head, 256-row tile, column chunk, split).
int pair_units(const BigParams& p) { return p.K * ((p.mtiles + 1) / 2) * p.nchunks * p.splits; }

// pair: the CTA-pair kernel, whose activation tensor map has a box of
// NB / 2 rows (one CTA's half of a chunk); otherwise the one-CTA kernel and
// a box of NB rows.
int launch_big(const CUtensorMap& A, const CUtensorMap& Bm, const BigParams& p, bool pair,
               int slots, cudaStream_t st) {
  cudaError_t e;
  if (pair) {
    BigParams p2 = p;
    p2.units = pair_units(p);
    const int pairs = p2.units < slots ? p2.units : slots;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM2;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, heads_big2_kernel, A, Bm, p2);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "heads_big2_kernel launch");
  }
  int rc = ensure_max_smem(heads_big_kernel, (int)SMEM, g_big_attr,
                           "cudaFuncSetAttribute(heads_big_kernel)");
  if (rc) return rc;
  const int grid = p.units < num_sms() ? p.units : num_sms();
  e = launch_pdl(heads_big_kernel, dim3(grid), dim3(kThreads), SMEM, st, A, Bm, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "heads_big_kernel launch");
}

}  // namespace

size_t heads_big_workspace(int B, int d, int V, int K, int s) {
  return make_big_plan(B, d, V, K, s).total;
}

int heads_big_launch(const HeadsArgs& a, cudaStream_t st) {
  const BigPlan P = make_big_plan(a.B, a.d, a.V, a.K, a.s);
  if (a.ws_bytes < P.total) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for heads");
  const int slots = big2_slots();
  const bool pair = slots > 0;
  // rows of one activation box: must equal what a CTA's B stage holds
  const uint32_t brows = pair ? (uint32_t)(NB / 2) : (uint32_t)NB;
  static_assert((NB / 2) * BK * 2 == B2_BYTES && NB * BK * 2 == B_BYTES,
                "activation boxes fill exactly one B stage of their kernel");
  uint8_t* ws = (uint8_t*)a.ws;
  __nv_bfloat16* u = (__nv_bfloat16*)(ws + P.off_u);
  float* part = (float*)(ws + P.off_p1);
  uint64_t* cand = (uint64_t*)(ws + P.off_cand);

  alignas(64) CUtensorMap mA1, mB1, mA2, mB2;
  {
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.K * a.d};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {BK, BM};
    int rc = make_tmap_bf16(&mA1, a.W1, 2, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.B};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {BK, brows};
    int rc = make_tmap_bf16(&mB1, a.h, 2, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.K * a.V};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {BK, BM};
    int rc = make_tmap_bf16(&mA2, a.W2, 2, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)2 * a.B, (uint64_t)a.K};
    const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)2 * a.B * a.d * 2};
    const uint32_t box[3] = {BK, brows, 1};
    int rc = make_tmap_bf16(&mB2, u, 3, dims, strides, box);
    if (rc) return rc;
  }

  BigParams p1{};
  p1.stage = 1;
  p1.K = a.K;
  p1.rows = a.d;
  p1.mtiles = P.mt1;
  p1.kchunks = P.kch;
  p1.splits = P.S1;
  p1.nchunks = P.nc1;
  p1.units = a.K * P.mt1 * P.nc1 * P.S1;
  p1.B = a.B;
  p1.d = a.d;
  p1.bcols = NB;
  p1.part = part;
  int rc = launch_big(mA1, mB1, p1, pair, slots, st);
  if (rc) return rc;
  {
    const size_t n = (size_t)a.K * a.B * a.d;
    cudaError_t e = launch_pdl(heads_big_silu_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256),
                               0, st, (const float*)part, P.S1, a.K, a.B, a.d,
                               (const __nv_bfloat16*)a.b1, (const __nv_bfloat16*)a.h, u);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "heads_big_silu_kernel launch");
  }
  BigParams p2 = p1;
  p2.stage = 2;
  p2.rows = a.V;
  p2.mtiles = P.mt2;
  p2.splits = 1;
  p2.nchunks = P.nc2;
  p2.units = a.K * P.mt2 * P.nc2;
  p2.bcols = NB / 2;
  p2.part = nullptr;
  p2.logits = a.logits;
  p2.cand = a.topk_idx ? cand : nullptr;
  p2.s = a.s;
  rc = launch_big(mA2, mB2, p2, pair, slots, st);
  if (rc) return rc;
  if (a.topk_idx)
    return topk_keys_launch(cand, a.B * a.K, P.mt2 * a.s, a.s, a.topk_idx, a.topk_val, st);
  return MEDUSA_OK;
}

}  // namespace medusa

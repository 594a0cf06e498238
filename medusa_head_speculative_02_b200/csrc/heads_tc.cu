// Medusa heads on the 5th-generation tensor cores (tcgen05), bf16.
//
// Source: Medusa paper digest ("論文解説: Medusa"), section
// "Medusa Headのアーキテクチャ": H_k(h) = Linear(SiLU(Linear(h)) + h), i.e.
//   stage 1:  u_k[b]      = SiLU(W1_k h[b] + b1_k) + h[b]      (d -> d)
//   stage 2:  logits_k[b] = W2_k u_k[b]                       (d -> V)
// followed by the per-head top-s of section "ツリーアテンションによる並列検証".
//
// At decode batch sizes (B <= 32) both stages are weight streams: every W
// byte is used for B multiply-adds, far below the B200 ridge point, so the
// kernel is designed around HBM throughput.  Weights are the MMA "A"
// operand (M = 128 output rows per tile, K-major, TMA 128-byte swizzle); the
// activations are the "B" operand with N = B (stage 1) or 2B (stage 2)
// columns padded to a multiple of 16 by TMA zero fill ("swap-AB").
// One persistent CTA per SM, warp-specialised:
//   warp 0     TMA producer (STAGES-deep ring of W/X tiles, weights marked
//              evict-first in L2, activations evict-last)
//   warp 1     single-thread tcgen05.mma issuer, fp32 accumulators in TMEM,
//              double-buffered so the epilogue of one tile overlaps the next
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (thread = output row)
// Work units are (head, 128-row tile, K-split), the split count chosen so
// the units fill the SMs' waves.  Stage 1 (few tiles: d rows per head)
// writes each split's partial sums with plain stores; heads_silu_kernel then
// sums the splits in order (deterministic) and applies bias + SiLU +
// residual, writing u as a bf16 hi/lo pair (u = hi + lo, columns 2b and
// 2b+1 of stage 2's B operand) so stage 2 sees u with ~16 significant bits.
// Stage 2 (many tiles) normally runs unsplit; when it is split, the CTA that
// completes a tile last (atomic ticket) sums the partials in split order.
// Its epilogue fuses the optional fp32 logits store and the top-s: a warp
// max over 64-bit keys (value desc, index asc) per 32-row slice, then the 4
// slices merged per 128-row tile in shared memory; a small kernel selects
// the final top-s of every (b, head) from the per-tile lists.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kThreads = 192;
constexpr int BM = 128;  // output rows per tile (MMA M)
constexpr int BK = 64;   // K elements per stage (one 128-byte swizzle row)
constexpr uint32_t A_BYTES = BM * BK * 2;

template <int NC>
struct TcCfg {
  static constexpr uint32_t B_BYTES = NC * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES;
  static constexpr uint32_t TMEM_COLS = (2 * NC < 32) ? 32 : 2 * NC;
  static constexpr uint32_t CBUF_BYTES = (NC / 2) * 4 * MEDUSA_MAX_S * 8;  // per-tile top-s lists
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 512 + CBUF_BYTES;
};

struct TcParams {
  int stage;    // 1 or 2
  int K;        // heads
  int rows;     // output rows per head: d (stage 1) or V (stage 2)
  int mtiles;   // ceil(rows / BM)
  int kchunks;  // ceil(d / BK)
  int splits;   // K-splits per tile
  int units;    // K * mtiles * splits
  int B;
  int d;
  int ncp;      // accumulator columns in use: B (stage 1) or 2B (stage 2)
  const __nv_bfloat16* b1;  // [K][d] or null
  const __nv_bfloat16* h;   // [B][d]
  __nv_bfloat16* u;         // [K][2B][d]
  float* logits;            // [B][K][V] or null
  uint64_t* cand;           // [B*K][mtiles*4][s] or null
  int s;
  float* part;              // [K*mtiles*splits][ncp][BM]
  int* counters;            // [K*mtiles]
};

__device__ __forceinline__ void unit_coords(const TcParams& p, int unit, int& tile, int& sp,
                                            int& kh, int& mt, int& k0, int& k1) {
  tile = unit / p.splits;
  sp = unit - tile * p.splits;
  kh = tile / p.mtiles;
  mt = tile - kh * p.mtiles;
  k0 = (int)((long long)sp * p.kchunks / p.splits);
  k1 = (int)((long long)(sp + 1) * p.kchunks / p.splits);
}

template <int NC>
__global__ void __launch_bounds__(kThreads, 1)
    heads_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const TcParams p) {
  using C = TcCfg<NC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)C::STAGES * A_BYTES;
  uint64_t* full = (uint64_t*)(sB + (size_t)C::STAGES * C::B_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* last_flag = (volatile int*)(tmem_slot + 2);
  uint64_t* cbuf = (uint64_t*)((uint8_t*)full + 512);  // [B][4 warps][s] candidate keys

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, C::TMEM_COLS);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      // The weight tiles of the first STAGES loads depend on no earlier
      // kernel: they are issued before waiting for the predecessor (whose
      // output is the activation operand), so the ring fills while it ends.
      uint32_t pre = 0;
      for (int unit = blockIdx.x; unit < p.units && pre < (uint32_t)C::STAGES; unit += gridDim.x) {
        int tile, sp, kh, mt, k0, k1;
        unit_coords(p, unit, tile, sp, kh, mt, k0, k1);
        const int row0 = kh * p.rows + mt * BM;
        for (int kc = k0; kc < k1 && pre < (uint32_t)C::STAGES; ++kc, ++pre) {
          mbar_arrive_expect_tx(&full[pre], C::STAGE_BYTES);
          tma_load_2d(sA + (size_t)pre * A_BYTES, &tmA, &full[pre], kc * BK, row0, pol_w);
        }
      }
      griddep_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x) {
        int tile, sp, kh, mt, k0, k1;
        unit_coords(p, unit, tile, sp, kh, mt, k0, k1);
        const int row0 = kh * p.rows + mt * BM;
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % C::STAGES);
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (it >= pre) {  // the first `pre` weight tiles are already on their way
            if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
            tma_load_2d(sA + (size_t)st * A_BYTES, &tmA, &full[st], kc * BK, row0, pol_w);
          }
          if (p.stage == 1)
            tma_load_2d(sB + (size_t)st * C::B_BYTES, &tmB, &full[st], kc * BK, 0, pol_x);
          else
            tma_load_3d(sB + (size_t)st * C::B_BYTES, &tmB, &full[st], kc * BK, 0, kh, pol_x);
        }
      }
      if (!ok) {
        // Aborted: let every load already issued land before the CTA exits.
        const uint32_t n = it < (uint32_t)C::STAGES ? it : (uint32_t)C::STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t last = it - 1 - j;
          mbar_wait(&full[last % C::STAGES], (last / C::STAGES) & 1u, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(BM, NC);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.units && ok; unit += gridDim.x, ++local) {
        int tile, sp, kh, mt, k0, k1;
        unit_coords(p, unit, tile, sp, kh, mt, k0, k1);
        const uint32_t acc = local & 1u;
        if (!mbar_wait(&tempty[acc], ((local >> 1) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + acc * NC;
        for (int kc = k0; kc < k1; ++kc, ++it) {
          const int st = (int)(it % C::STAGES);
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&full[st], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = umma_desc_sw128_kmajor(smem_u32(sA + (size_t)st * A_BYTES));
          const uint64_t bd = umma_desc_sw128_kmajor(smem_u32(sB + (size_t)st * C::B_BYTES));
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            umma_bf16(tmem_d, ad + 2u * j, bd + 2u * j, idesc, (kc > k0 || j > 0) ? 1u : 0u);
          umma_commit(&empty[st]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // All MMAs issued by this thread complete before TMEM is released.
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;
    uint32_t local = 0;
    for (int unit = blockIdx.x; unit < p.units; unit += gridDim.x, ++local) {
      int tile, sp, kh, mt, k0, k1;
      unit_coords(p, unit, tile, sp, kh, mt, k0, k1);
      const uint32_t acc = local & 1u;
      const bool good = mbar_wait(&tfull[acc], (local >> 1) & 1u, abort_flag);
      // The four epilogue warps leave together if any wait ran out (one
      // decision, the OR of every thread's view), so none can be left
      // behind at a named barrier.
      if (bar_red_or(1, 128, !good || *abort_flag)) break;
      tc_fence_after();
      float v[NC];
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += 16) {
        float t[16];
        tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + acc * NC + c0, t);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c0 + i] = t[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);

      const int m = mt * BM + r;  // output row within the head
      if (p.stage == 1) {
        // partial sums of this K-split, [split][head][b][d]; bias, SiLU and
        // the residual are applied by heads_silu_kernel once all splits land
        if (m < p.rows) {
          float* dst = p.part + (((size_t)sp * p.K + kh) * p.B) * p.d + m;
#pragma unroll
          for (int b = 0; b < NC; ++b)
            if (b < p.B) dst[(size_t)b * p.d] = v[b];
        }
        continue;
      }

      if (p.splits > 1) {
        float* mine = p.part + ((size_t)tile * p.splits + sp) * p.ncp * BM;
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (c < p.ncp) mine[(size_t)c * BM + r] = v[c];
        __threadfence();
        named_bar_sync(1, 128);
        if (warp == 2 && lane == 0) {
          const int old = atomicAdd(&p.counters[tile], 1);
          *last_flag = (old == p.splits - 1) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (!*last_flag) continue;
        __threadfence();
        const float* base = p.part + (size_t)tile * p.splits * p.ncp * BM;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          if (c < p.ncp) {
            float sum = 0.f;
            for (int s2 = 0; s2 < p.splits; ++s2)
              sum += __ldcg(base + ((size_t)s2 * p.ncp + c) * BM + r);
            v[c] = sum;
          }
        }
      }

      {
        const bool valid = m < p.rows;
#pragma unroll
        for (int b = 0; b < NC / 2; ++b) {
          if (b < p.B) {
            const float lg = v[2 * b] + v[2 * b + 1];
            if (p.logits && valid) p.logits[((size_t)b * p.K + kh) * p.rows + m] = lg;
            if (p.cand) {
              // this warp's 32 rows: s rounds of a warp max over 64-bit keys
              uint64_t key = valid ? make_key(lg, (uint32_t)m) : 0ull;
              uint64_t keep = 0ull;
              for (int j = 0; j < p.s; ++j) {
                const uint64_t mx = warp_max_u64(key);
                if (key == mx) key = 0ull;
                if (lane == j) keep = mx;
              }
              if (lane < p.s) cbuf[(b * 4 + q) * p.s + lane] = keep;
            }
          }
        }
        if (p.cand) {
          // merge the 4 warps' lists: the tile's top-s per column b
          named_bar_sync(1, 128);
          for (int b = warp - 2; b < p.B; b += 4) {
            uint64_t k0 = lane < 2 * p.s ? cbuf[b * 4 * p.s + lane] : 0ull;
            uint64_t k1 = lane < 2 * p.s ? cbuf[b * 4 * p.s + 2 * p.s + lane] : 0ull;
            uint64_t keep = 0ull;
            for (int j = 0; j < p.s; ++j) {
              const uint64_t mx = warp_max_u64(k0 > k1 ? k0 : k1);
              if (k0 == mx) k0 = 0ull;
              if (k1 == mx) k1 = 0ull;
              if (lane == j) keep = mx;
            }
            if (lane < p.s)
              p.cand[(((size_t)b * p.K + kh) * (size_t)p.mtiles + mt) * p.s + lane] = keep;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Splits per tile: the smallest S whose units fill the SMs' waves to >= 90%
// (each split keeps at least 4 K-chunks).
// u[k][b] = SiLU(sum of the K-split partials + b1[k]) + h[b], stored as the
// bf16 pair (hi, lo = u - hi) in rows 2b, 2b+1 of stage 2's B operand.
// It also zeroes the split counters of stage 2, which runs next.
__global__ void heads_silu_kernel(const float* __restrict__ part, int S, int K, int B, int d,
                                  const __nv_bfloat16* __restrict__ b1,
                                  const __nv_bfloat16* __restrict__ h,
                                  __nv_bfloat16* __restrict__ u, int* __restrict__ cnt2,
                                  int ncnt2) {
  griddep_launch_dependents();  // stage 2 may start streaming its weights
  griddep_wait();
  // one thread per (head, sequence, feature): i = (kh * B + b) * d + m
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long j = i; j < ncnt2; j += (long long)gridDim.x * blockDim.x) cnt2[j] = 0;
  if (i >= (long long)K * B * d) return;
  const int m = (int)(i % d);
  const int kb = (int)(i / d), kh = kb / B, b = kb - kh * B;
  float a = b1 ? __bfloat162float(b1[(size_t)kh * d + m]) : 0.f;
  for (int s2 = 0; s2 < S; ++s2) a += part[(((size_t)s2 * K + kh) * B + b) * d + m];
  const float uu = a / (1.f + expf(-a)) + __bfloat162float(h[(size_t)b * d + m]);
  const __nv_bfloat16 hi = __float2bfloat16_rn(uu);
  const __nv_bfloat16 lo = __float2bfloat16_rn(uu - __bfloat162float(hi));
  __nv_bfloat16* urow = u + ((size_t)kh * 2 * B + 2 * b) * d + m;
  urow[0] = hi;
  urow[d] = lo;
}

int choose_splits(int tiles, int kchunks, int sms, double want) {
  int best = 1;
  double best_eff = 0.0;
  for (int S = 1; S <= 16 && S <= kchunks / 4 + (S == 1); ++S) {
    const long long units = (long long)tiles * S;
    const long long waves = (units + sms - 1) / sms;
    const double eff = (double)units / (double)(waves * sms);
    if (eff >= want) return S;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = S;
    }
  }
  return best;
}

int ncols_for(int cols) { return cols <= 16 ? 16 : (cols <= 32 ? 32 : 64); }

struct TcPlan {
  int nc1, nc2, mt1, mt2, kch, S1, S2;
  size_t off_u, off_p1, off_p2, off_cnt, off_cand, total;
};

TcPlan make_plan(int B, int d, int V, int K, int s) {
  TcPlan P;
  const int sms = num_sms();
  P.nc1 = ncols_for(B);
  P.nc2 = ncols_for(2 * B);
  P.mt1 = (d + BM - 1) / BM;
  P.mt2 = (V + BM - 1) / BM;
  P.kch = (d + BK - 1) / BK;
  P.S1 = choose_splits(K * P.mt1, P.kch, sms, 0.9);
  P.S2 = choose_splits(K * P.mt2, P.kch, sms, 0.9);
  WsCarver w;
  P.off_u = w.take<__nv_bfloat16>((size_t)K * 2 * B * d);
  P.off_p1 = w.take<float>((size_t)P.S1 * K * B * d);
  P.off_p2 = w.take<float>(P.S2 > 1 ? (size_t)K * P.mt2 * P.S2 * 2 * B * BM : 0);
  P.off_cnt = w.take<int>((size_t)K * (P.mt1 + P.mt2));
  P.off_cand = w.take<uint64_t>((size_t)B * K * P.mt2 * s);
  P.total = w.total();
  return P;
}

template <int NC>
int launch_stage(const CUtensorMap& A, const CUtensorMap& Bm, const TcParams& p,
                 cudaStream_t st) {
  using C = TcCfg<NC>;
  static std::atomic<bool> attr_done[64];  // one per instantiation of NC
  int rc = ensure_max_smem(heads_tc_kernel<NC>, (int)C::SMEM, attr_done,
                           "cudaFuncSetAttribute(heads_tc_kernel)");
  if (rc) return rc;
  const int grid = p.units < num_sms() ? p.units : num_sms();
  cudaError_t e = launch_pdl(heads_tc_kernel<NC>, dim3(grid), dim3(kThreads), C::SMEM, st, A, Bm, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "heads_tc_kernel launch");
}

int dispatch_stage(int nc, const CUtensorMap& A, const CUtensorMap& Bm, const TcParams& p,
                   cudaStream_t st) {
  if (nc == 16) return launch_stage<16>(A, Bm, p, st);
  if (nc == 32) return launch_stage<32>(A, Bm, p, st);
  return launch_stage<64>(A, Bm, p, st);
}

}  // namespace

size_t heads_tc_workspace(int B, int d, int V, int K, int s) {
  return make_plan(B, d, V, K, s).total;
}

int heads_tc_launch(const HeadsArgs& a, cudaStream_t st) {
  const TcPlan P = make_plan(a.B, a.d, a.V, a.K, a.s);
  if (a.ws_bytes < P.total) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for heads");
  uint8_t* ws = (uint8_t*)a.ws;
  __nv_bfloat16* u = (__nv_bfloat16*)(ws + P.off_u);
  int* counters = (int*)(ws + P.off_cnt);
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
    const uint32_t box[2] = {BK, (uint32_t)P.nc1};
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
    const uint32_t box[3] = {BK, (uint32_t)P.nc2, 1};
    int rc = make_tmap_bf16(&mB2, u, 3, dims, strides, box);
    if (rc) return rc;
  }

  TcParams p1{};
  p1.stage = 1;
  p1.K = a.K;
  p1.rows = a.d;
  p1.mtiles = P.mt1;
  p1.kchunks = P.kch;
  p1.splits = P.S1;
  p1.units = a.K * P.mt1 * P.S1;
  p1.B = a.B;
  p1.d = a.d;
  p1.ncp = a.B;
  p1.b1 = (const __nv_bfloat16*)a.b1;
  p1.h = (const __nv_bfloat16*)a.h;
  p1.u = u;
  p1.part = (float*)(ws + P.off_p1);
  p1.counters = counters;
  int rc = dispatch_stage(P.nc1, mA1, mB1, p1, st);
  if (rc) return rc;
  {
    const long long n = (long long)a.K * a.B * a.d;
    cudaError_t e2 = launch_pdl(heads_silu_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                                st, p1.part,
                                P.S1, a.K, a.B, a.d, (const __nv_bfloat16*)a.b1,
                                (const __nv_bfloat16*)a.h, u, counters + (size_t)a.K * P.mt1,
                                a.K * P.mt2);
    if (e2 == cudaSuccess) e2 = cudaGetLastError();
    if (e2 != cudaSuccess) return cuda_fail(e2, "heads_silu_kernel launch");
  }

  TcParams p2 = p1;
  p2.stage = 2;
  p2.rows = a.V;
  p2.mtiles = P.mt2;
  p2.splits = P.S2;
  p2.units = a.K * P.mt2 * P.S2;
  p2.ncp = 2 * a.B;
  p2.logits = a.logits;
  p2.cand = a.topk_idx ? cand : nullptr;
  p2.s = a.s;
  p2.part = (float*)(ws + P.off_p2);
  p2.counters = counters + (size_t)a.K * P.mt1;
  rc = dispatch_stage(P.nc2, mA2, mB2, p2, st);
  if (rc) return rc;

  if (a.topk_idx)
    return topk_keys_launch(cand, a.B * a.K, P.mt2 * a.s, a.s, a.topk_idx, a.topk_val, st);
  return MEDUSA_OK;
}

}  // namespace medusa

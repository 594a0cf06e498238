// Tree attention on the 5th-generation tensor cores (tcgen05), bf16, dh = 128.
//
// Medusa paper digest ("論文解説: Medusa"), section "ツリーアテンションによる
// 並列検証": Mask_ij = 1 iff token j is an ancestor of token i, so all
// candidate paths are verified in one pass.  Node i of sequence b attends to
// the cached prefix (slots 0..L_b-1) and to the tree slots L_b + j of the
// nodes j on its root path (itself included).
//
// One CTA = (128 query rows, key chunk, sequence x kv-head).  The query rows
// of a kv-head are the tree nodes x the GQA group, packed so every K/V tile
// staged in shared memory serves all of them (the row tiles of one kv-head
// are adjacent in launch order and share tiles through L2).  Per 128-key
// tile:
//   S  = Q K^T        tcgen05.mma, Q and K K-major in smem, S in TMEM
//                     (double-buffered so S(j+1) overlaps softmax(j))
//   softmax           8 warps, two threads per query row (64 columns each):
//                     tcgen05.ld of the S half-row, prefix limit /
//                     ancestor-bitmask mask, tile max exchanged between the
//                     halves through TMEM, running max with lazy rescaling
//                     (the reference max moves only when it grows by more
//                     than 2^8, then the O row is rescaled in TMEM),
//                     P = 2^(scale*s - m) as bf16 into a double-buffered,
//                     128-byte-swizzled K-major smem tile
//   O += P V          tcgen05.mma, V is the MN-major operand straight from
//                     its TMA tile, O accumulates in TMEM
// Warp 0 issues the TMA loads (Q once, a 2-deep ring of K and V tiles),
// warp 1 issues all MMAs from one thread, warps 2-9 run the softmax and the
// epilogue.  Warps whose rows are all padding (fewer than 128 query rows)
// keep the barrier protocol but skip the arithmetic.  With one chunk the CTA
// writes the normalised output; with more it writes unnormalised partials
// (O, max, sum) for the combine kernel.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kThreads = 352;  // K producer, MMA issuer, 8 softmax warps, V producer
constexpr int kVWarp = 10;
constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int DH = 128;
constexpr uint32_t HALF = 128 * 64 * 2;  // one 64-column half of a 128-row bf16 tile
constexpr uint32_t TILE = 2 * HALF;      // 32 KB
constexpr int KV_STAGES = 3;
constexpr size_t SMEM = 1024 + (1 + 2 * KV_STAGES) * (size_t)TILE + 256;  // Q | K[3] | V[3] | barriers
constexpr float kRescale = 8.0f;  // log2 of the growth that forces a rescale

struct TcAttnParams {
  const int32_t* L;
  const uint32_t* anc;
  int B, N, W, Hq, Hkv, G, Lcap, R, P;
  float qscale;  // softmax scale * log2(e)
  __nv_bfloat16* out;
  float* po;
  float2* pml;
};

struct Range {
  int k_lo, k_hi, n_pre, n_tree;
};

__device__ __forceinline__ Range chunk_range(const TcAttnParams& p, int Lb, int chunk,
                                             bool seq_ok) {
  Range rg{0, 0, 0, 0};
  if (!seq_ok) return rg;
  int per = (Lb + p.P - 1) / p.P;
  per = (per + BN - 1) / BN * BN;
  rg.k_lo = min(Lb, chunk * per);
  rg.k_hi = min(Lb, rg.k_lo + per);
  rg.n_pre = (rg.k_hi - rg.k_lo + BN - 1) / BN;
  rg.n_tree = (chunk == p.P - 1) ? (p.N + BN - 1) / BN : 0;
  return rg;
}

// Writes columns [cb, cb + NCOL) of one query row: normalised bf16 output
// (one chunk) or the fp32 partial O plus, if write_ml, its (max, sum).
// o == nullptr writes an empty row (no visible key).
template <int NCOL>
__device__ __forceinline__ void write_row(const TcAttnParams& p, int b, int kvh, int chunk,
                                          int grow, int cb, float m, float l, const float* o,
                                          bool write_ml) {
  const int node = grow / p.G, g = grow - node * p.G;
  if (p.P == 1) {
    const float inv = (o && l > 0.f) ? 1.f / l : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(
        p.out + (((size_t)b * p.N + node) * p.Hq + (size_t)kvh * p.G + g) * DH + cb);
#pragma unroll
    for (int c = 0; c < NCOL / 8; ++c) {
      __align__(16) __nv_bfloat162 h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        h[e] = o ? __floats2bfloat162_rn(o[c * 8 + 2 * e] * inv, o[c * 8 + 2 * e + 1] * inv)
                 : __floats2bfloat162_rn(0.f, 0.f);
      dst[c] = *reinterpret_cast<const uint4*>(h);
    }
  } else {
    const size_t prow = ((size_t)(b * p.Hkv + kvh) * p.P + chunk) * p.R + grow;
    float4* dst = reinterpret_cast<float4*>(p.po + prow * DH + cb);
#pragma unroll
    for (int c = 0; c < NCOL / 4; ++c)
      dst[c] = o ? make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3])
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    if (write_ml) p.pml[prow] = make_float2(o ? m : -INFINITY, o ? l : 0.f);
  }
}

// Scores of one 64-column half (hf) of tile j with masked columns set to
// -inf: prefix tiles past the chunk end, tree tiles outside the row's
// ancestor set (am = its ancestor bitmask words).
__device__ __forceinline__ void mask_half(float (&v)[64], int hf, int j, const Range& rg, int N,
                                          const uint32_t (&am)[MEDUSA_MAX_N / 32]) {
  if (j < rg.n_pre) {
    const int lim = rg.k_hi - (rg.k_lo + j * BN) - hf * 64;
    if (lim < 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = (c < lim) ? v[c] : -INFINITY;
    }
  } else {
    const int tt = j - rg.n_pre;  // tree tile: nodes tt*128 .. tt*128+127
    // words of nodes tt*128 + 64*hf .. +63 (tt is 0 or 1 as N <= 256);
    // selects rather than a run-time index keep am[] in registers
    const uint32_t a0 = tt ? am[4] : am[0], a1 = tt ? am[5] : am[1];
    const uint32_t a2 = tt ? am[6] : am[2], a3 = tt ? am[7] : am[3];
    const uint32_t w0 = hf ? a2 : a0, w1 = hf ? a3 : a1;
    const int nvalid = N - tt * BN - hf * 64;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      const uint32_t word = c < 32 ? w0 : w1;
      const bool vis = c < nvalid && ((word >> (c & 31)) & 1u);
      v[c] = vis ? v[c] : -INFINITY;
    }
  }
}

__device__ __forceinline__ float max64(const float (&v)[64]) {
  float mx[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) mx[e] = v[e];
#pragma unroll
  for (int c = 8; c < 64; ++c) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
  return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TILE;                   // [KV_STAGES]
  uint8_t* sV = sm + (1 + KV_STAGES) * TILE;  // [KV_STAGES]
  uint64_t* bars = (uint64_t*)(sm + (1 + 2 * KV_STAGES) * TILE);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                    // [KV_STAGES]
  uint64_t* k_empty = k_full + KV_STAGES;         // [KV_STAGES]
  uint64_t* v_full = k_empty + KV_STAGES;         // [KV_STAGES]
  uint64_t* v_empty = v_full + KV_STAGES;         // [KV_STAGES]
  uint64_t* s_full = v_empty + KV_STAGES;         // [2]
  uint64_t* s_free = s_full + 2;                  // [2]
  uint64_t* p_full = s_free + 2;  // softmax wrote P (TMEM)
  uint64_t* o_done = p_full + 1;  // every P.V completed (P free, O stable)
  uint64_t* o_final = o_done + 1; // the last P.V completed
  uint64_t* mma_done = o_final + 1;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int mt = blockIdx.x, chunk = blockIdx.y, bk = blockIdx.z;
  const int b = bk / p.Hkv, kvh = bk - b * p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Lb = p.L[b];
  const bool seq_ok = Lb >= 0 && (long long)Lb + p.N <= p.Lcap;
  const Range rg = chunk_range(p, Lb, chunk, seq_ok);
  const int T = rg.n_pre + rg.n_tree;

  if (T == 0) {  // nothing to attend to in this chunk
    if (threadIdx.x < BM) {
      const int grow = mt * BM + threadIdx.x;
      if (grow < p.R) write_row<DH>(p, b, kvh, chunk, grow, 0, -INFINITY, 0.f, nullptr, true);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < KV_STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 256);
    }
    mbar_init(p_full, 8);
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, 512);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------------- TMA producers
    // warp 0 streams Q and the K tiles, warp 10 the V tiles, so a K tile is
    // requested as soon as its stage frees (after S), not after the P.V that
    // frees the V stage of the tile before.
    if (lane == 0) {
      const bool isK = warp == 0;
      const uint64_t pol = policy_evict_normal();
      if (isK) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        const int zq = b * p.N + mt * (BM / p.G);
        mbar_arrive_expect_tx(q_full, TILE);
        tma_load_3d(sQ, &tmQ, q_full, 0, kvh * p.G, zq, pol);
        tma_load_3d(sQ + HALF, &tmQ, q_full, 64, kvh * p.G, zq, pol);
      } else {
        prefetch_tmap(&tmV);
      }
      const CUtensorMap* map = isK ? &tmK : &tmV;
      uint64_t* emp = isK ? k_empty : v_empty;
      uint64_t* ful = isK ? k_full : v_full;
      uint8_t* buf = isK ? sK : sV;
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % KV_STAGES;
        const int key0 = j < rg.n_pre ? rg.k_lo + j * BN : Lb + (j - rg.n_pre) * BN;
        const int z = b * p.Lcap + key0;
        if (!mbar_wait(&emp[st], ((uint32_t)(j / KV_STAGES) & 1u) ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&ful[st], TILE);
        tma_load_3d(buf + st * TILE, map, &ful[st], 0, kvh, z, pol);
        tma_load_3d(buf + st * TILE + HALF, map, &ful[st], 64, kvh, z, pol);
        issued = j + 1;
      }
      if (issued < T) {
        // aborted: let the loads already issued land before the CTA exits
        if (isK) mbar_wait(q_full, 0u, nullptr);
        for (int j = (issued > KV_STAGES ? issued - KV_STAGES : 0); j < issued; ++j)
          mbar_wait(&ful[j % KV_STAGES], (uint32_t)(j / KV_STAGES) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16_f32(BM, BN);
      const uint32_t idesc_o = umma_idesc_bf16_f32_bmn(BM, DH);
      const uint32_t tO = tmem + 256;
      const uint32_t tP = tmem + 384;  // P: 64 columns of bf16 pairs
      bool ok = mbar_wait(q_full, 0u, abort_flag);
      for (int j = 0; j <= T && ok; ++j) {
        if (j < T) {
          const int ks = j % KV_STAGES;
          const int sb = j & 1;  // S buffer
          if (!mbar_wait(&k_full[ks], (uint32_t)(j / KV_STAGES) & 1u, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&s_free[sb], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tS = tmem + (uint32_t)sb * BN;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32u;
            umma_bf16(tS, umma_desc_sw128_kmajor(smem_u32(sQ) + off),
                      umma_desc_sw128_kmajor(smem_u32(sK + ks * TILE) + off), idesc_s,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(&k_empty[ks]);
          umma_commit(&s_full[sb]);
        }
        if (j >= 1) {
          // O += P V with P (bf16, written by the softmax warps) read from TMEM
          const int jj = j - 1;
          const int vs = jj % KV_STAGES;
          if (!mbar_wait(p_full, (uint32_t)(jj & 1), abort_flag)) { ok = false; break; }
          if (!mbar_wait(&v_full[vs], (uint32_t)(jj / KV_STAGES) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            umma_bf16_ts(tO, tP + (uint32_t)kk * 8u,
                         umma_desc_sw128(smem_u32(sV + vs * TILE) + (uint32_t)kk * 2048u, HALF,
                                         1024u),
                         idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&v_empty[vs]);
          umma_commit(o_done);
          if (jj == T - 1) umma_commit(o_final);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    // Two warpgroups share every S row: warps 2-5 take columns 0-63, warps
    // 6-9 columns 64-127 (two warps per SM sub-partition for latency
    // hiding).  The halves exchange their tile maxima and final sums through
    // spare TMEM columns (384 + ...), as the row's two threads sit in
    // different warps of the same TMEM lane quadrant.
    const int half = warp >= 6 ? 1 : 0;
    const int cb = half * 64;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int grow = mt * BM + r;
    const bool row_ok = grow < p.R;
    const bool warp_live = (mt * BM + q4 * 32) < p.R;  // warp-uniform
    const int node = min(grow / p.G, p.N - 1);
    uint32_t am[MEDUSA_MAX_N / 32];
#pragma unroll
    for (int w = 0; w < MEDUSA_MAX_N / 32; ++w) am[w] = (w < p.W) ? p.anc[(size_t)node * p.W + w] : 0u;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tx = tmem + lane_base + 448;  // exchange columns
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      bool good = ok && mbar_wait(&s_full[st], (j >> 1) & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, good)) {
        // no named barrier inside this loop: every wait is bounded, so the
        // other warps leave as soon as their own waits see the abort flag
        ok = false;
        break;
      }
      tc_fence_after();
      if (!warp_live) {
        // every row of this warp is padding past the last query row: keep
        // the barrier protocol, skip the arithmetic (its P rows are never
        // output; O rows are independent of each other).  Waiting for
        // PV(j-1) first keeps this arrival out of tile j-1's phase.
        tc_fence_before();
        mbar_arrive(&s_free[st]);
        if (j >= 1) {
          const bool w_ok = mbar_wait(o_done, (uint32_t)((j - 1) & 1), abort_flag);
          if (!__all_sync(0xffffffffu, w_ok)) { ok = false; continue; }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        continue;
      }
      // the whole row's max: the other half is read too (instead of trading
      // maxima with the other warpgroup), so the two halves never wait for
      // each other within a tile and their MUFU phases can drift apart
      float s[64];
      float omax;
      {
        float t[64];
        tmem_ld64(tmem + lane_base + (uint32_t)st * BN + (uint32_t)(64 - cb), t);
        mask_half(t, half ^ 1, j, rg, p.N, am);
        omax = max64(t);
      }
      tmem_ld64(tmem + lane_base + (uint32_t)st * BN + (uint32_t)cb, s);
      tc_fence_before();
      mbar_arrive(&s_free[st]);
      mask_half(s, half, j, rg, p.N, am);
      const float hmax = max64(s);
      const float tmax = fmaxf(hmax, omax) * p.qscale;  // scale > 0
      float corr = 1.f;
      bool rescale = false;
      if (tmax > m_used + kRescale) {
        corr = ex2_approx(m_used - tmax);  // 0 when m_used is -inf
        m_used = tmax;
        l *= corr;
        rescale = true;
      }
      // p = 2^(scale*s - m); a row with no visible key yet has m = -inf and
      // only -inf scores, for which 2^(-inf) = 0 with any finite offset
      const float moff = (m_used == -INFINITY) ? 0.f : m_used;
      float sum8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) sum8[e] = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float e = ex2_approx(fmaf(s[c], p.qscale, -moff));
        s[c] = e;
        sum8[c & 7] += e;
      }
      l += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));

      // P (TMEM) is free and O stable once PV(j-1) has completed; PV(j-2)
      // completed before this softmax's previous tile went on, so o_done is
      // at most one completion away from the awaited one
      if (j >= 1) {
        const bool w_ok = mbar_wait(o_done, (uint32_t)((j - 1) & 1), abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; continue; }
        tc_fence_after();
        // each half rescales its own 64 columns of the O row
        if (__any_sync(0xffffffffu, rescale)) {
          const uint32_t tO = tmem + lane_base + 256 + (uint32_t)cb;
#pragma unroll
          for (int c0 = 0; c0 < 64; c0 += 16) {
            float t[16];
            tmem_ld16(tO + c0, t);
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] *= corr;
            tmem_st16(tO + c0, t);
          }
        }
      }
      // my 64 keys of the P row -> TMEM columns 384 + 32*half, bf16 pairs
      {
        uint32_t pk[32];
#pragma unroll
        for (int c2 = 0; c2 < 32; ++c2) pk[c2] = pack_bf16x2_pos(s[2 * c2], s[2 * c2 + 1]);
        tmem_st32(tmem + lane_base + 384u + (uint32_t)(half * 32), pk);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // combine the halves' sums, then the epilogue (every softmax thread
    // reaches this barrier: the loop above leaves only all together)
    if (ok && warp_live) {
      tmem_st1(tx + 4u + (uint32_t)half, l);
      tc_fence_before();
    }
    const bool bad = bar_red_or(2, 256, !ok || *abort_flag);
    if (!bad && warp_live) {
      tc_fence_after();
      l += tmem_ld1(tx + 4u + (uint32_t)(half ^ 1));
      bool w_ok = mbar_wait(o_final, 0u, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (w_ok) {
        tc_fence_after();
        float o[64];
        tmem_ld64(tmem + lane_base + 256 + (uint32_t)cb, o);
        if (row_ok) write_row<64>(p, b, kvh, chunk, grow, cb, m_used, l, o, half == 0);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_tc_eligible(int dtype, int dh, int Hq, int Hkv) {
  const int G = Hq / Hkv;
  return dtype == MEDUSA_BF16 && dh == DH && G >= 1 && G <= BM && (BM % G) == 0;
}

int attention_tc_chunks(int B, int Hq, int Hkv, int N, int Lcap) {
  const int G = Hq / Hkv;
  const long long R = (long long)N * G;
  const long long units = (long long)B * Hkv * ((R + BM - 1) / BM);
  const int sms = num_sms();
  long long P = (3LL * sms + units - 1) / units;
  const long long max_p = ((long long)(Lcap - N) + 2 * BN - 1) / (2 * BN);  // >= 2 tiles each
  if (P > max_p) P = max_p;
  if (P < 1) P = 1;
  return (int)P;
}

int attention_tc_run(const AttnArgs& a, int P, float* po, float2* pml, cudaStream_t st) {
  const medusa_tree* t = a.tree;
  const int G = a.Hq / a.Hkv;
  const int R = t->N * G;
  const int mtiles = (R + BM - 1) / BM;
  alignas(64) CUtensorMap mQ, mK, mV;
  {
    const uint64_t dims[3] = {(uint64_t)DH, (uint64_t)a.Hq, (uint64_t)a.B * t->N};
    const uint64_t strides[2] = {(uint64_t)DH * 2, (uint64_t)a.Hq * DH * 2};
    const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)(BM / G)};
    int rc = make_tmap_bf16(&mQ, a.q, 3, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)DH, (uint64_t)a.Hkv, (uint64_t)a.B * a.Lcap};
    const uint64_t strides[2] = {(uint64_t)DH * 2, (uint64_t)a.Hkv * DH * 2};
    const uint32_t box[3] = {64, 1, BN};
    int rc = make_tmap_bf16(&mK, a.k, 3, dims, strides, box);
    if (rc) return rc;
    rc = make_tmap_bf16(&mV, a.v, 3, dims, strides, box);
    if (rc) return rc;
  }
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tree_attn_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tree_attn_tc_kernel)");
    attr_set[dev] = true;
  }
  TcAttnParams p;
  p.L = a.L;
  p.anc = t->d_anc;
  p.B = a.B;
  p.N = t->N;
  p.W = t->W;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = G;
  p.Lcap = a.Lcap;
  p.R = R;
  p.P = P;
  p.qscale = a.scale * 1.4426950408889634f;
  p.out = (__nv_bfloat16*)a.out;
  p.po = po;
  p.pml = pml;
  dim3 grid(mtiles, P, a.B * a.Hkv);
  tree_attn_tc_kernel<<<grid, kThreads, SMEM, st>>>(mQ, mK, mV, p);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "tree_attn_tc_kernel launch");
}

}  // namespace medusa

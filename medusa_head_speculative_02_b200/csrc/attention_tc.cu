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
//   softmax           4 warps, thread = query row: tcgen05.ld of its S row,
//                     scale to base 2, prefix limit / ancestor-bitmask mask,
//                     running max with lazy rescaling (the reference max
//                     moves only when it grows by more than 2^8, then the O
//                     row is rescaled in TMEM), P = 2^(s - m) as bf16 into a
//                     128-byte-swizzled K-major smem tile
//   O += P V          tcgen05.mma, V is the MN-major operand straight from
//                     its TMA tile, O accumulates in TMEM
// Warp 0 issues the TMA loads (Q once, a 2-deep ring of K and V tiles),
// warp 1 issues all MMAs from one thread, warps 2-5 run the softmax and the
// epilogue.  With one chunk the CTA writes the normalised output; with more
// it writes unnormalised partials (O, max, sum) for the combine kernel.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kThreads = 192;
constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int DH = 128;
constexpr uint32_t HALF = 128 * 64 * 2;  // one 64-column half of a 128-row bf16 tile
constexpr uint32_t TILE = 2 * HALF;      // 32 KB
constexpr size_t SMEM = 1024 + 7 * (size_t)TILE + 256;  // Q | K[2] | V[2] | P[2] | barriers
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

__device__ __forceinline__ void write_row(const TcAttnParams& p, int b, int kvh, int chunk,
                                          int grow, float m, float l, const float* o,
                                          bool normalise) {
  const int node = grow / p.G, g = grow - node * p.G;
  if (p.P == 1) {
    const float inv = (normalise && l > 0.f) ? 1.f / l : 0.f;
    uint4* dst = reinterpret_cast<uint4*>(
        p.out + (((size_t)b * p.N + node) * p.Hq + (size_t)kvh * p.G + g) * DH);
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) {
      __align__(16) __nv_bfloat16 h[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) h[e] = __float2bfloat16_rn(o ? o[c * 8 + e] * inv : 0.f);
      dst[c] = *reinterpret_cast<const uint4*>(h);
    }
  } else {
    const size_t prow = ((size_t)(b * p.Hkv + kvh) * p.P + chunk) * p.R + grow;
    float4* dst = reinterpret_cast<float4*>(p.po + prow * DH);
#pragma unroll
    for (int c = 0; c < DH / 4; ++c)
      dst[c] = o ? make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3])
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    p.pml[prow] = make_float2(o ? m : -INFINITY, o ? l : 0.f);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TILE;
  uint8_t* sV = sm + 3 * TILE;
  uint8_t* sP = sm + 5 * TILE;  // [2]
  uint64_t* bars = (uint64_t*)(sm + 7 * TILE);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* s_free = bars + 11;  // [2]
  uint64_t* p_full = bars + 13;  // [2] softmax wrote P buffer i
  uint64_t* p_free = bars + 15;  // [2] the P.V reading P buffer i completed
  uint64_t* o_done = bars + 17;  // every P.V completed (O stable for rescaling)
  uint64_t* o_final = bars + 18; // the last P.V completed
  uint64_t* mma_done = bars + 19;
  uint32_t* tmem_slot = (uint32_t*)(bars + 20);
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
      if (grow < p.R) write_row(p, b, kvh, chunk, grow, -INFINITY, 0.f, nullptr, false);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const uint64_t pol = policy_evict_normal();
      const int zq = b * p.N + mt * (BM / p.G);
      mbar_arrive_expect_tx(q_full, TILE);
      tma_load_3d(sQ, &tmQ, q_full, 0, kvh * p.G, zq, pol);
      tma_load_3d(sQ + HALF, &tmQ, q_full, 64, kvh * p.G, zq, pol);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < T && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1u;
        const int key0 = j < rg.n_pre ? rg.k_lo + j * BN : Lb + (j - rg.n_pre) * BN;
        const int z = b * p.Lcap + key0;
        if (!mbar_wait(&k_empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[st], TILE);
        tma_load_3d(sK + st * TILE, &tmK, &k_full[st], 0, kvh, z, pol);
        tma_load_3d(sK + st * TILE + HALF, &tmK, &k_full[st], 64, kvh, z, pol);
        if (!mbar_wait(&v_empty[st], ph ^ 1u, abort_flag)) { ok = false; issued = 2 * j + 1; break; }
        mbar_arrive_expect_tx(&v_full[st], TILE);
        tma_load_3d(sV + st * TILE, &tmV, &v_full[st], 0, kvh, z, pol);
        tma_load_3d(sV + st * TILE + HALF, &tmV, &v_full[st], 64, kvh, z, pol);
        issued = 2 * (j + 1);
      }
      if (!ok) {
        // let the loads already issued land before the CTA exits
        mbar_wait(q_full, 0u, nullptr);
        const int jk = (issued + 1) / 2;  // K tiles issued
        const int jv = issued / 2;        // V tiles issued
        for (int j = (jk > 2 ? jk - 2 : 0); j < jk; ++j)
          mbar_wait(&k_full[j & 1], (j >> 1) & 1u, nullptr);
        for (int j = (jv > 2 ? jv - 2 : 0); j < jv; ++j)
          mbar_wait(&v_full[j & 1], (j >> 1) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16_f32(BM, BN);
      const uint32_t idesc_o = umma_idesc_bf16_f32_bmn(BM, DH);
      const uint32_t tO = tmem + 256;
      bool ok = mbar_wait(q_full, 0u, abort_flag);
      for (int j = 0; j <= T && ok; ++j) {
        if (j < T) {
          const int st = j & 1;
          const uint32_t ph = (j >> 1) & 1u;
          if (!mbar_wait(&k_full[st], ph, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&s_free[st], ph ^ 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tS = tmem + (uint32_t)st * BN;
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32u;
            umma_bf16(tS, umma_desc_sw128_kmajor(smem_u32(sQ) + off),
                      umma_desc_sw128_kmajor(smem_u32(sK + st * TILE) + off), idesc_s,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(&k_empty[st]);
          umma_commit(&s_full[st]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj & 1;
          if (!mbar_wait(&p_full[jj & 1], (uint32_t)((jj >> 1) & 1), abort_flag)) { ok = false; break; }
          if (!mbar_wait(&v_full[st], (jj >> 1) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t aoff = (uint32_t)(kk >> 2) * HALF + (uint32_t)(kk & 3) * 32u;
            umma_bf16(tO, umma_desc_sw128_kmajor(smem_u32(sP + (jj & 1) * TILE) + aoff),
                      umma_desc_sw128(smem_u32(sV + st * TILE) + (uint32_t)kk * 2048u, HALF,
                                      1024u),
                      idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&v_empty[st]);
          umma_commit(&p_free[jj & 1]);
          umma_commit(o_done);
          if (jj == T - 1) umma_commit(o_final);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int grow = mt * BM + r;
    const bool row_ok = grow < p.R;
    const int node = min(grow / p.G, p.N - 1);
    uint32_t am[MEDUSA_MAX_N / 32];
#pragma unroll
    for (int w = 0; w < MEDUSA_MAX_N / 32; ++w) am[w] = (w < p.W) ? p.anc[(size_t)node * p.W + w] : 0u;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      ok = mbar_wait(&s_full[st], (j >> 1) & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[BN];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float t[32];
        tmem_ld32(tmem + lane_base + (uint32_t)st * BN + c0, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c0 + e] = t[e];
      }
      tc_fence_before();
      mbar_arrive(&s_free[st]);

      // mask (masked scores become -inf; full prefix tiles need none)
      if (j < rg.n_pre) {
        const int lim = rg.k_hi - (rg.k_lo + j * BN);
        if (lim < BN) {
#pragma unroll
          for (int c = 0; c < BN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
        }
      } else {
        const int tt = j - rg.n_pre;  // tree tile: nodes tt*128 .. tt*128+127
        uint32_t wsel[BN / 32];
#pragma unroll
        for (int w = 0; w < BN / 32; ++w) wsel[w] = tt == 0 ? am[w] : am[BN / 32 + w];
        const int nvalid = p.N - tt * BN;  // columns >= nvalid are past the last node
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          const bool vis = c < nvalid && ((wsel[c >> 5] >> (c & 31)) & 1u);
          s[c] = vis ? s[c] : -INFINITY;
        }
      }
      // raw row max (8 independent chains), then base 2: scale > 0
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = s[e];
#pragma unroll
      for (int c = 8; c < BN; ++c) mx[c & 7] = fmaxf(mx[c & 7], s[c]);
      const float tmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * p.qscale;
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
      for (int c = 0; c < BN; ++c) {
        const float e = ex2_approx(fmaf(s[c], p.qscale, -moff));
        s[c] = e;
        sum8[c & 7] += e;
      }
      l += ((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7]));

      // P buffer j&1 is free once PV(j-2) has read it
      if (j >= 2) {
        ok = mbar_wait(&p_free[st], (uint32_t)(((j >> 1) & 1) ^ 1), abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      }
      // rescaling O needs PV(j-1) complete (PV(j-2) is, so o_done is at most
      // one completion away from the awaited one)
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
        ok = mbar_wait(o_done, (uint32_t)((j - 1) & 1), abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        {
          const uint32_t tO = tmem + lane_base + 256;
#pragma unroll
          for (int c0 = 0; c0 < DH; c0 += 16) {
            float t[16];
            tmem_ld16(tO + c0, t);
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] *= corr;
            tmem_st16(tO + c0, t);
          }
        }
      }
      // P row -> smem, bf16, K-major with 128-byte swizzle
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          __align__(16) __nv_bfloat162 v2[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            v2[e] = __floats2bfloat162_rn(s[h * 64 + c8 * 8 + 2 * e], s[h * 64 + c8 * 8 + 2 * e + 1]);
          uint8_t* dst = sP + st * TILE + h * HALF + r * 128 + ((c8 ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(v2);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
    }
    if (ok) {
      ok = mbar_wait(o_final, 0u, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      float o[DH];
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 32) {
        float t[32];
        tmem_ld32(tmem + lane_base + 256 + c0, t);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c0 + e] = t[e];
      }
      if (row_ok) write_row(p, b, kvh, chunk, grow, m_used, l, o, true);
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

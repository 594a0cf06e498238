// Tree attention (verification pass of the candidate tree).
//
// Medusa paper digest ("論文解説: Medusa"), section "ツリーアテンションによる
// 並列検証": Mask_ij = 1 iff token j is an ancestor of token i in the tree, so
// every candidate path is scored in one pass; glossary ("Medusa",
// "Attention en arbre"): each node sees only its ancestors.  Node i of
// sequence b attends to the cached prefix (slots 0..L_b-1, unmasked) and to
// the tree slots L_b + j for the nodes j on its root path (itself included).
//
// Split-KV ("flash-decoding") layout: the keys of a (sequence, kv-head) are
// cut into P prefix chunks plus one tree chunk; every (row block, chunk)
// pair is an independent CTA producing unnormalised partial outputs with
// their running max / sum in base 2, and a combine kernel merges the chunks
// of every query row.  All query rows of a kv-head (tree nodes x the GQA
// group) share each staged K/V tile.  This SIMT kernel serves fp32 and
// dh = 64; attention_launch sends bf16 with dh = 128 to the tensor-core
// kernels of attention_tc.cu, whose launch shape (query tiles per CTA, key
// chunks, in-cluster merge) attention_tc_shape chooses.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int RB = 16;        // query rows per CTA
constexpr int TK = 32;        // keys per tile
constexpr int kThreads = 128; // 8 threads per query row

struct AttnPlan {
  int R;        // query rows per (b, kv-head) = N * G
  int rblocks;  // ceil(R / RB)
  int P;        // prefix chunks
  int chunks;   // P + 1 (tree chunk last)
  size_t off_o, off_ml, total;
};

AttnPlan make_plan(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap) {
  AttnPlan P;
  const int G = Hq / Hkv;
  P.R = t->N * G;
  P.rblocks = (P.R + RB - 1) / RB;
  const long long base = (long long)P.rblocks * B * Hkv;
  const int sms = num_sms();
  // >= ~4 CTAs per SM in total (an empty batch has nothing to split)
  long long want = base > 0 ? (4LL * sms + base - 1) / base : 1;
  const int max_p = (Lcap + 255) / 256;           // >= 256 keys per chunk
  if (want < 1) want = 1;
  if (want > max_p) want = max_p;
  if (want < 1) want = 1;
  P.P = (int)want;
  P.chunks = P.P + 1;
  WsCarver w;
  const size_t rows = (size_t)B * Hkv * P.chunks * P.R;
  P.off_o = w.take<float>(rows * dh);
  P.off_ml = w.take<float2>(rows);
  P.total = w.total();
  return P;
}

// grid: (rblocks, chunks, B*Hkv)
template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
    tree_attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ kc,
                          const T* __restrict__ vc, const int32_t* __restrict__ Lp,
                          const uint32_t* __restrict__ anc, int N, int W, int Hq, int Hkv,
                          int Lcap, float qscale, int P, int R, float* __restrict__ po,
                          float2* __restrict__ pml) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  __shared__ float qs[RB][DH];
  __shared__ float ks[TK][DH + 1];
  __shared__ float vs[TK][DH];
  __shared__ float ps[RB][TK];
  __shared__ uint32_t am[RB][MEDUSA_MAX_N / 32];

  const int rb = blockIdx.x, chunk = blockIdx.y;
  const int bk = blockIdx.z;
  const int b = bk / Hkv, kvh = bk - b * Hkv;
  const int G = Hq / Hkv;
  const int tid = threadIdx.x;
  const int i = tid >> 3;  // row within block
  const int sub = tid & 7;
  const int r = rb * RB + i;
  const bool row_ok = r < R;
  const int Lb = Lp[b];
  const bool seq_ok = Lb >= 0 && (long long)Lb + N <= Lcap;

  // stage the query rows (pre-scaled to base 2) and their ancestor masks
  for (int e = tid; e < RB * DH; e += kThreads) {
    const int ii = e / DH, dd = e - ii * DH;
    const int rr = rb * RB + ii;
    float val = 0.f;
    if (rr < R) {
      const int nn = rr / G, gg = rr - nn * G;
      val = to_f32(q[(((size_t)b * N + nn) * Hq + kvh * G + gg) * DH + dd]) * qscale;
    }
    qs[ii][dd] = val;
  }
  for (int e = tid; e < RB * W; e += kThreads) {
    const int ii = e / W, w = e - ii * W;
    const int rr = rb * RB + ii;
    am[ii][w] = rr < R ? anc[(size_t)(rr / G) * W + w] : 0u;
  }

  // key range of this chunk
  int k_lo, k_hi;
  const bool tree_chunk = chunk == P;
  if (!seq_ok) {
    k_lo = k_hi = 0;
  } else if (tree_chunk) {
    k_lo = 0;
    k_hi = N;  // node indices; slots Lb + j
  } else {
    int per = (Lb + P - 1) / P;
    per = (per + TK - 1) / TK * TK;
    k_lo = min(Lb, chunk * per);
    k_hi = min(Lb, k_lo + per);
  }
  const int slot0 = tree_chunk ? Lb : 0;

  float m = -INFINITY, l = 0.f;
  float o[DH / 8];
#pragma unroll
  for (int c = 0; c < DH / 8; ++c) o[c] = 0.f;

  for (int t0 = k_lo; t0 < k_hi; t0 += TK) {
    __syncthreads();
    for (int e = tid; e < TK * DH; e += kThreads) {
      const int j = e / DH, dd = e - j * DH;
      const int key = t0 + j;
      float kv = 0.f, vv = 0.f;
      if (key < k_hi && dbg_ok(slot0 + key < Lcap, DBG_ATTN_SLOT)) {
        const size_t off = (((size_t)b * Lcap + slot0 + key) * Hkv + kvh) * DH + dd;
        kv = to_f32(kc[off]);
        vv = to_f32(vc[off]);
      }
      ks[j][dd] = kv;
      vs[j][dd] = vv;
    }
    __syncthreads();
    // scores: this thread -> row i, keys sub + 8*jj
    float sc[TK / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < TK / 8; ++jj) {
      const int j = sub + 8 * jj;
      const int key = t0 + j;
      bool valid = row_ok && key < k_hi;
      if (valid && tree_chunk) valid = (am[i][key >> 5] >> (key & 31)) & 1u;
      float s = -INFINITY;
      if (valid) {
        float acc = 0.f;
#pragma unroll 8
        for (int dd = 0; dd < DH; ++dd) acc = fmaf(qs[i][dd], ks[j][dd], acc);
        s = acc;
      }
      sc[jj] = s;
      tmax = fmaxf(tmax, s);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
    const float m_new = fmaxf(m, tmax);
    const float corr = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
    float psum = 0.f;
#pragma unroll
    for (int jj = 0; jj < TK / 8; ++jj) {
      const float p = (sc[jj] == -INFINITY) ? 0.f : exp2f(sc[jj] - m_new);
      ps[i][sub + 8 * jj] = p;
      psum += p;
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
    l = l * corr + psum;
    m = m_new;
    __syncwarp();
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) {
      const int dd = sub + 8 * c;
      float acc = o[c] * corr;
#pragma unroll 8
      for (int j = 0; j < TK; ++j) acc = fmaf(ps[i][j], vs[j][dd], acc);
      o[c] = acc;
    }
  }

  if (row_ok) {
    const size_t prow = ((size_t)bk * (P + 1) + chunk) * R + r;
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) po[prow * DH + sub + 8 * c] = o[c];
    if (sub == 0) pml[prow] = make_float2(m, l);
  }
}

// One warp per output row (b, node, h): merge the chunks.
template <typename T, int DH>
__global__ void tree_attn_combine_kernel(const float* __restrict__ po,
                                         const float2* __restrict__ pml,
                                         const int32_t* __restrict__ Lp, int B, int N, int Hq,
                                         int Hkv, int Lcap, int chunks, int R,
                                         T* __restrict__ out) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= B * N * Hq) return;
  const int h = gw % Hq;
  const int bn = gw / Hq;
  const int b = bn / N, node = bn - b * N;
  const int G = Hq / Hkv;
  const int kvh = h / G, g = h - kvh * G;
  const int r = node * G + g;
  const size_t base = ((size_t)b * Hkv + kvh) * chunks;
  float M = -INFINITY;
  for (int c = 0; c < chunks; ++c) M = fmaxf(M, pml[(base + c) * R + r].x);
  float acc[DH / 32];
#pragma unroll
  for (int e = 0; e < DH / 32; ++e) acc[e] = 0.f;
  float Ls = 0.f;
  if (M != -INFINITY) {
    for (int c = 0; c < chunks; ++c) {
      const float2 ml = pml[(base + c) * R + r];
      if (ml.x == -INFINITY) continue;
      const float w = exp2f(ml.x - M);
      Ls += w * ml.y;
      const float* orow = po + ((base + c) * R + r) * DH;
#pragma unroll
      for (int e = 0; e < DH / 32; ++e) acc[e] = fmaf(w, orow[lane + 32 * e], acc[e]);
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
  T* orow = out + (((size_t)b * N + node) * Hq + h) * DH;
#pragma unroll
  for (int e = 0; e < DH / 32; ++e) orow[lane + 32 * e] = from_f32<T>(acc[e] * inv);
}

}  // namespace

namespace {
// Partial-output layout of the tensor-core path (only used with > 1 chunk).
struct TcPlan {
  int P;
  size_t off_o, off_ml, total;
};
TcPlan make_tc_plan(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap) {
  TcPlan P;
  P.P = attention_tc_chunks(B, Hq, Hkv, t->N, Lcap);
  WsCarver w;
  const size_t rows = P.P > 1 ? (size_t)B * Hkv * P.P * t->N * (Hq / Hkv) : 0;
  P.off_o = w.take<float>(rows * dh);
  P.off_ml = w.take<float2>(rows);
  P.total = w.total();
  return P;
}
}  // namespace

int attention_chunks(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap, int dtype) {
  if (attention_tc_eligible(dtype, dh, Hq, Hkv)) return attention_tc_shape(B, Hq, Hkv, t->N, Lcap).P;
  return make_plan(t, B, Hq, Hkv, dh, Lcap).chunks;
}

int attention_tiles_per_cta(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap,
                            int dtype) {
  if (!attention_tc_eligible(dtype, dh, Hq, Hkv)) return 1;
  return attention_tc_shape(B, Hq, Hkv, t->N, Lcap).tiles;
}

int attention_launches(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap, int dtype) {
  if (B == 0) return 0;
  if (attention_tc_eligible(dtype, dh, Hq, Hkv)) {
    const TcShape sh = attention_tc_shape(B, Hq, Hkv, t->N, Lcap);
    return (sh.P <= 1 || sh.fuse) ? 1 : 2;
  }
  return 2;  // SIMT kernel and its combine kernel
}

size_t attention_workspace(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap,
                           int dtype) {
  const size_t simt = make_plan(t, B, Hq, Hkv, dh, Lcap).total;
  const size_t tc = attention_tc_eligible(MEDUSA_BF16, dh, Hq, Hkv)
                        ? make_tc_plan(t, B, Hq, Hkv, dh, Lcap).total
                        : 0;
  if (dtype < 0) return simt > tc ? simt : tc;  // size query without a dtype
  return attention_tc_eligible(dtype, dh, Hq, Hkv) ? tc : simt;
}

int attention_launch(const AttnArgs& a, cudaStream_t st) {
  const medusa_tree* t = a.tree;
  if (attention_tc_eligible(a.dtype, a.dh, a.Hq, a.Hkv)) {
    const TcPlan P = make_tc_plan(t, a.B, a.Hq, a.Hkv, a.dh, a.Lcap);
    if (a.ws_bytes < P.total)
      return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for attention");
    if (a.B == 0) return MEDUSA_OK;
    float* po = (float*)((uint8_t*)a.ws + P.off_o);
    float2* pml = (float2*)((uint8_t*)a.ws + P.off_ml);
    const TcShape sh = attention_tc_shape(a.B, a.Hq, a.Hkv, t->N, a.Lcap);
    if (sh.P > 1 && !sh.fuse && sh.P > P.P)
      return fail(MEDUSA_ERR_INVALID_ARG, "attention plan exceeds its workspace");
    int rc = attention_tc_run(a, sh, po, pml, st);
    if (rc || sh.P == 1 || sh.fuse) return rc;
    const int R = t->N * (a.Hq / a.Hkv);
    const int rows = a.B * t->N * a.Hq;
    cudaError_t e = launch_pdl(tree_attn_combine_kernel<__nv_bfloat16, 128>, dim3((rows + 7) / 8),
                               dim3(256), 0, st, po, pml, a.L, a.B, t->N, a.Hq, a.Hkv, a.Lcap,
                               sh.P, R, (__nv_bfloat16*)a.out);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "tree attention combine launch");
  }
  const AttnPlan P = make_plan(t, a.B, a.Hq, a.Hkv, a.dh, a.Lcap);
  if (a.ws_bytes < P.total) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for attention");
  if (a.B == 0) return MEDUSA_OK;
  uint8_t* ws = (uint8_t*)a.ws;
  float* po = (float*)(ws + P.off_o);
  float2* pml = (float2*)(ws + P.off_ml);
  const float qscale = a.scale * kLog2e;
  dim3 g1(P.rblocks, P.chunks, a.B * a.Hkv);
  const int rows = a.B * t->N * a.Hq;
  const int cblocks = (rows + 7) / 8;
  cudaError_t le = cudaSuccess;
#define MEDUSA_ATT(T, DH)                                                                        \
  do {                                                                                           \
    le = launch_pdl(tree_attn_simt_kernel<T, DH>, g1, dim3(kThreads), 0, st, (const T*)a.q,      \
                    (const T*)a.k, (const T*)a.v, a.L, t->d_anc, t->N, t->W, a.Hq, a.Hkv, a.Lcap, \
                    qscale, P.P, P.R, po, pml);                                                  \
    if (le == cudaSuccess)                                                                       \
      le = launch_pdl(tree_attn_combine_kernel<T, DH>, dim3(cblocks), dim3(256), 0, st, po, pml, \
                      a.L, a.B, t->N, a.Hq, a.Hkv, a.Lcap, P.chunks, P.R, (T*)a.out);            \
  } while (0)
  if (a.dtype == MEDUSA_F32) {
    if (a.dh == 64) MEDUSA_ATT(float, 64);
    else MEDUSA_ATT(float, 128);
  } else {
    if (a.dh == 64) MEDUSA_ATT(__nv_bfloat16, 64);
    else MEDUSA_ATT(__nv_bfloat16, 128);
  }
#undef MEDUSA_ATT
  cudaError_t e = le != cudaSuccess ? le : cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "tree attention launch");
}

}  // namespace medusa

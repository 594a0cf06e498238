// Tree attention on the 5th-generation tensor cores (tcgen05), bf16, dh = 128.
//
// Medusa paper digest ("論文解説: Medusa"), section "ツリーアテンションによる
// 並列検証": Mask_ij = 1 iff token j is an ancestor of token i, so all
// candidate paths are verified in one pass.  Node i of sequence b attends to
// the cached prefix (slots 0..L_b-1) and to the tree slots L_b + j of the
// nodes j on its root path (itself included).
//
// Query rows of a (sequence, kv-head) are the tree nodes x the GQA group,
// packed 128 to an MMA tile.  A CTA takes one 128-row query tile and one key
// chunk of one (sequence, kv-head); the grid's slowest index runs over the
// sequences longest first (a permutation computed on the device), so the
// long CTAs start first and the tail of the launch is made of short ones.
// Per 128-key tile t:
//   S  = Q K^T      tcgen05.mma (M 128, N 128, K 128): Q and K K-major in
//                   smem (TMA, 128-byte swizzle), S into TMEM buffer t mod 3,
//                   issued while the softmax of tile t-1 runs
//   softmax         two warpgroups, one per 64-key half of the tile; a thread
//                   owns one query row of one half: one TMEM read of its 64
//                   scores, prefix limit / ancestor-bitmask mask, the row max
//                   of the tile from both halves (exchanged through smem),
//                   one running max per row with lazy rescaling (the
//                   reference max moves only when it grows by more than 2^8;
//                   the O row is then rescaled in TMEM once the previous P.V
//                   is done), P = 2^(scale*s - m) with packed fp32x2
//                   arithmetic, one pair in four of the exponentials on the
//                   FMA pipe (polynomial) and the rest on MUFU (all on MUFU
//                   in a key half with masked keys, so those weigh exactly
//                   0), written as bf16 pairs over the S columns just read;
//                   on a tile that reaches past slot L_b + N the softmax
//                   warps first zero those V rows in shared memory (cache
//                   slots the caller need not have written: NaN or Inf
//                   there would otherwise reach O through 0 * NaN)
//   O += P V        tcgen05.mma (M 128, N 128, K 128): A = P from TMEM, V
//                   the MN-major smem operand
// TMEM (512 columns): three S/P buffers and O, 128 columns each.  Warp 0
// streams Q and the K ring, warp 10 the V ring (3 stages of 128 keys each),
// warp 1 issues the MMAs, warps 2-5 / 6-9 are the softmax warpgroups of key
// halves 0 / 1; the two warps that share a TMEM lane quadrant meet at a
// named barrier once per tile.  With one chunk the CTA writes the
// normalised output.  With more, the chunks of a query tile either form a
// thread-block cluster (one CTA per chunk, when every cluster of the launch
// fits on the GPU at once): each CTA stages its unnormalised O rows and
// (max, sum) in its own shared memory, the K/V rings being free by then, and
// rank c merges rows [c R/P, (c+1) R/P) of the tile from all ranks through
// distributed shared memory; or they write the partials to the workspace for
// the combine kernel.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace cg = cooperative_groups;
namespace {

constexpr int kThreads = 352;  // K producer, MMA issuer, 2 x 4 softmax warps, V producer
constexpr int kVWarp = 10;
constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int DH = 128;
constexpr uint32_t HALF = 128 * 64 * 2;  // 64-column half of a 128-row bf16 tile: 16 KB
constexpr uint32_t TILE = 2 * HALF;      // 32 KB
constexpr int kStages = 3;
constexpr size_t kDataBytes = (1 + 2 * kStages) * (size_t)TILE;  // Q | K ring | V ring
constexpr size_t kXchBytes = 2 * 2 * BM * sizeof(uint16_t);  // row-max exchange
constexpr size_t SMEM = 1024 + kDataBytes + 256 + kXchBytes;
constexpr float kRescale = 8.0f;  // log2 of the growth that forces a rescale
constexpr int kMaxClusterChunks = 8;  // portable cluster size
// Staged O rows of the cluster merge: fp32, a row stride of DH + 4 floats, so
// the float4 stores of 8 consecutive rows fall in distinct banks.
constexpr int OST = DH + 4;
constexpr size_t kOStage = (size_t)BM * OST * sizeof(float);
static_assert(kOStage + BM * sizeof(float2) <= 2 * kStages * (size_t)TILE,
              "staged O rows and (max, sum) fit in the K/V rings");
static_assert(MEDUSA_MAX_N == 256, "ancestor words are selected for at most 4 x 64 nodes");

struct TcAttnParams {
  const int32_t* L;
  const uint32_t* anc;
  int B, N, W, Hq, Hkv, G, Lcap, R, P, mtiles;
  int fuse;      // 1: the P chunks of a query tile are one cluster and merge in the kernel
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
  per = (per + BN - 1) / BN * BN;  // whole 128-key tiles
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

// Scores of the 64-key half hf of 128-key tile j with masked columns set to
// -inf: prefix keys past the chunk end, tree slots outside the row's
// ancestor set (am = its ancestor bitmask words).
__device__ __forceinline__ void mask_half(float (&v)[64], int j, int hf, const Range& rg, int N,
                                          const uint32_t (&am)[MEDUSA_MAX_N / 32]) {
  if (j < rg.n_pre) {
    const int lim = rg.k_hi - (rg.k_lo + j * BN + hf * 64);
    if (lim < 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = (c < lim) ? v[c] : -INFINITY;
    }
  } else {
    // nodes 64q .. 64q+63, q < 4 as N <= 256; selects rather than a run-time
    // index keep am[] in registers
    const int q = 2 * (j - rg.n_pre) + hf;
    const uint32_t w0 = q == 0 ? am[0] : q == 1 ? am[2] : q == 2 ? am[4] : am[6];
    const uint32_t w1 = q == 0 ? am[1] : q == 1 ? am[3] : q == 2 ? am[5] : am[7];
    const int nvalid = N - q * 64;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      const uint32_t word = c < 32 ? w0 : w1;
      const bool vis = c < nvalid && ((word >> (c & 31)) & 1u);
      v[c] = vis ? v[c] : -INFINITY;
    }
  }
}

// P = 2^(qscale * s - m) for the 64 scores of one key half, packed as bf16
// pairs (pk[c] holds keys 2c, 2c+1); returns their fp32 sum.  kMasked: the
// half holds masked (-inf) scores, so every exponential goes to MUFU ex2,
// which gives exactly 0 there; otherwise one pair in four is taken on the
// FMA pipe (polynomial), which would give 2^-126 for -inf.
template <bool kMasked>
__device__ __forceinline__ float exp_pack64(const float (&v)[64], unsigned long long q2,
                                            unsigned long long m2, uint32_t (&pk)[32]) {
  unsigned long long sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c2 = 0; c2 < 32; ++c2) {
    float x0, x1, e0, e1;
    f2_unpack(f2_fma(f2_pack(v[2 * c2], v[2 * c2 + 1]), q2, m2), x0, x1);
    if (!kMasked && (c2 & 3) == 3) {
      exp2_fma2(x0, x1, e0, e1);
    } else {
      e0 = ex2_approx(x0);
      e1 = ex2_approx(x1);
    }
    sum2[c2 & 3] = f2_add(sum2[c2 & 3], f2_pack(e0, e1));
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(e0, e1);
    pk[c2] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  float a0, a1, b0, b1, c0f, c1f, d0, d1;
  f2_unpack(sum2[0], a0, a1);
  f2_unpack(sum2[1], b0, b1);
  f2_unpack(sum2[2], c0f, c1f);
  f2_unpack(sum2[3], d0, d1);
  return ((a0 + a1) + (b0 + b1)) + ((c0f + c1f) + (d0 + d1));
}

// True when the 64-key half hf of key tile j has masked columns: a tree
// tile, or the prefix tile that ends the chunk inside this half.
__device__ __forceinline__ bool half_masked(int j, int hf, const Range& rg) {
  return j >= rg.n_pre || rg.k_hi - (rg.k_lo + j * BN + hf * 64) < 64;
}

// First cache slot of key tile j (prefix tiles from the chunk start, then the
// tree tiles from slot L_b).
__device__ __forceinline__ int tile_key0(int j, int Lb, const Range& rg) {
  return j < rg.n_pre ? rg.k_lo + j * BN : Lb + (j - rg.n_pre) * BN;
}

// Zeroes rows [row0, BN) of a staged 128-key V tile (both 64-column halves;
// the 128-byte swizzle permutes 16-byte pieces within a row, so a whole row
// stays at bytes [128 row, 128 row + 128) of each half).  Those rows hold
// cache slots >= L_b + N, which the caller never has to write: their
// attention weight is exactly 0, and zero rows keep 0 * (NaN or Inf) out of
// the P.V product.  nthr threads, index i; the caller orders the stores
// before the tensor core's reads (proxy fence, then barrier).
__device__ __forceinline__ void zero_v_rows(uint8_t* tile, int row0, int i, int nthr) {
  const int n = (BN - row0) * 16;  // 16-byte pieces: 8 per row and half
  for (int e = i; e < n; e += nthr) {
    const int row = row0 + (e >> 4), pc = e & 15;
    *reinterpret_cast<uint4*>(tile + (pc >> 3) * HALF + row * 128 + (pc & 7) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

// bf16 bits of x rounded toward +inf (so the rounded value is >= x).
__device__ __forceinline__ uint32_t bf16_bits_up(float x) {
  uint32_t u = __float_as_uint(x);
  if (!(u & 0x80000000u)) u += 0xFFFFu;  // non-negative: away from zero
  return u >> 16;                          // negative: toward zero
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

// Merge of the P chunks of query tile qt of (sequence b, kv-head kvh) by the
// cluster they form (rank = chunk): every rank has staged its unnormalised O
// rows (so, row stride OST) and their (max, sum) in base 2 (sml; max = -inf:
// no visible key in that chunk) in its own shared memory.  Rank c takes rows
// [c per, (c+1) per) of the tile, one warp per row: the row max M over the
// chunks, weights 2^(m_c - M), and out = sum_c w_c O_c / sum_c w_c l_c as
// bf16 (0 for a row that sees no key).  Every thread of every rank calls it
// exactly once.
__device__ __forceinline__ void cluster_merge(float* so, float2* sml, int qt, int b, int kvh, int P,
                                              int R, int G, int N, int Hq,
                                              __nv_bfloat16* __restrict__ out) {
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();  // every rank's partial rows are in its shared memory
  const int rank = (int)cl.block_rank();
  const int live = min(BM, R - qt * BM);
  const int per = (live + P - 1) / P;
  const int r0 = rank * per, r1 = min(live, r0 + per);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = r0 + warp; r < r1; r += kThreads / 32) {
    const float2 ml = lane < P ? cl.map_shared_rank(sml, lane)[r] : make_float2(-INFINITY, 0.f);
    float M = ml.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w = (lane < P && ml.x != -INFINITY) ? exp2f(ml.x - M) : 0.f;
    float Ls = w * ml.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < P; ++c) {
      const float wc = __shfl_sync(0xffffffffu, w, c);
      if (wc != 0.f) {
        const float4 o = reinterpret_cast<const float4*>(cl.map_shared_rank(so, c) + (size_t)r * OST)[lane];
        acc.x = fmaf(wc, o.x, acc.x);
        acc.y = fmaf(wc, o.y, acc.y);
        acc.z = fmaf(wc, o.z, acc.z);
        acc.w = fmaf(wc, o.w, acc.w);
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    const int grow = qt * BM + r;
    const int node = grow / G, g = grow - node * G;
    __nv_bfloat16* dst = out + (((size_t)b * N + node) * Hq + (size_t)kvh * G + g) * DH + lane * 4;
    __align__(8) __nv_bfloat162 h[2] = {__floats2bfloat162_rn(acc.x * inv, acc.y * inv),
                                        __floats2bfloat162_rn(acc.z * inv, acc.w * inv)};
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(h);
  }
  cl.sync();  // every rank stays resident until the others have read its rows
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

  griddep_wait();  // prefix lengths and the K/V cache may come from the kernel ahead
  const int qt = blockIdx.x, chunk = blockIdx.y, bk = blockIdx.z;
  const int rank = bk / p.Hkv, kvh = bk - rank * p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* sQ = sm;
  uint8_t* sK = sm + TILE;
  uint8_t* sV = sK + kStages * TILE;
  uint64_t* bars = (uint64_t*)(sm + kDataBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;              // [kStages]
  uint64_t* k_empty = k_full + kStages;     // [kStages]
  uint64_t* v_full = k_empty + kStages;     // [kStages]
  uint64_t* v_empty = v_full + kStages;     // [kStages]
  uint64_t* s_full = v_empty + kStages;     // [S/P buffer]
  uint64_t* p_full = s_full + 3;            // [S/P buffer]
  uint64_t* pv_done = p_full + 3;           // [S/P buffer]
  uint64_t* mma_done = pv_done + 3;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* seq_slot = (int*)(tmem_slot + 2);
  // [tile parity][key half][row]: each half's tile row max, bf16 rounded up
  uint16_t* xch = (uint16_t*)(sm + kDataBytes + 256);

  // Sequence of this CTA: the one of rank `rank` by decreasing prefix length
  // (ties: lower index first).  Every CTA ranks the B lengths itself (one
  // thread per sequence); beyond kThreads sequences the order is the index.
  int b = rank;
  if (p.B > 1 && p.B <= kThreads) {
    if ((int)threadIdx.x < p.B) {
      const int i = threadIdx.x;
      const int li = p.L[i];
      int r = 0;
      for (int j = 0; j < p.B; ++j) {
        const int lj = p.L[j];
        r += (lj > li || (lj == li && j < i)) ? 1 : 0;
      }
      if (r == rank) *seq_slot = i;
    }
    __syncthreads();
    b = *seq_slot;
  }

  const int Lb = p.L[b];
  const bool seq_ok = Lb >= 0 && (long long)Lb + p.N <= p.Lcap;
  const Range rg = chunk_range(p, Lb, chunk, seq_ok);
  const int T = rg.n_pre + rg.n_tree;

  if (T == 0) {  // nothing to attend to in this chunk
    if (p.fuse) {
      float2* sml = (float2*)(sm + TILE + kOStage);
      if (threadIdx.x < BM) sml[threadIdx.x] = make_float2(-INFINITY, 0.f);
      griddep_launch_dependents();
      cluster_merge((float*)(sm + TILE), sml, qt, b, kvh, p.P, p.R, p.G, p.N, p.Hq, p.out);
      return;
    }
    if (threadIdx.x < BM) {
      const int grow = qt * BM + threadIdx.x;
      if (grow < p.R) write_row<DH>(p, b, kvh, chunk, grow, 0, -INFINITY, 0.f, nullptr, true);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);  // every softmax warp
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, 512);  // S/P 0 | S/P 1 | S/P 2 | O
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();  // TMEM taken: the next kernel may be scheduled

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------------- TMA producers
    // warp 0: the Q tile then the K ring; warp 10: the V ring
    if (lane == 0) {
      const bool isK = warp == 0;
      const uint64_t pol = policy_evict_normal();
      if (isK) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        mbar_arrive_expect_tx(q_full, TILE);
        const int zq = b * p.N + qt * (BM / p.G);
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
        const int st = j % kStages;
        const int key0 = j < rg.n_pre ? rg.k_lo + j * BN : Lb + (j - rg.n_pre) * BN;
        dbg_ok(key0 >= 0 && key0 < Lb + p.N && key0 < p.Lcap, DBG_ATTN_KEY_TILE);
        const int z = b * p.Lcap + key0;
        if (!mbar_wait(&emp[st], ((uint32_t)(j / kStages) & 1u) ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&ful[st], TILE);
        tma_load_3d(buf + st * TILE, map, &ful[st], 0, kvh, z, pol);
        tma_load_3d(buf + st * TILE + HALF, map, &ful[st], 64, kvh, z, pol);
        issued = j + 1;
      }
      if (issued < T) {
        // aborted: let the loads already issued land before the CTA exits
        if (isK) mbar_wait(q_full, 0u, nullptr);
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          mbar_wait(&ful[j % kStages], (uint32_t)(j / kStages) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // S(0), S(1), then for u = 0, 1, ...: P.V(u), S(u + 2).  S(u+2) reuses
    // the S/P buffer of tile u-1, whose P.V was issued one step earlier and
    // has normally completed by then, so the tensor pipe is not left idle
    // waiting for a completion; S still runs a tile ahead of the softmax.
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16_f32(BM, BN);
      const uint32_t idesc_o = umma_idesc_bf16_f32_bmn(BM, DH);
      // descriptors of the tile bases; a K step adds its byte offset / 16 to
      // the start-address field (no carry: shared addresses are < 2^18)
      const uint64_t dq = umma_desc_sw128_kmajor(smem_u32(sQ));
      const uint32_t tOacc = tmem + 384u;
      auto issue_s = [&](int t) -> bool {
        const int ks = t % kStages;
        const int bf = t % 3;
        if (!mbar_wait(&k_full[ks], (uint32_t)(t / kStages) & 1u, abort_flag)) return false;
        if (t >= 3 && !mbar_wait(&pv_done[bf], ((uint32_t)(t / 3) & 1u) ^ 1u, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dk = umma_desc_sw128_kmajor(smem_u32(sK + ks * TILE));
        const uint32_t dS = tmem + (uint32_t)bf * 128u;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * HALF + (kk & 3) * 32) >> 4);
          umma_bf16(dS, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&k_empty[ks]);
        umma_commit(&s_full[bf]);
        return true;
      };
      auto issue_pv = [&](int u) -> bool {
        const int vs = u % kStages;
        const int bf = u % 3;
        if (!mbar_wait(&p_full[bf], (uint32_t)(u / 3) & 1u, abort_flag)) return false;
        if (!mbar_wait(&v_full[vs], (uint32_t)(u / kStages) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dv = umma_desc_sw128(smem_u32(sV + vs * TILE), HALF, 1024u);
        const uint32_t aP = tmem + (uint32_t)bf * 128u;
        // keys 64 hf + 16 kk .. : P columns 32 hf + 8 kk of the buffer
        // (column c of a half holds keys 2c, 2c+1), V rows 64 hf + 16 kk
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tOacc, aP + (uint32_t)(hf * 64 + kk * 8),
                         dv + (uint64_t)((hf * 64 * 128 + kk * 16 * 128) >> 4), idesc_o,
                         (u > 0 || hf > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[vs]);
        umma_commit(&pv_done[bf]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0u, abort_flag);
      for (int t = 0; t < 2 && t < T && ok; ++t) ok = issue_s(t);
      for (int u = 0; u < T && ok; ++u) {
        ok = issue_pv(u);
        if (ok && u + 2 < T) ok = issue_s(u + 2);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    const int hf = (warp - 2) >> 2;  // key half of every tile
    const int q4 = warp & 3;         // TMEM lane quadrant of this warp (shared with its partner)
    const int r = q4 * 32 + lane;
    const int grow = qt * BM + r;
    const bool row_ok = grow < p.R;
    const bool warp_live = (qt * BM + q4 * 32) < p.R;  // warp-uniform, same for both partners
    const int node = min(grow / p.G, p.N - 1);
    uint32_t am[MEDUSA_MAX_N / 32];
#pragma unroll
    for (int w = 0; w < MEDUSA_MAX_N / 32; ++w) am[w] = (w < p.W) ? p.anc[(size_t)node * p.W + w] : 0u;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_base + 384u + (uint32_t)hf * 64u;  // this half's O columns
    const unsigned long long q2 = f2_pack(p.qscale, p.qscale);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // Every exit from the tile loop follows a pair barrier whose result is
    // the OR of both partners' error flags, so neither is left waiting.
    bool err = false;
    for (int t = 0; t < T; ++t) {
      const int bf = t % 3;
      const uint32_t tS = tmem + lane_base + (uint32_t)(bf * 128 + hf * 64);
      const bool good = mbar_wait(&s_full[bf], (uint32_t)(t / 3) & 1u, abort_flag);
      err = err || !__all_sync(0xffffffffu, good);
      // V rows of cache slots >= L_b + N in this tile (the tree tiles and the
      // prefix tile that ends the sequence): zeroed by the 256 softmax
      // threads once the tile has landed, before P(t) is released to P.V(t)
      const int zrow = Lb + p.N - tile_key0(t, Lb, rg);
      if (zrow < BN && !err) {
        const int vs = t % kStages;
        const bool vg = mbar_wait(&v_full[vs], (uint32_t)(t / kStages) & 1u, abort_flag);
        if (__all_sync(0xffffffffu, vg)) {
          zero_v_rows(sV + vs * TILE, zrow, (int)threadIdx.x - 64, 256);
          fence_proxy_async_smem();
        } else {
          err = true;
        }
      }
      float v[64];
      float tmax = -INFINITY;
      // Both halves of a row use max(round_up(max_0), round_up(max_1)): the
      // same value in both, and an upper bound of the row's tile max.  The
      // parity double buffer is free again two barriers later.
      uint16_t* xrow = xch + (size_t)(t & 1) * 2 * BM + r;
      if (!err && warp_live) {
        tc_fence_after();
        tmem_ld64(tS, v);
        mask_half(v, t, hf, rg, p.N, am);
        const uint32_t mine = bf16_bits_up(max64(v) * p.qscale);  // scale > 0
        tmax = __uint_as_float(mine << 16);
        xrow[hf * BM] = (uint16_t)mine;
      }
      if (bar_red_or(3 + q4, 64, err)) {
        ok = false;
        break;
      }
      if (!warp_live) {
        // rows past the last query row: keep the protocol, skip the work
        // (O rows are independent of each other, these are never output)
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[bf]);
        continue;
      }
      tmax = fmaxf(tmax, __uint_as_float((uint32_t)xrow[(hf ^ 1) * BM] << 16));
      const bool grow_m = tmax > m_used + kRescale;  // the same in both partners
      // warp-uniform branch: the TMEM accesses and the vote are collective
      if (__any_sync(0xffffffffu, grow_m)) {
        float corr = 1.f;
        if (grow_m) {
          corr = ex2_approx(m_used - tmax);  // 0 when m_used is -inf
          m_used = tmax;
          l *= corr;
        }
        if (t > 0) {
          // O must hold every P.V so far: wait for P.V(t-1)
          const bool w_ok = mbar_wait(&pv_done[(t - 1) % 3], (uint32_t)((t - 1) / 3) & 1u, abort_flag);
          if (__all_sync(0xffffffffu, w_ok)) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 16) {
              float o16[16];
              tmem_ld16(tO + c0, o16);
#pragma unroll
              for (int e = 0; e < 16; ++e) o16[e] *= corr;
              tmem_st16(tO + c0, o16);
            }
          } else {
            err = true;  // reported at the next pair barrier (or the final one)
          }
        }
      }
      // P = 2^(scale*s - m) in packed pairs (a row with no visible key yet
      // has m = -inf and only -inf scores, whose exponentials are zeroed)
      const float moff = (m_used == -INFINITY) ? 0.f : m_used;
      const unsigned long long m2 = f2_pack(-moff, -moff);
      uint32_t pk[32];
      // masked keys get exactly 0 (all-MUFU exponentials on masked halves)
      l += half_masked(t, hf, rg) ? exp_pack64<true>(v, q2, m2, pk)
                                  : exp_pack64<false>(v, q2, m2, pk);
      tmem_st32(tS, pk);  // P over the S columns just read
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[bf]);
    }
    ok = ok && !err;
    // last P.V complete (it commits after every earlier MMA)
    if (ok && warp_live) {
      const bool good = mbar_wait(&pv_done[(T - 1) % 3], (uint32_t)((T - 1) / 3) & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, good);
    }
    // row sum = both halves' partial sums: each publishes its own in column
    // hf of S/P buffer 0 (free now), then finishes its 64 output columns
    if (ok && warp_live) {
      tmem_st1(tmem + lane_base + (uint32_t)hf, l);
      tc_fence_before();
    }
    const bool bad = bar_red_or(2, 256, !ok || *abort_flag);
    if (p.fuse) {
      // stage this chunk's rows for the cluster merge: every MMA has completed
      // and every K/V load has landed, so the rings are free
      float* so = (float*)sK;
      float2* sml = (float2*)(sK + kOStage);
      const bool have = !bad && warp_live && row_ok && m_used != -INFINITY;
      float Ls = 0.f;
      if (!bad && warp_live) {
        tc_fence_after();
        Ls = l + tmem_ld1(tmem + lane_base + (uint32_t)(hf ^ 1));
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float a[32];
          tmem_ld32(tO + (uint32_t)c0, a);
          if (have) {
            float4* dst = reinterpret_cast<float4*>(so + (size_t)r * OST + hf * 64 + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(a[4 * e], a[4 * e + 1], a[4 * e + 2], a[4 * e + 3]);
          }
        }
      }
      if (hf == 0) sml[r] = have ? make_float2(m_used, Ls) : make_float2(-INFINITY, 0.f);
    } else if (!bad && warp_live) {
      tc_fence_after();
      const float Ls = l + tmem_ld1(tmem + lane_base + (uint32_t)(hf ^ 1));
      const int cb = hf * 64;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        float a[32];
        tmem_ld32(tO + (uint32_t)c0, a);
        if (row_ok) {
          if (m_used == -INFINITY)
            write_row<32>(p, b, kvh, chunk, grow, cb + c0, m_used, Ls, nullptr, hf == 0 && c0 == 0);
          else
            write_row<32>(p, b, kvh, chunk, grow, cb + c0, m_used, Ls, a, hf == 0 && c0 == 0);
        }
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
  if (p.fuse)
    cluster_merge((float*)sK, (float2*)(sK + kOStage), qt, b, kvh, p.P, p.R, p.G, p.N, p.Hq,
                  p.out);
}

// ---------------------------------------------------------------------------
// Two query tiles per CTA.  With at least two 128-row query tiles per
// (sequence, kv-head), a CTA takes tiles 2x and 2x+1 (the second may lie
// past the last row: computed, never written) and one key chunk, and both
// tiles read every K/V tile it stages.  With more than one chunk the chunks
// of a pair form a cluster and merge both tiles' rows in it, as
// tree_attn_tc_kernel's chunks do.  TMEM: S/P of tile a | S/P of tile b | O of a | O of b.
// One softmax warpgroup per tile, so each works on its tile while the
// tensor pipe runs the other tile's MMAs.  S_q(t) reuses the S/P columns of
// tile q, so it waits for P.V_q(t-1).
constexpr int kPairKStages = 3, kPairVStages = 2;
constexpr size_t kPairData = (2 + kPairKStages + kPairVStages) * (size_t)TILE;
constexpr size_t SMEM_PAIR = 1024 + kPairData + 256;
static_assert(2 * kOStage + 2 * BM * sizeof(float2) <=
                  (kPairKStages + kPairVStages) * (size_t)TILE,
              "both tiles' staged O rows and (max, sum) fit in the K/V rings");
static_assert(SMEM_PAIR <= 227 * 1024, "shared memory of the two-tile kernel");

// mask_half with the ancestor words of the row's node read from memory (two
// words, only for the tree tiles), so the kernel keeps no per-tile word sets
// in registers.
__device__ __forceinline__ void mask_half_mem(float (&v)[64], int j, int hf, const Range& rg,
                                              int N, int W, const uint32_t* __restrict__ anc_row) {
  if (j < rg.n_pre) {
    const int lim = rg.k_hi - (rg.k_lo + j * BN + hf * 64);
    if (lim < 64) {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = (c < lim) ? v[c] : -INFINITY;
    }
  } else {
    const int q = 2 * (j - rg.n_pre) + hf;  // nodes 64q .. 64q+63
    const uint32_t w0 = (2 * q < W) ? __ldg(anc_row + 2 * q) : 0u;
    const uint32_t w1 = (2 * q + 1 < W) ? __ldg(anc_row + 2 * q + 1) : 0u;
    const int nvalid = N - q * 64;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      const uint32_t word = c < 32 ? w0 : w1;
      const bool vis = c < nvalid && ((word >> (c & 31)) & 1u);
      v[c] = vis ? v[c] : -INFINITY;
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_tc_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                             const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV, const TcAttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

  griddep_wait();  // prefix lengths and the K/V cache may come from the kernel ahead
  const int qpair = blockIdx.x, chunk = blockIdx.y, bk = blockIdx.z;
  const int rank = bk / p.Hkv, kvh = bk - rank * p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* sQ = sm;  // tile a | tile b
  uint8_t* sK = sm + 2 * TILE;
  uint8_t* sV = sK + kPairKStages * TILE;
  uint64_t* bars = (uint64_t*)(sm + kPairData);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                  // [kPairKStages]
  uint64_t* k_empty = k_full + kPairKStages;    // [kPairKStages]
  uint64_t* v_full = k_empty + kPairKStages;    // [kPairVStages]
  uint64_t* v_empty = v_full + kPairVStages;    // [kPairVStages]
  uint64_t* s_full = v_empty + kPairVStages;    // [tile]
  uint64_t* p_full = s_full + 2;                // [tile]
  uint64_t* pv_done = p_full + 2;               // [tile]
  uint64_t* mma_done = pv_done + 2;
  uint32_t* tmem_slot = (uint32_t*)(mma_done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  int* seq_slot = (int*)(tmem_slot + 2);

  int b = rank;  // longest prefix first, as in tree_attn_tc_kernel
  if (p.B > 1 && p.B <= kThreads) {
    if ((int)threadIdx.x < p.B) {
      const int i = threadIdx.x;
      const int li = p.L[i];
      int r = 0;
      for (int j = 0; j < p.B; ++j) {
        const int lj = p.L[j];
        r += (lj > li || (lj == li && j < i)) ? 1 : 0;
      }
      if (r == rank) *seq_slot = i;
    }
    __syncthreads();
    b = *seq_slot;
  }

  const int Lb = p.L[b];
  const bool seq_ok = Lb >= 0 && (long long)Lb + p.N <= p.Lcap;
  const Range rg = chunk_range(p, Lb, chunk, seq_ok);
  const int T = rg.n_pre + rg.n_tree;
  const int qt0 = 2 * qpair;  // tile a; tile b = qt0 + 1
  const bool b_rows = (qt0 + 1) * BM < p.R;  // tile b has rows to write (uniform in a cluster)
  // in-cluster merge: staged O rows of tile q at so + q BM OST, (max, sum) at sml + q BM
  float* so = (float*)(sm + 2 * TILE);
  float2* sml = (float2*)(sm + 2 * TILE + 2 * kOStage);

  if (T == 0) {
    if (p.fuse) {  // a chunk with no key: (-inf, 0) for every row of both tiles
      if (threadIdx.x < 2 * BM) sml[threadIdx.x] = make_float2(-INFINITY, 0.f);
      griddep_launch_dependents();
      cluster_merge(so, sml, qt0, b, kvh, p.P, p.R, p.G, p.N, p.Hq, p.out);
      if (b_rows) cluster_merge(so + BM * OST, sml + BM, qt0 + 1, b, kvh, p.P, p.R, p.G, p.N, p.Hq, p.out);
      return;
    }
    for (int q = 0; q < 2; ++q) {
      const int grow = (qt0 + q) * BM + (int)threadIdx.x;
      if ((int)threadIdx.x < BM && grow < p.R)
        write_row<DH>(p, b, kvh, 0, grow, 0, -INFINITY, 0.f, nullptr, true);
    }
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kPairKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kPairVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);  // the tile's softmax warps
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    __syncwarp();
    tmem_alloc(tmem_slot, 512);  // S/P a | S/P b | O a | O b
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();  // TMEM taken: the next kernel may be scheduled

  if (warp == 0 || warp == kVWarp) {
    // ---------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const bool isK = warp == 0;
      const uint64_t pol = policy_evict_normal();
      if (isK) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        mbar_arrive_expect_tx(q_full, 2 * TILE);
        for (int q = 0; q < 2; ++q) {
          // rows past the tensor's end read as zero; rows of the next
          // sequence in tile b of the last pair are computed, never written
          const int zq = b * p.N + (qt0 + q) * (BM / p.G);
          tma_load_3d(sQ + q * TILE, &tmQ, q_full, 0, kvh * p.G, zq, pol);
          tma_load_3d(sQ + q * TILE + HALF, &tmQ, q_full, 64, kvh * p.G, zq, pol);
        }
      } else {
        prefetch_tmap(&tmV);
      }
      const int stages = isK ? kPairKStages : kPairVStages;
      const CUtensorMap* map = isK ? &tmK : &tmV;
      uint64_t* emp = isK ? k_empty : v_empty;
      uint64_t* ful = isK ? k_full : v_full;
      uint8_t* buf = isK ? sK : sV;
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int st = j % stages;
        const int key0 = j < rg.n_pre ? rg.k_lo + j * BN : Lb + (j - rg.n_pre) * BN;
        dbg_ok(key0 >= 0 && key0 < Lb + p.N && key0 < p.Lcap, DBG_ATTN_KEY_TILE);
        const int z = b * p.Lcap + key0;
        if (!mbar_wait(&emp[st], ((uint32_t)(j / stages) & 1u) ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&ful[st], TILE);
        tma_load_3d(buf + st * TILE, map, &ful[st], 0, kvh, z, pol);
        tma_load_3d(buf + st * TILE + HALF, map, &ful[st], 64, kvh, z, pol);
        issued = j + 1;
      }
      if (issued < T) {
        // aborted: let the loads already issued land before the CTA exits
        if (isK) mbar_wait(q_full, 0u, nullptr);
        for (int j = (issued > stages ? issued - stages : 0); j < issued; ++j)
          mbar_wait(&ful[j % stages], (uint32_t)(j / stages) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_bf16_f32(BM, BN);
      const uint32_t idesc_o = umma_idesc_bf16_f32_bmn(BM, DH);
      auto issue_s = [&](int t, int q) -> bool {
        const int ks = t % kPairKStages;
        if (q == 0 && !mbar_wait(&k_full[ks], (uint32_t)(t / kPairKStages) & 1u, abort_flag))
          return false;
        // the S/P columns of tile q hold P_q(t-1) until its P.V has run
        if (t > 0 && !mbar_wait(&pv_done[q], (uint32_t)(t - 1) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint64_t dq = umma_desc_sw128_kmajor(smem_u32(sQ + q * TILE));
        const uint64_t dk = umma_desc_sw128_kmajor(smem_u32(sK + ks * TILE));
        const uint32_t dS = tmem + (uint32_t)q * 128u;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * HALF + (kk & 3) * 32) >> 4);
          umma_bf16(dS, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        if (q == 1) umma_commit(&k_empty[ks]);  // both tiles have read K(t)
        umma_commit(&s_full[q]);
        return true;
      };
      auto issue_pv = [&](int u, int q) -> bool {
        const int vs = u % kPairVStages;
        if (!mbar_wait(&p_full[q], (uint32_t)u & 1u, abort_flag)) return false;
        if (q == 0 && !mbar_wait(&v_full[vs], (uint32_t)(u / kPairVStages) & 1u, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t dv = umma_desc_sw128(smem_u32(sV + vs * TILE), HALF, 1024u);
        const uint32_t aP = tmem + (uint32_t)q * 128u;
        const uint32_t tOq = tmem + 256u + (uint32_t)q * 128u;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tOq, aP + (uint32_t)(hf * 64 + kk * 8),
                         dv + (uint64_t)((hf * 64 * 128 + kk * 16 * 128) >> 4), idesc_o,
                         (u > 0 || hf > 0 || kk > 0) ? 1u : 0u);
        if (q == 1) umma_commit(&v_empty[vs]);  // both tiles have read V(u)
        umma_commit(&pv_done[q]);
        return true;
      };
      // S_a(0), S_b(0), then per key tile t: P.V_a(t), S_a(t+1), P.V_b(t),
      // S_b(t+1): each tile's next S follows its own P.V, so one tile's
      // chain (S, softmax, P.V) never waits for the other tile's softmax
      bool ok = mbar_wait(q_full, 0u, abort_flag) && issue_s(0, 0) && issue_s(0, 1);
      for (int t = 0; t < T && ok; ++t) {
        ok = issue_pv(t, 0);
        if (ok && t + 1 < T) ok = issue_s(t + 1, 0);
        if (ok) ok = issue_pv(t, 1);
        if (ok && t + 1 < T) ok = issue_s(t + 1, 1);
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0u, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- softmax warpgroups
    // warps 2-5: tile a, warps 6-9: tile b; a thread owns one query row and
    // all 128 keys of every key tile, taken as two 64-key halves under one
    // running max (lazy rescaling as in tree_attn_tc_kernel).  When the
    // second half raises the max, the first half's P (already in TMEM) is
    // rescaled with O.
    const int q = (warp - 2) >> 2;  // query tile of this warpgroup
    const int q4 = warp & 3;        // TMEM lane quadrant
    const int r = q4 * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)q * 128u;
    const uint32_t tO = tmem + lane_base + 256u + (uint32_t)q * 128u;
    const unsigned long long q2 = f2_pack(p.qscale, p.qscale);
    const int grow = (qt0 + q) * BM + r;
    const bool row_ok = grow < p.R;
    const bool live = ((qt0 + q) * BM + q4 * 32) < p.R;  // warp-uniform
    const uint32_t* anc_row = p.anc + (size_t)min(grow / p.G, p.N - 1) * p.W;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // Raises the running max to tmax when it grew by more than 2^kRescale:
    // rescales l, the O row (after P.V(t-1)) and, for the second half, the
    // first half's P.  Warp-collective (TMEM accesses): every lane calls it.
    auto maybe_rescale = [&](float tmax, int t, bool p_half0) -> bool {
      const bool grow_m = tmax > m_used + kRescale;
      if (!__any_sync(0xffffffffu, grow_m)) return true;
      float corr = 1.f;
      if (grow_m) {
        corr = ex2_approx(m_used - tmax);  // 0 when m_used is -inf
        m_used = tmax;
        l *= corr;
      }
      if (t > 0) {
        const bool w_ok = mbar_wait(&pv_done[q], (uint32_t)(t - 1) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < DH; c0 += 16) {
          float o16[16];
          tmem_ld16(tO + (uint32_t)c0, o16);
#pragma unroll
          for (int e = 0; e < 16; ++e) o16[e] *= corr;
          tmem_st16(tO + (uint32_t)c0, o16);
        }
      }
      if (p_half0) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < 32; c0 += 16) {
          float w16[16];
          tmem_ld16(tS + (uint32_t)c0, w16);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&w16[e]);
            const float2 f = __bfloat1622float2(h2);
            h2 = __floats2bfloat162_rn(f.x * corr, f.y * corr);
            w16[e] = *reinterpret_cast<const float*>(&h2);
          }
          tmem_st16(tS + (uint32_t)c0, w16);
        }
      }
      return true;
    };
    for (int t = 0; t < T && ok; ++t) {
      const bool good = mbar_wait(&s_full[q], (uint32_t)t & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, good)) {
        ok = false;
        break;
      }
      // V rows of cache slots >= L_b + N in this tile: zeroed by tile a's
      // warpgroup before P_a(t) is released; the MMA thread issues P.V_b(t)
      // after P.V_a(t), so both products read the zeroed rows
      const int zrow = Lb + p.N - tile_key0(t, Lb, rg);
      if (q == 0 && zrow < BN) {
        const int vs = t % kPairVStages;
        const bool vg = mbar_wait(&v_full[vs], (uint32_t)(t / kPairVStages) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, vg)) {
          ok = false;
          break;
        }
        zero_v_rows(sV + vs * TILE, zrow, (int)threadIdx.x - 64, 128);
        fence_proxy_async_smem();
      }
      if (live) {
#pragma unroll 1
        for (int hf = 0; hf < 2 && ok; ++hf) {
          float v[64];
          tc_fence_after();
          tmem_ld64(tS + (uint32_t)(hf * 64), v);
          mask_half_mem(v, t, hf, rg, p.N, p.W, anc_row);
          if (!maybe_rescale(max64(v) * p.qscale, t, hf == 1)) {
            ok = false;
            break;
          }
          // P = 2^(scale*s - m) in packed pairs (a row with no visible key
          // yet has m = -inf and only -inf scores, whose exponentials are zeroed)
          const float moff = (m_used == -INFINITY) ? 0.f : m_used;
          const unsigned long long m2 = f2_pack(-moff, -moff);
          uint32_t pk[32];
          // masked keys get exactly 0 (all-MUFU exponentials on masked halves)
          l += half_masked(t, hf, rg) ? exp_pack64<true>(v, q2, m2, pk)
                                      : exp_pack64<false>(v, q2, m2, pk);
          tmem_st32(tS + (uint32_t)(hf * 64), pk);  // P over the S columns just read
        }
        if (!ok) break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[q]);
    }
    // this tile's last P.V complete
    if (ok && live) {
      const bool good = mbar_wait(&pv_done[q], (uint32_t)(T - 1) & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, good);
    }
    const bool bad = bar_red_or(2, 256, !ok || *abort_flag);
    if (p.fuse) {
      // stage this chunk's rows for the cluster merge: every MMA has completed
      // and every K/V load has landed, so the rings are free
      const bool have = !bad && live && row_ok && m_used != -INFINITY;
      if (!bad && live) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < DH; c0 += 32) {
          float a[32];
          tmem_ld32(tO + (uint32_t)c0, a);
          if (have) {
            float4* dst = reinterpret_cast<float4*>(so + ((size_t)q * BM + r) * OST + c0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(a[4 * e], a[4 * e + 1], a[4 * e + 2], a[4 * e + 3]);
          }
        }
      }
      sml[q * BM + r] = have ? make_float2(m_used, l) : make_float2(-INFINITY, 0.f);
    } else if (!bad && live) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < DH; c0 += 32) {
        float a[32];
        tmem_ld32(tO + (uint32_t)c0, a);
        if (row_ok) {
          if (m_used == -INFINITY)
            write_row<32>(p, b, kvh, 0, grow, c0, m_used, l, nullptr, c0 == 0);
          else
            write_row<32>(p, b, kvh, 0, grow, c0, m_used, l, a, c0 == 0);
        }
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
  if (p.fuse) {
    cluster_merge(so, sml, qt0, b, kvh, p.P, p.R, p.G, p.N, p.Hq, p.out);
    if (b_rows) cluster_merge(so + BM * OST, sml + BM, qt0 + 1, b, kvh, p.P, p.R, p.G, p.N, p.Hq, p.out);
  }
}

std::atomic<bool> g_smem_attr[64];  // per device: the kernel's shared-memory limit raised
std::atomic<bool> g_smem_attr_pair[64];

// Clusters of P CTAs of the one-tile (pair = false) or two-tile kernel that
// can be resident at once on the current device (0 when the query fails),
// cached per device, kernel and P.
int max_active_clusters(bool pair, int P) {
  static std::atomic<int> cache[2][64][kMaxClusterChunks + 1];
  int dev = 0;
  if (P < 1 || P > kMaxClusterChunks || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 0;
  }
  const int v = cache[pair][dev][P].load(std::memory_order_relaxed);
  if (v) return v - 1;
  const void* fn = pair ? (const void*)tree_attn_tc_pair_kernel : (const void*)tree_attn_tc_kernel;
  const size_t smem = pair ? SMEM_PAIR : SMEM;
  if (pair ? ensure_max_smem(tree_attn_tc_pair_kernel, (int)SMEM_PAIR, g_smem_attr_pair,
                             "cudaFuncSetAttribute(tree_attn_tc_pair_kernel)")
           : ensure_max_smem(tree_attn_tc_kernel, (int)SMEM, g_smem_attr,
                             "cudaFuncSetAttribute(tree_attn_tc_kernel)"))
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, P, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = P;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();  // not an error of the caller's stream: no in-cluster merge
    return 0;
  }
  cache[pair][dev][P].store(n + 1, std::memory_order_relaxed);
  return n;
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
  if (units <= 0) return 1;  // empty batch: nothing to split
  const int sms = num_sms();
  long long P = (2LL * sms + units - 1) / units;
  const long long max_p = ((long long)(Lcap - N) + 4 * BN - 1) / (4 * BN);  // >= 4 tiles each
  if (P > max_p) P = max_p;
  if (P < 1) P = 1;
  return (int)P;
}

TcShape attention_tc_shape(int B, int Hq, int Hkv, int N, int Lcap) {
  TcShape sh;
  sh.P = attention_tc_chunks(B, Hq, Hkv, N, Lcap);
  sh.tiles = 1;
  sh.fuse = false;
  if (B <= 0) return sh;
  const long long R = (long long)N * (Hq / Hkv);
  const long long mtiles = (R + BM - 1) / BM;
  const long long units = (long long)B * Hkv * mtiles;
  if (sh.P >= 2 && sh.P <= kMaxClusterChunks) {
    // the chunks of a query tile merge in-cluster when every cluster fits at once
    const int n = max_active_clusters(false, sh.P);
    sh.fuse = n > 0 && units <= n;
  }
  if (mtiles < 2) return sh;
  // Cost in (waves of CTAs) x (key tiles per CTA).  A CTA with two query
  // tiles takes about 1.8 times as long per key tile as a CTA with one
  // (measured on the 8B-GQA and long-context shapes: 2.32-2.35 us against
  // 1.29-1.34 us).  Two-tile plans split the keys into P2 chunks only where
  // the chunks can merge in-cluster.
  const long long sms = num_sms();
  const long long T = (Lcap - N + BN - 1) / BN + (N + BN - 1) / BN;
  const long long cost1 = ((units * sh.P + sms - 1) / sms) * ((T + sh.P - 1) / sh.P);
  const long long pairs = (long long)B * Hkv * ((mtiles + 1) / 2);
  const long long max_p = ((long long)(Lcap - N) + 4 * BN - 1) / (4 * BN);  // >= 4 tiles each
  long long best = cost1 * 10;
  int bestP = 0;
  for (int P2 = 1; P2 <= 4; P2 *= 2) {
    if (P2 > 1 && P2 > max_p) break;
    long long waves;
    if (P2 == 1) {
      waves = (pairs + sms - 1) / sms;
    } else {
      const int n = max_active_clusters(true, P2);
      if (n <= 0) break;
      waves = (pairs + n - 1) / n;
    }
    const long long cost2 = 18 * waves * ((T + P2 - 1) / P2);
    if (cost2 < best) {
      best = cost2;
      bestP = P2;
    }
  }
  if (bestP > 0) {
    sh.P = bestP;
    sh.tiles = 2;
    sh.fuse = bestP > 1;
  }
  return sh;
}

int attention_tc_run(const AttnArgs& a, const TcShape& sh, float* po, float2* pml,
                     cudaStream_t st) {
  const int P = sh.P;
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
    const uint32_t box[3] = {64, 1, BN};  // 64 dh x 1 head x 128 keys
    int rc = make_tmap_bf16(&mK, a.k, 3, dims, strides, box);
    if (rc) return rc;
    rc = make_tmap_bf16(&mV, a.v, 3, dims, strides, box);
    if (rc) return rc;
  }
  int rc = ensure_max_smem(tree_attn_tc_kernel, (int)SMEM, g_smem_attr,
                           "cudaFuncSetAttribute(tree_attn_tc_kernel)");
  if (rc) return rc;
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
  p.mtiles = mtiles;
  p.fuse = (sh.fuse && P >= 2 && P <= kMaxClusterChunks) ? 1 : 0;
  p.qscale = a.scale * 1.4426950408889634f;
  p.out = (__nv_bfloat16*)a.out;
  p.po = po;
  p.pml = pml;
  cudaError_t e;
  const bool pair = sh.tiles == 2;
  if (pair && P > 1 && !p.fuse) return fail(MEDUSA_ERR_UNSUPPORTED, "two-tile plan without merge");
  if (pair) {
    rc = ensure_max_smem(tree_attn_tc_pair_kernel, (int)SMEM_PAIR, g_smem_attr_pair,
                         "cudaFuncSetAttribute(tree_attn_tc_pair_kernel)");
    if (rc) return rc;
  }
  dim3 grid(pair ? (mtiles + 1) / 2 : mtiles, P, a.B * a.Hkv);
  if (p.fuse) {
    // the P chunks of a query tile (grid y) are one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = P;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (pair) {
      cfg.dynamicSmemBytes = SMEM_PAIR;
      e = cudaLaunchKernelEx(&cfg, tree_attn_tc_pair_kernel, mQ, mK, mV, p);
    } else {
      e = cudaLaunchKernelEx(&cfg, tree_attn_tc_kernel, mQ, mK, mV, p);
    }
  } else if (pair) {
    e = launch_pdl(tree_attn_tc_pair_kernel, grid, dim3(kThreads), SMEM_PAIR, st, mQ, mK, mV, p);
  } else {
    e = launch_pdl(tree_attn_tc_kernel, grid, dim3(kThreads), SMEM, st, mQ, mK, mV, p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "tree_attn_tc_kernel launch");
}

}  // namespace medusa

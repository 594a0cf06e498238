// Acceptance of the verified tree.
//
// Medusa paper digest ("論文解説: Medusa"), section "候補選択：Typical
// Acceptance": a candidate x is accepted iff p(x) > min(eps, delta *
// exp(-H(p))), H(p) = -sum p log p; with temperature 0 the check is an argmax
// comparison.  Explainer ("メドゥーサ デコーディング ヘッド", "ディープダイブ")
// and glossary ("Medusa", "Attention en arbre"): the longest path whose
// tokens are all valid is accepted.
//
// Phase 1 (row_reduce_kernel, HBM stream): every verify row [V] is split
// into chunks; each CTA reduces its chunk to the 64-bit argmax key (value
// desc, index asc) and, for typical acceptance, the base-2 online softmax
// statistics of z = l * log2(e) / T:  m = max z, Z = sum 2^(z-m),
// S = sum 2^(z-m) (z-m).  Natural-log entropy: H = ln Z - ln2 * S / Z.
// A thread folds one 16-byte load at a time: one max per load, the first
// index recomputed only when that max improves, and the softmax statistics
// rescaled at most once per load.  -inf logits add nothing; NaN logits are
// outside the contract (they never win the argmax and add nothing).
// Phase 2 (accept_walk_kernel, one CTA per sequence, one thread per node):
// merge the chunks of the N rows, decide every node's own condition against
// its parent row,
// accept a node iff its whole root path satisfies the condition (ancestor
// bitmask test), take the deepest accepted node (ties: lowest index) and
// emit its path and the argmax of its row.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kRedThreads = 256;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;

// Per-depth scale of typical acceptance: z[D] = log2(e) / T_D for the
// candidates of depth D = 1..K (z[0] = z[1]); a row at depth d is reduced at
// the scale of its children, z[min(d + 1, K)].
struct ZTab {
  float z[MEDUSA_MAX_K + 1];
};

struct RowPart {
  uint64_t key;
  float m, Z, S, pad;
};

struct Soft {
  float m, Z, S;
};

__device__ __forceinline__ Soft soft_merge(Soft a, Soft b) {
  if (b.Z == 0.f) return a;
  if (a.Z == 0.f) return b;
  const float M = fmaxf(a.m, b.m);
  const float ta = a.m - M, tb = b.m - M;
  const float ca = exp2f(ta), cb = exp2f(tb);
  Soft r;
  r.m = M;
  r.Z = ca * a.Z + cb * b.Z;
  r.S = ca * fmaf(ta, a.Z, a.S) + cb * fmaf(tb, b.Z, b.S);
  return r;
}

// Eight bf16 or four fp32 logits of one 16-byte load, as floats.
template <typename T> struct Lanes;
template <> struct Lanes<__nv_bfloat16> {
  static constexpr int n = 8;
  static __device__ __forceinline__ void get(const uint4& w, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(u[i] << 16);
      x[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
};
template <> struct Lanes<float> {
  static constexpr int n = 4;
  static __device__ __forceinline__ void get(const uint4& w, float (&x)[4]) {
    x[0] = __uint_as_float(w.x);
    x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z);
    x[3] = __uint_as_float(w.w);
  }
};

// Running per-thread state of the row reduction: the argmax (value, first
// index) and, for typical acceptance, (m, Z, S) of z = x * zscale in base 2,
// Z and S kept as two packed fp32 lanes (even / odd columns of each load)
// so the sums run as two independent chains of f32x2 operations; folded
// into sf at the end.
struct RedState {
  float bv;
  int bi;
  Soft sf;
  unsigned long long Z2, S2;
};

__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Folds NV consecutive logits starting at column `base` (indices increase
// from call to call within a thread, so a strict > keeps the first maximum).
template <bool TYPICAL, int NV>
__device__ __forceinline__ void red_consume(RedState& st, const float (&x)[NV], int base,
                                            float zscale) {
  float vm = x[0];
#pragma unroll
  for (int j = 1; j < NV; ++j) vm = fmaxf(vm, x[j]);
  if (vm > st.bv) {
    int jj = NV - 1;
#pragma unroll
    for (int j = NV - 1; j >= 0; --j) jj = (x[j] == vm) ? j : jj;
    st.bv = vm;
    st.bi = base + jj;
  }
  if (TYPICAL) {
    const float vz = vm * zscale;  // zscale > 0: the max of the scaled values
    if (vz > st.sf.m) {
      if (st.sf.m != -INFINITY) {
        // S <- c (d Z + S), Z <- c Z on both lanes, c = 2^d (d < 0)
        const float d = st.sf.m - vz;
        const float c = ex2_approx(d);
        const unsigned long long d2 = f2_pack(d, d), c2 = f2_pack(c, c);
        st.S2 = f2_mul(c2, f2_fma(d2, st.Z2, st.S2));
        st.Z2 = f2_mul(c2, st.Z2);
      }
      st.sf.m = vz;
    }
    if (st.sf.m != -INFINITY) {  // else every value so far is -inf: nothing to add
      const unsigned long long zs2 = f2_pack(zscale, zscale);
      const unsigned long long nm2 = f2_pack(-st.sf.m, -st.sf.m);
      if constexpr (NV == 1) {  // unaligned rows: one logit at a time, on lane 0
        const float t = fmaxf(fmaf(x[0], zscale, -st.sf.m), -200.f);
        const float e = ex2_approx(t);
        st.Z2 = f2_add(st.Z2, f2_pack(e, 0.f));
        st.S2 = f2_fma(f2_pack(e, 0.f), f2_pack(t, 0.f), st.S2);
      } else {
#pragma unroll
        for (int j = 0; j + 1 < NV; j += 2) {
          // t <= 0; clamped so that a -inf (or NaN) logit adds 0 to Z and S
          float t0, t1;
          f2_unpack(f2_fma(f2_pack(x[j], x[j + 1]), zs2, nm2), t0, t1);
          t0 = fmaxf(t0, -200.f);
          t1 = fmaxf(t1, -200.f);
          const unsigned long long e2 = f2_pack(ex2_approx(t0), ex2_approx(t1));
          st.Z2 = f2_add(st.Z2, e2);
          st.S2 = f2_fma(e2, f2_pack(t0, t1), st.S2);
        }
      }
    }
  }
}

// Chunk sp of verify row `row` reduced by one CTA: the argmax key and, with
// TYPICAL, the softmax statistics at scale zscale.
template <typename T, bool TYPICAL>
__device__ __forceinline__ void row_reduce_chunk(const T* __restrict__ vlog, int V, int chunk,
                                                 int splits, float zscale, size_t row, int sp,
                                                 RowPart* __restrict__ parts) {
  const int lo = sp * chunk;
  const int hi = min(V, lo + chunk);
  const T* xr = vlog + row * (size_t)V;
  constexpr int VEC = Lanes<T>::n;
  RedState st{-INFINITY, 0x7FFFFFFF, Soft{-INFINITY, 0.f, 0.f}, 0ull, 0ull};
  const bool vec_ok = ((((uintptr_t)(xr + lo)) & 15u) == 0) && ((hi - lo) % VEC == 0);
  if (vec_ok) {
    const uint4* p = reinterpret_cast<const uint4*>(xr + lo);
    const int nv = (hi - lo) / VEC;
    // a thread whose values are all -inf reports its first column
    if ((int)threadIdx.x < nv) st.bi = lo + (int)threadIdx.x * VEC;
    // four 16-byte loads in flight per thread (enough bytes in flight per SM
    // to cover the memory latency), folded in index order
    constexpr int kUnroll = 4;
    for (int i = threadIdx.x; i < nv; i += kUnroll * kRedThreads) {
      uint4 w[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int iu = i + u * kRedThreads;
        w[u] = iu < nv ? __ldcs(p + iu) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int iu = i + u * kRedThreads;
        if (iu < nv) {
          float x[VEC];
          Lanes<T>::get(w[u], x);
          red_consume<TYPICAL, VEC>(st, x, lo + iu * VEC, zscale);
        }
      }
    }
  } else {
    if (lo + (int)threadIdx.x < hi) st.bi = lo + (int)threadIdx.x;
    for (int i = lo + threadIdx.x; i < hi; i += kRedThreads) {
      const float x[1] = {to_f32(xr[i])};
      red_consume<TYPICAL, 1>(st, x, i, zscale);
    }
  }
  uint64_t best = make_key(st.bv, (uint32_t)st.bi);
  Soft sf = st.sf;
  if (TYPICAL) {  // both lanes share sf.m
    float z0, z1, s0, s1;
    f2_unpack(st.Z2, z0, z1);
    f2_unpack(st.S2, s0, s1);
    sf.Z = z0 + z1;
    sf.S = s0 + s1;
  }
  // block reduction
  best = warp_max_u64(best);
  if (TYPICAL) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Soft other;
      other.m = __shfl_xor_sync(0xffffffffu, sf.m, o);
      other.Z = __shfl_xor_sync(0xffffffffu, sf.Z, o);
      other.S = __shfl_xor_sync(0xffffffffu, sf.S, o);
      sf = soft_merge(sf, other);
    }
  }
  __shared__ uint64_t sk[kRedThreads / 32];
  __shared__ Soft ss[kRedThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sk[warp] = best;
    ss[warp] = sf;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kRedThreads / 32; ++w) {
      best = sk[w] > best ? sk[w] : best;
      if (TYPICAL) sf = soft_merge(sf, ss[w]);
    }
    RowPart rp;
    rp.key = best;
    rp.m = sf.m;
    rp.Z = sf.Z;
    rp.S = sf.S;
    rp.pad = 0.f;
    parts[row * splits + sp] = rp;
  }
}

// Typical acceptance tests a node against its parent's row only, so the
// softmax statistics are needed for the rows of nodes that have children;
// a leaf's row is reduced to its argmax alone (the next token when that
// leaf ends the accepted path) and reports (m, Z, S) = (-inf, 0, 0).
template <typename T, bool TYPICAL>
__global__ void __launch_bounds__(kRedThreads)
    row_reduce_kernel(const T* __restrict__ vlog, int V, int chunk, int splits, ZTab zt,
                      const int32_t* __restrict__ depth, const int32_t* __restrict__ nchild,
                      int N, int K, RowPart* __restrict__ parts) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  // typical: rows taken node-major (node 0 of every sequence, then node 1,
  // ...): the nodes with children, whose rows cost the exponentials, come
  // first in (depth, lexicographic) order, so the launch ends on cheap rows
  const unsigned nseq = gridDim.x / (unsigned)N;
  const size_t row = TYPICAL ? (size_t)(blockIdx.x % nseq) * N + blockIdx.x / nseq
                             : (size_t)blockIdx.x;
  const int sp = blockIdx.y;
  if (TYPICAL) {
    const int node = (int)(row % (size_t)N);
    if (nchild[node] > 0) {  // CTA-uniform
      const int dc = depth[node] + 1;
      row_reduce_chunk<T, true>(vlog, V, chunk, splits, zt.z[dc < K ? dc : K], row, sp, parts);
      return;
    }
  }
  row_reduce_chunk<T, false>(vlog, V, chunk, splits, 0.f, row, sp, parts);
}

// One CTA per sequence, one thread per tree node (blockDim = N rounded up to
// a whole warp, <= MEDUSA_MAX_N).
template <typename T, bool TYPICAL>
__global__ void __launch_bounds__(MEDUSA_MAX_N)
    accept_walk_kernel(const T* __restrict__ vlog, const RowPart* __restrict__ parts, int splits,
                       const int32_t* __restrict__ tok, const int32_t* __restrict__ parent,
                       const int32_t* __restrict__ depth, const uint32_t* __restrict__ anc, int N,
                       int W, int K, int V, ZTab zt, float eps, float delta,
                       int32_t* __restrict__ accept_len, int32_t* __restrict__ accept_nodes,
                       int32_t* __restrict__ next_tok) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int32_t amax[MEDUSA_MAX_N];
  __shared__ float mrow[MEDUSA_MAX_N], zrow[MEDUSA_MAX_N], thr[MEDUSA_MAX_N];
  __shared__ uint32_t cond[MEDUSA_MAX_N / 32];
  __shared__ uint32_t wkey[MEDUSA_MAX_N / 32];
  const int b = blockIdx.x;
  const int n = threadIdx.x;
  const int warp = n >> 5, lane = n & 31;

  // merge the chunks of row n: argmax and (typical) the acceptance threshold
  if (n < N) {
    const RowPart* pr = parts + ((size_t)b * N + n) * splits;
    uint64_t best = 0ull;
    Soft sf{-INFINITY, 0.f, 0.f};
    for (int s2 = 0; s2 < splits; ++s2) {
      const RowPart rp = pr[s2];
      best = rp.key > best ? rp.key : best;
      if (TYPICAL) sf = soft_merge(sf, Soft{rp.m, rp.Z, rp.S});
    }
    amax[n] = (int32_t)key_index(best);
    if (TYPICAL) {
      mrow[n] = sf.m;
      zrow[n] = sf.Z;
      const float H = logf(sf.Z) - kLn2 * sf.S / sf.Z;
      thr[n] = fminf(eps, delta * expf(-H));
    }
  }
  __syncthreads();

  // node n's own condition against its parent's row (root: true)
  bool c = (n == 0);
  if (n > 0 && n < N) {
    const int par = parent[n];
    const int t = tok[(size_t)b * N + n];
    dbg_ok(t >= 0 && t < V, DBG_ACCEPT_TOKEN);  // a token outside the vocabulary never matches
    if (!dbg_ok(par >= 0 && par < n, DBG_ACCEPT_PARENT)) {
      c = false;
    } else if (TYPICAL) {
      if (t >= 0 && t < V) {
        const float x = to_f32(vlog[((size_t)b * N + par) * V + t]);
        // the parent's row was reduced at the scale of n's depth
        const float p = exp2f(x * zt.z[depth[n]] - mrow[par]) / zrow[par];
        c = p > thr[par];
      }
    } else {
      c = (amax[par] == t);
    }
  }
  const uint32_t bits = __ballot_sync(0xffffffffu, c);
  if (lane == 0) cond[warp] = bits;
  __syncthreads();

  // accepted iff every node on the root path satisfies its condition;
  // deepest accepted node wins, ties to the lowest index.
  uint32_t key = 0u;
  if (n < N) {
    bool ok = true;
    for (int w = 0; w < W; ++w) ok = ok && ((anc[(size_t)n * W + w] & ~cond[w]) == 0u);
    if (ok) key = ((uint32_t)depth[n] << 16) | (0xFFFFu - (uint32_t)n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t other = __shfl_xor_sync(0xffffffffu, key, o);
    key = other > key ? other : key;
  }
  if (lane == 0) wkey[warp] = key;
  __syncthreads();
  if (n == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) key = wkey[w] > key ? wkey[w] : key;
    const int best = (int)(0xFFFFu - (key & 0xFFFFu));
    const int D = (int)(key >> 16);
    accept_len[b] = D;
    next_tok[b] = amax[best];
    int j = 0;
    for (int w = 0; w < W; ++w) {
      uint32_t bitsw = anc[(size_t)best * W + w];
      while (bitsw) {
        const int i = __ffs(bitsw) - 1;
        bitsw &= bitsw - 1;
        if (j <= K) accept_nodes[(size_t)b * (K + 1) + j] = w * 32 + i;
        ++j;
      }
    }
    for (; j <= K; ++j) accept_nodes[(size_t)b * (K + 1) + j] = -1;
  }
}

struct AccPlan {
  int splits, chunk;
  size_t total;
};

AccPlan make_plan(int rows, int V) {
  AccPlan P;
  const int target = 4 * num_sms();
  int splits = (target + rows - 1) / (rows > 0 ? rows : 1);
  const int max_splits = (V + 2047) / 2048;  // keep >= ~2K elements per CTA
  splits = splits < 1 ? 1 : (splits > max_splits ? max_splits : splits);
  splits = splits < 1 ? 1 : splits;
  int chunk = (V + splits - 1) / splits;
  chunk = (chunk + 7) & ~7;  // 16-byte aligned chunk starts for bf16 rows
  splits = (V + chunk - 1) / chunk;
  P.splits = splits;
  P.chunk = chunk;
  WsCarver w;
  w.take<RowPart>((size_t)rows * splits);
  P.total = w.total();
  return P;
}

}  // namespace

size_t accept_workspace(const medusa_tree* t, int B, int V) {
  return make_plan(B * t->N, V).total;
}

int accept_launch(const AcceptArgs& a, cudaStream_t st) {
  const int N = a.tree->N;
  const int rows = a.B * N;
  if (rows == 0) return MEDUSA_OK;
  const AccPlan P = make_plan(rows, a.V);
  if (a.ws_bytes < P.total) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for accept");
  RowPart* parts = (RowPart*)a.ws;
  ZTab zt;
  for (int D = 0; D <= MEDUSA_MAX_K; ++D) {
    const int i = D < 1 ? 0 : (D > a.tree->K ? a.tree->K - 1 : D - 1);
    zt.z[D] = a.typical && a.tree->K > 0 ? kLog2e / a.temps[i < 0 ? 0 : i] : 0.f;
  }
  dim3 g1(rows, P.splits);
  const int walk_threads = (N + 31) / 32 * 32;
  const medusa_tree* t = a.tree;
  cudaError_t le = cudaSuccess;
#define MEDUSA_ACC(T, TYP)                                                                     \
  do {                                                                                         \
    le = launch_pdl(row_reduce_kernel<T, TYP>, g1, dim3(kRedThreads), 0, st, (const T*)a.vlog, \
                    a.V, P.chunk, P.splits, zt, t->d_depth, t->d_nchild, N, t->K, parts);    \
    if (le == cudaSuccess)                                                                     \
      le = launch_pdl(accept_walk_kernel<T, TYP>, dim3(a.B), dim3(walk_threads), 0, st,        \
                      (const T*)a.vlog, parts, P.splits, a.tok, t->d_parent, t->d_depth,       \
                      t->d_anc, N, t->W, t->K, a.V, zt, a.eps, a.delta, a.accept_len,          \
                      a.accept_nodes, a.next_tok);                                             \
  } while (0)
  // greedy results from the typical pass's row reduction (its keys hold
  // every row's argmax)
#define MEDUSA_ACC_GREEDY(T)                                                                     \
  do {                                                                                           \
    if (le == cudaSuccess && a.typical && a.g_accept_len)                                        \
      le = launch_pdl(accept_walk_kernel<T, false>, dim3(a.B), dim3(walk_threads), 0, st,        \
                      (const T*)a.vlog, parts, P.splits, a.tok, t->d_parent, t->d_depth,         \
                      t->d_anc, N, t->W, t->K, a.V, zt, 0.f, 0.f, a.g_accept_len,                \
                      a.g_accept_nodes, a.g_next_tok);                                           \
  } while (0)
  if (a.dtype == MEDUSA_F32) {
    if (a.typical) MEDUSA_ACC(float, true);
    else MEDUSA_ACC(float, false);
    MEDUSA_ACC_GREEDY(float);
  } else {
    if (a.typical) MEDUSA_ACC(__nv_bfloat16, true);
    else MEDUSA_ACC(__nv_bfloat16, false);
    MEDUSA_ACC_GREEDY(__nv_bfloat16);
  }
#undef MEDUSA_ACC_GREEDY
#undef MEDUSA_ACC
  cudaError_t e = le != cudaSuccess ? le : cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "accept kernels launch");
}

// ---------------------------------------------------------------------------
// Greedy acceptance whose scratch is owned by the library, for callers that
// cannot allocate device memory.  The per-row-chunk results of the verify
// row reduction go to this fixed array instead of a caller workspace:
// MEDUSA_NOALLOC_ACCEPT_PARTS entries x 24 bytes (1.5 MiB), held by every
// GPU that loads the library until the process exits.  Every call writes
// each entry it reads before reading it, so nothing has to start at zero;
// calls that overlap on the GPU share the array and race.
static __device__ __align__(256) RowPart g_accept_scratch[MEDUSA_NOALLOC_ACCEPT_PARTS];

namespace {
std::mutex g_scratch_mu;
RowPart* g_scratch_addr[64] = {nullptr};
unsigned long long g_scratch_ctx[64] = {0};  // id of the context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the CUDA context current on this thread (the driver never reuses an
// id within a process, unlike a context handle); false when no context is
// current yet or the driver entry points are unavailable.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (CtxGetCurrentFn)p;
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)p;
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_accept_scratch on the current device.  Looked up with
// that device current on its first call, and again whenever the device's
// context has changed since (a cudaDeviceReset destroys the context the
// cached address belonged to); otherwise the cached address is used.
int scratch_address(RowPart** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MEDUSA_ERR_UNSUPPORTED, "device ordinal >= 64");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  const bool have_id = current_context_id(&id);
  if (!g_scratch_addr[dev] || !have_id || id != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_accept_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_accept_scratch)");
    g_scratch_addr[dev] = (RowPart*)p;
    g_scratch_ctx[dev] = current_context_id(&id) ? id : 0ull;
  }
  *out = g_scratch_addr[dev];
  return MEDUSA_OK;
}
}  // namespace

int accept_greedy_noalloc_launch(const void* vlog, int dtype, const int32_t* tok,
                                 const medusa_tree* t, int B, int V, int32_t* accept_len,
                                 int32_t* accept_nodes, int32_t* next_tok, cudaStream_t st) {
  const int N = t->N;
  const long long rows = (long long)B * N;
  if (rows == 0) return MEDUSA_OK;
  if (rows > MEDUSA_NOALLOC_ACCEPT_PARTS)
    return fail(MEDUSA_ERR_INVALID_ARG,
                "medusa_accept_greedy_noalloc: B*N exceeds its static scratch "
                "(MEDUSA_NOALLOC_ACCEPT_PARTS rows)");
  const AccPlan P = make_plan((int)rows, V);
  // make_plan splits rows only while rows < 4 x SMs, so rows x splits stays
  // below 4 x SMs + rows, far inside the array for any device
  if (rows * P.splits > MEDUSA_NOALLOC_ACCEPT_PARTS)
    return fail(MEDUSA_ERR_UNSUPPORTED,
                "medusa_accept_greedy_noalloc: row chunks exceed the static scratch");
  RowPart* parts = nullptr;
  int rc = scratch_address(&parts);
  if (rc) return rc;
  dim3 g1((unsigned)rows, P.splits);
  const int walk_threads = (N + 31) / 32 * 32;
  const ZTab zt0 = {};  // greedy: no scale
  cudaError_t le = cudaSuccess;
#define MEDUSA_ACC_STATIC(T)                                                                     \
  do {                                                                                           \
    le = launch_pdl(row_reduce_kernel<T, false>, g1, dim3(kRedThreads), 0, st, (const T*)vlog, V, \
                    P.chunk, P.splits, zt0, t->d_depth, t->d_nchild, N, t->K, parts);            \
    if (le == cudaSuccess)                                                                       \
      le = launch_pdl(accept_walk_kernel<T, false>, dim3(B), dim3(walk_threads), 0, st,          \
                      (const T*)vlog,                                                            \
                      parts, P.splits, tok, t->d_parent, t->d_depth, t->d_anc, N, t->W, t->K, V, \
                      zt0, 0.f, 0.f, accept_len, accept_nodes, next_tok);                        \
  } while (0)
  if (dtype == MEDUSA_F32)
    MEDUSA_ACC_STATIC(float);
  else
    MEDUSA_ACC_STATIC(__nv_bfloat16);
#undef MEDUSA_ACC_STATIC
  cudaError_t e = le != cudaSuccess ? le : cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "accept kernels launch (static scratch)");
}

}  // namespace medusa

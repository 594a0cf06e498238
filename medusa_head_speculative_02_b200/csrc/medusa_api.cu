// Host side of libmedusa: the C ABI declared in include/medusa.h, argument
// validation, the tree plan, TMA descriptor encoding and the device status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstring>
#include <cmath>
#include <map>
#include <queue>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace medusa {

__device__ unsigned int g_dev_status = 0u;
__device__ unsigned int g_dev_debug_site = 0u;

namespace {
thread_local std::string t_last_error;

// CUDA driver entry point of cuTensorMapEncodeTiled, fetched through the
// runtime so the library needs no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
}  // namespace

int fail(int code, const std::string& msg) {
  t_last_error = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MEDUSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// NVTX range around one ABI call (shows the call by name in Nsight Systems
// and Nsight Compute range filters); a no-op unless a tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
      cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
  }
  return 148;
}

int make_tmap_bf16(void* map, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MEDUSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn((CUtensorMap*)map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                  const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MEDUSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")");
  return MEDUSA_OK;
}

// ---------------------------------------------------------------- tree plan
namespace {

struct Tup {
  std::vector<int> r;
  int S = 0;
  int D() const { return (int)r.size(); }
};

// 5^n for n <= 16
uint64_t pow5(int n) {
  uint64_t v = 1;
  for (int i = 0; i < n; ++i) v *= 5;
  return v;
}

// Sign of score(D1,S1) - score(D2,S2) with score = 0.8^D 0.5^S = 2^(2D-S) / 5^D,
// computed exactly: compare 2^e * 5^D2 with 5^D1, e = (2D1-S1) - (2D2-S2).
int cmp_score(int D1, int S1, int D2, int S2) {
  const int e = (2 * D1 - S1) - (2 * D2 - S2);
  const uint64_t a5 = pow5(D2), b5 = pow5(D1);  // < 2^38 for D <= 16
  if (e >= 0) {
    if (e >= 24) return 1;  // 2^24 * 5^D2 >= 2^24 > 5^8 >= 5^D1
    const uint64_t x = a5 << e;
    return x > b5 ? 1 : (x < b5 ? -1 : 0);
  }
  if (-e >= 24) return -1;
  const uint64_t y = b5 << (-e);
  return a5 > y ? 1 : (a5 < y ? -1 : 0);
}

// true iff a precedes b in the selection order (score desc, depth asc, lex asc)
bool precedes(const Tup& a, const Tup& b) {
  const int c = cmp_score(a.D(), a.S, b.D(), b.S);
  if (c != 0) return c > 0;
  if (a.D() != b.D()) return a.D() < b.D();
  return a.r < b.r;
}

struct Later {
  bool operator()(const Tup& a, const Tup& b) const { return precedes(b, a); }
};

int plan_host(int K, int s, int N, medusa_tree* t) {
  if (K < 1 || K > MEDUSA_MAX_K) return fail(MEDUSA_ERR_INVALID_ARG, "K out of [1, MEDUSA_MAX_K]");
  if (s < 1 || s > MEDUSA_MAX_S) return fail(MEDUSA_ERR_INVALID_ARG, "s out of [1, MEDUSA_MAX_S]");
  if (N < 1 || N > MEDUSA_MAX_N) return fail(MEDUSA_ERR_INVALID_ARG, "N out of [1, MEDUSA_MAX_N]");
  double total = 0, p = 1;
  for (int D = 0; D <= K; ++D, p *= s) total += p;
  if ((double)N > total) return fail(MEDUSA_ERR_INVALID_ARG, "N exceeds 1 + s + ... + s^K");

  // Best-first enumeration: a tuple's first child and its next sibling both
  // score strictly lower than it, so popping in order yields the global order.
  std::priority_queue<Tup, std::vector<Tup>, Later> pq;
  pq.push(Tup{});
  std::vector<Tup> chosen;
  while ((int)chosen.size() < N) {
    Tup t0 = pq.top();
    pq.pop();
    if (t0.D() < K) {
      Tup c = t0;
      c.r.push_back(0);
      pq.push(c);
    }
    if (t0.D() >= 1 && t0.r.back() + 1 < s) {
      Tup sib = t0;
      sib.r.back() += 1;
      sib.S += 1;
      pq.push(sib);
    }
    chosen.push_back(std::move(t0));
  }
  std::sort(chosen.begin(), chosen.end(), [](const Tup& a, const Tup& b) {
    if (a.D() != b.D()) return a.D() < b.D();
    return a.r < b.r;
  });
  std::map<std::vector<int>, int> index;
  for (int i = 0; i < N; ++i) index[chosen[i].r] = i;

  t->K = K;
  t->s = s;
  t->N = N;
  t->W = (N + 31) / 32;
  t->parent.assign(N, -1);
  t->depth.assign(N, 0);
  t->rank_path.assign((size_t)N * K, -1);
  t->head_rank.assign(N, -1);
  t->anc.assign((size_t)N * t->W, 0u);
  for (int i = 0; i < N; ++i) {
    const std::vector<int>& r = chosen[i].r;
    const int D = (int)r.size();
    t->depth[i] = D;
    for (int j = 0; j < D; ++j) t->rank_path[(size_t)i * K + j] = r[j];
    if (D > 0) {
      std::vector<int> pr(r.begin(), r.end() - 1);
      t->parent[i] = index.at(pr);
      t->head_rank[i] = (D - 1) * s + r[D - 1];
    }
  }
  for (int i = 0; i < N; ++i)
    for (int j = i; j >= 0; j = t->parent[j]) t->anc[(size_t)i * t->W + j / 32] |= 1u << (j % 32);
  return MEDUSA_OK;
}

int check_tree(const medusa_tree* t) {
  if (!t || !t->d_block) return fail(MEDUSA_ERR_INVALID_ARG, "tree is NULL");
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != t->device) return fail(MEDUSA_ERR_INVALID_ARG, "tree was created on another device");
  return MEDUSA_OK;
}

bool dtype_ok(int dt) { return dt == MEDUSA_F32 || dt == MEDUSA_BF16; }

}  // namespace
}  // namespace medusa

using namespace medusa;

namespace medusa {
namespace selftest {
// One thread waits for phase 0 of a barrier that no thread arrives at.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0u, &abort_flag, limit_ns);
}
}  // namespace selftest
}  // namespace medusa

extern "C" {

int medusa_selftest_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 2000)
    return fail(MEDUSA_ERR_INVALID_ARG, "limit_ms must be in [1, 2000]");
  selftest::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
      (unsigned long long)limit_ms * 1000000ull);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "selftest_wait_kernel launch");
}

const char* medusa_last_error(void) { return t_last_error.c_str(); }

#ifdef MEDUSA_DEBUG
const char* medusa_version(void) { return "medusa-b200 0.2 (sm_100a, MEDUSA_DEBUG index checks)"; }
#else
const char* medusa_version(void) { return "medusa-b200 0.2 (sm_100a)"; }
#endif

int medusa_device_status(int* status, int clear) {
  if (!status) return fail(MEDUSA_ERR_INVALID_ARG, "status is NULL");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  unsigned int v = 0, site = 0;
  e = cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&site, g_dev_debug_site, sizeof(site));
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  if (clear) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_dev_status, &z, sizeof(z));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_dev_debug_site, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_fail(e, "clear device status");
  }
  if (v & DEV_BOUNDS) {
    *status = MEDUSA_ERR_BOUNDS;
    fail(MEDUSA_ERR_BOUNDS, "device index check failed, first at site " + std::to_string(site));
  } else {
    *status = (v & DEV_TIMEOUT) ? MEDUSA_ERR_TIMEOUT : MEDUSA_OK;
  }
  return MEDUSA_OK;
}

int medusa_tree_plan_host(int K, int s, int N, int32_t* parent, int32_t* depth,
                          int32_t* rank_path, uint32_t* anc_mask) {
  try {
    medusa_tree t;
    int rc = plan_host(K, s, N, &t);
    if (rc) return rc;
    if (parent) std::copy(t.parent.begin(), t.parent.end(), parent);
    if (depth) std::copy(t.depth.begin(), t.depth.end(), depth);
    if (rank_path) std::copy(t.rank_path.begin(), t.rank_path.end(), rank_path);
    if (anc_mask) std::copy(t.anc.begin(), t.anc.end(), anc_mask);
    return MEDUSA_OK;
  } catch (...) {
    return fail(MEDUSA_ERR_INVALID_ARG, "tree plan construction failed");
  }
}

int medusa_tree_create(int K, int s, int N, medusa_tree_t** out) {
  medusa::NvtxRange nvtx_range("medusa_tree_create");
  if (!out) return fail(MEDUSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  medusa_tree* t = nullptr;
  try {
    t = new medusa_tree();
    int rc = plan_host(K, s, N, t);
    if (rc) {
      delete t;
      return rc;
    }
    cudaError_t e = cudaGetDevice(&t->device);
    if (e != cudaSuccess) {
      delete t;
      return cuda_fail(e, "cudaGetDevice");
    }
    t->nchild.assign(N, 0);
    for (int c = 1; c < N; ++c) t->nchild[t->parent[c]]++;
    const size_t n4 = (size_t)N * 4;
    const size_t bytes = 4 * n4 + (size_t)N * t->W * 4;
    e = cudaMalloc(&t->d_block, bytes);
    if (e != cudaSuccess) {
      delete t;
      return cuda_fail(e, "cudaMalloc(tree plan)");
    }
    std::vector<uint8_t> host(bytes);
    memcpy(host.data(), t->parent.data(), n4);
    memcpy(host.data() + n4, t->depth.data(), n4);
    memcpy(host.data() + 2 * n4, t->head_rank.data(), n4);
    memcpy(host.data() + 3 * n4, t->nchild.data(), n4);
    memcpy(host.data() + 4 * n4, t->anc.data(), (size_t)N * t->W * 4);
    e = cudaMemcpy(t->d_block, host.data(), bytes, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(t->d_block);
      delete t;
      return cuda_fail(e, "upload tree plan");
    }
    uint8_t* d = (uint8_t*)t->d_block;
    t->d_parent = (const int32_t*)d;
    t->d_depth = (const int32_t*)(d + n4);
    t->d_head_rank = (const int32_t*)(d + 2 * n4);
    t->d_nchild = (const int32_t*)(d + 3 * n4);
    t->d_anc = (const uint32_t*)(d + 4 * n4);
    *out = t;
    return MEDUSA_OK;
  } catch (...) {
    delete t;
    return fail(MEDUSA_ERR_INVALID_ARG, "tree creation failed");
  }
}

int medusa_tree_destroy(medusa_tree_t* t) {
  if (!t) return MEDUSA_OK;
  if (t->d_block) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != t->device) cudaSetDevice(t->device);
    cudaFree(t->d_block);
    if (cur != t->device && cur >= 0) cudaSetDevice(cur);
  }
  delete t;
  return MEDUSA_OK;
}

int medusa_tree_info(const medusa_tree_t* t, int* K, int* s, int* N, int32_t* parent,
                     int32_t* depth, int32_t* rank_path, uint32_t* anc_mask) {
  if (!t) return fail(MEDUSA_ERR_INVALID_ARG, "tree is NULL");
  if (K) *K = t->K;
  if (s) *s = t->s;
  if (N) *N = t->N;
  if (parent) std::copy(t->parent.begin(), t->parent.end(), parent);
  if (depth) std::copy(t->depth.begin(), t->depth.end(), depth);
  if (rank_path) std::copy(t->rank_path.begin(), t->rank_path.end(), rank_path);
  if (anc_mask) std::copy(t->anc.begin(), t->anc.end(), anc_mask);
  return MEDUSA_OK;
}

size_t medusa_heads_workspace_size(int B, int d, int V, int K, int s, int dtype) {
  if (B <= 0 || d <= 0 || V <= 0 || K <= 0 || s < 0) return 0;
  if (s == 0) s = 1;
  if (dtype != MEDUSA_BF16) return heads_simt_workspace(B, d, V, K, s);
  return B > 32 ? heads_big_workspace(B, d, V, K, s) : heads_tc_workspace(B, d, V, K, s);
}

int medusa_heads_forward(const void* h, const void* W1, const void* b1, const void* W2, int B,
                         int d, int V, int K, int dtype, float* logits, int s,
                         int32_t* topk_idx, float* topk_val, void* ws, size_t ws_bytes,
                         void* stream) {
  medusa::NvtxRange nvtx_range("medusa_heads_forward");
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || d <= 0 || V <= 0 || K < 1 || K > MEDUSA_MAX_K)
    return fail(MEDUSA_ERR_INVALID_ARG, "bad heads shape");
  if (d % 8 != 0) return fail(MEDUSA_ERR_UNSUPPORTED, "d must be a multiple of 8");
  if (!h || !W1 || !W2) return fail(MEDUSA_ERR_INVALID_ARG, "h, W1 and W2 must be non-NULL");
  if (!logits && !topk_idx) return fail(MEDUSA_ERR_INVALID_ARG, "nothing to compute");
  if (topk_idx && (s < 1 || s > MEDUSA_MAX_S || s > V))
    return fail(MEDUSA_ERR_INVALID_ARG, "s out of [1, min(V, MEDUSA_MAX_S)]");
  if (!topk_idx) s = 1;
  if (!aligned16(h) || !aligned16(W1) || !aligned16(W2) || (b1 && !aligned16(b1)) ||
      !aligned16(ws))
    return fail(MEDUSA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (dtype == MEDUSA_BF16 && B > MEDUSA_MAX_HEADS_B)
    return fail(MEDUSA_ERR_UNSUPPORTED, "bf16 heads: B <= MEDUSA_MAX_HEADS_B");
  if (dtype == MEDUSA_F32 && B > 16) return fail(MEDUSA_ERR_UNSUPPORTED, "fp32 heads: B <= 16");
  if (B == 0) return MEDUSA_OK;
  const size_t need = medusa_heads_workspace_size(B, d, V, K, s, dtype);
  if (!ws || ws_bytes < need) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small");
  HeadsArgs a{h, W1, b1, W2, B, d, V, K, dtype, logits, s, topk_idx, topk_val, ws, ws_bytes};
  cudaStream_t st = (cudaStream_t)stream;
  if (dtype != MEDUSA_BF16) return heads_simt_launch(a, st);
  return B > 32 ? heads_big_launch(a, st) : heads_tc_launch(a, st);
}

int medusa_topk(const void* logits, int dtype, int R, int V, int s, int32_t* idx, float* val,
                void* stream) {
  medusa::NvtxRange nvtx_range("medusa_topk");
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (R < 0 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (s < 1 || s > MEDUSA_MAX_S || s > V)
    return fail(MEDUSA_ERR_INVALID_ARG, "s out of [1, min(V, MEDUSA_MAX_S)]");
  if (R > 0 && (!logits || !idx)) return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return topk_rows_launch(logits, dtype, R, V, s, idx, val, (cudaStream_t)stream);
}

int medusa_build_tree(const medusa_tree_t* tree, const int32_t* root_tok,
                      const int32_t* topk_idx, const int32_t* prefix_len, int B,
                      int32_t* tree_tok, int32_t* tree_pos, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_build_tree");
  int rc = check_tree(tree);
  if (rc) return rc;
  if (B < 0) return fail(MEDUSA_ERR_INVALID_ARG, "B < 0");
  if (B > 0 && (!root_tok || !topk_idx || !tree_tok || (tree_pos && !prefix_len)))
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return build_tree_launch(tree, root_tok, topk_idx, prefix_len, B, tree_tok, tree_pos,
                           (cudaStream_t)stream);
}

size_t medusa_tree_attention_workspace_size(const medusa_tree_t* tree, int B, int Hq, int Hkv,
                                            int dh, int Lcap) {
  if (!tree || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lcap < 0) return 0;
  return attention_workspace(tree, B, Hq, Hkv, dh, Lcap, -1);
}

int medusa_tree_attention_chunks(const medusa_tree_t* tree, int B, int Hq, int Hkv, int dh,
                                 int Lcap, int dtype) {
  if (!tree || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lcap < tree->N || !dtype_ok(dtype))
    return fail(MEDUSA_ERR_INVALID_ARG, "bad attention shape");
  return attention_chunks(tree, B, Hq, Hkv, dh, Lcap, dtype);
}

int medusa_tree_attention_tiles_per_cta(const medusa_tree_t* tree, int B, int Hq, int Hkv,
                                        int dh, int Lcap, int dtype) {
  if (!tree || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lcap < tree->N || !dtype_ok(dtype))
    return fail(MEDUSA_ERR_INVALID_ARG, "bad attention shape");
  return attention_tiles_per_cta(tree, B, Hq, Hkv, dh, Lcap, dtype);
}

int medusa_tree_attention_launches(const medusa_tree_t* tree, int B, int Hq, int Hkv, int dh,
                                   int Lcap, int dtype) {
  if (!tree || B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lcap < tree->N || !dtype_ok(dtype))
    return fail(MEDUSA_ERR_INVALID_ARG, "bad attention shape");
  return attention_launches(tree, B, Hq, Hkv, dh, Lcap, dtype);
}

int medusa_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                          const int32_t* prefix_len, const medusa_tree_t* tree, int B, int Hq,
                          int Hkv, int dh, int Lcap, float scale, int dtype, void* out, void* ws,
                          size_t ws_bytes, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_tree_attention");
  int rc = check_tree(tree);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0)
    return fail(MEDUSA_ERR_INVALID_ARG, "need Hq % Hkv == 0 and positive head counts");
  if (dh != 64 && dh != 128) return fail(MEDUSA_ERR_UNSUPPORTED, "dh must be 64 or 128");
  if (Lcap < tree->N) return fail(MEDUSA_ERR_INVALID_ARG, "Lcap < N");
  if (!(std::isfinite(scale) && scale > 0.f))
    return fail(MEDUSA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (B == 0) return MEDUSA_OK;
  if (!q || !k_cache || !v_cache || !prefix_len || !out)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  const size_t need = attention_workspace(tree, B, Hq, Hkv, dh, Lcap, dtype);
  if (!ws || ws_bytes < need) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small");
  AttnArgs a{q, k_cache, v_cache, prefix_len, tree, B, Hq, Hkv, dh, Lcap, scale, dtype, out,
             ws, ws_bytes};
  return attention_launch(a, (cudaStream_t)stream);
}

size_t medusa_accept_workspace_size(const medusa_tree_t* tree, int B, int V) {
  if (!tree || B < 0 || V <= 0) return 0;
  return accept_workspace(tree, B, V);
}

// temps: host array of the per-depth temperatures (K entries) or NULL for
// the single temperature T.
static int accept_common(const void* vlogits, int dtype, const int32_t* tree_tok,
                         const medusa_tree_t* tree, int B, int V, bool typical, float T,
                         const float* temps, float eps, float delta, int32_t* accept_len,
                         int32_t* accept_nodes, int32_t* next_tok, void* ws, size_t ws_bytes,
                         void* stream, int32_t* g_accept_len = nullptr,
                         int32_t* g_accept_nodes = nullptr, int32_t* g_next_tok = nullptr) {
  int rc = check_tree(tree);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  float tk[MEDUSA_MAX_K];
  for (int i = 0; i < MEDUSA_MAX_K; ++i) tk[i] = (temps && i < tree->K) ? temps[i] : T;
  if (typical) {
    bool good = std::isfinite(eps) && std::isfinite(delta);
    for (int i = 0; i < tree->K; ++i) good = good && tk[i] > 0.f && std::isfinite(tk[i]);
    if (!good)
      return fail(MEDUSA_ERR_INVALID_ARG,
                  "typical acceptance needs temperatures > 0 and finite eps, delta");
  }
  if (B == 0) return MEDUSA_OK;
  if (!vlogits || !tree_tok || !accept_len || !accept_nodes || !next_tok)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  const size_t need = accept_workspace(tree, B, V);
  if (!ws || ws_bytes < need) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small");
  AcceptArgs a{};
  a.vlog = vlogits;
  a.dtype = dtype;
  a.tok = tree_tok;
  a.tree = tree;
  a.B = B;
  a.V = V;
  a.typical = typical;
  for (int i = 0; i < MEDUSA_MAX_K; ++i) a.temps[i] = tk[i];
  a.eps = eps;
  a.delta = delta;
  a.accept_len = accept_len;
  a.accept_nodes = accept_nodes;
  a.next_tok = next_tok;
  a.g_accept_len = g_accept_len;
  a.g_accept_nodes = g_accept_nodes;
  a.g_next_tok = g_next_tok;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  return accept_launch(a, (cudaStream_t)stream);
}

int medusa_accept_greedy(const void* vlogits, int dtype, const int32_t* tree_tok,
                         const medusa_tree_t* tree, int B, int V, int32_t* accept_len,
                         int32_t* accept_nodes, int32_t* next_tok, void* ws, size_t ws_bytes,
                         void* stream) {
  medusa::NvtxRange nvtx_range("medusa_accept_greedy");
  return accept_common(vlogits, dtype, tree_tok, tree, B, V, false, 1.f, nullptr, 0.f, 0.f,
                       accept_len, accept_nodes, next_tok, ws, ws_bytes, stream);
}

int medusa_accept_typical(const void* vlogits, int dtype, const int32_t* tree_tok,
                          const medusa_tree_t* tree, int B, int V, float temperature, float eps,
                          float delta, int32_t* accept_len, int32_t* accept_nodes,
                          int32_t* next_tok, void* ws, size_t ws_bytes, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_accept_typical");
  return accept_common(vlogits, dtype, tree_tok, tree, B, V, true, temperature, nullptr, eps,
                       delta, accept_len, accept_nodes, next_tok, ws, ws_bytes, stream);
}

int medusa_accept_greedy_typical(const void* vlogits, int dtype, const int32_t* tree_tok,
                                 const medusa_tree_t* tree, int B, int V, float temperature,
                                 float eps, float delta, int32_t* g_accept_len,
                                 int32_t* g_accept_nodes, int32_t* g_next_tok,
                                 int32_t* t_accept_len, int32_t* t_accept_nodes,
                                 int32_t* t_next_tok, void* ws, size_t ws_bytes, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_accept_greedy_typical");
  if (B > 0 && (!g_accept_len || !g_accept_nodes || !g_next_tok))
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  if (B > 0 && (g_accept_len == t_accept_len || g_accept_nodes == t_accept_nodes ||
                g_next_tok == t_next_tok))
    return fail(MEDUSA_ERR_INVALID_ARG, "greedy and typical outputs overlap");
  return accept_common(vlogits, dtype, tree_tok, tree, B, V, true, temperature, nullptr, eps,
                       delta, t_accept_len, t_accept_nodes, t_next_tok, ws, ws_bytes, stream,
                       g_accept_len, g_accept_nodes, g_next_tok);
}

int medusa_accept_typical_per_head(const void* vlogits, int dtype, const int32_t* tree_tok,
                                   const medusa_tree_t* tree, int B, int V,
                                   const float* temperatures, float eps, float delta,
                                   int32_t* accept_len, int32_t* accept_nodes, int32_t* next_tok,
                                   void* ws, size_t ws_bytes, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_accept_typical_per_head");
  if (!temperatures) return fail(MEDUSA_ERR_INVALID_ARG, "temperatures is NULL");
  return accept_common(vlogits, dtype, tree_tok, tree, B, V, true, 1.f, temperatures, eps,
                       delta, accept_len, accept_nodes, next_tok, ws, ws_bytes, stream);
}

int medusa_accept_greedy_noalloc(const void* vlogits, int dtype, const int32_t* tree_tok,
                                 const medusa_tree_t* tree, int B, int V, int32_t* accept_len,
                                 int32_t* accept_nodes, int32_t* next_tok, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_accept_greedy_noalloc");
  int rc = check_tree(tree);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || V < 1) return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (B == 0) return MEDUSA_OK;
  if (!vlogits || !tree_tok || !accept_len || !accept_nodes || !next_tok)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return accept_greedy_noalloc_launch(vlogits, dtype, tree_tok, tree, B, V, accept_len,
                                      accept_nodes, next_tok, (cudaStream_t)stream);
}

int medusa_kv_compact(void* k_cache, void* v_cache, const int32_t* prefix_len,
                      const int32_t* accept_len, const int32_t* accept_nodes, int B, int Hkv,
                      int dh, int Lcap, int K, int dtype, int32_t* new_len, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_kv_compact");
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || Hkv <= 0 || dh <= 0 || Lcap <= 0 || K < 0 || K > MEDUSA_MAX_K)
    return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (((size_t)Hkv * dh * (dtype == MEDUSA_F32 ? 4 : 2)) % 4 != 0)
    return fail(MEDUSA_ERR_UNSUPPORTED, "slot size must be a multiple of 4 bytes");
  if (B == 0) return MEDUSA_OK;
  if (!k_cache || !v_cache || !prefix_len || !accept_len || !accept_nodes)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return kv_compact_launch(k_cache, v_cache, prefix_len, accept_len, accept_nodes, B, Hkv, dh,
                           Lcap, K, dtype, new_len, (cudaStream_t)stream);
}

int medusa_kv_compact_layers(void* k_caches, void* v_caches, int n_layers,
                             long long layer_stride, const int32_t* prefix_len,
                             const int32_t* accept_len, const int32_t* accept_nodes, int B,
                             int Hkv, int dh, int Lcap, int K, int dtype, int32_t* new_len,
                             void* stream) {
  medusa::NvtxRange nvtx_range("medusa_kv_compact_layers");
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (n_layers < 0 || B < 0 || Hkv <= 0 || dh <= 0 || Lcap <= 0 || K < 0 || K > MEDUSA_MAX_K)
    return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (((size_t)Hkv * dh * (dtype == MEDUSA_F32 ? 4 : 2)) % 4 != 0)
    return fail(MEDUSA_ERR_UNSUPPORTED, "slot size must be a multiple of 4 bytes");
  if (n_layers > 1 && layer_stride < (long long)B * Lcap * Hkv * dh)
    return fail(MEDUSA_ERR_INVALID_ARG, "layer_stride smaller than one layer's cache");
  if (B == 0 || n_layers == 0) return MEDUSA_OK;
  if (!k_caches || !v_caches || !prefix_len || !accept_len || !accept_nodes)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return kv_compact_launch(k_caches, v_caches, prefix_len, accept_len, accept_nodes, B, Hkv, dh,
                           Lcap, K, dtype, new_len, (cudaStream_t)stream, n_layers,
                           n_layers > 1 ? layer_stride : 0);
}

int medusa_topk_merge(const float* val, const int32_t* idx, long long shard_stride,
                      const int32_t* v0, int G, int R, int c, int s, int32_t* out_idx,
                      float* out_val, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_topk_merge");
  if (G < 1 || R < 0 || c < 1 || s < 1 || s > MEDUSA_MAX_S || (long long)G * c > (1LL << 30))
    return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (shard_stride < (long long)R * c) return fail(MEDUSA_ERR_INVALID_ARG, "shard_stride < R * c");
  if (R == 0) return MEDUSA_OK;
  if (!val || !idx || !out_idx) return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return topk_merge_launch(val, idx, shard_stride, v0, G, R, c, s, out_idx, out_val,
                           (cudaStream_t)stream);
}

int medusa_sample_next(const void* vlogits, int dtype, const int32_t* accept_len,
                       const int32_t* accept_nodes, int B, int N, int V, int K,
                       float temperature, uint64_t seed, uint64_t offset,
                       const uint64_t* offset_dev, int32_t* next_tok, void* stream) {
  medusa::NvtxRange nvtx_range("medusa_sample_next");
  if (!dtype_ok(dtype)) return fail(MEDUSA_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || N <= 0 || N > MEDUSA_MAX_N || V <= 0 || K < 0 || K > MEDUSA_MAX_K)
    return fail(MEDUSA_ERR_INVALID_ARG, "bad shape");
  if (!(temperature >= 0.f) || !std::isfinite(temperature))
    return fail(MEDUSA_ERR_INVALID_ARG, "temperature must be finite and >= 0");
  if (B == 0) return MEDUSA_OK;
  if (!vlogits || !accept_len || !accept_nodes || !next_tok)
    return fail(MEDUSA_ERR_INVALID_ARG, "NULL pointer");
  return sample_next_launch(vlogits, dtype, accept_len, accept_nodes, B, N, V, K, temperature,
                            seed, offset, offset_dev, next_tok, (cudaStream_t)stream);
}

}  // extern "C"

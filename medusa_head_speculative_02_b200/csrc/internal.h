// Internal declarations shared by the host API and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <string>
#include <vector>

#include "../../include/medusa.h"

struct medusa_tree {
  int K = 0, s = 0, N = 0, W = 0;  // W = 32-bit words per ancestor-mask row
  int device = -1;
  std::vector<int32_t> parent, depth, rank_path, head_rank;
  std::vector<int32_t> nchild;  // children of every node (0: a leaf)
  std::vector<uint32_t> anc;
  // device copies (one allocation owned by the plan)
  void* d_block = nullptr;
  const int32_t* d_parent = nullptr;
  const int32_t* d_depth = nullptr;
  const int32_t* d_head_rank = nullptr;  // (D-1)*s + r_D, -1 for the root
  const int32_t* d_nchild = nullptr;
  const uint32_t* d_anc = nullptr;
};

namespace medusa {

// Thread-local error message plumbing (defined in medusa_api.cu).
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);
int num_sms();

// Raises `kernel`'s dynamic shared-memory limit to `bytes` once per device;
// `done` is the call site's own per-device flag array (safe to call from
// several host threads).
template <typename K>
int ensure_max_smem(K* kernel, int bytes, std::atomic<bool> (&done)[64], const char* what) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MEDUSA_ERR_UNSUPPORTED, "device ordinal >= 64");
  if (!done[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    done[dev].store(true, std::memory_order_release);
  }
  return MEDUSA_OK;
}

// Launches a kernel of this library with programmatic stream serialization:
// it may be scheduled before the kernel ahead of it in the stream has
// finished, once every CTA of that kernel has signalled
// griddepcontrol.launch_dependents (or exited).  Every kernel launched this
// way executes griddepcontrol.wait before its first access to memory that
// another kernel of the library writes, and signals its dependents only
// after taking its TMEM, so a waiting CTA never holds resources its
// predecessor still needs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Carves 256-byte-aligned segments out of a caller workspace.
struct WsCarver {
  size_t off = 0;
  template <typename T>
  size_t take(size_t count) {
    off = (off + 255) & ~(size_t)255;
    size_t at = off;
    off += count * sizeof(T);
    return at;
  }
  size_t total() const { return (off + 255) & ~(size_t)255; }
};

// ---------------------------------------------------------------- heads
struct HeadsArgs {
  const void* h;
  const void* W1;
  const void* b1;
  const void* W2;
  int B, d, V, K, dtype;
  float* logits;
  int s;
  int32_t* topk_idx;
  float* topk_val;
  void* ws;
  size_t ws_bytes;
};
size_t heads_tc_workspace(int B, int d, int V, int K, int s);
int heads_tc_launch(const HeadsArgs& a, cudaStream_t st);
// large batch (bf16, B > 32): compute-bound GEMMs with N = 256 (csrc/heads_big.cu)
size_t heads_big_workspace(int B, int d, int V, int K, int s);
int heads_big_launch(const HeadsArgs& a, cudaStream_t st);
size_t heads_simt_workspace(int B, int d, int V, int K, int s);
int heads_simt_launch(const HeadsArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- top-s
int topk_rows_launch(const void* x, int dtype, int R, int V, int s, int32_t* idx, float* val,
                     cudaStream_t st);
int topk_keys_launch(const uint64_t* keys, int R, int C, int s, int32_t* idx, float* val,
                     cudaStream_t st);

// ---------------------------------------------------------------- tree
int build_tree_launch(const medusa_tree* t, const int32_t* root, const int32_t* topk,
                      const int32_t* L, int B, int32_t* tok, int32_t* pos, cudaStream_t st);

// ---------------------------------------------------------------- attention
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* L;
  const medusa_tree* tree;
  int B, Hq, Hkv, dh, Lcap;
  float scale;
  int dtype;
  void* out;
  void* ws;
  size_t ws_bytes;
};
size_t attention_workspace(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap,
                           int dtype);
int attention_launch(const AttnArgs& a, cudaStream_t st);
int attention_chunks(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap, int dtype);
int attention_launches(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap, int dtype);
int attention_tiles_per_cta(const medusa_tree* t, int B, int Hq, int Hkv, int dh, int Lcap,
                            int dtype);
// tcgen05 path (bf16, dh = 128, GQA group dividing 128)
bool attention_tc_eligible(int dtype, int dh, int Hq, int Hkv);
int attention_tc_chunks(int B, int Hq, int Hkv, int N, int Lcap);
// Launch shape of the tensor-core attention: P key chunks per query tile,
// `tiles` (1 or 2) 128-row query tiles per CTA, and whether the chunks of a
// query tile run as one thread-block cluster and merge inside the kernel
// (else, with P > 1, the combine kernel merges them; two-tile shapes with
// P > 1 always merge in-cluster).
struct TcShape {
  int P;
  int tiles;
  bool fuse;
};
TcShape attention_tc_shape(int B, int Hq, int Hkv, int N, int Lcap);
int attention_tc_run(const AttnArgs& a, const TcShape& sh, float* po, float2* pml,
                     cudaStream_t st);

// ---------------------------------------------------------------- acceptance
struct AcceptArgs {
  const void* vlog;
  int dtype;
  const int32_t* tok;
  const medusa_tree* tree;
  int B, V;
  bool typical;
  float temps[MEDUSA_MAX_K];  // typical: temperature of the candidates of depth 1..K
  float eps, delta;
  int32_t* accept_len;
  int32_t* accept_nodes;
  int32_t* next_tok;
  // typical only: also the greedy results from the same row reduction
  // (null: none)
  int32_t* g_accept_len = nullptr;
  int32_t* g_accept_nodes = nullptr;
  int32_t* g_next_tok = nullptr;
  void* ws;
  size_t ws_bytes;
};
size_t accept_workspace(const medusa_tree* t, int B, int V);
int accept_launch(const AcceptArgs& a, cudaStream_t st);
int accept_greedy_noalloc_launch(const void* vlog, int dtype, const int32_t* tok,
                                 const medusa_tree* t, int B, int V, int32_t* accept_len,
                                 int32_t* accept_nodes, int32_t* next_tok, cudaStream_t st);

// ---------------------------------------------------------------- compaction
// layers caches, layer_stride elements apart (1 layer: stride unused)
int kv_compact_launch(void* k, void* v, const int32_t* L, const int32_t* alen,
                      const int32_t* anodes, int B, int Hkv, int dh, int Lcap, int K,
                      int dtype, int32_t* new_len, cudaStream_t st, int layers = 1,
                      long long layer_stride = 0);

// ---------------------------------------------------------------- TMA descriptors
// Encodes a bf16 tensor map (dims innermost first) with 128-byte swizzling.
// merge of per-shard top-s candidate lists (csrc/topk.cu)
int topk_merge_launch(const float* val, const int32_t* idx, long long gs, const int32_t* v0, int G,
                      int R, int c, int s, int32_t* out_idx, float* out_val, cudaStream_t st);

// sampled next token (csrc/sample.cu)
int sample_next_launch(const void* vlog, int dtype, const int32_t* alen, const int32_t* anodes,
                       int B, int N, int V, int K, float temperature, uint64_t seed,
                       uint64_t offset, const uint64_t* offset_dev, int32_t* next_tok,
                       cudaStream_t st);

int make_tmap_bf16(void* map /* CUtensorMap* */, const void* base, int rank,
                   const uint64_t* dims, const uint64_t* strides_bytes,
                   const uint32_t* box);

}  // namespace medusa

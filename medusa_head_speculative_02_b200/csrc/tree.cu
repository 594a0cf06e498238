// Tree expansion.  Medusa paper digest ("論文解説: Medusa"), section
// "ツリーアテンションによる並列検証": the tree nodes are rank tuples over the
// heads' top-s candidates.  Node n at depth D >= 1 with last rank r_D takes
// the rank-r_D token of head D-1 (0-based; head D-1 predicts depth D), the
// root keeps the token already produced; position = prefix length + depth.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

__global__ void build_tree_kernel(const int32_t* __restrict__ head_rank,
                                  const int32_t* __restrict__ depth,
                                  const int32_t* __restrict__ root,
                                  const int32_t* __restrict__ topk,
                                  const int32_t* __restrict__ L, int B, int N, int Ks,
                                  int32_t* __restrict__ tok, int32_t* __restrict__ pos) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * N) return;
  const int b = i / N, n = i - b * N;
  const int hr = head_rank[n];
  if (!dbg_ok(hr >= -1 && hr < Ks, DBG_TREE_HEAD_RANK)) return;
  tok[i] = hr < 0 ? root[b] : topk[(size_t)b * Ks + hr];
  if (pos) pos[i] = L[b] + depth[n];
}

}  // namespace

int build_tree_launch(const medusa_tree* t, const int32_t* root, const int32_t* topk,
                      const int32_t* L, int B, int32_t* tok, int32_t* pos, cudaStream_t st) {
  const int total = B * t->N;
  if (total == 0) return MEDUSA_OK;
  cudaError_t e = launch_pdl(build_tree_kernel, dim3((total + 255) / 256), dim3(256), 0, st,
                             t->d_head_rank, t->d_depth, root, topk, L, B, t->N, t->K * t->s, tok,
                             pos);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "build_tree_kernel launch");
}

}  // namespace medusa

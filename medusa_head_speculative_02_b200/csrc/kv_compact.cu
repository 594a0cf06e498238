// KV-cache compaction of the accepted path.  The verified tree's K/V sit at
// slots L_b..L_b+N-1 (node j at L_b + j); after acceptance the path nodes
// n_1..n_a must become the contiguous continuation L_b+1..L_b+a of the root
// (explainer "メドゥーサ デコーディング ヘッド", "ディープダイブ": the longest
// matching prefix is kept).
//
// Copies are bit-exact.  Each thread owns one 16-byte (or 4-byte) column of
// the slot and walks j = 1..a in order; since n_j >= j for a path in a
// topologically numbered tree, a slot is always read before it is
// overwritten within that column, so no cross-thread ordering is needed.
// With several layers (grid z), every layer's cache gets the same moves:
// the tree is verified by every layer of the base model, and the accepted
// path is kept in each of them.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

template <typename VecT>
__global__ void kv_compact_kernel(VecT* __restrict__ kc, VecT* __restrict__ vc,
                                  const int32_t* __restrict__ L,
                                  const int32_t* __restrict__ alen,
                                  const int32_t* __restrict__ anodes, int Lcap, int K,
                                  size_t slot_vecs, size_t layer_vecs,
                                  int32_t* __restrict__ new_len) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  const int b = blockIdx.y;
  const int layer = blockIdx.z;
  const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int a = alen[b];
  const int Lb = L[b];
  const bool valid = a >= 0 && a <= K && Lb >= 0;
  if (x == 0 && layer == 0 && new_len) new_len[b] = valid ? Lb + 1 + a : -1;
  if (!valid || x >= slot_vecs) return;
  VecT* kb = kc + (size_t)layer * layer_vecs + (size_t)b * Lcap * slot_vecs + x;
  VecT* vb = vc + (size_t)layer * layer_vecs + (size_t)b * Lcap * slot_vecs + x;
  for (int j = 1; j <= a; ++j) {
    const int n = anodes[(size_t)b * (K + 1) + j];
    const long long src = (long long)Lb + n, dst = (long long)Lb + j;
    const bool in_range = n >= j && src < Lcap && dst < Lcap;
    if (x == 0) dbg_ok(in_range, DBG_COMPACT_NODE);  // debug builds: record the bad entry
    if (!in_range) continue;
    kb[dst * slot_vecs] = kb[src * slot_vecs];
    vb[dst * slot_vecs] = vb[src * slot_vecs];
  }
}

}  // namespace

int kv_compact_launch(void* k, void* v, const int32_t* L, const int32_t* alen,
                      const int32_t* anodes, int B, int Hkv, int dh, int Lcap, int K, int dtype,
                      int32_t* new_len, cudaStream_t st, int layers, long long layer_stride) {
  if (B == 0 || layers == 0) return MEDUSA_OK;
  const size_t esize = dtype == MEDUSA_F32 ? 4 : 2;
  const size_t slot_bytes = (size_t)Hkv * dh * esize;
  const size_t layer_bytes = (size_t)layer_stride * esize;
  const bool v16 = (slot_bytes % 16 == 0) && (layer_bytes % 16 == 0) &&
                   ((((uintptr_t)k) | ((uintptr_t)v)) % 16 == 0);
  cudaError_t e;
  if (v16) {
    const size_t nv = slot_bytes / 16;
    dim3 grid((unsigned)((nv + 127) / 128), B, layers);
    e = launch_pdl(kv_compact_kernel<uint4>, grid, dim3(128), 0, st, (uint4*)k, (uint4*)v, L, alen,
                   anodes, Lcap, K, nv, layer_bytes / 16, new_len);
  } else {
    const size_t nv = slot_bytes / 4;
    dim3 grid((unsigned)((nv + 127) / 128), B, layers);
    e = launch_pdl(kv_compact_kernel<uint32_t>, grid, dim3(128), 0, st, (uint32_t*)k, (uint32_t*)v,
                   L, alen, anodes, Lcap, K, nv, layer_bytes / 4, new_len);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "kv_compact_kernel launch");
}

}  // namespace medusa

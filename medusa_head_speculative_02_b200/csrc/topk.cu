// Top-s selection.  Medusa paper digest ("論文解説: Medusa"), section
// "ツリーアテンションによる並列検証": each head contributes its s most likely
// tokens.  Order: value descending, ties to the lower index, encoded in one
// 64-bit key per element so a single unsigned compare decides.
//
// One CTA per row: every thread keeps a sorted register list of its best s
// keys while streaming its strided share of the row (16-byte vector loads
// when the row is aligned), then s rounds of a block-wide max pop the winners.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kSmax = MEDUSA_MAX_S;
constexpr int kThreads = 256;

// s rounds: block max of every thread's best remaining key; the owner pops it.
__device__ __forceinline__ void block_select(uint64_t (&k)[kSmax], int s, uint64_t* red, int32_t* idx_out,
                             float* val_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j = 0; j < s; ++j) {
    const uint64_t m = warp_max_u64(k[0]);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    uint64_t best = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) best = red[w] > best ? red[w] : best;
    if (best != 0ull && k[0] == best) topk_pop<kSmax>(k);
    if (threadIdx.x == 0) {
      idx_out[j] = best ? (int32_t)key_index(best) : -1;
      if (val_out) val_out[j] = best ? key_value(best) : __int_as_float(0x7fc00000);
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) topk_rows_kernel(const T* __restrict__ x, int V, int s,
                                                             int32_t* __restrict__ idx,
                                                             float* __restrict__ val) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint64_t red[kThreads / 32];
  const size_t row = blockIdx.x;
  const T* xr = x + row * (size_t)V;
  uint64_t k[kSmax];
#pragma unroll
  for (int i = 0; i < kSmax; ++i) k[i] = 0ull;
  uint64_t kth = 0ull;
  constexpr int VEC = 16 / sizeof(T);
  if ((V % VEC) == 0 && (((uintptr_t)xr) & 15u) == 0) {
    const int nv = V / VEC;
    for (int i = threadIdx.x; i < nv; i += kThreads) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(xr) + i);
      const T* e = reinterpret_cast<const T*>(&w);
#pragma unroll
      for (int j = 0; j < VEC; ++j) {
        const uint64_t key = make_key(to_f32(e[j]), (uint32_t)(i * VEC + j));
        if (key > kth) topk_insert<kSmax>(k, s, key, kth);
      }
    }
  } else {
    for (int i = threadIdx.x; i < V; i += kThreads) {
      const uint64_t key = make_key(to_f32(xr[i]), (uint32_t)i);
      if (key > kth) topk_insert<kSmax>(k, s, key, kth);
    }
  }
  block_select(k, s, red, idx + row * s, val ? val + row * s : nullptr);
}

// Rows of pre-built candidate keys (0 = empty).
__global__ void __launch_bounds__(kThreads) topk_keys_kernel(const uint64_t* __restrict__ keys,
                                                             int C, int s,
                                                             int32_t* __restrict__ idx,
                                                             float* __restrict__ val) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint64_t red[kThreads / 32];
  const size_t row = blockIdx.x;
  const uint64_t* kr = keys + row * (size_t)C;
  uint64_t k[kSmax];
#pragma unroll
  for (int i = 0; i < kSmax; ++i) k[i] = 0ull;
  uint64_t kth = 0ull;
  // 8 independent loads in flight per thread before any insertion
  for (int base = threadIdx.x; base < C; base += 8 * kThreads) {
    uint64_t kk[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * kThreads;
      kk[u] = i < C ? __ldcg(kr + i) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (kk[u] > kth) topk_insert<kSmax>(k, s, kk[u], kth);
  }
  block_select(k, s, red, idx + row * s, val ? val + row * s : nullptr);
}

// Candidate lists of G shards: shard g's list for row r is val / idx
// [g * gs + r * c .. + c) (index < 0: empty slot).  The row's s best by value
// descending, ties to the lower index; shard g's indices are offset by v0[g]
// (device array) when v0 is given.
__global__ void __launch_bounds__(kThreads)
    topk_merge_kernel(const float* __restrict__ val, const int32_t* __restrict__ idx,
                      long long gs, const int32_t* __restrict__ v0, int G, int R, int c, int s,
                      int32_t* __restrict__ out_idx, float* __restrict__ out_val) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint64_t red[kThreads / 32];
  const int row = blockIdx.x;
  uint64_t k[kSmax];
#pragma unroll
  for (int i = 0; i < kSmax; ++i) k[i] = 0ull;
  uint64_t kth = 0ull;
  const int C = G * c;
  for (int t = threadIdx.x; t < C; t += kThreads) {
    const int g = t / c, j = t - g * c;
    const size_t o = (size_t)g * (size_t)gs + (size_t)row * c + j;
    const int i = idx[o];
    if (i < 0) {
      dbg_ok(i == -1, DBG_MERGE_SHARD);  // -1 marks an empty slot; lower ids are malformed
      continue;
    }
    const uint64_t key = make_key(val[o], (uint32_t)(i + (v0 ? v0[g] : 0)));
    if (key > kth) topk_insert<kSmax>(k, s, key, kth);
  }
  block_select(k, s, red, out_idx + (size_t)row * s, out_val ? out_val + (size_t)row * s : nullptr);
}

}  // namespace

int topk_merge_launch(const float* val, const int32_t* idx, long long gs, const int32_t* v0, int G,
                      int R, int c, int s, int32_t* out_idx, float* out_val, cudaStream_t st) {
  if (R == 0) return MEDUSA_OK;
  cudaError_t e = launch_pdl(topk_merge_kernel, dim3(R), dim3(kThreads), 0, st, val, idx, gs, v0, G,
                             R, c, s, out_idx, out_val);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "topk_merge_kernel launch");
}

int topk_rows_launch(const void* x, int dtype, int R, int V, int s, int32_t* idx, float* val,
                     cudaStream_t st) {
  if (R == 0) return MEDUSA_OK;
  cudaError_t e;
  if (dtype == MEDUSA_F32)
    e = launch_pdl(topk_rows_kernel<float>, dim3(R), dim3(kThreads), 0, st, (const float*)x, V, s,
                   idx, val);
  else
    e = launch_pdl(topk_rows_kernel<__nv_bfloat16>, dim3(R), dim3(kThreads), 0, st,
                   (const __nv_bfloat16*)x, V, s, idx, val);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "topk_rows_kernel launch");
}

int topk_keys_launch(const uint64_t* keys, int R, int C, int s, int32_t* idx, float* val,
                     cudaStream_t st) {
  if (R == 0) return MEDUSA_OK;
  cudaError_t e = launch_pdl(topk_keys_kernel, dim3(R), dim3(kThreads), 0, st, keys, C, s, idx, val);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "topk_keys_kernel launch");
}

}  // namespace medusa

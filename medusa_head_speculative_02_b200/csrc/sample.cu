// Sampled next token.
//
// Page "Medusa：基于多Token预测的LLM推理加速", section "3.3 贪婪vs采样验证":
// greedy verification takes the argmax of the logits, sampling verification
// draws the token from softmax(logits / temperature).  The token is drawn
// from the verify row of the last accepted node n_a = accept_nodes[b][a],
// a = accept_len[b].
//
// The draw is the Gumbel-max construction: argmax_v (l_v / T + G_v) with
// G_v = -log(-log(U_v)) i.i.d. standard Gumbel is distributed exactly as
// softmax(l / T).  U_v comes from the counter-based SplitMix64 generator
// (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
// OOPSLA 2014): output number ((offset * B) + b) * V + v of the generator
// started at `seed`, its top 23 bits t mapped to (t + 1/2) * 2^-23, exact in
// fp32 and strictly inside (0, 1).  Every vocabulary entry has its own
// counter, so the draw needs no prefix sum: a cluster of 8 CTAs per sequence
// streams its row once, z_v = fl(fl(l_v * (1/T)) + G_v) in fp32, and the
// argmax (lowest index on ties) is merged through distributed shared memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace medusa {
namespace {

constexpr int kThreads = 512;
constexpr int kCluster = 8;  // CTAs per sequence (portable cluster size)

__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t idx) {
  uint64_t z = seed + (idx + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Grid (B, kCluster): the kCluster CTAs of one sequence form a thread-block
// cluster; each folds one slice of the row, then CTA rank 0 of the cluster
// reads the others' best keys from their shared memory (DSMEM).
template <typename T>
__global__ void __launch_bounds__(kThreads)
    sample_next_kernel(const T* __restrict__ vlog, const int32_t* __restrict__ alen,
                       const int32_t* __restrict__ anodes, int B, int N, int V, int K,
                       int greedy, float inv_t, uint64_t seed, uint64_t offset,
                       const uint64_t* __restrict__ offset_dev, int32_t* __restrict__ next_tok) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  if (offset_dev) offset += *offset_dev;
  __shared__ uint64_t red[kThreads / 32];
  __shared__ uint64_t cta_best;
  cg::cluster_group cluster = cg::this_cluster();
  const int b = blockIdx.x;
  const int part = (int)cluster.block_rank();
  const int a = alen[b];
  const int node = (a >= 0 && a <= K) ? anodes[(size_t)b * (K + 1) + a] : -1;
  const bool valid = node >= 0 && node < N;  // uniform over the cluster
  if (part == 0 && threadIdx.x == 0) dbg_ok(valid, DBG_SAMPLE_NODE);
  uint64_t best = 0ull;
  if (valid) {
    const T* row = vlog + ((size_t)b * N + node) * (size_t)V;
    const uint64_t base = (offset * (uint64_t)B + (uint64_t)b) * (uint64_t)V;
    const int per = (V + kCluster - 1) / kCluster;
    const int lo = part * per, hi = min(V, lo + per);
    // independent entries: unrolled so their generator / log chains overlap
#pragma unroll 4
    for (int v = lo + (int)threadIdx.x; v < hi; v += kThreads) {
      const float x = to_f32(row[v]);
      float z = x;
      if (!greedy) {
        const uint32_t t = (uint32_t)(splitmix64_at(seed, base + (uint64_t)v) >> 41);
        const float u = ((float)t + 0.5f) * 1.1920928955078125e-07f;  // 2^-23
        const float g = -logf(-logf(u));
        z = __fadd_rn(__fmul_rn(x, inv_t), g);
      }
      const uint64_t key = make_key(z, (uint32_t)v);
      best = key > best ? key : best;
    }
  }
  best = warp_max_u64(best);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kThreads / 32; ++w) best = red[w] > best ? red[w] : best;
    cta_best = best;
  }
  cluster.sync();  // every CTA's best key is in its shared memory
  if (part == 0 && threadIdx.x == 0) {
    uint64_t k = 0ull;
    for (int r = 0; r < kCluster; ++r) {
      const uint64_t other = *cluster.map_shared_rank(&cta_best, r);
      k = other > k ? other : k;
    }
    next_tok[b] = valid ? (int32_t)key_index(k) : -1;
  }
  cluster.sync();  // the peers' shared memory stays live until rank 0 has read it
}

}  // namespace

int sample_next_launch(const void* vlog, int dtype, const int32_t* alen, const int32_t* anodes,
                       int B, int N, int V, int K, float temperature, uint64_t seed,
                       uint64_t offset, const uint64_t* offset_dev, int32_t* next_tok,
                       cudaStream_t st) {
  if (B == 0) return MEDUSA_OK;
  const int greedy = temperature == 0.f ? 1 : 0;
  const float inv_t = greedy ? 0.f : 1.f / temperature;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B, kCluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = kCluster;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  if (dtype == MEDUSA_F32)
    e = cudaLaunchKernelEx(&cfg, sample_next_kernel<float>, (const float*)vlog, alen, anodes, B, N,
                           V, K, greedy, inv_t, seed, offset, offset_dev, next_tok);
  else
    e = cudaLaunchKernelEx(&cfg, sample_next_kernel<__nv_bfloat16>, (const __nv_bfloat16*)vlog,
                           alen, anodes, B, N, V, K, greedy, inv_t, seed, offset, offset_dev,
                           next_tok);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MEDUSA_OK : cuda_fail(e, "sample_next_kernel launch");
}

}  // namespace medusa

// Medusa heads in fp32 (SIMT).  Medusa paper digest ("論文解説: Medusa"),
// section "Medusa Headのアーキテクチャ":
//   u_k[b] = SiLU(W1_k h[b] + b1_k) + h[b],   logits_k[b] = W2_k u_k[b].
// One warp per output row (all B batch columns at once, float4 loads of the
// weight row), then the row top-s kernel over the logits.  The fp32 path
// serves small models; bf16 goes through the tcgen05 kernels.
#include "common.cuh"
#include "internal.h"

namespace medusa {
namespace {

constexpr int kBmax = 16;
constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// rows: `nrow` weight rows of length d (W[kh] block of `rows_per_head`);
// x: [K][B][d] activations (stride_k = 0 when shared by every head).
// stage 1 writes u[kh][b][m] = SiLU(acc + b1) + h; stage 2 writes
// logits[b][kh][m] = acc.
__global__ void __launch_bounds__(kWarps * 32)
    heads_simt_kernel(int stage, const float* __restrict__ W, const float* __restrict__ x,
                      size_t x_stride_k, const float* __restrict__ b1,
                      const float* __restrict__ h, float* __restrict__ out, int B, int d,
                      int rows_per_head, int K) {
  // nothing in this kernel runs ahead of its predecessor
  griddep_launch_dependents();
  griddep_wait();
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= K * rows_per_head) return;
  const int kh = gw / rows_per_head, m = gw - kh * rows_per_head;
  const float4* wr = reinterpret_cast<const float4*>(W + (size_t)gw * d);
  const float* xk = x + (size_t)kh * x_stride_k;
  float acc[kBmax];
#pragma unroll
  for (int b = 0; b < kBmax; ++b) acc[b] = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 w = __ldg(wr + i);
#pragma unroll
    for (int b = 0; b < kBmax; ++b) {
      if (b < B) {
        const float4 xv = __ldg(reinterpret_cast<const float4*>(xk + (size_t)b * d) + i);
        acc[b] += w.x * xv.x + w.y * xv.y + w.z * xv.z + w.w * xv.w;
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kBmax; ++b) {
    if (b < B) {
      const float a = warp_sum(acc[b]);
      if (lane == 0) {
        if (stage == 1) {
          const float z = a + (b1 ? b1[(size_t)kh * d + m] : 0.f);
          out[((size_t)kh * B + b) * d + m] = z / (1.f + expf(-z)) + h[(size_t)b * d + m];
        } else {
          out[((size_t)b * K + kh) * rows_per_head + m] = a;
        }
      }
    }
  }
}

struct SimtPlan {
  size_t off_u, off_logits, total;
};

SimtPlan make_plan(int B, int d, int V, int K) {
  SimtPlan P;
  WsCarver w;
  P.off_u = w.take<float>((size_t)K * B * d);
  P.off_logits = w.take<float>((size_t)B * K * V);
  P.total = w.total();
  return P;
}

}  // namespace

size_t heads_simt_workspace(int B, int d, int V, int K, int /*s*/) {
  return make_plan(B, d, V, K).total;
}

int heads_simt_launch(const HeadsArgs& a, cudaStream_t st) {
  if (a.B > kBmax) return fail(MEDUSA_ERR_UNSUPPORTED, "fp32 heads support B <= 16");
  const SimtPlan P = make_plan(a.B, a.d, a.V, a.K);
  if (a.ws_bytes < P.total) return fail(MEDUSA_ERR_INVALID_ARG, "workspace too small for heads");
  uint8_t* ws = (uint8_t*)a.ws;
  float* u = (float*)(ws + P.off_u);
  float* logits = a.logits ? a.logits : (float*)(ws + P.off_logits);
  const int rows1 = a.K * a.d, rows2 = a.K * a.V;
  cudaError_t e = launch_pdl(heads_simt_kernel, dim3((rows1 + kWarps - 1) / kWarps),
                             dim3(kWarps * 32), 0, st, 1, (const float*)a.W1, (const float*)a.h,
                             (size_t)0, (const float*)a.b1, (const float*)a.h, u, a.B, a.d, a.d,
                             a.K);
  if (e == cudaSuccess)
    e = launch_pdl(heads_simt_kernel, dim3((rows2 + kWarps - 1) / kWarps), dim3(kWarps * 32), 0, st,
                   2, (const float*)a.W2, (const float*)u, (size_t)a.B * a.d,
                   (const float*)nullptr, (const float*)nullptr, logits, a.B, a.d, a.V, a.K);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "heads_simt_kernel launch");
  if (a.topk_idx)
    return topk_rows_launch(logits, MEDUSA_F32, a.B * a.K, a.V, a.s, a.topk_idx, a.topk_val, st);
  return MEDUSA_OK;
}

}  // namespace medusa

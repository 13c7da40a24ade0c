// Grouped GEMM on CUDA cores for fp32 layers.  The tensor cores have no
// full-fp32 multiply (tf32 keeps 10 mantissa bits), so fp32 layers take this
// path: one thread per output element, fp32 FMA over k = 0..K-1 in order.
// Same epilogues as the tensor-core engine (ReLU / SwiGLU for the first
// projection, gate scaling for the second).  Meant for small fp32 layers.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__device__ __forceinline__ int expert_of_row(const int32_t* __restrict__ offsets, int E, int r) {
  int lo = 0, hi = E;  // offsets[lo] <= r < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= r) lo = mid; else hi = mid;
  }
  return lo;
}

template <int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(int E, int N, int K, const float* __restrict__ A,
                                                        const float* __restrict__ B0, const float* __restrict__ B1,
                                                        float* __restrict__ out, const int32_t* __restrict__ offsets,
                                                        const float* __restrict__ row_gate) {
  const int n = blockIdx.x * 32 + threadIdx.x;
  const int r = blockIdx.y * 8 + threadIdx.y;
  pdl_wait();
  pdl_trigger();
  if (r >= offsets[E] || n >= N) return;
  const int e = expert_of_row(offsets, E, r);
  const float* a = A + static_cast<int64_t>(r) * K;
  const float* w = B0 + (static_cast<int64_t>(e) * N + n) * K;
  float acc = 0.f;
  for (int c = 0; c < K; ++c) acc = fmaf(a[c], w[c], acc);
  float v;
  if (EPI == EPI_RELU_BF16) {
    v = fmaxf(acc, 0.f);
  } else if (EPI == EPI_SWIGLU_BF16) {
    const float* w3 = B1 + (static_cast<int64_t>(e) * N + n) * K;
    float b = 0.f;
    for (int c = 0; c < K; ++c) b = fmaf(a[c], w3[c], b);
    v = acc / (1.f + expf(-acc)) * b;
  } else {
    v = acc * row_gate[r];
  }
  out[static_cast<int64_t>(r) * N + n] = v;
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs& g, int64_t s_max, cudaStream_t s) {
  const dim3 block(32, 8);
  const dim3 grid(static_cast<unsigned>((g.N + 31) / 32), static_cast<unsigned>((s_max + 7) / 8));
  const float* A = static_cast<const float*>(g.A);
  const float* B0 = static_cast<const float*>(g.B0);
  const float* B1 = static_cast<const float*>(g.B1);
  float* out = static_cast<float*>(g.out);
  switch (g.epi) {
    case EPI_RELU_BF16:
      return launch_pdl(simt_gemm_kernel<EPI_RELU_BF16>, grid, block, 0, s, g.E, g.N, g.K, A, B0, B1, out, g.offsets,
                        g.row_gate);
    case EPI_SWIGLU_BF16:
      return launch_pdl(simt_gemm_kernel<EPI_SWIGLU_BF16>, grid, block, 0, s, g.E, g.N, g.K, A, B0, B1, out,
                        g.offsets, g.row_gate);
    default:
      return launch_pdl(simt_gemm_kernel<EPI_GATE_F32>, grid, block, 0, s, g.E, g.N, g.K, A, B0, B1, out, g.offsets,
                        g.row_gate);
  }
}

}  // namespace moe

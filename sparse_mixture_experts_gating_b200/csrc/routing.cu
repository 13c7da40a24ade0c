// Routing kernels of the MoE layer forward pass:
//   router   - fp32 router logits h = W_r x (+ b), softmax, log-sum-exp, top-k
//              (ties -> lower expert index), gates, per-block counts and sums
//   scan     - per-expert totals, stable per-block rank bases, capacity,
//              expert offsets, tile prefix, aux loss and z-loss
//   dispatch - slot rank of each (token, choice) in token order, drop mask,
//              permute of the kept token rows into expert-sorted order
//   combine  - y_t = sum over kept choices j (in order j) of the gated expert rows
// Layer definition: "Mixture of experts" (rayaq.ca), sections "Replacing the
// feed-forward block", "Top-k gating", "The load-balancing loss", "Capacity
// and dropped tokens", "Implementation".
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BT = kRouterTokens;  // tokens per router block
constexpr int KC = 32;             // d-chunk staged in shared memory
constexpr int KP = KC + 4;         // padded row (keeps 16-byte alignment)
constexpr int TT = 4;              // tokens per thread in the logits tile
constexpr int RT = 128;            // router threads

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Router.  One block = BT tokens.  Phase 1: the [BT x E] logits tile on CUDA
// cores in fp32 (each logit summed over c = 0..d-1 in order).  Phase 2: one
// warp per token for softmax, log-sum-exp, top-k and gates.
// TE = experts per thread (E padded to 16*TE); NQ = logits per lane in phase 2.
template <typename XT, int TE>
__global__ void __launch_bounds__(RT) router_kernel(RoutingArgs a) {
  constexpr int EP = 16 * TE;
  constexpr int NQ = (EP + 31) / 32;
  constexpr int LP = EP + 1;
  extern __shared__ __align__(16) float sm[];
  float* x_s = sm;                       // [BT][KP]
  float* w_s = x_s + BT * KP;            // [EP][KP]
  float* l_s = w_s + EP * KP;            // [BT][LP]
  float* ps_s = l_s + BT * LP;           // [4][EP]
  float* lse2_s = ps_s + 4 * EP;         // [4]
  int* cnt1_s = reinterpret_cast<int*>(lse2_s + 4);  // [EP]
  int* hist_s = cnt1_s + EP;                          // [EP]

  const int tid = threadIdx.x;
  const int E = a.E, d = a.d, k = a.k;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * BT;
  const int nt = static_cast<int>((a.T - t0) < BT ? (a.T - t0) : BT);
  const XT* x = static_cast<const XT*>(a.x);

  for (int e = tid; e < EP; e += RT) { cnt1_s[e] = 0; hist_s[e] = 0; }

  if (a.logits_in == nullptr) {
    const int tg = tid >> 4, eg = tid & 15;
    float acc[TT][TE];
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
      for (int j = 0; j < TE; ++j) acc[i][j] = 0.f;

    for (int c0 = 0; c0 < d; c0 += KC) {
      for (int i = tid; i < BT * KC; i += RT) {
        const int t = i / KC, c = i % KC;
        float v = 0.f;
        if (t < nt && c0 + c < d) v = to_f32(x[(t0 + t) * d + c0 + c]);
        x_s[t * KP + c] = v;
      }
      for (int i = tid; i < EP * KC; i += RT) {
        const int e = i / KC, c = i % KC;
        float v = 0.f;
        if (e < E && c0 + c < d) v = a.W_r[static_cast<int64_t>(e) * d + c0 + c];
        w_s[e * KP + c] = v;
      }
      __syncthreads();
#pragma unroll
      for (int cc = 0; cc < KC; cc += 4) {
        float4 xv[TT], wv[TE];
#pragma unroll
        for (int i = 0; i < TT; ++i) xv[i] = *reinterpret_cast<const float4*>(&x_s[(tg * TT + i) * KP + cc]);
#pragma unroll
        for (int j = 0; j < TE; ++j) wv[j] = *reinterpret_cast<const float4*>(&w_s[(eg + 16 * j) * KP + cc]);
#pragma unroll
        for (int i = 0; i < TT; ++i)
#pragma unroll
          for (int j = 0; j < TE; ++j) {
            float s = acc[i][j];
            s = fmaf(xv[i].x, wv[j].x, s);
            s = fmaf(xv[i].y, wv[j].y, s);
            s = fmaf(xv[i].z, wv[j].z, s);
            s = fmaf(xv[i].w, wv[j].w, s);
            acc[i][j] = s;
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TT; ++i)
#pragma unroll
      for (int j = 0; j < TE; ++j) {
        const int e = eg + 16 * j;
        float v = acc[i][j];
        if (a.b_r != nullptr && e < E) v += a.b_r[e];
        l_s[(tg * TT + i) * LP + e] = v;
      }
  } else {
    for (int i = tid; i < BT * EP; i += RT) {
      const int t = i / EP, e = i % EP;
      l_s[t * LP + e] = (t < nt && e < E) ? a.logits_in[(t0 + t) * E + e] : 0.f;
    }
  }
  __syncthreads();

  // ---- phase 2: one warp per token
  const int warp = tid >> 5, lane = tid & 31;
  float psum[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) psum[q] = 0.f;
  float lse2 = 0.f;
  for (int t = warp; t < nt; t += RT / 32) {
    float v[NQ];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = lane + 32 * q;
      const float lv = (e < E) ? l_s[t * LP + e] : -INFINITY;
      v[q] = (lv != lv) ? -INFINITY : lv;  // NaN logits (out of contract) rank last
      m = fmaxf(m, v[q]);
    }
    m = warp_max(m);
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) s += (lane + 32 * q < E) ? expf(v[q] - m) : 0.f;
    s = warp_sum(s);
    const float lse = m + logf(s);
    const float inv_s = 1.f / s;
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (lane + 32 * q < E) psum[q] += expf(v[q] - m) * inv_s;
    lse2 += lse * lse;
    const int64_t tok = t0 + t;
    if (a.logits_out != nullptr) {
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (lane + 32 * q < E) a.logits_out[tok * E + lane + 32 * q] = v[q];
    }
    if (a.lse_out != nullptr && lane == 0) a.lse_out[tok] = lse;

    // top-k: k rounds of a warp arg-max over (value desc, index asc); lane j
    // keeps choice j.
    uint32_t picked = 0;
    float top0 = 0.f, den = 0.f, my_g = 0.f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int e = lane + 32 * q;
        if (e < E && !((picked >> q) & 1u) && (be == 0x7fffffff || v[q] > bv || (v[q] == bv && e < be))) {
          bv = v[q];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
      }
      if ((be & 31) == lane) picked |= 1u << (be >> 5);
      float g;
      if (a.gate_mode == 0) {
        g = expf(bv - m) * inv_s;  // Switch: the full-softmax probability
      } else {
        if (j == 0) top0 = bv;
        g = expf(bv - top0);       // renormalised: divided by the sum below
        den += g;
      }
      if (lane == j) { my_g = g; my_e = be; }
      if (lane == 0) {
        atomicAdd(&hist_s[be], 1);
        if (j == 0) atomicAdd(&cnt1_s[be], 1);
      }
    }
    if (lane < k) {
      a.topk_idx[tok * k + lane] = my_e;
      a.topk_gate[tok * k + lane] = (a.gate_mode == 0) ? my_g : my_g / den;
    }
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q)
    if (lane + 32 * q < EP) ps_s[warp * EP + lane + 32 * q] = psum[q];
  if (lane == 0) lse2_s[warp] = lse2;
  __syncthreads();
  const int nb = a.nblk;
  for (int e = tid; e < E; e += RT) {
    a.part_hist[e * nb + blockIdx.x] = hist_s[e];
    a.part_cnt1[e * nb + blockIdx.x] = cnt1_s[e];
    a.part_psum[e * nb + blockIdx.x] = ((ps_s[e] + ps_s[EP + e]) + ps_s[2 * EP + e]) + ps_s[3 * EP + e];
  }
  if (tid == 0) a.part_lse2[blockIdx.x] = ((lse2_s[0] + lse2_s[1]) + lse2_s[2]) + lse2_s[3];
}

template <typename XT, int TE>
cudaError_t launch_router_t(const RoutingArgs& a, cudaStream_t s) {
  constexpr int EP = 16 * TE;
  const size_t smem = sizeof(float) * (BT * KP + EP * KP + BT * (EP + 1) + 4 * EP + 4) + sizeof(int) * 2 * EP;
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(&router_kernel<XT, TE>), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  router_kernel<XT, TE><<<a.nblk, RT, smem, s>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <typename XT>
cudaError_t launch_router_x(const RoutingArgs& a, cudaStream_t s) {
  if (a.E <= 16) return launch_router_t<XT, 1>(a, s);
  if (a.E <= 32) return launch_router_t<XT, 2>(a, s);
  if (a.E <= 64) return launch_router_t<XT, 4>(a, s);
  if (a.E <= 128) return launch_router_t<XT, 8>(a, s);
  return launch_router_t<XT, 16>(a, s);
}

// ---------------------------------------------------------------------------
// Scan: one block of 1024 threads.  Warp w owns experts w, w+32, ...
__global__ void __launch_bounds__(1024) scan_kernel(RoutingArgs a) {
  __shared__ int s_counts[256];
  __shared__ int s_cnt1[256];
  __shared__ float s_psum[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, nb = a.nblk;
  pdl_wait();
  pdl_trigger();
  constexpr int V = 8;  // blocks per lane loaded ahead of the dependent scan steps
  for (int e = warp; e < E; e += 32) {
    int run = 0, c1 = 0;
    float ps = 0.f;
    for (int g0 = 0; g0 < nb; g0 += 32 * V) {
      int hv[V], cv[V];
      float pv[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {  // independent loads first
        const int b = g0 + v * 32 + lane;
        const bool in = b < nb;
        hv[v] = in ? a.part_hist[e * nb + b] : 0;
        cv[v] = in ? a.part_cnt1[e * nb + b] : 0;
        pv[v] = in ? a.part_psum[e * nb + b] : 0.f;
      }
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int b = g0 + v * 32 + lane;
        if (g0 + v * 32 >= nb) break;
        int incl = hv[v];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        if (b < nb) a.blockoff[e * nb + b] = run + incl - hv[v];
        run += __shfl_sync(0xffffffffu, incl, 31);
        c1 += warp_sum_i(cv[v]);
        ps += warp_sum(pv[v]);
      }
    }
    if (lane == 0) { s_counts[e] = run; s_cnt1[e] = c1; s_psum[e] = ps; }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0, tiles = 0, drop = 0;
    double auxp = 0.0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int cnt = e < E ? s_counts[e] : 0;
      const int kept = (a.capacity < 0) ? cnt : static_cast<int>((int64_t)cnt < a.capacity ? (int64_t)cnt : a.capacity);
      const int mt = (kept + kTileM - 1) / kTileM;
      int ik = kept, im = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, ik, o);
        const int w = __shfl_up_sync(0xffffffffu, im, o);
        if (lane >= o) { ik += u; im += w; }
      }
      if (e < E) {
        a.counts[e] = cnt;
        a.offsets[e] = base + ik - kept;
        a.mprefix[e] = tiles + im - mt;
        if (a.offsets_out != nullptr) a.offsets_out[e] = base + ik - kept;
        auxp += static_cast<double>(s_cnt1[e]) * static_cast<double>(s_psum[e]);
      }
      base += __shfl_sync(0xffffffffu, ik, 31);
      tiles += __shfl_sync(0xffffffffu, im, 31);
      drop += warp_sum_i(cnt - kept);
    }
    auxp = warp_sum_d(auxp);
    if (lane == 0) {
      a.offsets[E] = base;
      a.mprefix[E] = tiles;
      if (a.offsets_out != nullptr) a.offsets_out[E] = base;
      *a.dropped = drop;
      const double T = static_cast<double>(a.T);
      *a.aux = static_cast<float>(static_cast<double>(E) * auxp / (T * T));
    }
  } else if (warp == 1) {
    double zs = 0.0;
    for (int b = lane; b < nb; b += 32) zs += static_cast<double>(a.part_lse2[b]);
    zs = warp_sum_d(zs);
    if (lane == 0) *a.z = static_cast<float>(zs / static_cast<double>(a.T));
  }
}

// ---------------------------------------------------------------------------
// Dispatch: one block per router block of BT tokens.  Warp 0 assigns the slot
// rank of every (token, choice) of the block in token-major order (stable:
// base = number of earlier assignments to the same expert in earlier blocks);
// then all warps copy the kept rows of x into the expert-sorted buffer.
template <typename XT>
__global__ void __launch_bounds__(256) dispatch_kernel(RoutingArgs a) {
  __shared__ int run_s[256];
  __shared__ int dest_s[BT * 8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, d = a.d, nb = a.nblk;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * BT;
  const int nt = static_cast<int>((a.T - t0) < BT ? (a.T - t0) : BT);
  const int nA = nt * k;
  pdl_wait();
  pdl_trigger();
  for (int e = tid; e < E; e += 256) run_s[e] = a.blockoff[e * nb + blockIdx.x];
  __syncthreads();
  if (warp == 0) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int a0 = 0; a0 < nA; a0 += 32) {
      const int ai = a0 + lane;
      const bool valid = ai < nA;
      int e = valid ? a.topk_idx[t0 * k + ai] : -1;
      if (e < 0 || e >= E) e = -1;  // never produced by the router; keeps smem indexing in range
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const bool ok = valid && e >= 0;
      const int base = ok ? run_s[e] : 0;
      const int rank = base + __popc(peers & lt);
      __syncwarp();
      if (ok && lane == __ffs(peers) - 1) run_s[e] = base + __popc(peers);
      __syncwarp();
      if (valid && !ok) {
        dest_s[ai] = -1;
        a.dest_row[t0 * k + ai] = -1;
      } else if (valid) {
        const bool kept = a.capacity < 0 || rank < a.capacity;
        const int dest = kept ? a.offsets[e] + rank : -1;
        dest_s[ai] = dest;
        a.dest_row[t0 * k + ai] = dest;
        if (a.drop_mask != nullptr) a.drop_mask[t0 * k + ai] = kept ? 0 : 1;
        if (kept) {
          a.row_token[dest] = static_cast<int32_t>(t0 + ai / k);
          a.row_gate[dest] = a.topk_gate[t0 * k + ai];
        }
      }
    }
  }
  __syncthreads();
  const XT* x = static_cast<const XT*>(a.x);
  XT* Xp = static_cast<XT*>(a.Xp);
  XT* yz = static_cast<XT*>(a.y_zero_dropped);
  const bool vec = (static_cast<size_t>(d) * sizeof(XT)) % 16 == 0;
  for (int ai = warp; ai < nA; ai += 8) {
    const int dest = dest_s[ai];
    const int64_t tok = t0 + ai / k;
    if (dest >= 0) {
      if (vec) {
        const uint4* src = reinterpret_cast<const uint4*>(x + tok * d);
        uint4* dst = reinterpret_cast<uint4*>(Xp + static_cast<int64_t>(dest) * d);
        const int nv = static_cast<int>(static_cast<size_t>(d) * sizeof(XT) / 16);
        int v = lane;
        for (; v + 96 < nv; v += 128) {  // four independent 16-byte loads in flight per lane
          const uint4 a0 = src[v], a1 = src[v + 32], a2 = src[v + 64], a3 = src[v + 96];
          dst[v] = a0;
          dst[v + 32] = a1;
          dst[v + 64] = a2;
          dst[v + 96] = a3;
        }
        for (; v < nv; v += 32) dst[v] = src[v];
      } else {
        for (int c = lane; c < d; c += 32) Xp[static_cast<int64_t>(dest) * d + c] = x[tok * d + c];
      }
    } else if (yz != nullptr) {  // k == 1: a dropped token's output row is zero
      for (int c = lane; c < d; c += 32) yz[tok * d + c] = XT(0.f);
      if (a.yf_zero_dropped != nullptr)
        for (int c = lane; c < d; c += 32) a.yf_zero_dropped[tok * d + c] = 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// Combine: y_t = sum over kept choices j (ascending) of the slot's row of Yp
// (summed over its K-range partials in order).  One thread per token and
// group of 4 columns, so small batches still spread over many warps.
template <typename YT>
__global__ void __launch_bounds__(256) combine_kernel(int64_t T, int k, int d, const int32_t* __restrict__ dest_row,
                                                      const float* __restrict__ Yp, int ksplit, int64_t split_stride,
                                                      YT* __restrict__ y, float* __restrict__ yf) {
  pdl_wait();
  pdl_trigger();
  const uint32_t vpr = static_cast<uint32_t>(d) >> 2;  // float4 groups per row (d % 4 == 0 on this path)
  const uint32_t i = blockIdx.x * 256u + threadIdx.x;    // T * d / 4 < 2^32 (checked on the host)
  if (i >= static_cast<uint32_t>(T) * vpr) return;
  const uint32_t t32 = i / vpr;
  const int64_t t = t32;
  const int v = static_cast<int>(i - t32 * vpr);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ksplit == 1) {
    float4 u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // all loads first (independent), then the ordered sum
      const int dst = j < k ? dest_row[t * k + j] : -1;
      u[j] = dst >= 0 ? reinterpret_cast<const float4*>(Yp + static_cast<int64_t>(dst) * d)[v]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      acc.x += u[j].x; acc.y += u[j].y; acc.z += u[j].z; acc.w += u[j].w;
    }
  } else {
    for (int j = 0; j < k; ++j) {
      const int dst = dest_row[t * k + j];
      if (dst < 0) continue;
      float4 sj = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int ks = 0; ks < ksplit; ++ks) {
        const float4 u = reinterpret_cast<const float4*>(Yp + static_cast<int64_t>(ks) * split_stride +
                                                         static_cast<int64_t>(dst) * d)[v];
        sj.x += u.x; sj.y += u.y; sj.z += u.z; sj.w += u.w;
      }
      acc.x += sj.x; acc.y += sj.y; acc.z += sj.z; acc.w += sj.w;
    }
  }
  if (yf != nullptr) reinterpret_cast<float4*>(yf + t * d)[v] = acc;
  if constexpr (sizeof(YT) == 2) {
    uint2 o;
    o.x = pack_bf16x2(acc.x, acc.y);
    o.y = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2*>(y + t * d)[v] = o;
  } else {
    reinterpret_cast<float4*>(y + t * d)[v] = acc;
  }
}

// Scalar combine for rows whose width is not a multiple of 4 (fp32 layers).
template <typename YT>
__global__ void __launch_bounds__(256) combine_scalar_kernel(int64_t T, int k, int d,
                                                             const int32_t* __restrict__ dest_row,
                                                             const float* __restrict__ Yp, int ksplit,
                                                             int64_t split_stride, YT* __restrict__ y,
                                                             float* __restrict__ yf) {
  pdl_wait();
  pdl_trigger();
  const uint32_t i = blockIdx.x * 256u + threadIdx.x;  // T * d < 2^32 (checked on the host)
  if (i >= static_cast<uint32_t>(T) * static_cast<uint32_t>(d)) return;
  const uint32_t t32 = i / static_cast<uint32_t>(d);
  const int64_t t = t32;
  const int c = static_cast<int>(i - t32 * static_cast<uint32_t>(d));
  float acc = 0.f;
  for (int j = 0; j < k; ++j) {
    const int dst = dest_row[t * k + j];
    if (dst < 0) continue;
    float sj = 0.f;
    for (int ks = 0; ks < ksplit; ++ks) sj += Yp[static_cast<int64_t>(ks) * split_stride + static_cast<int64_t>(dst) * d + c];
    acc += sj;
  }
  y[t * d + c] = YT(acc);
  if (yf != nullptr) yf[t * d + c] = acc;
}

// ---------------------------------------------------------------------------
// Failure-path self-test: wait on an mbarrier that nothing ever arrives on.
__global__ void selftest_timeout_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    if (!mbar_wait(&bar, 0, limit_ns)) record_error(err, DEV_ERR_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_router(const RoutingArgs& a, cudaStream_t s) {
  return a.x_is_bf16 ? launch_router_x<__nv_bfloat16>(a, s) : launch_router_x<float>(a, s);
}

cudaError_t launch_scan(const RoutingArgs& a, cudaStream_t s) {
  return launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, a);
}

cudaError_t launch_dispatch(const RoutingArgs& a, cudaStream_t s) {
  if (a.x_is_bf16) return launch_pdl(dispatch_kernel<__nv_bfloat16>, dim3(a.nblk), dim3(256), 0, s, a);
  return launch_pdl(dispatch_kernel<float>, dim3(a.nblk), dim3(256), 0, s, a);
}

cudaError_t launch_combine(int64_t T, int k, int d, int y_is_bf16, const int32_t* dest_row, const float* Yp,
                           int ksplit, int64_t split_stride, void* y, float* y_f32, cudaStream_t s) {
  if ((d & 3) == 0) {
    const dim3 grid(static_cast<unsigned>((T * (d / 4) + 255) / 256));
    if (y_is_bf16)
      return launch_pdl(combine_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, T, k, d, dest_row, Yp, ksplit,
                        split_stride, static_cast<__nv_bfloat16*>(y), y_f32);
    return launch_pdl(combine_kernel<float>, grid, dim3(256), 0, s, T, k, d, dest_row, Yp, ksplit, split_stride,
                      static_cast<float*>(y), y_f32);
  }
  const dim3 grid(static_cast<unsigned>((T * d + 255) / 256));
  if (y_is_bf16)
    return launch_pdl(combine_scalar_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, T, k, d, dest_row, Yp, ksplit,
                      split_stride, static_cast<__nv_bfloat16*>(y), y_f32);
  return launch_pdl(combine_scalar_kernel<float>, grid, dim3(256), 0, s, T, k, d, dest_row, Yp, ksplit,
                    split_stride, static_cast<float*>(y), y_f32);
}

cudaError_t launch_selftest_timeout(unsigned int* err, int64_t limit_ns, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(err, static_cast<uint64_t>(limit_ns));
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

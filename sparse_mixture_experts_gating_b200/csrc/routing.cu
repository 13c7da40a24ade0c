// Routing kernels of the MoE layer forward pass:
//   router   - fp32 router logits h = W_r x (+ b), softmax, log-sum-exp, top-k
//              (ties -> lower expert index), gates, per-block counts and sums
//   scan     - per-expert totals and stable per-block rank bases
//   dispatch - capacity and expert offsets from the totals, slot rank of each
//              (token, choice) in token order, drop mask, permute of the kept
//              token rows into expert-sorted order; one extra block finalises
//              the scan (offsets and tile prefix for the GEMMs, dropped count,
//              aux loss, z-loss and the other balance statistics)
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
#include "scan_dispatch.h"

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
// Scan: one block per expert e.  Each thread takes a contiguous run of the
// router blocks, so the exclusive prefix of e's per-block counts (the stable
// rank base of each block, in token order) is one block-wide scan; e's totals
// (routed count, first-choice count, probability sum) go to the workspace,
// where the dispatch launch turns them into capacity, expert offsets, tile
// prefix, dropped count, aux loss and z-loss (scan_finalize), all summed in a
// fixed order.
constexpr int SCAN_T = 256;
constexpr int kScanSingleBlocks = 8;  // up to 256 tokens: one block, one expert per thread

__device__ __forceinline__ int block_exscan_int(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < SCAN_T / 32 ? s_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < SCAN_T / 32) s_warp[lane] = wi - w;  // exclusive warp bases
    if (lane == SCAN_T / 32 - 1) s_warp[SCAN_T / 32] = wi;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  total = s_warp[SCAN_T / 32];
  __syncthreads();
  return r;
}

// Sum over the block in a fixed tree order (deterministic).
template <typename F>
__device__ __forceinline__ F block_sum(F v, F* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
  __syncthreads();
  F t = 0;
  if (threadIdx.x == 0)
    for (int w = 0; w < SCAN_T / 32; ++w) t += s_red[w];
  __syncthreads();
  return t;  // valid in thread 0
}

// N sums over the block at once, in a fixed tree order; every thread adds the
// per-warp partials itself in the same order, so all get the same totals.
template <int N>
__device__ __forceinline__ void block_sums(double (&v)[N], double* s_red /* [SCAN_T / 32][N] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < N; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  }
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) s_red[warp * N + i] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    double t = 0.0;
    for (int w = 0; w < SCAN_T / 32; ++w) t += s_red[w * N + i];
    v[i] = t;
  }
  __syncthreads();
}

// Exclusive prefix sums of two ints over the block (thread order), and their totals.
__device__ __forceinline__ void block_exscan_int2(int a0, int a1, int* s_warp2 /* [2][SCAN_T / 32 + 1] */,
                                                  int& r0, int& r1, int& t0, int& t1) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int W = SCAN_T / 32;
  int i0 = a0, i1 = a1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u0 = __shfl_up_sync(0xffffffffu, i0, o);
    const int u1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) { i0 += u0; i1 += u1; }
  }
  if (lane == 31) { s_warp2[warp] = i0; s_warp2[W + 1 + warp] = i1; }
  __syncthreads();
  int b0 = 0, b1 = 0;
  t0 = t1 = 0;
  for (int w = 0; w < W; ++w) {
    const int w0 = s_warp2[w], w1 = s_warp2[W + 1 + w];
    if (w < warp) { b0 += w0; b1 += w1; }
    t0 += w0;
    t1 += w1;
  }
  r0 = b0 + i0 - a0;
  r1 = b1 + i1 - a1;
  __syncthreads();
}

// Capacity, expert offsets, tile prefix, dropped count, aux loss, z-loss and
// the alternative balance statistics from the per-expert totals (thread e < E
// holds routed expert e's; threads E .. E + n_shared - 1 stand for the shared
// experts' groups of T rows, which take no part in capacity, counts or
// losses), by all SCAN_T threads of one block.  Sums run in double, in a
// fixed order.
__device__ __forceinline__ void scan_finalize(const RoutingArgs& a, int cnt, int c1, float ps, int* s_warp2,
                                              double* s_red) {
  const int tid = threadIdx.x, E = a.E, nb = a.nblk;
  const int groups = E + a.n_shared;
  const bool routed = tid < E;
  double zs = 0.0;  // this thread's share of sum lse^2 (loaded before the scans below)
  for (int b = tid; b < nb; b += SCAN_T) zs += static_cast<double>(a.part_lse2[b]);
  int kept = 0;
  if (routed) kept = (a.capacity < 0) ? cnt : static_cast<int>((int64_t)cnt < a.capacity ? (int64_t)cnt : a.capacity);
  else if (tid < groups) kept = static_cast<int>(a.T);
  const int mt = (kept + kTileM - 1) / kTileM;
  int off, mp, total_rows, total_tiles;
  block_exscan_int2(kept, mt, s_warp2, off, mp, total_rows, total_tiles);
  if (routed) a.counts[tid] = cnt;
  if (tid < groups) {
    a.offsets[tid] = off;
    a.mprefix[tid] = mp;
  }
  // the debug copy holds the routed experts' offsets [E + 1] (offsets[E] = kept routed
  // rows: the total without shared experts, else thread E's prefix; E < 256 then)
  if (a.offsets_out != nullptr) {
    if (tid < E) a.offsets_out[tid] = off;
    if (a.n_shared == 0 ? tid == 0 : tid == E) a.offsets_out[E] = a.n_shared == 0 ? total_rows : off;
  }
  const double T = static_cast<double>(a.T);
  const double c = routed ? static_cast<double>(cnt) : 0.0;
  const double Pe = routed ? static_cast<double>(ps) / T : 0.0;  // mean router probability of e
  // dropped, sum f1*P (first choices), sum of counts, sum of P, sum counts*P, sum lse^2
  double v[6] = {routed ? static_cast<double>(cnt - kept) : 0.0,
                 routed ? static_cast<double>(c1) * static_cast<double>(ps) : 0.0, c, Pe, c * Pe, zs};
  block_sums<6>(v, s_red);
  // population moments over the E experts
  const double mean_c = v[2] / E, mean_p = v[3] / E;
  const double dc = routed ? c - mean_c : 0.0, dp = routed ? Pe - mean_p : 0.0;
  double m2[2] = {dc * dc, dp * dp};
  block_sums<2>(m2, s_red);
  if (tid == 0) {
    a.offsets[groups] = total_rows;
    a.mprefix[groups] = total_tiles;
    *a.dropped = static_cast<int>(v[0]);
    *a.aux = static_cast<float>(static_cast<double>(E) * v[1] / (T * T));
    *a.z = static_cast<float>(v[5] / T);
    a.balance_out[0] = static_cast<float>(E * v[4] / (T * a.k));
    a.balance_out[1] = static_cast<float>(mean_c > 0.0 ? sqrt(m2[0] / E) / mean_c : 0.0);
    a.balance_out[2] = static_cast<float>(mean_p > 0.0 ? (m2[1] / E) / (mean_p * mean_p) : 0.0);
  }
}

// SINGLE (few router blocks): one block, thread e walks expert e's blocks in
// order, then finalises.  Otherwise one block per expert as described above
// (the dispatch launch finalises).
template <bool SINGLE>
__global__ void __launch_bounds__(SCAN_T) scan_kernel(RoutingArgs a) {
  __shared__ int s_warp[2 * (SCAN_T / 32 + 1)];
  __shared__ float s_redf[SCAN_T / 32];
  __shared__ int s_redi[SCAN_T / 32];
  __shared__ double s_redd[6 * (SCAN_T / 32)];
  const int tid = threadIdx.x;
  const int E = a.E, nb = a.nblk;
  pdl_wait();
  pdl_trigger();
  if constexpr (SINGLE) {
    int cnt = 0, c1 = 0;
    float ps = 0.f;
    if (tid < E) {
      const int64_t row = static_cast<int64_t>(tid) * nb;
#pragma unroll 4
      for (int b = 0; b < nb; ++b) {
        a.blockoff[row + b] = cnt;
        cnt += a.part_hist[row + b];
        c1 += a.part_cnt1[row + b];
        ps += a.part_psum[row + b];
      }
    }
    scan_finalize(a, cnt, c1, ps, s_warp, s_redd);
    return;
  }
  const int e = blockIdx.x;
  // this thread's run of router blocks [b0, b1)
  const int per = (nb + SCAN_T - 1) / SCAN_T;
  const int b0 = min(nb, tid * per), b1 = min(nb, b0 + per);
  const int32_t* hist = a.part_hist + static_cast<int64_t>(e) * nb;
  int h_run = 0, c1 = 0;
  float ps = 0.f;
  for (int b = b0; b < b1; ++b) {
    h_run += hist[b];
    c1 += a.part_cnt1[static_cast<int64_t>(e) * nb + b];
    ps += a.part_psum[static_cast<int64_t>(e) * nb + b];
  }
  int count = 0;
  int base = block_exscan_int(h_run, s_warp, count);
  for (int b = b0; b < b1; ++b) {
    a.blockoff[static_cast<int64_t>(e) * nb + b] = base;
    base += hist[b];
  }
  const int c1_tot = block_sum<int>(c1, s_redi);
  const float ps_tot = block_sum<float>(ps, s_redf);
  if (tid == 0) {  // the totals; the dispatch launch finalises (scan_finalize) alongside its copies
    a.counts[e] = count;
    a.tot_cnt1[e] = c1_tot;
    a.tot_psum[e] = ps_tot;
  }
}

// One warp zeroes row `tok` of y (16-byte stores where the row allows).
template <typename XT>
__device__ __forceinline__ void zero_row(XT* __restrict__ y, int d, int64_t tok, int lane) {
  if ((static_cast<size_t>(d) * sizeof(XT)) % 16 == 0) {
    uint4* dst = reinterpret_cast<uint4*>(y + tok * d);
    const int nv = static_cast<int>(static_cast<size_t>(d) * sizeof(XT) / 16);
    for (int v = lane; v < nv; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
  } else {
    for (int c = lane; c < d; c += 32) y[tok * d + c] = XT(0.f);
  }
}

// ---------------------------------------------------------------------------
// One warp copies row `tok` of x to row `dest` of the expert-sorted buffer
// (rows of 16-byte multiples: up to eight 16-byte loads in flight per lane).
template <typename XT>
__device__ __forceinline__ void copy_x_row(const XT* __restrict__ x, XT* __restrict__ Xp, int d, int64_t tok,
                                           int64_t dest, int lane) {
  if ((static_cast<size_t>(d) * sizeof(XT)) % 16 == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(x + tok * d);
    uint4* dst = reinterpret_cast<uint4*>(Xp + dest * d);
    const int nv = static_cast<int>(static_cast<size_t>(d) * sizeof(XT) / 16);
    for (int v0 = lane; v0 < nv; v0 += 256) {
      uint4 c[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (v0 + 32 * q < nv) c[q] = src[v0 + 32 * q];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (v0 + 32 * q < nv) dst[v0 + 32 * q] = c[q];
    }
  } else {
    for (int c = lane; c < d; c += 32) Xp[dest * d + c] = x[tok * d + c];
  }
}

// ---------------------------------------------------------------------------
// Dispatch: one block per router block of BT tokens.  The block derives the
// group offsets from the scan's per-expert counts itself (as scan_finalize
// does), while its (token, choice) experts and gates, and its per-expert rank
// bases, load alongside.  Warp 0 assigns the slot rank of every (token,
// choice) of the block in token-major order (stable: base = number of earlier
// assignments to the same expert in earlier blocks); then all warps copy the
// kept rows of x into the expert-sorted buffer.  With `finalize` one more
// block, nblk, runs scan_finalize (offsets and tile prefix for the GEMMs,
// counts, losses and statistics) beside them.
template <typename XT>
__global__ void __launch_bounds__(256) dispatch_kernel(RoutingArgs a) {
  __shared__ int run_s[256];
  __shared__ int off_s[256];
  __shared__ int dest_s[BT * 8];
  __shared__ int e_s[BT * 8];
  __shared__ float g_s[BT * 8];
  __shared__ int s_warp[2 * (SCAN_T / 32 + 1)];
  __shared__ double s_red[6 * (SCAN_T / 32)];
  static_assert(SCAN_T == 256, "the dispatch block is the scan's block size");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, d = a.d, nb = a.nblk;
  pdl_wait();
  pdl_trigger();
  if (static_cast<int>(blockIdx.x) == nb) {  // the scan's finalisation
    scan_finalize(a, tid < E ? a.counts[tid] : 0, tid < E ? a.tot_cnt1[tid] : 0, tid < E ? a.tot_psum[tid] : 0.f,
                  s_warp, s_red);
    return;
  }
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * BT;
  const int nt = static_cast<int>((a.T - t0) < BT ? (a.T - t0) : BT);
  const int nA = nt * k;
  {
    const int groups = E + a.n_shared;
    int kept = 0;
    if (tid < E) {
      const int cnt = a.counts[tid];
      run_s[tid] = a.blockoff[tid * nb + blockIdx.x];
      kept = (a.capacity < 0) ? cnt : static_cast<int>((int64_t)cnt < a.capacity ? (int64_t)cnt : a.capacity);
    } else if (tid < groups) {
      kept = static_cast<int>(a.T);
    }
    for (int i = tid; i < nA; i += 256) {
      e_s[i] = a.topk_idx[t0 * k + i];
      g_s[i] = a.topk_gate[t0 * k + i];
    }
    int off, mp, total_rows, total_tiles;
    block_exscan_int2(kept, (kept + kTileM - 1) / kTileM, s_warp, off, mp, total_rows, total_tiles);  // syncs
    if (tid < groups) off_s[tid] = off;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int a0 = 0; a0 < nA; a0 += 32) {
      const int ai = a0 + lane;
      const bool valid = ai < nA;
      int e = valid ? e_s[ai] : -1;
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
        const int dest = kept ? off_s[e] + rank : -1;
        dest_s[ai] = dest;
        a.dest_row[t0 * k + ai] = dest;
        if (a.drop_mask != nullptr) a.drop_mask[t0 * k + ai] = kept ? 0 : 1;
        if (kept) {
          a.row_token[dest] = static_cast<int32_t>(t0 + ai / k);
          a.row_gate[dest] = g_s[ai];
        }
      }
    }
  }
  __syncthreads();
  const XT* x = static_cast<const XT*>(a.x);
  XT* Xp = static_cast<XT*>(a.Xp);
  XT* yz = static_cast<XT*>(a.y_zero_dropped);
  auto copy_row = [&](int64_t tok, int64_t dest) { copy_x_row(x, Xp, d, tok, dest, lane); };
  for (int ai = warp; ai < nA; ai += 8) {
    const int dest = dest_s[ai];
    const int64_t tok = t0 + ai / k;
    if (dest >= 0) {
      copy_row(tok, dest);
    } else if (yz != nullptr) {  // k == 1: a dropped token's output row is zero
      zero_row(yz, d, tok, lane);
      if (a.yf_zero_dropped != nullptr)
        for (int c = lane; c < d; c += 32) a.yf_zero_dropped[tok * d + c] = 0.f;
    }
  }
  // shared experts: every token of the block, gate 1, rows offsets[E] + s * T + t
  if (a.n_shared > 0) {
    const int64_t base = off_s[E];
    for (int q = warp; q < nt * a.n_shared; q += 8) {
      const int si = q / nt;
      const int64_t tok = t0 + (q - si * nt);
      const int64_t row = base + si * a.T + tok;
      if (lane == 0) {
        a.row_token[row] = static_cast<int32_t>(tok);
        a.row_gate[row] = 1.f;
      }
      copy_row(tok, row);
    }
  }
}

// ---------------------------------------------------------------------------
// Scan and dispatch in one launch, for few experts times router blocks (each
// warp loads at most kFusedLoads histogram entries per lane): block
// (b, part) derives every expert's total and its prefix over the router
// blocks before b itself (a warp per expert row, lanes over consecutive
// blocks, four rows' loads in flight), takes the capacity-capped group sizes
// and offsets the way scan_finalize does, ranks router block b's assignments
// and copies its share of their rows (the warps of the gridDim.y parts stride
// over them).  One more block, (nblk, 0), writes the scan's tables and
// statistics (scan_finalize) alongside.  No per-block offsets table and no
// second launch.
constexpr int kFusedLoads = 16;  // (the Switch layer's 64 experts x 256 blocks, 64 loads per lane, ran no faster fused)
constexpr int kFusedRows = 4;  // expert rows per batch of loads

// Totals of kFusedRows expert rows e0, e0 + 8, ... (warp-uniform; rows past
// E count zero) of a per-block table [E][nb], and their parts before block
// blk: lanes over consecutive blocks, 256 blocks of every row per batch.
template <typename V>
__device__ __forceinline__ void rows_sums(const V* __restrict__ tab, int E, int nb, int e0, int blk, int lane,
                                          V (&tot)[kFusedRows], V (&pre)[kFusedRows]) {
#pragma unroll
  for (int u = 0; u < kFusedRows; ++u) { tot[u] = V(0); pre[u] = V(0); }
#pragma unroll 1
  for (int c0 = 0; c0 < nb; c0 += 256) {
    V v[kFusedRows][8];
#pragma unroll
    for (int u = 0; u < kFusedRows; ++u) {
      const int e = e0 + 8 * u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int b = c0 + 32 * j + lane;
        v[u][j] = (e < E && b < nb) ? tab[static_cast<int64_t>(e) * nb + b] : V(0);
      }
    }
#pragma unroll
    for (int u = 0; u < kFusedRows; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        tot[u] += v[u][j];
        if (c0 + 32 * j + lane < blk) pre[u] += v[u][j];
      }
  }
}

template <typename V>
__device__ __forceinline__ V warp_total(V v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename XT>
__global__ void __launch_bounds__(SCAN_T) scan_dispatch_kernel(RoutingArgs a) {
  __shared__ int s_tot[256], s_pre[256], s_c1[256], s_off[257];
  __shared__ float s_ps[256];
  __shared__ int s_dest[BT * 8];
  __shared__ int s_warp[2 * (SCAN_T / 32 + 1)];
  __shared__ double s_red[6 * (SCAN_T / 32)];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, d = a.d, nb = a.nblk;
  const int blk = blockIdx.x;
  const bool stats = blk == nb;  // the block of the scan's tables and statistics
  const int64_t t0 = static_cast<int64_t>(blk) * BT;
  const int nt = stats ? 0 : static_cast<int>((a.T - t0) < BT ? (a.T - t0) : BT);
  const int nA = nt * k;
  pdl_wait();
  pdl_trigger();
  if (stats && blockIdx.y != 0) return;
  // warp w: expert rows w + 8 i, kFusedRows of them per batch
#pragma unroll 1
  for (int e0 = warp; e0 < E; e0 += 8 * kFusedRows) {
    int tot[kFusedRows], pre[kFusedRows];
    rows_sums(a.part_hist, E, nb, e0, blk, lane, tot, pre);
#pragma unroll
    for (int u = 0; u < kFusedRows; ++u) {
      const int t = warp_total(tot[u]), p = warp_total(pre[u]);
      if (lane == 0 && e0 + 8 * u < E) { s_tot[e0 + 8 * u] = t; s_pre[e0 + 8 * u] = p; }
    }
    if (stats) {  // first-choice counts and probability sums for the statistics
      int c1[kFusedRows], c1p[kFusedRows];
      float ps[kFusedRows], psp[kFusedRows];
      rows_sums(a.part_cnt1, E, nb, e0, 0, lane, c1, c1p);
      rows_sums(a.part_psum, E, nb, e0, 0, lane, ps, psp);
#pragma unroll
      for (int u = 0; u < kFusedRows; ++u) {
        const int c = warp_total(c1[u]);
        const float q = warp_total(ps[u]);
        if (lane == 0 && e0 + 8 * u < E) { s_c1[e0 + 8 * u] = c; s_ps[e0 + 8 * u] = q; }
      }
    }
  }
  __syncthreads();
  if (stats) {
    scan_finalize(a, tid < E ? s_tot[tid] : 0, tid < E ? s_c1[tid] : 0, tid < E ? s_ps[tid] : 0.f, s_warp, s_red);
    return;
  }
  {  // group offsets, as scan_finalize computes them
    const int groups = E + a.n_shared;
    int kept = 0;
    if (tid < E)
      kept = (a.capacity < 0) ? s_tot[tid]
                              : static_cast<int>((int64_t)s_tot[tid] < a.capacity ? (int64_t)s_tot[tid] : a.capacity);
    else if (tid < groups)
      kept = static_cast<int>(a.T);
    int off, mp, total_rows, total_tiles;
    block_exscan_int2(kept, (kept + kTileM - 1) / kTileM, s_warp, off, mp, total_rows, total_tiles);
    if (tid < groups) s_off[tid] = off;
    if (tid == 0) s_off[groups] = total_rows;
  }
  __syncthreads();
  const bool writer = blockIdx.y == 0;  // one part writes the block's routing tables
  if (warp == 0) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int a0 = 0; a0 < nA; a0 += 32) {
      const int ai = a0 + lane;
      const bool valid = ai < nA;
      int e = valid ? a.topk_idx[t0 * k + ai] : -1;
      if (e < 0 || e >= E) e = -1;  // never produced by the router; keeps smem indexing in range
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      const bool ok = valid && e >= 0;
      const int base = ok ? s_pre[e] : 0;
      const int rank = base + __popc(peers & lt);
      __syncwarp();
      if (ok && lane == __ffs(peers) - 1) s_pre[e] = base + __popc(peers);
      __syncwarp();
      if (valid && !ok) {
        s_dest[ai] = -1;
        if (writer) a.dest_row[t0 * k + ai] = -1;
      } else if (valid) {
        const bool kept = a.capacity < 0 || rank < a.capacity;
        const int dest = kept ? s_off[e] + rank : -1;
        s_dest[ai] = dest;
        if (writer) {
          a.dest_row[t0 * k + ai] = dest;
          if (a.drop_mask != nullptr) a.drop_mask[t0 * k + ai] = kept ? 0 : 1;
          if (kept) {
            a.row_token[dest] = static_cast<int32_t>(t0 + ai / k);
            a.row_gate[dest] = a.topk_gate[t0 * k + ai];
          }
        }
      }
    }
  }
  __syncthreads();
  const XT* x = static_cast<const XT*>(a.x);
  XT* Xp = static_cast<XT*>(a.Xp);
  XT* yz = static_cast<XT*>(a.y_zero_dropped);
  const int gw = static_cast<int>(blockIdx.y) * (SCAN_T / 32) + warp, nw = static_cast<int>(gridDim.y) * (SCAN_T / 32);
  for (int ai = gw; ai < nA; ai += nw) {
    const int dest = s_dest[ai];
    const int64_t tok = t0 + ai / k;
    if (dest >= 0) {
      copy_x_row(x, Xp, d, tok, dest, lane);
    } else if (yz != nullptr) {  // k == 1: a dropped token's output row is zero
      zero_row(yz, d, tok, lane);
      if (a.yf_zero_dropped != nullptr)
        for (int c = lane; c < d; c += 32) a.yf_zero_dropped[tok * d + c] = 0.f;
    }
  }
  // shared experts: every token of the block, gate 1, rows offsets[E] + s * T + t
  if (a.n_shared > 0) {
    const int64_t base = s_off[E];
    for (int q = gw; q < nt * a.n_shared; q += nw) {
      const int si = q / nt;
      const int64_t tok = t0 + (q - si * nt);
      const int64_t row = base + si * a.T + tok;
      if (lane == 0) {
        a.row_token[row] = static_cast<int32_t>(tok);
        a.row_gate[row] = 1.f;
      }
      copy_x_row(x, Xp, d, tok, row, lane);
    }
  }
}

// ---------------------------------------------------------------------------
// Small batches (T <= 32: one router block).  Two kernels replace the router,
// scan and dispatch:
//   route_small_dot_kernel  grid (DS, E): block (ds, e) sums W_r[e][c] x[t][c]
//                           over its d-chunk for every token t (fp32, a fixed
//                           block-tree order) into partial[ds][t][e];
//   route_small_kernel      one block of SCAN_T threads: logits = the DS
//                           partials in order (+ bias), then softmax,
//                           log-sum-exp, top-k and gates (a warp per token,
//                           lanes over experts), the per-expert totals, the
//                           scan's capacity / offsets / losses (scan_finalize),
//                           slot ranks in token order, and the row copies.
constexpr int SMALL_T = 32;
constexpr int SMALL_DS_MAX = 16;

template <typename XT>
__global__ void __launch_bounds__(256) route_small_dot_kernel(RoutingArgs a, int chunk, float* __restrict__ partial) {
  __shared__ float s_red[8][SMALL_T];
  const int ds = blockIdx.x, e = blockIdx.y, tid = threadIdx.x;
  const int T = static_cast<int>(a.T), d = a.d;
  const XT* x = static_cast<const XT*>(a.x);
  const float* w = a.W_r + static_cast<int64_t>(e) * d;
  const int c0 = ds * chunk, c1 = min(d, c0 + chunk);
  float acc[SMALL_T];
#pragma unroll
  for (int t = 0; t < SMALL_T; ++t) acc[t] = 0.f;
  for (int c = c0 + tid; c < c1; c += 256) {
    const float wv = w[c];
#pragma unroll
    for (int t = 0; t < SMALL_T; ++t)
      if (t < T) acc[t] = fmaf(wv, to_f32(x[static_cast<int64_t>(t) * d + c]), acc[t]);
  }
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int t = 0; t < SMALL_T; ++t) {
    if (t < T) {
      float v = acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) s_red[warp][t] = v;
    }
  }
  __syncthreads();
  if (tid < T) {
    float v = 0.f;
#pragma unroll
    for (int wi = 0; wi < 8; ++wi) v += s_red[wi][tid];
    partial[(static_cast<int64_t>(ds) * T + tid) * a.E + e] = v;
  }
}

template <typename XT>
__global__ void __launch_bounds__(SCAN_T) route_small_kernel(RoutingArgs a, int n_ds, const float* __restrict__ partial) {
  extern __shared__ __align__(16) float sm_h[];  // [T][E]: logits, then probabilities
  __shared__ int s_idx[SMALL_T * 8];
  __shared__ float s_gate[SMALL_T * 8];
  __shared__ int s_hist[256], s_cnt1[256], s_dest[SMALL_T * 8];
  __shared__ float s_lse2[SMALL_T];
  __shared__ int s_warp[2 * (SCAN_T / 32 + 1)];
  __shared__ double s_red[6 * (SCAN_T / 32)];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = static_cast<int>(a.T), E = a.E, k = a.k, d = a.d;
  pdl_wait();
  pdl_trigger();
  for (int e = tid; e < 256; e += SCAN_T) { s_hist[e] = 0; s_cnt1[e] = 0; }
  // logits: partials in d-chunk order, then the bias
  for (int i = tid; i < T * E; i += SCAN_T) {
    const int t = i / E, e = i - t * E;
    float h;
    if (a.logits_in != nullptr) {
      h = a.logits_in[i];
    } else {
      float pv[SMALL_DS_MAX];  // all chunk loads in flight, then the sum in chunk order
#pragma unroll
      for (int ds = 0; ds < SMALL_DS_MAX; ++ds)
        pv[ds] = ds < n_ds ? partial[(static_cast<int64_t>(ds) * T + t) * E + e] : 0.f;
      h = 0.f;
#pragma unroll
      for (int ds = 0; ds < SMALL_DS_MAX; ++ds)
        if (ds < n_ds) h += pv[ds];
      if (a.b_r != nullptr) h += a.b_r[e];
    }
    if (h != h) h = -INFINITY;  // NaN logits (out of contract) rank last
    sm_h[i] = h;
    if (a.logits_out != nullptr) a.logits_out[i] = h;
  }
  __syncthreads();
  // a warp per token: max, log-sum-exp, top-k (value desc, index asc), gates
  for (int t = warp; t < T; t += SCAN_T / 32) {
    float* h = sm_h + t * E;
    float m = -INFINITY;
    for (int e = lane; e < E; e += 32) m = fmaxf(m, h[e]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sl = 0.f;
    for (int e = lane; e < E; e += 32) sl += expf(h[e] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
    const float inv_s = 1.f / sl;
    const float lse = m + logf(sl);
    uint32_t picked = 0;  // bit i: this lane's expert lane + 32 i is taken
    float tv0 = 0.f, den = 0.f;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7fffffff, bi = -1;
      for (int i = 0, e = lane; e < E; ++i, e += 32)
        if (!((picked >> i) & 1u) && (be == 0x7fffffff || h[e] > bv)) { bv = h[e]; be = e; bi = i; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
      }
      if (bi >= 0 && lane + 32 * bi == be) picked |= 1u << bi;
      if (j == 0) tv0 = bv;
      const float gsw = expf(bv - m) * inv_s;
      const float ren = expf(bv - tv0);
      den += ren;
      if (lane == 0) {
        s_idx[t * k + j] = be;
        s_gate[t * k + j] = a.gate_mode == 0 ? gsw : ren;  // renormalised below
        a.topk_idx[t * k + j] = be;
        atomicAdd(&s_hist[be], 1);
        if (j == 0) atomicAdd(&s_cnt1[be], 1);
      }
    }
    if (lane == 0) {
      for (int j = 0; j < k; ++j) {
        if (a.gate_mode != 0) s_gate[t * k + j] /= den;
        a.topk_gate[t * k + j] = s_gate[t * k + j];
      }
      if (a.lse_out != nullptr) a.lse_out[t] = lse;
      s_lse2[t] = lse * lse;
    }
    __syncwarp();
    for (int e = lane; e < E; e += 32) h[e] = expf(h[e] - m) * inv_s;  // probabilities
  }
  __syncthreads();
  // per-expert totals in token order; z from the token lse^2 in order
  int cnt = 0, c1 = 0;
  float ps = 0.f;
  if (tid < E) {
    cnt = s_hist[tid];
    c1 = s_cnt1[tid];
    for (int t = 0; t < T; ++t) ps += sm_h[t * E + tid];
  }
  if (tid == 0) {
    float z2 = 0.f;
    for (int t = 0; t < T; ++t) z2 += s_lse2[t];
    a.part_lse2[0] = z2;
  }
  __syncthreads();
  scan_finalize(a, cnt, c1, ps, s_warp, s_red);  // counts, offsets, tile prefix, dropped, losses
  // slot ranks in token order (assignment i = t * k + j), kept flags, destinations
  const int nA = T * k;
  for (int i = tid; i < nA; i += SCAN_T) {
    const int e = s_idx[i];
    int rank = 0;
    for (int i2 = 0; i2 < i; ++i2) rank += s_idx[i2] == e;
    const bool kept = a.capacity < 0 || rank < a.capacity;
    const int dest = kept ? a.offsets[e] + rank : -1;
    s_dest[i] = dest;
    a.dest_row[i] = dest;
    if (a.drop_mask != nullptr) a.drop_mask[i] = kept ? 0 : 1;
    if (kept) {
      a.row_token[dest] = i / k;
      a.row_gate[dest] = s_gate[i];
    }
  }
  __syncthreads();
  // row copies (a warp per row): kept assignments, then the shared experts' rows
  const XT* x = static_cast<const XT*>(a.x);
  XT* Xp = static_cast<XT*>(a.Xp);
  XT* yz = static_cast<XT*>(a.y_zero_dropped);
  auto copy_row = [&](int64_t tok, int64_t dest) { copy_x_row(x, Xp, d, tok, dest, lane); };
  for (int i = warp; i < nA; i += SCAN_T / 32) {
    const int64_t tok = i / k;
    if (s_dest[i] >= 0) {
      copy_row(tok, s_dest[i]);
    } else if (yz != nullptr) {  // k == 1: a dropped token's output row is zero
      zero_row(yz, d, tok, lane);
      if (a.yf_zero_dropped != nullptr)
        for (int c = lane; c < d; c += 32) a.yf_zero_dropped[tok * d + c] = 0.f;
    }
  }
  if (a.n_shared > 0) {
    const int64_t base = a.offsets[E];
    for (int q = warp; q < T * a.n_shared; q += SCAN_T / 32) {
      const int si = q / T;
      const int64_t tok = q - si * T;
      const int64_t row = base + si * static_cast<int64_t>(T) + tok;
      if (lane == 0) {
        a.row_token[row] = static_cast<int32_t>(tok);
        a.row_gate[row] = 1.f;
      }
      copy_row(tok, row);
    }
  }
}

// ---------------------------------------------------------------------------
// Combine: y_t = sum over kept choices j (ascending) of the slot's row of Yp
// (summed over its K-range partials in order), then the shared experts' rows.
// A block takes one token at a time (grid-stride over tokens) and the
// columns [blockIdx.y * cpb, +cpb) of it (small batches split a row over
// several blocks): the token's destination rows are block-wide constants, so
// each thread only streams its groups of 4 columns (VU of them per pass, all
// loads issued before the ordered sums).
template <typename YT, int K, int VU>
__global__ void __launch_bounds__(256, 4) combine_kernel(int64_t T, int d, const int32_t* __restrict__ dest_row,
                                                      int n_shared, const int32_t* __restrict__ shared_base,
                                                      const float* __restrict__ Yp, int ksplit, int64_t split_stride,
                                                      int cpb, YT* __restrict__ y, float* __restrict__ yf) {
  pdl_wait();
  pdl_trigger();
  const int vpr = d >> 2;  // float4 groups per row (d % 4 == 0 on this path)
  const int c_end = min(vpr, static_cast<int>(blockIdx.y + 1) * cpb);
  const float4* Y4 = reinterpret_cast<const float4*>(Yp);
  const int64_t sb = n_shared > 0 ? *shared_base : 0;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    int64_t base[K];  // first float4 of each kept choice's row (-1: dropped)
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const int dst = dest_row[t * K + j];
      base[j] = dst >= 0 ? static_cast<int64_t>(dst) * vpr : -1;
    }
    for (int v0 = static_cast<int>(blockIdx.y) * cpb + threadIdx.x; v0 < c_end; v0 += 256 * VU) {
      float4 acc[VU];
      if (ksplit == 1) {
        float4 r[VU][K];
#pragma unroll
        for (int u = 0; u < VU; ++u) {
          const int v = v0 + u * 256;
#pragma unroll
          for (int j = 0; j < K; ++j)
            r[u][j] = (v < c_end && base[j] >= 0) ? Y4[base[j] + v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < VU; ++u) {
          acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int j = 0; j < K; ++j) {
            acc[u].x += r[u][j].x; acc[u].y += r[u][j].y; acc[u].z += r[u][j].z; acc[u].w += r[u][j].w;
          }
        }
      } else if constexpr (VU == 1) {  // (the host launches K-range partials with VU = 1)
        // K-range partials: each choice's ranges summed in order, then the
        // choices in order.  Up to three choices: KU ranges of every choice
        // in flight at a time; more: one choice at a time, four ranges.
        constexpr int KC = K <= 3 ? K : 1;       // choices loaded together
        constexpr int KU = K <= 3 ? 8 / K : 4;   // ranges loaded together
        const int64_t ss4 = split_stride >> 2;
        acc[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (v0 < c_end) {
#pragma unroll
          for (int j0 = 0; j0 < K; j0 += KC) {
            float4 sj[KC];
#pragma unroll
            for (int j = 0; j < KC; ++j) sj[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int ks0 = 0; ks0 < ksplit; ks0 += KU) {
              float4 q[KU][KC];
#pragma unroll
              for (int i = 0; i < KU; ++i)
#pragma unroll
                for (int j = 0; j < KC; ++j)
                  q[i][j] = (ks0 + i < ksplit && base[j0 + j] >= 0) ? Y4[(ks0 + i) * ss4 + base[j0 + j] + v0]
                                                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int i = 0; i < KU; ++i)
#pragma unroll
                for (int j = 0; j < KC; ++j) {
                  sj[j].x += q[i][j].x; sj[j].y += q[i][j].y; sj[j].z += q[i][j].z; sj[j].w += q[i][j].w;
                }
            }
#pragma unroll
            for (int j = 0; j < KC; ++j) {
              acc[0].x += sj[j].x; acc[0].y += sj[j].y; acc[0].z += sj[j].z; acc[0].w += sj[j].w;
            }
          }
        }
      } else {
#pragma unroll
        for (int u = 0; u < VU; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      // shared experts' rows (offsets[E] + s * T + t), after the routed sum, in order s
      for (int si = 0; si < n_shared; ++si) {
        const int64_t rb = (sb + static_cast<int64_t>(si) * T + t) * vpr;
#pragma unroll
        for (int u = 0; u < VU; ++u) {
          const int v = v0 + u * 256;
          if (v >= c_end) continue;
          float4 sj = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
          for (int ks = 0; ks < ksplit; ++ks) {
            const float4 q = Y4[ks * (split_stride >> 2) + rb + v];
            sj.x += q.x; sj.y += q.y; sj.z += q.z; sj.w += q.w;
          }
          acc[u].x += sj.x; acc[u].y += sj.y; acc[u].z += sj.z; acc[u].w += sj.w;
        }
      }
#pragma unroll
      for (int u = 0; u < VU; ++u) {
        const int v = v0 + u * 256;
        if (v >= c_end) continue;
        if (yf != nullptr) reinterpret_cast<float4*>(yf + t * d)[v] = acc[u];
        if constexpr (sizeof(YT) == 2) {
          uint2 o;
          o.x = pack_bf16x2(acc[u].x, acc[u].y);
          o.y = pack_bf16x2(acc[u].z, acc[u].w);
          reinterpret_cast<uint2*>(y + t * d)[v] = o;
        } else {
          reinterpret_cast<float4*>(y + t * d)[v] = acc[u];
        }
      }
    }
  }
}

// Scalar combine for rows whose width is not a multiple of 4 (fp32 layers).
template <typename YT>
__global__ void __launch_bounds__(256) combine_scalar_kernel(int64_t T, int k, int d,
                                                             const int32_t* __restrict__ dest_row, int n_shared,
                                                             const int32_t* __restrict__ shared_base,
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
  for (int si = 0; si < n_shared; ++si) {  // shared experts after the routed sum
    const int64_t row = *shared_base + static_cast<int64_t>(si) * T + t;
    float sj = 0.f;
    for (int ks = 0; ks < ksplit; ++ks) sj += Yp[static_cast<int64_t>(ks) * split_stride + row * d + c];
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

int route_small_chunks(int E, int d) {
  int ds = (d + 255) / 256;
  const int want = (2 * 148 + E - 1) / E;  // about two blocks per SM over all experts
  if (ds > want) ds = want;
  if (ds > SMALL_DS_MAX) ds = SMALL_DS_MAX;
  return ds < 1 ? 1 : ds;
}

size_t route_small_partials_bytes(int E) {
  return static_cast<size_t>(SMALL_DS_MAX) * SMALL_T * E * sizeof(float);
}

cudaError_t launch_route_small(const RoutingArgs& a, void* partials, cudaStream_t s) {
  const int n_ds = route_small_chunks(a.E, a.d);
  const int chunk = (a.d + n_ds - 1) / n_ds;
  float* part = static_cast<float*>(partials);
  const size_t smem = static_cast<size_t>(a.T) * a.E * sizeof(float);
  cudaError_t e;
  if (a.logits_in == nullptr) {  // the first kernel of the forward: an ordinary launch
    if (a.x_is_bf16)
      route_small_dot_kernel<__nv_bfloat16><<<dim3(n_ds, a.E), 256, 0, s>>>(a, chunk, part);
    else
      route_small_dot_kernel<float><<<dim3(n_ds, a.E), 256, 0, s>>>(a, chunk, part);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.x_is_bf16)
      return launch_pdl(route_small_kernel<__nv_bfloat16>, dim3(1), dim3(SCAN_T), smem, s, a, n_ds,
                        static_cast<const float*>(part));
    return launch_pdl(route_small_kernel<float>, dim3(1), dim3(SCAN_T), smem, s, a, n_ds,
                      static_cast<const float*>(part));
  }
  if (a.x_is_bf16)
    route_small_kernel<__nv_bfloat16><<<1, SCAN_T, smem, s>>>(a, 0, part);
  else
    route_small_kernel<float><<<1, SCAN_T, smem, s>>>(a, 0, part);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_scan(const RoutingArgs& a, cudaStream_t s) {
  if (a.nblk <= kScanSingleBlocks) return launch_pdl(scan_kernel<true>, dim3(1), dim3(SCAN_T), 0, s, a);
  return launch_pdl(scan_kernel<false>, dim3(a.E), dim3(SCAN_T), 0, s, a);
}

bool scan_dispatch_fits(const RoutingArgs& a) {
  // histogram loads per lane: ceil(E / 8) rows of ceil(nblk / 32) entries
  const int64_t loads = static_cast<int64_t>((a.E + 7) / 8) * ((a.nblk + 31) / 32);
  return a.E <= 256 && loads <= kFusedLoads;
}

cudaError_t launch_scan_dispatch(const RoutingArgs& a, cudaStream_t s) {
  // few router blocks: split each block's rows over up to 8 parts (about two
  // blocks per SM in all)
  int parts = (2 * 148) / (a.nblk > 0 ? a.nblk : 1);
  parts = parts < 1 ? 1 : (parts > 8 ? 8 : parts);
  const dim3 grid(static_cast<unsigned>(a.nblk + 1), static_cast<unsigned>(parts));  // + the statistics block
  if (a.x_is_bf16) return launch_pdl(scan_dispatch_kernel<__nv_bfloat16>, grid, dim3(SCAN_T), 0, s, a);
  return launch_pdl(scan_dispatch_kernel<float>, grid, dim3(SCAN_T), 0, s, a);
}

cudaError_t launch_dispatch(const RoutingArgs& a, cudaStream_t s) {
  // one more block finalises the scan when its per-expert blocks did not
  // (the single-block scan finalises itself)
  const unsigned grid = static_cast<unsigned>(a.nblk + (a.nblk > kScanSingleBlocks ? 1 : 0));
  if (a.x_is_bf16) return launch_pdl(dispatch_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s, a);
  return launch_pdl(dispatch_kernel<float>, dim3(grid), dim3(256), 0, s, a);
}

namespace {
template <int K>
cudaError_t launch_combine_k(int64_t T, int d, int y_is_bf16, const int32_t* dest_row, int n_shared,
                             const int32_t* shared_base, const float* Yp, int ksplit, int64_t split_stride, void* y,
                             float* y_f32, cudaStream_t s) {
  const int64_t blocks = T < 148 * 16 ? T : 148 * 16;
  // few tokens: split each row's groups of 4 columns over up to yc blocks
  // (about two blocks per SM in all, at least 256 groups per block)
  const int vpr = d / 4;
  int yc = static_cast<int>((2 * 148 + blocks - 1) / (blocks > 0 ? blocks : 1));
  const int yc_max = (vpr + 255) / 256;
  if (yc > yc_max) yc = yc_max;
  if (yc < 1) yc = 1;
  const int cpb = (vpr + yc - 1) / yc;
  const dim3 grid(static_cast<unsigned>(blocks > 0 ? blocks : 1), static_cast<unsigned>(yc));
  // column groups per thread and pass: two for up to four choices, one where
  // the loads of K-range partials take the registers
  if (ksplit > 1 || K > 4) {
    if (y_is_bf16)
      return launch_pdl(combine_kernel<__nv_bfloat16, K, 1>, grid, dim3(256), 0, s, T, d, dest_row, n_shared,
                        shared_base, Yp, ksplit, split_stride, cpb, static_cast<__nv_bfloat16*>(y), y_f32);
    return launch_pdl(combine_kernel<float, K, 1>, grid, dim3(256), 0, s, T, d, dest_row, n_shared, shared_base,
                      Yp, ksplit, split_stride, cpb, static_cast<float*>(y), y_f32);
  }
  if (y_is_bf16)
    return launch_pdl(combine_kernel<__nv_bfloat16, K, 2>, grid, dim3(256), 0, s, T, d, dest_row, n_shared,
                      shared_base, Yp, ksplit, split_stride, cpb, static_cast<__nv_bfloat16*>(y), y_f32);
  return launch_pdl(combine_kernel<float, K, 2>, grid, dim3(256), 0, s, T, d, dest_row, n_shared, shared_base, Yp,
                    ksplit, split_stride, cpb, static_cast<float*>(y), y_f32);
}
}  // namespace

cudaError_t launch_combine(int64_t T, int k, int d, int y_is_bf16, const int32_t* dest_row, int n_shared,
                           const int32_t* shared_base, const float* Yp, int ksplit, int64_t split_stride, void* y,
                           float* y_f32, cudaStream_t s) {
  if ((d & 3) == 0) {
    switch (k) {
      case 1:
        return launch_combine_k<1>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 2:
        return launch_combine_k<2>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 3:
        return launch_combine_k<3>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 4:
        return launch_combine_k<4>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 5:
        return launch_combine_k<5>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 6:
        return launch_combine_k<6>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      case 7:
        return launch_combine_k<7>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
      default:
        return launch_combine_k<8>(T, d, y_is_bf16, dest_row, n_shared, shared_base, Yp, ksplit, split_stride, y,
                                     y_f32, s);
    }
  }
  const dim3 grid(static_cast<unsigned>((T * d + 255) / 256));
  if (y_is_bf16)
    return launch_pdl(combine_scalar_kernel<__nv_bfloat16>, grid, dim3(256), 0, s, T, k, d, dest_row, n_shared,
                      shared_base, Yp, ksplit, split_stride, static_cast<__nv_bfloat16*>(y), y_f32);
  return launch_pdl(combine_scalar_kernel<float>, grid, dim3(256), 0, s, T, k, d, dest_row, n_shared, shared_base,
                    Yp, ksplit, split_stride, static_cast<float*>(y), y_f32);
}

cudaError_t launch_selftest_timeout(unsigned int* err, int64_t limit_ns, cudaStream_t s) {
  selftest_timeout_kernel<<<1, 32, 0, s>>>(err, static_cast<uint64_t>(limit_ns));
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

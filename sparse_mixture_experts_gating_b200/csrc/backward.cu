// Backward pass of the MoE layer: fp32 accumulation throughout.
//
// Gradients of L = sum_t <dy_t, y_t> + aux_coef * aux + z_coef * z
// ("Mixture of experts", rayaq.ca: section "Replacing the feed-forward
// block" -- the router learns only through the gate values, the choice of
// experts being discrete; section "The load-balancing loss" -- f_i is a count
// without gradient, P_i has one, and the z-loss is the mean of lse^2).  The
// routing of the forward pass (top-k, capacity drops, slots) is held fixed and
// read from its workspace.  Per kept row r of expert e (token t, gate g):
//   a1 = W1_e x_t, a3 = W3_e x_t (recomputed), hid = act(a1, a3)
//   u = W2_e^T dy_t;  dg_r = <u, hid>;  dhid = g u
//   ReLU: da1 = dhid [a1 > 0];  SwiGLU: da3 = dhid silu(a1),
//         da1 = dhid a3 (s + a1 s (1 - s)), s = logistic(a1)
//   dXp_r = W1_e^T da1 + W3_e^T da3;  dW2_e += g dy_t hid^T;  dW1_e += da1 x_t^T
// and per token: dx_t = sum of its kept rows' dXp (and the shared experts'
// rows) + W_r^T dh_t, with dh_t from the gates, the load-balancing loss and
// the z-loss (Switch: through the full softmax; renormalised: through the
// softmax over the chosen logits).  Every sum runs in a fixed order, so the
// results are deterministic.
//
// For fp32 layers the contractions run as tiled fp32 GEMMs on CUDA cores
// (64 x 64 tiles, 16-deep k-steps, 4 x 4 outputs per thread) over the expert
// groups of the sorted buffers.  For bf16 layers every product of the experts
// runs on the forward's tensor-core grouped GEMM with its fp32 epilogue (gate
// 1).  The row-grouped ones (w1 x
// and w3 x again, W2^T dy, W1^T da1 + W3^T da3): the weights are transposed
// per expert into K-major copies, dy is gathered into expert-sorted rows, and
// da1 / da3 enter as hi + lo bf16 planes (about 16 significant bits) like the
// forward's hidden activation.  The weight gradients reduce over each
// expert's ragged rows: every expert's rows are packed transposed and
// zero-padded to k_pad, so each gradient is a product of groups of d_ff rows
// over K = k_pad (dW2 comes out transposed and is turned once more).  The
// router's gradient dW_r, a sum over all tokens, runs on CUDA cores in chunks
// of tokens whose partials are summed in chunk order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "backward.h"
#include "common.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;
constexpr int THREADS = 256;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i) {
  return to_f32(p[i]);
}

// Rows of group e; without offsets, one group of single_rows rows cut into
// chunks of `chunk` rows (0: whole), e being the chunk.
__device__ __forceinline__ void group_rows(const int32_t* offsets, int e, int64_t single_rows, int64_t chunk,
                                           int64_t& r0, int64_t& r1) {
  if (offsets != nullptr) { r0 = offsets[e]; r1 = offsets[e + 1]; return; }
  if (chunk <= 0) { r0 = 0; r1 = single_rows; return; }
  r0 = e * chunk;
  r1 = r0 + chunk < single_rows ? r0 + chunk : single_rows;
}

// 4 x 4 outputs per thread from shared tiles As[TK][TM], Bs[TK][TN].
__device__ __forceinline__ void tile_fma(const float (*As)[TM + 4], const float (*Bs)[TN + 4], int ty, int tx,
                                         float (&acc)[4][4]) {
#pragma unroll
  for (int kk = 0; kk < TK; ++kk) {
    float av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// Row-grouped GEMM: C[r][n] = sum_k A(r, k) B_e(n, k) for the rows r of
// group e = blockIdx.z, k over K0 terms of (A0, B0) then K1 terms of (A1, B1).
//   A(r, k) = A0[ar * K0 + k] (A1[ar * K1 + k - K0]), ar = GATHER ? row_token[r] : r
//   B_e(n, k) = KMAJOR ? B0[(e N + n) K0 + k] : B0[(e K0 + k) N + n]   (B1 likewise with K1)
struct RowGemm {
  int N, K0, K1;
  const void* A0;
  const void* A1;
  const void* B0;
  const void* B1;
  float* C;  // [rows][N]
  const int32_t* offsets;
  const int32_t* row_token;
};

template <typename TA, typename TB, bool KMAJOR, bool GATHER>
__global__ void __launch_bounds__(THREADS) bw_rowgemm_kernel(RowGemm g) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int e = blockIdx.z;
  int64_t g0, g1;
  group_rows(g.offsets, e, 0, 0, g0, g1);
  const int64_t r0 = g0 + static_cast<int64_t>(blockIdx.y) * TM;
  if (r0 >= g1) return;
  const int n0 = blockIdx.x * TN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int K = g.K0 + g.K1;
  const TA* A0 = static_cast<const TA*>(g.A0);
  const TA* A1 = static_cast<const TA*>(g.A1);
  const TB* B0 = static_cast<const TB*>(g.B0);
  const TB* B1 = static_cast<const TB*>(g.B1);
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
#pragma unroll
    for (int q = 0; q < (TM * TK) / THREADS; ++q) {  // A tile, k fastest
      const int el = tid + q * THREADS;
      const int i = el / TK, kk = el % TK;
      const int64_t r = r0 + i;
      const int k = k0 + kk;
      float v = 0.f;
      if (r < g1 && k < K) {
        const int64_t ar = GATHER ? g.row_token[r] : r;
        v = k < g.K0 ? ldf(A0, ar * g.K0 + k) : ldf(A1, ar * g.K1 + (k - g.K0));
      }
      As[kk][i] = v;
    }
#pragma unroll
    for (int q = 0; q < (TN * TK) / THREADS; ++q) {  // B tile, along its contiguous index
      const int el = tid + q * THREADS;
      const int j = KMAJOR ? el / TK : el % TN;
      const int kk = KMAJOR ? el % TK : el / TN;
      const int n = n0 + j, k = k0 + kk;
      float v = 0.f;
      if (n < g.N && k < K) {
        if (k < g.K0)
          v = KMAJOR ? ldf(B0, (static_cast<int64_t>(e) * g.N + n) * g.K0 + k)
                     : ldf(B0, (static_cast<int64_t>(e) * g.K0 + k) * g.N + n);
        else
          v = KMAJOR ? ldf(B1, (static_cast<int64_t>(e) * g.N + n) * g.K1 + (k - g.K0))
                     : ldf(B1, (static_cast<int64_t>(e) * g.K1 + (k - g.K0)) * g.N + n);
      }
      Bs[kk][j] = v;
    }
    __syncthreads();
    tile_fma(As, Bs, ty, tx, acc);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty * 4 + i;
    if (r >= g1) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < g.N) g.C[r * g.N + n] = acc[i][j];
    }
  }
}

// Gradient of a weight per group: C_e[m][n] = sum over the rows r of group e
// of P(r, m) Q(r, n), rows in order; P(r, m) = P[pr * M + m] (times
// row_gate[r] and pr = row_token[r] with GATHER_SCALE, else pr = r),
// Q(r, n) = Q[r * N + n].  offsets NULL: one group of `rows` rows, cut into
// chunks of `chunk` rows whose partial products go to C + chunk * M * N (0:
// whole).  Groups without rows get zeros.
struct WGrad {
  int M, N;
  int64_t rows, chunk;
  const void* P;
  const void* Q;
  float* C;  // [groups][M][N]
  const int32_t* offsets;
  const int32_t* row_token;
  const float* row_gate;
};

template <typename TP, typename TQ, bool GATHER_SCALE>
__global__ void __launch_bounds__(THREADS) bw_wgrad_kernel(WGrad g) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int e = blockIdx.z;
  int64_t g0, g1;
  group_rows(g.offsets, e, g.rows, g.chunk, g0, g1);
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const TP* P = static_cast<const TP*>(g.P);
  const TQ* Q = static_cast<const TQ*>(g.Q);
  float acc[4][4] = {};
  for (int64_t k0 = g0; k0 < g1; k0 += TK) {
#pragma unroll
    for (int q = 0; q < (TM * TK) / THREADS; ++q) {  // P tile, m fastest
      const int el = tid + q * THREADS;
      const int i = el % TM, kk = el / TM;
      const int64_t r = k0 + kk;
      const int m = m0 + i;
      float v = 0.f;
      if (r < g1 && m < g.M) {
        if (GATHER_SCALE) v = ldf(P, static_cast<int64_t>(g.row_token[r]) * g.M + m) * g.row_gate[r];
        else v = ldf(P, r * g.M + m);
      }
      As[kk][i] = v;
    }
#pragma unroll
    for (int q = 0; q < (TN * TK) / THREADS; ++q) {  // Q tile, n fastest
      const int el = tid + q * THREADS;
      const int j = el % TN, kk = el / TN;
      const int64_t r = k0 + kk;
      const int n = n0 + j;
      Bs[kk][j] = (r < g1 && n < g.N) ? ldf(Q, r * g.N + n) : 0.f;
    }
    __syncthreads();
    tile_fma(As, Bs, ty, tx, acc);
    __syncthreads();
  }
  float* C = g.C + static_cast<int64_t>(e) * g.M * g.N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < g.N) C[static_cast<int64_t>(m) * g.N + n] = acc[i][j];
    }
  }
}

// Block-wide sum of one float per thread, in a fixed order.
__device__ __forceinline__ float block_sum_f(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < THREADS / 32; ++w) t += s_red[w];
  return t;
}

// One block per sorted row: the hidden activation (into A1), the gradients of
// w1 x (into U) and w3 x (into A3), and dg_r = <W2^T dy_t, hid>.
template <bool SWIGLU>
__global__ void __launch_bounds__(THREADS) bw_act_kernel(int d_ff, const int32_t* offsets, int groups,
                                                         const float* row_gate, float* A1, float* A3, float* U,
                                                         float* dg, __nv_bfloat16* dA1p, __nv_bfloat16* dA3p,
                                                         int64_t plane) {
  __shared__ float s_red[THREADS / 32];
  const int64_t r = blockIdx.x;
  if (r >= offsets[groups]) return;
  const float g = row_gate[r];
  float part = 0.f;
  for (int n = threadIdx.x; n < d_ff; n += THREADS) {
    const int64_t i = r * d_ff + n;
    const float a1 = A1[i], u = U[i];
    const float dhid = g * u;
    float da1, da3 = 0.f;
    if (SWIGLU) {
      const float a3 = A3[i];
      const float s = 1.f / (1.f + expf(-a1));
      const float silu = a1 * s;
      const float hid = silu * a3;
      part = fmaf(u, hid, part);
      A1[i] = hid;
      da3 = dhid * silu;
      da1 = dhid * a3 * (s + a1 * s * (1.f - s));
      A3[i] = da3;
    } else {
      const float hid = fmaxf(a1, 0.f);
      part = fmaf(u, hid, part);
      A1[i] = hid;
      da1 = a1 > 0.f ? dhid : 0.f;
    }
    U[i] = da1;
    if (dA1p != nullptr) {  // hi = RNE(v), lo = RNE(v - hi)
      const __nv_bfloat16 h1 = __float2bfloat16_rn(da1);
      dA1p[i] = h1;
      dA1p[plane + i] = __float2bfloat16_rn(da1 - __bfloat162float(h1));
      if (SWIGLU) {
        const __nv_bfloat16 h3 = __float2bfloat16_rn(da3);
        dA3p[i] = h3;
        dA3p[plane + i] = __float2bfloat16_rn(da3 - __bfloat162float(h3));
      }
    }
  }
  const float t = block_sum_f(part, s_red);
  if (threadIdx.x == 0) dg[r] = t;
}

// First-choice counts f_i * T (integer, so order-free).
__global__ void bw_cnt1_kernel(int64_t T, int k, const int32_t* topk_idx, int32_t* cnt1) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  if (t < T) atomicAdd(cnt1 + topk_idx[t * k], 1);
}

// One block per token: the router logits (given: the forward's router kernel
// run again, the same fp32 values; else recomputed here, fp32, bias added
// last), the softmax and log-sum-exp, and the gradient reaching the logits.
template <typename XT>
__global__ void __launch_bounds__(THREADS) bw_router_kernel(BackwardArgs a) {
  __shared__ float s_h[256], s_dp[256], s_dh[256];
  __shared__ float s_red[THREADS / 32];
  __shared__ float s_dgj[8];
  const int64_t t = blockIdx.x;
  const int E = a.E, d = a.d, k = a.k, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const XT* x = static_cast<const XT*>(a.x) + t * d;
  if (a.logits != nullptr) {  // computed again by the forward's router kernel
    for (int e = tid; e < E; e += THREADS) s_h[e] = a.logits[t * E + e];
  } else {
    for (int e = warp; e < E; e += THREADS / 32) {
      const float* w = a.W_r + static_cast<int64_t>(e) * d;
      float s = 0.f;
      for (int c = lane; c < d; c += 32) s = fmaf(w[c], to_f32(x[c]), s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) s_h[e] = a.b_r != nullptr ? s + a.b_r[e] : s;
    }
  }
  if (tid < k) {
    const int dst = a.dest_row[t * k + tid];
    s_dgj[tid] = dst >= 0 ? a.dg[dst] : 0.f;  // a dropped choice passes nothing
  }
  __syncthreads();
  float m = -INFINITY;
  for (int e = tid; e < E; e += THREADS) m = fmaxf(m, s_h[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  m = -INFINITY;
  for (int w = 0; w < THREADS / 32; ++w) m = fmaxf(m, s_red[w]);
  float z = 0.f;
  for (int e = tid; e < E; e += THREADS) z += expf(s_h[e] - m);
  const float Z = block_sum_f(z, s_red);
  const float lse = m + logf(Z);
  const float inv_T = 1.f / static_cast<float>(a.T);
  // dp (Switch gates and the load-balancing loss) and the renormalised gates' direct part
  for (int e = tid; e < E; e += THREADS) {
    float dp = a.aux_coef * static_cast<float>(E) * static_cast<float>(a.cnt1[e]) * inv_T * inv_T;
    float dh = 0.f;
    for (int j = 0; j < k; ++j) {
      if (a.topk_idx[t * k + j] != e) continue;
      if (a.gate_mode == MOE_GATE_SWITCH) {
        dp += s_dgj[j];
      } else {
        float sg = 0.f;
        for (int i = 0; i < k; ++i) sg = fmaf(a.topk_gate[t * k + i], s_dgj[i], sg);
        dh = a.topk_gate[t * k + j] * (s_dgj[j] - sg);
      }
    }
    s_dp[e] = dp;
    s_dh[e] = dh;
  }
  __syncthreads();
  float pd = 0.f;
  for (int e = tid; e < E; e += THREADS) pd = fmaf(expf(s_h[e] - m) / Z, s_dp[e], pd);
  const float dpp = block_sum_f(pd, s_red);
  for (int e = tid; e < E; e += THREADS) {
    const float p = expf(s_h[e] - m) / Z;
    a.dh[t * E + e] = s_dh[e] + p * (s_dp[e] - dpp) + a.z_coef * 2.f * inv_T * lse * p;
  }
}

// dx for 128 tokens x 128 columns per block (16 x 16 threads, 8 x 8 outputs
// each): the router term W_r^T dh_t from 32-expert chunks of dh (transposed)
// and W_r staged in shared memory, experts in order, then the same sum as
// bw_dx_kernel (kept rows' dXp, choices in order, then the shared experts'
// rows) plus that term: the same operations in the same order.  Needs
// d % 8 == 0, E % 4 == 0 and 16-byte aligned dh, W_r, dXp and dx.
__global__ void __launch_bounds__(256) bw_dx_tiled_kernel(BackwardArgs a, int parts) {
  __shared__ __align__(16) float s_h[32][132];  // [expert][token]
  __shared__ __align__(16) float s_w[32][132];  // [expert][column]
  const int E = a.E, d = a.d, k = a.k;
  const int64_t T = a.T;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int c0 = blockIdx.x * 128;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int ne = min(32, E - e0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // dh [128 tokens][32 experts] -> s_h[expert][token]
      const int id = tid + 256 * q, t = id >> 3, e4 = (id & 7) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t0 + t < T && e4 < ne) v = *reinterpret_cast<const float4*>(a.dh + (t0 + t) * E + e0 + e4);
      s_h[e4][t] = v.x;
      s_h[e4 + 1][t] = v.y;
      s_h[e4 + 2][t] = v.z;
      s_h[e4 + 3][t] = v.w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // W_r [32 experts][128 columns]
      const int id = tid + 256 * q, e = id >> 5, c = (id & 31) * 4;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < ne && c0 + c < d) w = *reinterpret_cast<const float4*>(a.W_r + static_cast<int64_t>(e0 + e) * d + c0 + c);
      *reinterpret_cast<float4*>(&s_w[e][c]) = w;
    }
    __syncthreads();
    for (int e = 0; e < ne; ++e) {
      const float4 h0 = *reinterpret_cast<const float4*>(&s_h[e][ty * 8]);
      const float4 h1 = *reinterpret_cast<const float4*>(&s_h[e][ty * 8 + 4]);
      const float4 w0 = *reinterpret_cast<const float4*>(&s_w[e][tx * 8]);
      const float4 w1 = *reinterpret_cast<const float4*>(&s_w[e][tx * 8 + 4]);
      const float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
      const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(h[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int c = c0 + tx * 8;
  if (c >= d) return;
  const int64_t pstride = a.s_max * d;  // between the W1 and W3 parts of dXp
  const int64_t sbase = a.n_shared > 0 ? a.offsets[E] : 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + ty * 8 + i;
    if (t >= T) break;
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
    auto add_row = [&](int64_t row) {
      const float4* p = reinterpret_cast<const float4*>(a.dXp + row * d + c);
      const float4 p0 = p[0], p1 = p[1];
      v[0] += p0.x; v[1] += p0.y; v[2] += p0.z; v[3] += p0.w;
      v[4] += p1.x; v[5] += p1.y; v[6] += p1.z; v[7] += p1.w;
      if (parts == 2) {
        const float4* p2 = reinterpret_cast<const float4*>(a.dXp + pstride + row * d + c);
        const float4 q0 = p2[0], q1 = p2[1];
        v[0] += q0.x; v[1] += q0.y; v[2] += q0.z; v[3] += q0.w;
        v[4] += q1.x; v[5] += q1.y; v[6] += q1.z; v[7] += q1.w;
      }
    };
    for (int j = 0; j < k; ++j) {
      const int dst = a.dest_row[t * k + j];
      if (dst >= 0) add_row(dst);
    }
    for (int si = 0; si < a.n_shared; ++si) add_row(sbase + si * T + t);
    float4* o = reinterpret_cast<float4*>(a.dx + t * d + c);
    o[0] = make_float4(v[0] + acc[i][0], v[1] + acc[i][1], v[2] + acc[i][2], v[3] + acc[i][3]);
    o[1] = make_float4(v[4] + acc[i][4], v[5] + acc[i][5], v[6] + acc[i][6], v[7] + acc[i][7]);
  }
}

// One block per token: dx_t = its kept rows' dXp (choices in order), then the
// shared experts' rows, then W_r^T dh_t (experts in order).
__global__ void __launch_bounds__(THREADS) bw_dx_kernel(BackwardArgs a, int parts) {
  __shared__ float s_dh[256];
  const int64_t t = blockIdx.x;
  const int E = a.E, d = a.d, k = a.k;
  const int64_t pstride = a.s_max * d;  // between the W1 and W3 parts of dXp
  for (int e = threadIdx.x; e < E; e += THREADS) s_dh[e] = a.dh[t * E + e];
  __syncthreads();
  const int64_t sbase = a.n_shared > 0 ? a.offsets[E] : 0;
  for (int c = threadIdx.x; c < d; c += THREADS) {
    float v = 0.f;
    for (int j = 0; j < k; ++j) {
      const int dst = a.dest_row[t * k + j];
      if (dst < 0) continue;
      v += a.dXp[static_cast<int64_t>(dst) * d + c];
      if (parts == 2) v += a.dXp[pstride + static_cast<int64_t>(dst) * d + c];
    }
    for (int si = 0; si < a.n_shared; ++si) {
      const int64_t row = sbase + si * a.T + t;
      v += a.dXp[row * d + c];
      if (parts == 2) v += a.dXp[pstride + row * d + c];
    }
    float r = 0.f;
    for (int e = 0; e < E; ++e) r = fmaf(s_dh[e], a.W_r[static_cast<int64_t>(e) * d + c], r);
    a.dx[t * d + c] = v + r;
  }
}

// out[i] = sum over z < nz of part[z * n + i], z in order.
__global__ void bw_sum_parts_kernel(int64_t n, int nz, const float* __restrict__ part, float* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= n) return;
  float v = 0.f;
  for (int z = 0; z < nz; ++z) v += part[z * n + i];
  out[i] = v;
}

// db_e = sum over tokens of dh[t][e], tokens in a fixed order.
__global__ void __launch_bounds__(THREADS) bw_db_kernel(int64_t T, int E, const float* dh, float* db) {
  __shared__ float s_red[THREADS / 32];
  const int e = blockIdx.x;
  float s = 0.f;
  for (int64_t t = threadIdx.x; t < T; t += THREADS) s += dh[t * E + e];
  const float tot = block_sum_f(s, s_red);
  if (threadIdx.x == 0) db[e] = tot;
}

// dy rows into expert-sorted order (a warp per row, 16-byte copies).
__global__ void __launch_bounds__(256) bw_gather_dy_kernel(int d, const int32_t* offsets, int groups,
                                                           const int32_t* row_token, const uint4* dy, uint4* dYs) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= offsets[groups]) return;
  const int nv = d / 8;  // 16-byte groups of a bf16 row
  const int64_t t = row_token[r];
  for (int v = lane; v < nv; v += 32) dYs[r * nv + v] = dy[t * nv + v];
}

// One tensor-core grouped GEMM with the fp32 epilogue (gate 1):
// out[r][n] = sum_k A[r][k] B_e[n][k] over the expert-sorted rows.
cudaError_t tc_product(const BackwardArgs& a, const void* A, const void* A_lo, const void* B, int N, int K, float* out,
                       cudaStream_t s, const int32_t* offsets = nullptr, const int32_t* mprefix = nullptr,
                       int64_t a_rows = 0, int max_rows = 0, const int32_t* k_rows = nullptr) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.epi = EPI_GATE_F32;
  g.E = a.E + a.n_shared;
  g.N = N;
  g.K = K;
  g.a_rows = offsets != nullptr ? a_rows : a.s_max;
  g.max_group_rows = offsets != nullptr ? max_rows : a.max_group_rows;
  g.A = A;
  g.A2 = A_lo;
  g.split = A_lo != nullptr;
  g.B0 = B;
  g.out = out;
  g.ksplit = 1;
  g.offsets = offsets != nullptr ? offsets : a.offsets;
  g.mprefix = offsets != nullptr ? mprefix : a.mprefix;
  g.row_gate = a.ones;
  g.row_token = a.row_token;
  g.err = a.err;
  g.k_rows = k_rows;
  TcGemmPlan plan;
  const char* why = nullptr;
  cudaError_t e = plan_gemm_tc(g, &plan, &why);
  if (e != cudaSuccess) return e;
  return launch_gemm_tc(plan, a.num_sms, s);
}

// The per-expert product with a single-plane A and B as hi + lo planes
// (EPI_GATE_F32_B2, gate 1): out[r][n] = sum_k A[r][k] (B_hi + B_lo)_e[n][k]
// over groups of max_rows rows (offsets / mprefix), group e's K = its rows
// in k_rows.
cudaError_t tc_product_b2(const BackwardArgs& a, const void* A, const void* B_hi, const void* B_lo, int N, int K,
                          float* out, cudaStream_t s, const int32_t* offsets, const int32_t* mprefix, int64_t a_rows,
                          int max_rows, const int32_t* k_rows) {
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.epi = EPI_GATE_F32_B2;
  g.E = a.E + a.n_shared;
  g.N = N;
  g.K = K;
  g.a_rows = a_rows;
  g.max_group_rows = max_rows;
  g.A = A;
  g.B0 = B_hi;
  g.B1 = B_lo;
  g.out = out;
  g.ksplit = 1;
  g.offsets = offsets;
  g.mprefix = mprefix;
  g.row_gate = a.ones;
  g.row_token = a.row_token;
  g.err = a.err;
  g.k_rows = k_rows;
  TcGemmPlan plan;
  const char* why = nullptr;
  cudaError_t e = plan_gemm_tc(g, &plan, &why);
  if (e != cudaSuccess) return e;
  return launch_gemm_tc(plan, a.num_sms, s);
}

// bf16 [G][R][C] -> [G][C][R] with R and C even: 64 x 64 tiles, pairs of
// columns read and pairs of rows written as 4-byte words.
__global__ void __launch_bounds__(256) bw_transpose_bf16x2_kernel(const __nv_bfloat16* __restrict__ in,
                                                                  __nv_bfloat16* __restrict__ out, int R, int C) {
  __shared__ __nv_bfloat16 tile[64][66];
  const int64_t g = blockIdx.z;
  const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const __nv_bfloat16* src = in + g * R * C;
  __nv_bfloat16* dst = out + g * R * C;
  for (int i = ty; i < 64; i += 8) {
    const int r = r0 + i, c = c0 + 2 * tx;
    if (r < R && c < C) {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(src + static_cast<int64_t>(r) * C + c);
      tile[i][2 * tx] = v.x;
      tile[i][2 * tx + 1] = v.y;
    }
  }
  __syncthreads();
  for (int i = ty; i < 64; i += 8) {
    const int c = c0 + i, r = r0 + 2 * tx;
    if (c < C && r < R) {
      __nv_bfloat162 v;
      v.x = tile[2 * tx][i];
      v.y = tile[2 * tx + 1][i];
      *reinterpret_cast<__nv_bfloat162*>(dst + static_cast<int64_t>(c) * R + r) = v;
    }
  }
}

// [G][R][C] -> [G][C][R] for elements of 2 or 4 bytes (T = uint16_t / float)
// with R and C multiples of 16 / sizeof(T) and 16-byte aligned buffers: 64 x
// 64 tiles, 16-byte reads along the input rows; each 16-byte write holds
// 16 / sizeof(T) consecutive input rows of one input column, and the threads
// of a warp write whole output row segments (64 elements) side by side.
template <typename T>
__global__ void __launch_bounds__(256) bw_transpose16_kernel(const T* __restrict__ in, T* __restrict__ out, int R,
                                                             int C) {
  constexpr int V = 16 / static_cast<int>(sizeof(T));  // elements per 16-byte word
  constexpr int NW = 64 * 64 / V / 256;                // words per thread and phase
  __shared__ T tile[64][64 + 4 / static_cast<int>(sizeof(T))];  // rows padded by one 4-byte word
  const int64_t g = blockIdx.z;
  const int c0 = blockIdx.x * 64, r0 = blockIdx.y * 64;
  const T* src = in + g * R * C;
  T* dst = out + g * R * C;
  uint4 v[NW];
#pragma unroll
  for (int p = 0; p < NW; ++p) {  // word p of this thread: row id / (64 / V), column chunk id % (64 / V)
    const int id = threadIdx.x + 256 * p;
    const int r = id / (64 / V), c = (id % (64 / V)) * V;
    v[p] = (r0 + r < R && c0 + c < C)
               ? *reinterpret_cast<const uint4*>(src + static_cast<int64_t>(r0 + r) * C + c0 + c)
               : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int p = 0; p < NW; ++p) {
    const int id = threadIdx.x + 256 * p;
    const int r = id / (64 / V), c = (id % (64 / V)) * V;
    const uint32_t w[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint32_t*>(&tile[r][c + j * (4 / sizeof(T))]) = w[j];
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < NW; ++p) {  // output row c0 + oc, input rows r0 + q V .. + V - 1
    const int id = threadIdx.x + 256 * p;
    const int oc = id / (64 / V), q = id % (64 / V);
    if (c0 + oc < C && r0 + q * V < R) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if constexpr (sizeof(T) == 2)
          w[j] = static_cast<uint32_t>(tile[q * V + 2 * j][oc]) | (static_cast<uint32_t>(tile[q * V + 2 * j + 1][oc]) << 16);
        else
          w[j] = __float_as_uint(tile[q * V + j][oc]);
      }
      *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(c0 + oc) * R + r0 + q * V) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

bool aligned16(const void* a, const void* b) {
  return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15) == 0;
}

cudaError_t transpose_bf16(const void* in, void* out, int G, int R, int C, cudaStream_t s) {
  const dim3 grid((C + 63) / 64, (R + 63) / 64, G);
  if (aligned16(in, out) && R % 8 == 0 && C % 8 == 0)
    bw_transpose16_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(in), static_cast<uint16_t*>(out),
                                                        R, C);
  else
    bw_transpose_bf16x2_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in),
                                                    static_cast<__nv_bfloat16*>(out), R, C);
  count_launch();
  return cudaGetLastError();
}


// Per-expert operand of a weight gradient: out[e][f][kk] = v(off_e + kk, f)
// for kk below the group's row count, 0 up to the next multiple of 64 (the
// product's k-blocks; no further than k_pad), where v(r, f) =
// src[r][f] (times scale[r] when given); bf16, with SPLIT a lo plane at
// out + plane holding v - hi.  32 x 32 tiles: rows read along f, written
// along kk.
template <typename ST, bool SPLIT>
__global__ void __launch_bounds__(256) bw_pack_kernel(const ST* __restrict__ src, int F,
                                                      const int32_t* __restrict__ offsets,
                                                      const float* __restrict__ scale, int k_pad,
                                                      __nv_bfloat16* __restrict__ out, int64_t plane) {
  __shared__ float tile[32][33];
  const int e = blockIdx.z;
  const int f0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int64_t off = offsets[e];
  const int rows = static_cast<int>(offsets[e + 1] - off);
  if (k0 >= (rows + 63) / 64 * 64) return;  // the product reads k-blocks of 64 below the group's rows only
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int kk = k0 + i, f = f0 + threadIdx.x;
    float v = 0.f;
    if (kk < rows && f < F) {
      v = to_f32(src[(off + kk) * F + f]);
      if (scale != nullptr) v *= scale[off + kk];
    }
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int f = f0 + i, kk = k0 + threadIdx.x;
    if (f < F && kk < k_pad) {
      const float v = tile[threadIdx.x][i];
      const int64_t o = (static_cast<int64_t>(e) * F + f) * k_pad + kk;
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      out[o] = h;
      if (SPLIT) out[plane + o] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// The same operand in 64 (kk) x 64 (f) tiles with 16-byte accesses: rows of
// src read along f (fp32 tile in shared memory), 16-byte writes of eight
// consecutive kk of one f, the threads of a warp writing whole 128-byte row
// segments.  Needs F % 8 == 0, k_pad % 8 == 0 and 16-byte aligned buffers.
template <typename ST, bool SPLIT>
__global__ void __launch_bounds__(256) bw_pack16_kernel(const ST* __restrict__ src, int F,
                                                        const int32_t* __restrict__ offsets,
                                                        const float* __restrict__ scale, int k_pad,
                                                        __nv_bfloat16* __restrict__ out, int64_t plane) {
  constexpr int V = 16 / static_cast<int>(sizeof(ST));  // source elements per 16-byte load
  constexpr int NL = 64 * 64 / V / 256;                  // loads per thread
  __shared__ float tile[64][65];
  const int e = blockIdx.z;
  const int f0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  const int64_t off = offsets[e];
  const int rows = static_cast<int>(offsets[e + 1] - off);
  if (k0 >= (rows + 63) / 64 * 64) return;  // the product reads k-blocks of 64 below the group's rows only
#pragma unroll
  for (int p = 0; p < NL; ++p) {
    const int id = threadIdx.x + 256 * p;
    const int r = id / (64 / V), c = (id % (64 / V)) * V;
    float v[V];
    if (k0 + r < rows && f0 + c < F) {
      const uint4 u = *reinterpret_cast<const uint4*>(src + (off + k0 + r) * F + f0 + c);
      const float sc = scale != nullptr ? scale[off + k0 + r] : 1.f;
      if constexpr (sizeof(ST) == 2) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[2 * j] = __uint_as_float(w[j] << 16);
          v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      } else {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
      }
      if (scale != nullptr)
#pragma unroll
        for (int j = 0; j < V; ++j) v[j] *= sc;
    } else {
#pragma unroll
      for (int j = 0; j < V; ++j) v[j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < V; ++j) tile[r][c + j] = v[j];
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < 2; ++p) {  // output row f0 + oc, kk = k0 + 8 q .. + 7
    const int id = threadIdx.x + 256 * p;
    const int oc = id / 8, q = id % 8;
    if (f0 + oc >= F || k0 + 8 * q >= k_pad) continue;
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = tile[8 * q + 2 * j][oc], b = tile[8 * q + 2 * j + 1][oc];
      const __nv_bfloat16 ha = __float2bfloat16_rn(a), hb = __float2bfloat16_rn(b);
      hi[j] = static_cast<uint32_t>(__bfloat16_as_ushort(ha)) | (static_cast<uint32_t>(__bfloat16_as_ushort(hb)) << 16);
      if (SPLIT) {
        const __nv_bfloat16 la = __float2bfloat16_rn(a - __bfloat162float(ha));
        const __nv_bfloat16 lb = __float2bfloat16_rn(b - __bfloat162float(hb));
        lo[j] = static_cast<uint32_t>(__bfloat16_as_ushort(la)) | (static_cast<uint32_t>(__bfloat16_as_ushort(lb)) << 16);
      }
    }
    const int64_t o = (static_cast<int64_t>(e) * F + f0 + oc) * k_pad + k0 + 8 * q;
    *reinterpret_cast<uint4*>(out + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (SPLIT) *reinterpret_cast<uint4*>(out + plane + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

template <typename ST, bool SPLIT>
cudaError_t pack(const void* src, int F, const int32_t* offsets, const float* scale, int G, int k_pad, void* out,
                 int64_t plane, cudaStream_t s) {
  const bool wide = F % 8 == 0 && k_pad % 8 == 0 && plane % 8 == 0 &&
                    ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  if (wide) {
    const dim3 grid((F + 63) / 64, (k_pad + 63) / 64, G);
    bw_pack16_kernel<ST, SPLIT><<<grid, 256, 0, s>>>(static_cast<const ST*>(src), F, offsets, scale, k_pad,
                                                     static_cast<__nv_bfloat16*>(out), plane);
  } else {
    const dim3 grid((F + 31) / 32, (k_pad + 31) / 32, G);
    bw_pack_kernel<ST, SPLIT><<<grid, dim3(32, 8), 0, s>>>(static_cast<const ST*>(src), F, offsets, scale, k_pad,
                                                           static_cast<__nv_bfloat16*>(out), plane);
  }
  count_launch();
  return cudaGetLastError();
}

// Gate 1 for n rows, and the group tables of the per-expert products
// (groups of F rows each: offsets e F, m-tile prefix e ceil(F / 128)), for
// F = F1 and F = F2.
__global__ void bw_tables_kernel(int64_t n, float* ones, int G, int F1, int32_t* woff1, int32_t* wpre1, int F2,
                                 int32_t* woff2, int32_t* wpre2) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i < n) ones[i] = 1.f;
  if (i <= G) {
    woff1[i] = static_cast<int32_t>(i * F1);
    wpre1[i] = static_cast<int32_t>(i * ((F1 + kTileM - 1) / kTileM));
    woff2[i] = static_cast<int32_t>(i * F2);
    wpre2[i] = static_cast<int32_t>(i * ((F2 + kTileM - 1) / kTileM));
  }
}

template <typename TA, typename TB, bool KMAJOR, bool GATHER>
cudaError_t rowgemm(const RowGemm& g, int groups, int max_rows, cudaStream_t s) {
  const dim3 grid((g.N + TN - 1) / TN, (max_rows + TM - 1) / TM, groups);
  bw_rowgemm_kernel<TA, TB, KMAJOR, GATHER><<<grid, THREADS, 0, s>>>(g);
  count_launch();
  return cudaGetLastError();
}

template <typename TP, typename TQ, bool GATHER_SCALE>
cudaError_t wgrad(const WGrad& g, int groups, cudaStream_t s) {
  const dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM, groups);
  bw_wgrad_kernel<TP, TQ, GATHER_SCALE><<<grid, THREADS, 0, s>>>(g);
  count_launch();
  return cudaGetLastError();
}

template <typename XT>
cudaError_t backward_t(const BackwardArgs& a, cudaStream_t s) {
  const int groups = a.E + a.n_shared;
  const bool swiglu = a.act == MOE_ACT_SWIGLU;
  cudaError_t e;
  // first-choice counts for the load-balancing loss's gradient
  if ((e = cudaMemsetAsync(a.cnt1, 0, sizeof(int32_t) * a.E, s)) != cudaSuccess) return e;
  bw_cnt1_kernel<<<static_cast<unsigned>((a.T + THREADS - 1) / THREADS), THREADS, 0, s>>>(a.T, a.k, a.topk_idx,
                                                                                          a.cnt1);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const bool tc = a.x_is_bf16 != 0;
  const int64_t plane = a.s_max * static_cast<int64_t>(a.d_ff);
  if (tc) {
    // K-major copies of the weights for the transposed products, dy in sorted rows
    if ((e = transpose_bf16(a.W2, a.W2t, groups, a.d, a.d_ff, s)) != cudaSuccess) return e;
    if ((e = transpose_bf16(a.W1, a.W1t, groups, a.d_ff, a.d, s)) != cudaSuccess) return e;
    if (swiglu && (e = transpose_bf16(a.W3, a.W3t, groups, a.d_ff, a.d, s)) != cudaSuccess) return e;
    const int64_t n_ones = std::max<int64_t>(a.s_max, static_cast<int64_t>(groups) * std::max(a.d_ff, a.d));
    bw_tables_kernel<<<static_cast<unsigned>((std::max<int64_t>(n_ones, groups + 1) + 255) / 256), 256, 0, s>>>(
        n_ones, a.ones, groups, a.d_ff, a.woff, a.wpre, a.d, a.woff_d, a.wpre_d);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bw_gather_dy_kernel<<<static_cast<unsigned>((a.s_max + 7) / 8), 256, 0, s>>>(
        a.d, a.offsets, groups, a.row_token, static_cast<const uint4*>(a.dy), static_cast<uint4*>(a.dYs));
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // a1 = W1 x, a3 = W3 x, u = W2^T dy
    if ((e = tc_product(a, a.Xp, nullptr, a.W1, a.d_ff, a.d, a.A1, s)) != cudaSuccess) return e;
    if (swiglu && (e = tc_product(a, a.Xp, nullptr, a.W3, a.d_ff, a.d, a.A3, s)) != cudaSuccess) return e;
    if ((e = tc_product(a, a.dYs, nullptr, a.W2t, a.d_ff, a.d, a.U, s)) != cudaSuccess) return e;
  } else {
    // a1 = W1 x, a3 = W3 x
    RowGemm g{};
    g.N = a.d_ff;
    g.K0 = a.d;
    g.A0 = a.Xp;
    g.B0 = a.W1;
    g.C = a.A1;
    g.offsets = a.offsets;
    g.row_token = a.row_token;
    if ((e = rowgemm<XT, XT, true, false>(g, groups, a.max_group_rows, s)) != cudaSuccess) return e;
    if (swiglu) {
      g.B0 = a.W3;
      g.C = a.A3;
      if ((e = rowgemm<XT, XT, true, false>(g, groups, a.max_group_rows, s)) != cudaSuccess) return e;
    }
    // u = W2^T dy_t
    g.K0 = a.d;
    g.A0 = a.dy;
    g.B0 = a.W2;
    g.C = a.U;
    if ((e = rowgemm<XT, XT, false, true>(g, groups, a.max_group_rows, s)) != cudaSuccess) return e;
  }
  // hidden activation, its gradients, dg
  __nv_bfloat16* p1 = tc ? static_cast<__nv_bfloat16*>(a.dA1p) : nullptr;
  __nv_bfloat16* p3 = tc && swiglu ? static_cast<__nv_bfloat16*>(a.dA3p) : nullptr;
  if (swiglu)
    bw_act_kernel<true><<<static_cast<unsigned>(a.s_max), THREADS, 0, s>>>(a.d_ff, a.offsets, groups, a.row_gate,
                                                                            a.A1, a.A3, a.U, a.dg, p1, p3, plane);
  else
    bw_act_kernel<false><<<static_cast<unsigned>(a.s_max), THREADS, 0, s>>>(a.d_ff, a.offsets, groups, a.row_gate,
                                                                             a.A1, a.A3, a.U, a.dg, p1, p3, plane);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dXp = W1^T da1 (+ W3^T da3)
  int parts = 1;
  if (tc) {
    if ((e = tc_product(a, p1, p1 + plane, a.W1t, a.d, a.d_ff, a.dXp, s)) != cudaSuccess) return e;
    if (swiglu) {
      if ((e = tc_product(a, p3, p3 + plane, a.W3t, a.d, a.d_ff, a.dXp + a.s_max * a.d, s)) != cudaSuccess)
        return e;
      parts = 2;
    }
  } else {
    RowGemm gx{};
    gx.N = a.d;
    gx.K0 = a.d_ff;
    gx.K1 = swiglu ? a.d_ff : 0;
    gx.A0 = a.U;
    gx.A1 = a.A3;
    gx.B0 = a.W1;
    gx.B1 = a.W3;
    gx.C = a.dXp;
    gx.offsets = a.offsets;
    if ((e = rowgemm<float, XT, false, false>(gx, groups, a.max_group_rows, s)) != cudaSuccess) return e;
  }
  // weight gradients
  if (tc) {
    // per expert: dW1_e = da1^T x, dW3_e = da3^T x, dW2_e^T = (g hid)^T dy over
    // its rows, zero-padded to k_pad, as products of F-row groups
    const int kp = a.k_pad;
    const int64_t pl = static_cast<int64_t>(groups) * a.d_ff * kp;  // between the hi and lo planes
    const int64_t arows = static_cast<int64_t>(groups) * a.d_ff;
    auto* P1 = static_cast<__nv_bfloat16*>(a.P1);
    auto* P3 = static_cast<__nv_bfloat16*>(a.P3);
    auto* PH = static_cast<__nv_bfloat16*>(a.PH);
    if ((e = pack<__nv_bfloat16, false>(a.Xp, a.d, a.offsets, nullptr, groups, kp, a.XT, 0, s)) != cudaSuccess)
      return e;
    if ((e = pack<__nv_bfloat16, false>(a.dYs, a.d, a.offsets, nullptr, groups, kp, a.DT, 0, s)) != cudaSuccess)
      return e;
    if ((e = pack<float, true>(a.U, a.d_ff, a.offsets, nullptr, groups, kp, P1, pl, s)) != cudaSuccess) return e;
    if ((e = pack<float, true>(a.A1, a.d_ff, a.offsets, a.row_gate, groups, kp, PH, pl, s)) != cudaSuccess) return e;
    if ((e = tc_product(a, P1, P1 + pl, a.XT, a.d, kp, a.dW1, s, a.woff, a.wpre, arows, a.d_ff, a.offsets)) != cudaSuccess)
      return e;
    if (swiglu) {
      if ((e = pack<float, true>(a.A3, a.d_ff, a.offsets, nullptr, groups, kp, P3, pl, s)) != cudaSuccess) return e;
      if ((e = tc_product(a, P3, P3 + pl, a.XT, a.d, kp, a.dW3, s, a.woff, a.wpre, arows, a.d_ff, a.offsets)) != cudaSuccess)
        return e;
    }
    // dW2_e [d][d_ff] directly: A = dy^T (d rows per expert), B = (g hid)^T as hi + lo planes
    if ((e = tc_product_b2(a, a.DT, PH, PH + pl, a.d_ff, kp, a.dW2, s, a.woff_d, a.wpre_d,
                           static_cast<int64_t>(groups) * a.d, a.d, a.offsets)) != cudaSuccess)
      return e;
  } else {
  WGrad w{};
  w.offsets = a.offsets;
  w.row_token = a.row_token;
  w.row_gate = a.row_gate;
  w.M = a.d;  // dW2_e = sum_r (g_r dy_t) hid_r^T
  w.N = a.d_ff;
  w.P = a.dy;
  w.Q = a.A1;
  w.C = a.dW2;
  if ((e = wgrad<XT, float, true>(w, groups, s)) != cudaSuccess) return e;
  w.M = a.d_ff;  // dW1_e = sum_r da1_r x_r^T
  w.N = a.d;
  w.P = a.U;
  w.Q = a.Xp;
  w.C = a.dW1;
  if ((e = wgrad<float, XT, false>(w, groups, s)) != cudaSuccess) return e;
  if (swiglu) {
    w.P = a.A3;
    w.C = a.dW3;
    if ((e = wgrad<float, XT, false>(w, groups, s)) != cudaSuccess) return e;
  }
  }
  // router: dh, then dx, dW_r, db_r
  bw_router_kernel<XT><<<static_cast<unsigned>(a.T), THREADS, 0, s>>>(a);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const bool tiled = a.d % 8 == 0 && a.E % 4 == 0 && (a.T + 127) / 128 <= 65535 &&
                     ((reinterpret_cast<uintptr_t>(a.W_r) | reinterpret_cast<uintptr_t>(a.dXp) |
                       reinterpret_cast<uintptr_t>(a.dx) | reinterpret_cast<uintptr_t>(a.dh)) & 15) == 0;
  if (tiled)
    bw_dx_tiled_kernel<<<dim3(static_cast<unsigned>((a.d + 127) / 128), static_cast<unsigned>((a.T + 127) / 128)), 256,
                         0, s>>>(a, parts);
  else
    bw_dx_kernel<<<static_cast<unsigned>(a.T), THREADS, 0, s>>>(a, parts);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // dW_r = sum_t dh_t x_t^T: K = T cut into a.wr_chunks chunks of partials, summed in order
  WGrad wr{};
  wr.M = a.E;
  wr.N = a.d;
  wr.rows = a.T;
  wr.chunk = (a.T + a.wr_chunks - 1) / a.wr_chunks;
  wr.P = a.dh;
  wr.Q = a.x;
  wr.C = a.wr_part;
  if ((e = wgrad<float, XT, false>(wr, a.wr_chunks, s)) != cudaSuccess) return e;
  const int64_t nwr = static_cast<int64_t>(a.E) * a.d;
  bw_sum_parts_kernel<<<static_cast<unsigned>((nwr + 255) / 256), 256, 0, s>>>(nwr, a.wr_chunks, a.wr_part, a.dW_r);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.db_r != nullptr) {
    bw_db_kernel<<<a.E, THREADS, 0, s>>>(a.T, a.E, a.dh, a.db_r);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s) {
  return a.x_is_bf16 ? backward_t<__nv_bfloat16>(a, s) : backward_t<float>(a, s);
}

}  // namespace moe

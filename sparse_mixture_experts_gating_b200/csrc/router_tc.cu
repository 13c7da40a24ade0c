// Router of bf16 layers on the tensor cores, with fp32 arithmetic:
//   h = W_r x (+ b)  ("Mixture of experts", rayaq.ca, section "Replacing the
//   feed-forward block"; the router stays float32 per section "Implementation").
//
// W_r (fp32) is split exactly into three bf16 planes w0 + w1 + w2 = W_r (each
// plane takes the next 8 significant bits of the residual; 3 x 8 = 24 bits =
// an fp32 significand).  x is bf16, so every product x_c * w_p,c is exact and
// the tcgen05 MMA accumulates all 3d of them in fp32 in TMEM: an fp32 dot
// product, not a reduced-precision one.  With dyadic inputs whose partial sums
// are all representable, the logits are exact in any order.
//
// One CTA per 128-token tile (persistent over tiles): warp 0 issues TMA (x box
// 128 x 64, three plane boxes E_pad x 64), warp 1 issues the MMAs (M 128,
// N E_pad, K 16; 4 per plane per k-block), and 4 NP epilogue warps take each
// token (TMEM lane) with NP threads, one per part of the experts (NP = 2, or 4
// for E_pad 64 and 128): bias, max, one-pass top-k (ties to the lower expert index),
// log-sum-exp, gates, and the per-32-token partial counts and sums that the
// scan kernel reduces (the warps of one TMEM lane quarter own one 32-token
// router block, the same partition as the CUDA-core router).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
// Epilogue threads per token (expert parts) and block size: two parts of up
// to 16 experts (E_pad 16, 32); for E_pad 64 and 128, four parts of 16 or 32,
// so that each thread keeps its logits in registers and the top-k and
// exponential chains stay short.
template <int EP>
struct RtShape {
  static constexpr int NP = EP >= 64 ? 4 : 2;
  static constexpr int THREADS = 64 + 128 * NP;  // producer, MMA, 4 NP epilogue warps
};
constexpr int A_BYTES = BM * BK * 2;
constexpr int MAX_STAGES = 8;  // small router tiles: a deep ring hides the TMA round trip

struct RtParams {
  int64_t T;
  int E, k, d, gate_mode, num_kb, nblk, n_tiles;
  int ksplit, kb_per;   // K ranges per tile (1: no split) and k-blocks per range
  float* partials;      // [n_tiles][ksplit][128][EP] fp32 partial logits
  int* tickets;         // [n_tiles] ranges finished (zeroed by the split kernel)
  const float* b_r;
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* part_hist;
  int32_t* part_cnt1;
  float* part_psum;
  float* part_lse2;
  float* logits_out;
  float* lse_out;
  unsigned int* err;
  uint64_t limit_ns;
};

template <int NP, int K>
struct RtCtl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  volatile int abort;
  int last;  // this CTA finished the last K range of the tile
  int hist[4][kRouterTcMaxE];
  int cnt1[4][kRouterTcMaxE];
  float xm[4][NP][32];           // per lane quarter and part: partial max of each token
  float xs[4][NP][32];           // partial exp sums
  float xtv[4][NP - 1][K][32];   // parts 1.. : their top-k lists (values, indices)
  int xte[4][NP - 1][K][32];
  float bias[kRouterTcMaxE];
};

template <int EP, int K>
struct RtGeo {
  static constexpr int B_PLANE = EP * BK * 2;  // one plane box: EP rows x 128 B
  static constexpr int STAGE_BYTES = A_BYTES + 3 * B_PLANE;
  // as many stages as fit beside the control block (E_pad 128: three of 64 KB)
  using Ctl = RtCtl<RtShape<EP>::NP, K>;
  static constexpr int FIT = static_cast<int>((227 * 1024 - 1024 - sizeof(Ctl)) / STAGE_BYTES);
  static constexpr int STAGES = FIT < MAX_STAGES ? FIT : MAX_STAGES;
  static constexpr uint32_t TMEM_COLS = (2 * EP) <= 32 ? 32 : (2 * EP) <= 64 ? 64 : (2 * EP) <= 128 ? 128
                                        : (2 * EP) <= 256 ? 256 : 512;
  static constexpr size_t SMEM = STAGES * STAGE_BYTES + sizeof(Ctl) + 1024;
};

// Sums of 16 columns over the 32 lanes of a warp: step b (offsets 16, 8, 4,
// 2) keeps the half of the columns selected by lane bit b and adds the other
// lane's copy of it, so after four steps lane l holds its 16-lane partial of
// column l >> 1; the last step (offset 1) completes it.  Returns column
// (lane >> 1)'s sum.
__device__ __forceinline__ float column_sums16(const float (&v)[16], int lane) {
  float a[8], b[4], c[2];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = (lane & 16) != 0;
    a[i] = (up ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, up ? v[i] : v[i + 8], 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = (lane & 8) != 0;
    b[i] = (up ? a[i + 4] : a[i]) + __shfl_xor_sync(0xffffffffu, up ? a[i] : a[i + 4], 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = (lane & 4) != 0;
    c[i] = (up ? b[i + 2] : b[i]) + __shfl_xor_sync(0xffffffffu, up ? b[i] : b[i + 2], 4);
  }
  const bool up = (lane & 2) != 0;
  const float d = (up ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, up ? c[0] : c[1], 2);
  return d + __shfl_xor_sync(0xffffffffu, d, 1);
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Split W_r (fp32 [E][d]) into bf16 planes [3][EP][d]; rows E..EP-1 are zero.
__global__ void __launch_bounds__(256) split_router_kernel(const float* __restrict__ W, int E, int EP, int d,
                                                           __nv_bfloat16* __restrict__ planes, int* tickets,
                                                           int n_tickets) {
  const int64_t n = static_cast<int64_t>(EP) * d;
  pdl_trigger();  // the router may be scheduled at once (it waits for this grid before reading)
  if (tickets != nullptr)
    for (int i = blockIdx.x * 256 + threadIdx.x; i < n_tickets; i += gridDim.x * 256) tickets[i] = 0;
  for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < n; i += static_cast<int64_t>(gridDim.x) * 256) {
    const int e = static_cast<int>(i / d);
    const float w = e < E ? W[i] : 0.f;
    const __nv_bfloat16 w0 = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(w0);
    const __nv_bfloat16 w1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(w1);
    planes[i] = w0;
    planes[n + i] = w1;
    planes[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

// K (= top-k) is a template parameter so the running k-best list is indexed
// statically and lives in registers.
template <int EP, int K>
__global__ void __launch_bounds__(RtShape<EP>::THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const RtParams p) {
  using G = RtGeo<EP, K>;
  using RtCtlT = typename G::Ctl;
  constexpr int NP = RtShape<EP>::NP;
  constexpr int NUM_THREADS = RtShape<EP>::THREADS;
  constexpr int STAGES = G::STAGES;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, EP);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* stages = smem_raw + pad;
  RtCtlT* ctl = reinterpret_cast<RtCtlT*>(stages + STAGES * G::STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&ctl->tfull[a], 1); mbar_init(&ctl->tempty[a], 128 * NP); }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  for (int i = threadIdx.x; i < 4 * kRouterTcMaxE; i += NUM_THREADS) {
    (&ctl->hist[0][0])[i] = 0;
    (&ctl->cnt1[0][0])[i] = 0;
  }
  for (int e = threadIdx.x; e < kRouterTcMaxE; e += NUM_THREADS)
    ctl->bias[e] = (p.b_r != nullptr && e < p.E) ? p.b_r[e] : 0.f;
  if (warp == 1) tmem_alloc(&ctl->tmem_slot, G::TMEM_COLS);
  pdl_wait();  // the W_r planes and tickets come from the split kernel
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;  // per-stage bits: a copy was issued / its phase
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_tiles * p.ksplit && ok; u += gridDim.x) {
        const int tile = u / p.ksplit, ks = u - tile * p.ksplit;
        const int kb0 = ks * p.kb_per, kb1 = min(p.num_kb, kb0 + p.kb_per);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_or_abort(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.err, p.limit_ns)) {
            ok = false;
            break;
          }
          uint8_t* sa = stages + stage * G::STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl->full[stage], G::STAGE_BYTES);
          tma_load_2d(sa, &tmX, &ctl->full[stage], kb * BK, tile * BM);
          if (3 * EP <= 256) {  // the three planes in one box
            tma_load_2d(sa + A_BYTES, &tmW, &ctl->full[stage], kb * BK, 0);
          } else {
#pragma unroll
            for (int pl = 0; pl < 3; ++pl)
              tma_load_2d(sa + A_BYTES + pl * G::B_PLANE, &tmW, &ctl->full[stage], kb * BK, pl * EP);
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (issued_phase >> s) & 1u, p.limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------- MMA issuer
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_tiles * p.ksplit && ok; u += gridDim.x) {
        if (!mbar_wait_or_abort(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, p.err, p.limit_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * EP);
        const int ks = u % p.ksplit;
        const int kb0 = ks * p.kb_per, kb1 = min(p.num_kb, kb0 + p.kb_per);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_or_abort(&ctl->full[stage], phase, &ctl->abort, p.err, p.limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * G::STAGE_BYTES);
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {
            const uint32_t sb = sa + A_BYTES + pl * G::B_PLANE;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16(d_tmem, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), IDESC,
                        (kb != kb0 || pl != 0 || k != 0) ? 1u : 0u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      umma_commit(&ctl->drain);
      mbar_wait(&ctl->drain, 0, p.limit_ns);
    }
  } else {  // ---------------------------------------------------------- epilogue
    // 4 NP warps, NP per TMEM lane quarter q (= 32-token router block of the
    // tile).  Warp part hf takes expert columns [c_lo, c_lo + H): the parts
    // split the experts and exchange, per token, the partial max, the partial
    // top-k lists (parts 1.. -> part 0) and the partial exp sums through shared
    // memory; lower-expert parts go first in every merge and sum, so ties and
    // summation order are fixed.
    const int wi = warp - 2;       // 0 .. 4 NP - 1
    const int q = warp & 3;        // TMEM lane quarter
    const int hf = wi >> 2;        // expert part: 0 = lowest experts
    constexpr int H = EP / NP < 16 ? 16 : EP / NP;  // columns per part (EP = 16: part 1 has none)
    const int c_lo = hf * H;
    const bool has_cols = c_lo < EP;
    const int pair_bar = 2 + q;    // named barrier of the quarter's NP warps
    int acc = 0;
    uint32_t acc_phase = 0;
    const int E = p.E;
    for (int u = blockIdx.x; u < p.n_tiles * p.ksplit; u += gridDim.x) {
      const int tile = u / p.ksplit, ks = u - tile * p.ksplit;
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait_or_abort(&ctl->tfull[acc], acc_phase, &ctl->abort, p.err, p.limit_ns));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * EP);
      if (p.ksplit > 1) {
        // Publish this K range's partial logits of this half's columns (row =
        // TMEM lane); the CTA that finishes a tile's last range sums all
        // ranges in order back into its accumulator; the others release it.
        // Rows past T carry no token: they neither publish nor read partials.
        const bool row_live = static_cast<int64_t>(tile) * BM + q * 32 + lane < p.T;
        float* prow = p.partials + ((static_cast<int64_t>(tile) * p.ksplit + ks) * BM + q * 32 + lane) * EP;
        if (has_cols) {
#pragma unroll 1
          for (int c0 = c_lo; c0 < c_lo + H; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(tq + c0, r);
            tmem_ld_wait();
            if (row_live) {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(prow + c0 + i) =
                    make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]),
                                __uint_as_float(r[i + 3]));
            }
          }
        }
        __threadfence();
        named_barrier(1, 128 * NP);  // all 128 rows of this range are written
        if (threadIdx.x == 64) ctl->last = (atomicAdd(p.tickets + tile, 1) == p.ksplit - 1) ? 1 : 0;
        named_barrier(1, 128 * NP);
        if (!ctl->last) {
          tc_fence_before();
          mbar_arrive(&ctl->tempty[acc]);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
          continue;
        }
        __threadfence();
        const float* prow0 = p.partials + (static_cast<int64_t>(tile) * p.ksplit * BM + q * 32 + lane) * EP;
        if (has_cols) {
#pragma unroll 1
          for (int c0 = c_lo; c0 < c_lo + H; c0 += 16) {
            uint32_t r[16];
            float sum[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) sum[i] = 0.f;
            // ranges in ascending order (deterministic), four loads in flight per batch
#pragma unroll 1
            for (int s0 = 0; row_live && s0 < p.ksplit; s0 += 4) {
              float4 v[4][4];
#pragma unroll
              for (int u2 = 0; u2 < 4; ++u2) {
                const float* src = prow0 + static_cast<int64_t>(s0 + u2) * BM * EP + c0;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  v[u2][i] = s0 + u2 < p.ksplit ? __ldcg(reinterpret_cast<const float4*>(src + 4 * i))
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
              for (int u2 = 0; u2 < 4; ++u2) {
                if (s0 + u2 < p.ksplit) {
#pragma unroll
                  for (int i = 0; i < 4; ++i) {
                    sum[4 * i] += v[u2][i].x;
                    sum[4 * i + 1] += v[u2][i].y;
                    sum[4 * i + 2] += v[u2][i].z;
                    sum[4 * i + 3] += v[u2][i].w;
                  }
                }
              }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(sum[i]);
            tmem_st16(tq + c0, r);
          }
          tmem_st_wait();
        }
      }
      const int64_t tok = static_cast<int64_t>(tile) * BM + q * 32 + lane;
      const bool valid = tok < p.T;
      const int blk = tile * 4 + q;
      const bool blk_valid = blk < p.nblk;

      // 1. this part's logits: up to 32 columns (every E_pad at NP parts) in
      // one batch of TMEM loads into registers, after which the accumulator is
      // released; wider parts would take passes over 16-column chunks that
      // re-read TMEM
      constexpr bool REG = H <= 32;
      float h[REG ? H : 1];
      if constexpr (REG) {
        if (has_cols) {
          uint32_t hr[H / 16][16];
#pragma unroll
          for (int c = 0; c < H / 16; ++c) tmem_ld16(tq + c_lo + c * 16, hr[c]);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < H; ++i) h[i] = __uint_as_float(hr[i / 16][i % 16]);
        }
        tc_fence_before();
        mbar_arrive(&ctl->tempty[acc]);  // accumulator consumed: the next tile's MMAs may start
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // logit of column i of this half (from registers or a chunk just loaded)
      auto logit = [&](float raw, int e) {
        float v = raw + ctl->bias[e];
        return v != v ? -INFINITY : v;  // NaN logits (out of contract) rank last
      };

      // 2. bias, partial max and partial top-k (value desc, index asc): the k
      // best are kept sorted; a candidate enters by compare-and-swap down the
      // list (strict >, so an equal logit never displaces the lower index seen
      // first; once an entry moves, the rest of the list shifts down behind it)
      float m = -INFINITY;
      float tv[K];
      int te[K];
#pragma unroll
      for (int j = 0; j < K; ++j) { tv[j] = -INFINITY; te[j] = 0x7fffffff; }
      auto consider = [&](float v, int e) {
        if (valid && p.logits_out != nullptr) p.logits_out[tok * E + e] = v;
        m = fmaxf(m, v);
        if (v > tv[K - 1] || te[K - 1] == 0x7fffffff) {
          float cv = v;
          int ce = e;
          bool shifting = false;
#pragma unroll
          for (int j = 0; j < K; ++j) {
            if (shifting || cv > tv[j] || te[j] == 0x7fffffff) {
              shifting = true;
              const float tvj = tv[j];
              const int tej = te[j];
              tv[j] = cv;
              te[j] = ce;
              cv = tvj;
              ce = tej;
            }
          }
        }
      };
      if constexpr (REG) {
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const int e = c_lo + i;
          if (has_cols && e < E) {
            h[i] = logit(h[i], e);
            consider(h[i], e);
          }
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < H; c0 += 32) {  // 32 columns per wait
          uint32_t r[2][16];
          tmem_ld16(tq + c_lo + c0, r[0]);
          tmem_ld16(tq + c_lo + c0 + 16, r[1]);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = c_lo + c0 + i;
            if (e < E) consider(logit(__uint_as_float(r[i / 16][i % 16]), e), e);
          }
        }
      }
      // 3. exchange: every part's max; the lists of parts 1.. to part 0, which
      // merges them in part order (lower parts hold the lower expert indices,
      // so the earlier list wins equal values)
      ctl->xm[q][hf][lane] = m;
      if (hf > 0) {
#pragma unroll
        for (int j = 0; j < K; ++j) { ctl->xtv[q][hf - 1][j][lane] = tv[j]; ctl->xte[q][hf - 1][j][lane] = te[j]; }
      }
      named_barrier(pair_bar, 32 * NP);
      m = ctl->xm[q][0][lane];
#pragma unroll
      for (int pp = 1; pp < NP; ++pp) m = fmaxf(m, ctl->xm[q][pp][lane]);
#pragma unroll
      for (int pp = 1; pp < NP; ++pp) {
        if (hf != 0) break;
        float bv[K];
        int be[K];
#pragma unroll
        for (int j = 0; j < K; ++j) { bv[j] = ctl->xtv[q][pp - 1][j][lane]; be[j] = ctl->xte[q][pp - 1][j][lane]; }
        float mv[K];
        int me[K];
        int ia = 0, ib = 0;
#pragma unroll
        for (int j = 0; j < K; ++j) {
          // take from A unless B's head is strictly larger (or A is exhausted/empty)
          float av = -INFINITY, bvh = -INFINITY;
          int ae = 0x7fffffff, beh = 0x7fffffff;
#pragma unroll
          for (int t = 0; t < K; ++t) {
            if (t == ia) { av = tv[t]; ae = te[t]; }
            if (t == ib) { bvh = bv[t]; beh = be[t]; }
          }
          const bool take_b = ia >= K || (ib < K && beh != 0x7fffffff &&
                                          (ae == 0x7fffffff || bvh > av));
          mv[j] = take_b ? bvh : av;
          me[j] = take_b ? beh : ae;
          if (take_b) ++ib; else ++ia;
        }
#pragma unroll
        for (int j = 0; j < K; ++j) { tv[j] = mv[j]; te[j] = me[j]; }
      }
      // 4. s = sum_e exp(h - m): four partial sums per part in a fixed order,
      // then the parts in order (registers: each exponential once, kept in h)
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (REG) {
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float x = (has_cols && c_lo + i < E) ? expf(h[i] - m) : 0.f;
          h[i] = x;
          s4[i & 3] += x;
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < H; c0 += 32) {  // 32 columns per wait
          uint32_t r[2][16];
          tmem_ld16(tq + c_lo + c0, r[0]);
          tmem_ld16(tq + c_lo + c0 + 16, r[1]);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int e = c_lo + c0 + i;
            s4[i & 3] += e < E ? expf(logit(__uint_as_float(r[i / 16][i % 16]), e) - m) : 0.f;
          }
        }
      }
      ctl->xs[q][hf][lane] = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      named_barrier(pair_bar, 32 * NP);
      float s = ctl->xs[q][0][lane];
#pragma unroll
      for (int pp = 1; pp < NP; ++pp) s += ctl->xs[q][pp][lane];
      const float inv_s = 1.f / s;
      const float lse = m + logf(s);
      // 5. per-expert probability sums of this 32-token block for this part's
      // experts, 16 at a time: a fixed shuffle tree over the 32 tokens (lanes),
      // halving the columns at each step, leaves column lane / 2 in lanes
      // 2c and 2c + 1 (deterministic)
#pragma unroll
      for (int c0 = 0; c0 < H; c0 += 16) {
        float pv[16];
        if constexpr (REG) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pv[i] = (valid && has_cols && c_lo + c0 + i < E) ? h[(c0 + i) & (H - 1)] * inv_s : 0.f;
        } else {
          uint32_t r[16];
          tmem_ld16(tq + c_lo + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int e = c_lo + c0 + i;
            pv[i] = (valid && e < E) ? expf(logit(__uint_as_float(r[i]), e) - m) * inv_s : 0.f;
          }
        }
        const float ps = column_sums16(pv, lane);
        const int e = c_lo + c0 + (lane >> 1);
        if ((lane & 1) == 0 && has_cols && e < E && blk_valid) p.part_psum[e * p.nblk + blk] = ps;
      }
      if constexpr (!REG) {
        tc_fence_before();
        mbar_arrive(&ctl->tempty[acc]);  // accumulator consumed
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (hf != 0) continue;  // part 0 alone writes the outputs

      // 6. (part 0) gates, outputs and block counts
      if (valid) {
        float den = 0.f;
        if (p.gate_mode != 0) {
#pragma unroll
          for (int j = 0; j < K; ++j) den += expf(tv[j] - tv[0]);
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
          const float g = (p.gate_mode == 0) ? expf(tv[j] - m) * inv_s : expf(tv[j] - tv[0]) / den;
          p.topk_idx[tok * K + j] = te[j];
          p.topk_gate[tok * K + j] = g;
        }
        if (p.lse_out != nullptr) p.lse_out[tok] = lse;
      }
      // block counts: per choice j, one shared-memory update per distinct
      // expert by the lowest lane choosing it (no contended atomics)
#pragma unroll
      for (int j = 0; j < K; ++j) {
        const int e = valid ? ((te[j] >= 0 && te[j] < E) ? te[j] : 0) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) {
          const int n = __popc(peers);
          ctl->hist[q][e] += n;
          if (j == 0) ctl->cnt1[q][e] += n;
        }
        __syncwarp();
      }
      const float l2 = warp_sum_f(valid ? lse * lse : 0.f);
      __syncwarp();
      if (blk_valid) {
        if (lane == 0) p.part_lse2[blk] = l2;
        for (int e = lane; e < E; e += 32) {
          p.part_hist[e * p.nblk + blk] = ctl->hist[q][e];
          p.part_cnt1[e * p.nblk + blk] = ctl->cnt1[q][e];
        }
      }
      __syncwarp();
      for (int e = lane; e < E; e += 32) { ctl->hist[q][e] = 0; ctl->cnt1[q][e] = 0; }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, G::TMEM_COLS);
  }
}

template <int EP, int K>
cudaError_t launch_ep(const RoutingArgs& a, void* wsplit, void* partials, int num_sms, unsigned int* err,
                      cudaStream_t s, const char** why) {
  using G = RtGeo<EP, K>;
  static_assert(G::STAGES >= 2, "router stages");
  CUtensorMap mx, mw;
  if (!make_map_bf16(&mx, a.x, static_cast<uint64_t>(a.T), static_cast<uint64_t>(a.d), BM) ||
      !make_map_bf16(&mw, wsplit, static_cast<uint64_t>(3 * EP), static_cast<uint64_t>(a.d),
                     3 * EP <= 256 ? 3 * EP : EP)) {
    *why = "router: cuTensorMapEncodeTiled failed";
    return cudaErrorInvalidValue;
  }
  RtParams p;
  p.T = a.T;
  p.E = a.E;
  p.k = a.k;
  p.d = a.d;
  p.gate_mode = a.gate_mode;
  p.num_kb = (a.d + BK - 1) / BK;
  p.nblk = a.nblk;
  p.n_tiles = static_cast<int>((a.T + BM - 1) / BM);
  p.ksplit = router_ksplit(a.T, a.d);
  p.kb_per = (p.num_kb + p.ksplit - 1) / p.ksplit;
  p.partials = static_cast<float*>(partials);
  p.tickets = reinterpret_cast<int*>(static_cast<uint8_t*>(partials) +
                                     static_cast<size_t>(p.n_tiles) * p.ksplit * BM * EP * sizeof(float));
  p.b_r = a.b_r;
  p.topk_idx = a.topk_idx;
  p.topk_gate = a.topk_gate;
  p.part_hist = a.part_hist;
  p.part_cnt1 = a.part_cnt1;
  p.part_psum = a.part_psum;
  p.part_lse2 = a.part_lse2;
  p.logits_out = a.logits_out;
  p.lse_out = a.lse_out;
  p.err = err;
  p.limit_ns = kWaitLimitNs;

  const int64_t n = static_cast<int64_t>(EP) * a.d;
  const int sblocks = static_cast<int>((n + 255) / 256 < 4 * num_sms ? (n + 255) / 256 : 4 * num_sms);
  split_router_kernel<<<sblocks, 256, 0, s>>>(a.W_r, a.E, EP, a.d, static_cast<__nv_bfloat16*>(wsplit),
                                              p.ksplit > 1 ? p.tickets : nullptr, p.n_tiles);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = set_smem_limit_once(reinterpret_cast<const void*>(&router_tc_kernel<EP, K>), static_cast<int>(G::SMEM));
  if (e != cudaSuccess) return e;
  const int units = p.n_tiles * p.ksplit;
  const int grid = units < num_sms ? units : num_sms;
  return launch_pdl(router_tc_kernel<EP, K>, dim3(grid), dim3(RtShape<EP>::THREADS), G::SMEM, s, mx, mw, p);
}

template <int EP>
cudaError_t launch_k(const RoutingArgs& a, void* wsplit, void* partials, int num_sms, unsigned int* err,
                     cudaStream_t s, const char** why) {
  switch (a.k) {
    case 1: return launch_ep<EP, 1>(a, wsplit, partials, num_sms, err, s, why);
    case 2: return launch_ep<EP, 2>(a, wsplit, partials, num_sms, err, s, why);
    case 3: return launch_ep<EP, 3>(a, wsplit, partials, num_sms, err, s, why);
    case 4: return launch_ep<EP, 4>(a, wsplit, partials, num_sms, err, s, why);
    case 5: return launch_ep<EP, 5>(a, wsplit, partials, num_sms, err, s, why);
    case 6: return launch_ep<EP, 6>(a, wsplit, partials, num_sms, err, s, why);
    case 7: return launch_ep<EP, 7>(a, wsplit, partials, num_sms, err, s, why);
    default: return launch_ep<EP, 8>(a, wsplit, partials, num_sms, err, s, why);
  }
}

}  // namespace

int router_ksplit(int64_t T, int d) {
  const int64_t tiles = (T + BM - 1) / BM;
  const int64_t num_kb = (d + BK - 1) / BK;
  if (tiles <= 0) return 1;
  // Up to one wave of tiles with a long K (d >= 4096): two K ranges per tile
  // fill the idle SMs and halve each CTA's MMAs (prefill d 4096, 64 tiles:
  // 57 -> 41 us); with a shorter K the exchange costs more than it saves
  // (d 768, 64 tiles: 21.5 -> 25.4 us; d 2048, 128 tiles: 52 -> 77 us).
  if (tiles > 16) return (tiles <= kSplitTargetCtas && num_kb >= 64) ? 2 : 1;
  int64_t ks = kSplitTargetCtas / tiles;
  if (ks > 16) ks = 16;
  if (ks > num_kb / 2) ks = num_kb / 2;
  if (ks <= 1) return 1;
  const int64_t per = (num_kb + ks - 1) / ks;  // no empty K range
  return static_cast<int>((num_kb + per - 1) / per);
}

size_t router_partials_bytes(int64_t T, int E, int d) {
  // the largest need over every batch size up to T, so a workspace sized for
  // some T serves every smaller batch too
  size_t best = 0;
  const int64_t max_tiles = (T + BM - 1) / BM;
  for (int64_t tiles = 1; tiles <= max_tiles && tiles <= kSplitTargetCtas; ++tiles) {
    const int ks = router_ksplit(tiles * BM, d);
    if (ks <= 1) continue;
    const size_t need = static_cast<size_t>(tiles) * ks * BM * router_pad_e(E) * sizeof(float) +
                        static_cast<size_t>(tiles) * 4;
    if (need > best) best = need;
  }
  return best;
}

cudaError_t launch_router_tc(const RoutingArgs& a, void* wsplit, void* partials, int num_sms, unsigned int* err,
                             cudaStream_t s, const char** why) {
  *why = nullptr;
  const int EP = router_pad_e(a.E);
  if (EP <= 16) return launch_k<16>(a, wsplit, partials, num_sms, err, s, why);
  if (EP <= 32) return launch_k<32>(a, wsplit, partials, num_sms, err, s, why);
  if (EP <= 64) return launch_k<64>(a, wsplit, partials, num_sms, err, s, why);
  if (EP <= 128) return launch_k<128>(a, wsplit, partials, num_sms, err, s, why);
  *why = "router: tensor-core router supports at most 128 experts";
  return cudaErrorInvalidValue;
}

}  // namespace moe

// Grouped GEMM with 4-bit expert weights on the tcgen05 tensor cores, for
// the weight-streaming batches of decoding ("Mixture of experts", rayaq.ca,
// section "Total versus active parameters": at small batch sizes decoding is
// limited by reading weights; "Mixture of Experts (MoE)", inferensys.com,
// inference-optimization glossary: 4-bit post-training quantization of the
// experts' weights).
//
// Weights arrive as 4-bit codes with one bf16 scale per 128 consecutive
// elements of a row (format in include/moe.h, moe_quantize_int4), stored in
// tiles of 128 rows x 64 elements so that every k-block of a weight tile is
// one contiguous 4 KB copy (a row-major layout would fetch 32-byte pieces of
// 128 rows 2 KB or more apart).  The
// product runs transposed: D[f][n] = sum_k W[f][k] X[n][k], with the weight
// rows f as the M = 128 operand and the (few) activation rows n of the
// expert as the N operand (16, 32 or 64 columns).  Dequantized weights never
// touch shared or global memory: dequantizing warps turn each k-block of
// codes into bf16 rows held in tensor memory (tcgen05.st), which the MMA
// reads as its A operand, while the activation tile comes from shared memory
// through TMA.  HBM then carries the codes and scales only.
//
// Warp roles (736 threads, one CTA per SM):
//   warp 0        code producer: bulk copies of KS = 4 consecutive k-blocks of
//                 each code tile (NQ x 16 KB per stage, one contiguous copy
//                 per weight matrix) into a ring of stages that only the
//                 dequantizing warps release, so the HBM stream keeps about
//                 96 KB in flight per SM, independent of the MMAs
//   warp 22       activation producer: the [NB rows x 64] activation tile of
//                 every k-block by TMA (hi and lo planes of the hidden
//                 activation for the second projection) into a ring the MMAs
//                 release, up to 32 stages deep: these small copies have the
//                 same latency as the code stream, and a shallow ring of them
//                 (6 stages) held the whole pipeline to a third of its rate
//   warp 1        TMEM allocator; lane 0 issues the MMAs (M 128, N NB, K 16)
//   warps 2..17   dequantize: warp w owns TMEM lanes 32 (w % 4) .. + 31 (one
//                 weight row per lane) and quarter (w - 2) / 4 of each
//                 k-block (16 elements, 8 TMEM columns); it prefetches the
//                 next scale group and keeps one k-block's tensor-memory
//                 stores in flight while it dequantizes the next
//   warps 18..21  epilogue: activation (first projection) or gate (second)
//                 and the stores, one weight row (output column) per lane
// The dequantized values are exact: (code - 8) * scale with a scale of at
// most 5 significant bits fits bf16 exactly, and both steps are exact bf16x2
// operations.  Every wait is bounded as in the bf16 grouped GEMM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int WBM = 128;                 // weight rows per tile (TMEM lanes)
constexpr int WBK = 64;                  // K per k-block
constexpr int Q_TILE = WBM * WBK / 2;    // bytes of codes per weight tile and k-block (4 KB)
constexpr int MAX_A_STAGES = 8;          // TMEM A ring
constexpr int KS = 4;                    // k-blocks per code stage
constexpr int MAX_Q_STAGES = 8;
constexpr int MAX_X_STAGES = 32;
constexpr int Q_RING_BYTES = 96 * 1024;
constexpr int X_RING_BYTES = 96 * 1024;
constexpr int DQ_WARPS = 16;
constexpr int EPI_WARP0 = 2 + DQ_WARPS;
constexpr int XPROD_WARP = EPI_WARP0 + 4;
constexpr int W4_THREADS = 32 * (XPROD_WARP + 1);
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_G = 256;

template <int MODE>
struct W4Geo {
  static constexpr int NQ = MODE == W4_SWIGLU ? 2 : 1;      // weight matrices per tile (W1 and W3)
  static constexpr int PLANES = MODE == W4_GATE ? 2 : 1;    // activation planes (hidden hi + lo)
};

// TMEM: two accumulators of NQ x NB columns, the rest (up to 8 stages of
// NQ x 32 columns) for the dequantized A ring.
template <int MODE, int NB>
struct W4Tmem {
  static constexpr int NQ = W4Geo<MODE>::NQ;
  static constexpr int FREE = (static_cast<int>(TMEM_COLS) - 2 * NQ * NB) / (NQ * 32);
  static constexpr int A_STAGES = FREE < MAX_A_STAGES ? FREE : MAX_A_STAGES;
  static constexpr uint32_t ACC0 = A_STAGES * NQ * 32;  // first accumulator column
  static_assert(A_STAGES >= 2, "tensor memory too small for the A ring");
};

// Two shared-memory rings: code stages (KS k-blocks of every weight matrix of
// the tile) and activation stages (one k-block).
template <int MODE, int NB>
struct W4Stage {
  static constexpr int Q_BYTES = W4Geo<MODE>::NQ * KS * Q_TILE;
  static constexpr int QN = (Q_RING_BYTES / Q_BYTES) < MAX_Q_STAGES ? (Q_RING_BYTES / Q_BYTES) : MAX_Q_STAGES;
  static constexpr int X_BYTES = W4Geo<MODE>::PLANES * NB * 128;
  static constexpr int XN = (X_RING_BYTES / X_BYTES) < MAX_X_STAGES ? (X_RING_BYTES / X_BYTES) : MAX_X_STAGES;
  static constexpr int BYTES = QN * Q_BYTES + XN * X_BYTES;
};

struct W4Ctl {
  uint64_t qfull[MAX_Q_STAGES];
  uint64_t qempty[MAX_Q_STAGES];
  uint64_t xfull[MAX_X_STAGES];
  uint64_t xempty[MAX_X_STAGES];
  uint64_t afull[MAX_A_STAGES];
  uint64_t aempty[MAX_A_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  volatile int abort;
  int nprefix[MAX_G + 1];  // prefix over groups of their n-tiles
  int offsets[MAX_G + 1];
};

template <int MODE, int NB>
constexpr size_t w4_smem_bytes() {
  return W4Stage<MODE, NB>::BYTES + sizeof(W4Ctl) + 1024;
}


// unit -> (group, m-tile over weight rows, n-tile over activation rows, K range)
struct W4Item {
  int e, mt, nt, ks, kb0, kb1;
};

__device__ __forceinline__ bool w4_item(const W4Ctl* c, const W4Params& p, int u, W4Item& w) {
  const int units = c->nprefix[p.G] * p.m_tiles * p.ksplit;
  if (u >= units) return false;
  const int tile = u / p.ksplit;
  w.ks = u - tile * p.ksplit;
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (c->nprefix[mid] * p.m_tiles <= tile) lo = mid; else hi = mid;
  }
  w.e = lo;
  const int local = tile - c->nprefix[lo] * p.m_tiles;
  const int nts = c->nprefix[lo + 1] - c->nprefix[lo];
  w.mt = local / nts;
  w.nt = local - w.mt * nts;
  w.kb0 = w.ks * p.kb_per;
  w.kb1 = min(p.num_kb, w.kb0 + p.kb_per);
  return true;
}

__device__ __forceinline__ bool w4_wait(W4Ctl* c, uint64_t* bar, uint32_t parity, const W4Params& p) {
  return mbar_wait_or_abort(bar, parity, &c->abort, p.err, p.limit_ns);
}

// A operand read from TMEM: D[tmem] (+)= A[tmem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void umma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Eight codes of one 32-bit word (element 2j in bits 4j.., element 2j+1 in
// bits 4j+16.., codes offset by 8) -> four bf16 pairs (code - 8) * s, exact.
__device__ __forceinline__ void dequant_word(uint32_t w, __nv_bfloat162 s2, uint32_t* out) {
  __nv_bfloat162_raw braw;  // 136 as bits: no conversion instruction
  braw.x = 0x4308;
  braw.y = 0x4308;
  const __nv_bfloat162 bias(braw);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // bf16 pair 128 + code
    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&t);
    v = __hmul2(__hsub2(v, bias), s2);
    out[j] = *reinterpret_cast<const uint32_t*>(&v);
  }
}

template <int MODE, int NB>
__global__ void __launch_bounds__(W4_THREADS, 1)
    w4_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const W4Params p) {
  using Geo = W4Geo<MODE>;
  using St = W4Stage<MODE, NB>;
  constexpr int NQ = Geo::NQ, PLANES = Geo::PLANES;
  constexpr int QN = St::QN, XN = St::XN, Q_BYTES = St::Q_BYTES, X_BYTES = St::X_BYTES;
  constexpr int A_STAGES = W4Tmem<MODE, NB>::A_STAGES;
  constexpr uint32_t ACC0 = W4Tmem<MODE, NB>::ACC0;
  constexpr uint32_t IDESC = idesc_bf16_f32(WBM, NB);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* xring = smem_raw + pad;          // activation stages first: 1024-byte aligned for the swizzle
  uint8_t* qring = xring + XN * X_BYTES;
  W4Ctl* ctl = reinterpret_cast<W4Ctl*>(qring + QN * Q_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QN; ++s) { mbar_init(&ctl->qfull[s], 1); mbar_init(&ctl->qempty[s], DQ_WARPS); }
    for (int s = 0; s < XN; ++s) { mbar_init(&ctl->xfull[s], 1); mbar_init(&ctl->xempty[s], 1); }
    for (int a = 0; a < A_STAGES; ++a) { mbar_init(&ctl->afull[a], DQ_WARPS); mbar_init(&ctl->aempty[a], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&ctl->tfull[a], 1); mbar_init(&ctl->tempty[a], 128); }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) tmem_alloc(&ctl->tmem_slot, TMEM_COLS);
  pdl_wait();  // group offsets and the activation rows come from the kernels before
  pdl_trigger();
  if (threadIdx.x == 0) {
    ctl->nprefix[0] = 0;
    for (int g = 0; g < p.G; ++g) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      ctl->offsets[g] = o0;
      ctl->nprefix[g + 1] = ctl->nprefix[g] + (o1 - o0 + NB - 1) / NB;
    }
    ctl->offsets[p.G] = p.offsets[p.G];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_phase = 0;
      bool ok = true;
      W4Item w;
      for (int u = blockIdx.x; ok && w4_item(ctl, p, u, w); u += gridDim.x) {
        // tile row (e, mt): its k-blocks are Q_TILE apart, contiguous
        const int64_t qtile = (static_cast<int64_t>(w.e) * p.m_tiles + w.mt) * p.num_kb * Q_TILE;
        for (int kb = w.kb0; kb < w.kb1; kb += KS) {
          const int nkb = min(KS, w.kb1 - kb);
          if (!w4_wait(ctl, &ctl->qempty[stage], phase ^ 1u, p)) { ok = false; break; }
          uint8_t* st = qring + stage * Q_BYTES;
          const uint32_t bytes = static_cast<uint32_t>(nkb * Q_TILE);
          mbar_arrive_expect_tx(&ctl->qfull[stage], NQ * bytes);
          bulk_load(st, p.Q0 + qtile + static_cast<int64_t>(kb) * Q_TILE, bytes, &ctl->qfull[stage]);
          if (NQ == 2)
            bulk_load(st + KS * Q_TILE, p.Q1 + qtile + static_cast<int64_t>(kb) * Q_TILE, bytes, &ctl->qfull[stage]);
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == QN) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < QN; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->qfull[s], (issued_phase >> s) & 1u, p.limit_ns);
    }
  } else if (warp == XPROD_WARP) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_phase = 0;
      bool ok = true;
      W4Item w;
      for (int u = blockIdx.x; ok && w4_item(ctl, p, u, w); u += gridDim.x) {
        const int xrow = ctl->offsets[w.e] + w.nt * NB;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!w4_wait(ctl, &ctl->xempty[stage], phase ^ 1u, p)) { ok = false; break; }
          uint8_t* st = xring + stage * X_BYTES;
          mbar_arrive_expect_tx(&ctl->xfull[stage], X_BYTES);
          if (PLANES == 2) tma_load_3d(st, &tmX, &ctl->xfull[stage], kb * WBK, xrow, 0);
          else tma_load_2d(st, &tmX, &ctl->xfull[stage], kb * WBK, xrow);
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == XN) { stage = 0; phase ^= 1u; }
        }
      }
      for (int s = 0; s < XN; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->xfull[s], (issued_phase >> s) & 1u, p.limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, astage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0, acc_phase = 0;
      bool ok = true;
      W4Item w;
      for (int u = blockIdx.x; ok && w4_item(ctl, p, u, w); u += gridDim.x) {
        if (!w4_wait(ctl, &ctl->tempty[acc], acc_phase ^ 1u, p)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + ACC0 + static_cast<uint32_t>(acc * NQ * NB);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!w4_wait(ctl, &ctl->xfull[stage], phase, p) || !w4_wait(ctl, &ctl->afull[astage], aphase, p)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sx = smem_u32(xring + stage * X_BYTES);
          const uint32_t a0 = tmem_base + static_cast<uint32_t>(astage * NQ * 32);
#pragma unroll
          for (int kk = 0; kk < WBK / 16; ++kk) {
            const uint32_t acc_in = (kb != w.kb0 || kk != 0) ? 1u : 0u;
            const uint64_t bd = sdesc_k_sw128(sx + kk * 32);
            umma_tmem_a(d0, a0 + kk * 8, bd, IDESC, acc_in);
            if (NQ == 2) umma_tmem_a(d0 + NB, a0 + 32 + kk * 8, bd, IDESC, acc_in);
            if (PLANES == 2) umma_tmem_a(d0, a0 + kk * 8, sdesc_k_sw128(sx + NB * 128 + kk * 32), IDESC, 1u);
          }
          umma_commit(&ctl->xempty[stage]);
          umma_commit(&ctl->aempty[astage]);
          if (++stage == XN) { stage = 0; phase ^= 1u; }
          if (++astage == A_STAGES) { astage = 0; aphase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      umma_commit(&ctl->drain);
      mbar_wait(&ctl->drain, 0, p.limit_ns);
    }
  } else if (warp < EPI_WARP0) {
    // ------------------------------------------------------------ dequantize
    const int q = warp & 3, part = (warp - 2) >> 2;  // 16 elements (8 columns) of each k-block
    const int r = q * 32 + lane;  // weight row within the tile
    const int groups = p.K / W4_GROUP;
    const __nv_bfloat16 zero = __float2bfloat16(0.f);
    int stage = 0, astage = 0, held = -1;  // held: A stage whose stores are still in flight
    uint32_t phase = 0, aphase = 0;
    bool ok = true;
    W4Item w;
    for (int u = blockIdx.x; ok && w4_item(ctl, p, u, w); u += gridDim.x) {
      // scales of tile row (e, mt): [groups][128], this lane's row r
      const int64_t sbase = (static_cast<int64_t>(w.e) * p.m_tiles + w.mt) * groups * WBM + r;
      const __nv_bfloat16* s0p = p.S0 + sbase;
      const __nv_bfloat16* s1p = p.S1 + sbase;
      // scales of this k-block's group and the next one, loaded one group ahead
      int g_cur = (w.kb0 * WBK + part * 16) / W4_GROUP;
      __nv_bfloat16 sc0 = s0p[g_cur * WBM], sc1 = NQ == 2 ? s1p[g_cur * WBM] : zero;
      __nv_bfloat16 nx0 = g_cur + 1 < groups ? s0p[(g_cur + 1) * WBM] : zero;
      __nv_bfloat16 nx1 = (NQ == 2 && g_cur + 1 < groups) ? s1p[(g_cur + 1) * WBM] : zero;
      for (int kb = w.kb0; kb < w.kb1; ++kb) {
        const int j = (kb - w.kb0) % KS;  // k-block within the code stage
        if (j == 0 && !__all_sync(0xffffffffu, w4_wait(ctl, &ctl->qfull[stage], phase, p))) { ok = false; break; }
        const int grp = (kb * WBK + part * 16) / W4_GROUP;
        if (grp != g_cur) {
          g_cur = grp;
          sc0 = nx0;
          sc1 = nx1;
          nx0 = grp + 1 < groups ? s0p[(grp + 1) * WBM] : zero;
          if (NQ == 2) nx1 = grp + 1 < groups ? s1p[(grp + 1) * WBM] : zero;
        }
        if (!__all_sync(0xffffffffu, w4_wait(ctl, &ctl->aempty[astage], aphase ^ 1u, p))) { ok = false; break; }
        tc_fence_after();
        const uint8_t* st = qring + stage * Q_BYTES + j * Q_TILE;
        uint32_t v[NQ][8];
#pragma unroll
        for (int m = 0; m < NQ; ++m) {
          const uint2 words = *reinterpret_cast<const uint2*>(st + m * KS * Q_TILE + r * 32 + part * 8);
          const __nv_bfloat162 s2 = __bfloat162bfloat162(m == 0 ? sc0 : sc1);
          dequant_word(words.x, s2, v[m]);
          dequant_word(words.y, s2, v[m] + 4);
        }
        // the code stage is read once its last k-block's codes are in registers
        if (j == KS - 1 || kb + 1 == w.kb1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->qempty[stage]);
          if (++stage == QN) { stage = 0; phase ^= 1u; }
        }
        // the previous k-block's stores completed: hand that A stage to the MMA
        if (held >= 0) {
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->afull[held]);
        }
        const uint32_t tcol = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>(astage * NQ * 32 + part * 8);
#pragma unroll
        for (int m = 0; m < NQ; ++m) tmem_st8(tcol + m * 32, v[m]);
        held = astage;
        if (++astage == A_STAGES) { astage = 0; aphase ^= 1u; }
      }
    }
    if (held >= 0) {
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&ctl->afull[held]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    W4Item w;
    for (int u = blockIdx.x; w4_item(ctl, p, u, w); u += gridDim.x) {
      const bool got = __all_sync(0xffffffffu, w4_wait(ctl, &ctl->tfull[acc], acc_phase, p));
      if (!got) break;
      tc_fence_after();
      const int f = w.mt * WBM + r;  // weight row = output column of this lane
      const bool vcol = f < p.N;
      const int g0 = ctl->offsets[w.e], grows = ctl->offsets[w.e + 1] - g0;
      const int n0 = w.nt * NB;
      const int nvalid = min(NB, grows - n0);
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ACC0 +
                          static_cast<uint32_t>(acc * NQ * NB);
#pragma unroll 1
      for (int c = 0; c < NB; c += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld16(tb + c, ra);
        if (NQ == 2) tmem_ld16(tb + NB + c, rb);
        tmem_ld_wait();
        if (vcol) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c + i;
            if (n >= nvalid) break;
            const int64_t row = g0 + n0 + n;  // expert-sorted row
            const float a = __uint_as_float(ra[i]);
            if (MODE == W4_GATE) {
              float* out = static_cast<float*>(p.out) + static_cast<int64_t>(w.ks) * p.split_stride;
              out[row * p.N + f] = a * p.row_gate[row];
            } else {
              const float h = MODE == W4_SWIGLU ? __fdividef(a, 1.f + __expf(-a)) * __uint_as_float(rb[i])
                                                : fmaxf(a, 0.f);
              const __nv_bfloat16 hi = __float2bfloat16_rn(h);
              const __nv_bfloat16 lo = __float2bfloat16_rn(h - __bfloat162float(hi));
              static_cast<__nv_bfloat16*>(p.out)[row * p.N + f] = hi;
              static_cast<__nv_bfloat16*>(p.out_lo)[row * p.N + f] = lo;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Quantizer: one warp per (row, group of 128 elements).  Lane l holds
// elements 4l .. 4l+3 of the group; scale = max|w| / 7 in fp32, rounded up to
// 5 significant bits; code = round-half-even(w / scale) + 8 (0 if scale = 0).
__device__ __forceinline__ uint32_t round_up_5_bits(float s) {
  uint32_t u = __float_as_uint(s);
  if (u & 0x7FFFFu) u = (u | 0x7FFFFu) + 1u;
  return u;
}

__global__ void __launch_bounds__(256) quantize_int4_kernel(const __nv_bfloat16* __restrict__ W, int64_t rows,
                                                            int K, uint32_t* __restrict__ codes,
                                                            __nv_bfloat16* __restrict__ scales) {
  const int groups = K / W4_GROUP;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= rows * groups) return;
  const int lane = threadIdx.x & 31;
  const int64_t row = gw / groups;
  const int grp = static_cast<int>(gw - row * groups);
  const __nv_bfloat16* src = W + row * K + grp * W4_GROUP + lane * 4;
  const uint2 raw = *reinterpret_cast<const uint2*>(src);
  float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u), __uint_as_float(raw.y << 16),
                __uint_as_float(raw.y & 0xFFFF0000u)};
  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __uint_as_float(round_up_5_bits(__fdiv_rn(amax, 7.f)));
  uint32_t u[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float qf = s > 0.f ? rintf(__fdiv_rn(v[i], s)) : 0.f;
    u[i] = static_cast<uint32_t>(static_cast<int>(fminf(fmaxf(qf, -8.f), 7.f)) + 8);
  }
  // word m holds elements 8m .. 8m+7: element 2j in nibble j, element 2j+1 in nibble j + 4
  const uint32_t part = (lane & 1) == 0 ? (u[0] | (u[1] << 16) | (u[2] << 4) | (u[3] << 20))
                                        : ((u[0] << 8) | (u[1] << 24) | (u[2] << 12) | (u[3] << 28));
  const uint32_t word = part | __shfl_xor_sync(0xffffffffu, part, 1);
  // tiled layout: tile (row / 128, k-block), 128 rows x 8 words each
  const int m = lane / 2;                      // word of the group, 0 .. 15
  const int64_t trow = row / 128, rin = row % 128;
  const int64_t kb = 2 * grp + m / 8;          // k-block of 64 elements
  if ((lane & 1) == 0) codes[((trow * (K / 64) + kb) * 128 + rin) * 8 + (m % 8)] = word;
  if (lane == 0) scales[(trow * groups + grp) * 128 + rin] = __float2bfloat16_rn(s);
}


template <int MODE, int NB>
cudaError_t launch_w4_t(const W4Plan& pl, int num_sms, cudaStream_t s) {
  constexpr size_t bytes = w4_smem_bytes<MODE, NB>();
  static_assert(bytes <= 227 * 1024, "4-bit grouped GEMM shared memory");
  cudaError_t e =
      set_smem_limit_once(reinterpret_cast<const void*>(&w4_gemm_kernel<MODE, NB>), static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  return launch_pdl(w4_gemm_kernel<MODE, NB>, dim3(num_sms), dim3(W4_THREADS), bytes, s, pl.x, pl.p);
}

template <int MODE>
cudaError_t launch_w4_nb(const W4Plan& pl, int num_sms, cudaStream_t s) {
  if (pl.nb == 16) return launch_w4_t<MODE, 16>(pl, num_sms, s);
  if (pl.nb == 32) return launch_w4_t<MODE, 32>(pl, num_sms, s);
  return launch_w4_t<MODE, 64>(pl, num_sms, s);
}

}  // namespace

int w4_rows_per_tile(int64_t max_group_rows) { return max_group_rows <= 16 ? 16 : max_group_rows <= 32 ? 32 : 64; }

cudaError_t plan_w4_gemm(const W4Args& g, W4Plan* pl, const char** why) {
  *why = nullptr;
  if (g.G > MAX_G) { *why = "4-bit grouped GEMM supports at most 256 expert groups"; return cudaErrorInvalidValue; }
  if (g.K % W4_GROUP != 0) { *why = "4-bit weights need the input dimension to be a multiple of 128"; return cudaErrorInvalidValue; }
  if (g.N % WBM != 0) { *why = "4-bit weights need d and d_ff to be multiples of 128"; return cudaErrorInvalidValue; }
  if (((reinterpret_cast<uintptr_t>(g.Q0) | reinterpret_cast<uintptr_t>(g.mode == W4_SWIGLU ? g.Q1 : g.Q0)) & 15) != 0) {
    *why = "4-bit codes must be 16-byte aligned";
    return cudaErrorInvalidValue;
  }
  pl->nb = w4_rows_per_tile(g.max_group_rows);
  bool ok = true;
  if (g.mode == W4_GATE) {
    const intptr_t stride = static_cast<const uint8_t*>(g.X_lo) - static_cast<const uint8_t*>(g.X);
    if (stride <= 0 || stride % 16 != 0) { *why = "4-bit grouped GEMM: lo plane must follow the hi plane"; return cudaErrorInvalidValue; }
    ok = ok && make_map_planes_bf16(&pl->x, g.X, static_cast<uint64_t>(stride), static_cast<uint64_t>(g.x_rows),
                                    static_cast<uint64_t>(g.K), static_cast<uint32_t>(pl->nb));
  } else {
    ok = ok && make_map_bf16(&pl->x, g.X, static_cast<uint64_t>(g.x_rows), static_cast<uint64_t>(g.K),
                             static_cast<uint32_t>(pl->nb));
  }
  if (!ok) { *why = "cuTensorMapEncodeTiled failed for the 4-bit grouped GEMM"; return cudaErrorInvalidValue; }
  W4Params& p = pl->p;
  p.G = g.G;
  p.N = g.N;
  p.K = g.K;
  p.m_tiles = (g.N + WBM - 1) / WBM;
  p.num_kb = g.K / WBK;
  p.ksplit = g.mode == W4_GATE ? (g.ksplit < 1 ? 1 : (g.ksplit > p.num_kb ? p.num_kb : g.ksplit)) : 1;
  p.kb_per = (p.num_kb + p.ksplit - 1) / p.ksplit;
  p.ksplit = (p.num_kb + p.kb_per - 1) / p.kb_per;  // no empty K range
  p.split_stride = g.split_stride;
  p.Q0 = static_cast<const uint8_t*>(g.Q0);
  p.Q1 = static_cast<const uint8_t*>(g.mode == W4_SWIGLU ? g.Q1 : g.Q0);
  p.S0 = static_cast<const __nv_bfloat16*>(g.S0);
  p.S1 = static_cast<const __nv_bfloat16*>(g.mode == W4_SWIGLU ? g.S1 : g.S0);
  p.out = g.out;
  p.out_lo = g.out_lo;
  p.offsets = g.offsets;
  p.row_gate = g.row_gate;
  p.err = g.err;
  p.limit_ns = kWaitLimitNs;
  pl->mode = g.mode;
  return cudaSuccess;
}

cudaError_t launch_w4_gemm(const W4Plan& pl, int num_sms, cudaStream_t s) {
  if (pl.mode == W4_SWIGLU) return launch_w4_nb<W4_SWIGLU>(pl, num_sms, s);
  if (pl.mode == W4_RELU) return launch_w4_nb<W4_RELU>(pl, num_sms, s);
  return launch_w4_nb<W4_GATE>(pl, num_sms, s);
}

cudaError_t launch_quantize_int4(const void* W, int64_t rows, int K, void* codes, void* scales, cudaStream_t s) {
  const int64_t warps = rows * (K / W4_GROUP);
  if (warps <= 0) return cudaSuccess;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 2147483647LL) return cudaErrorInvalidValue;
  quantize_int4_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(W), rows, K, static_cast<uint32_t*>(codes),
      static_cast<__nv_bfloat16*>(scales));
  count_launch();
  return cudaGetLastError();
}

}  // namespace moe

// Expert products with 4-bit weights for batches of at most 64 tokens
// ("Mixture of experts", rayaq.ca, section "Total versus active parameters":
// decoding a few tokens is bound by reading the active experts' weights).
//
// With a few activation rows per expert the products are a handful of
// matrix-vector products.  The tcgen05 path (gemm_w4.cu) cycles every
// dequantized k-block through tensor memory and waits for the MMA's commit
// before reusing it; at these sizes that round trip, not HBM, sets its pace.
// Here the dequantized codes never leave registers: each warp turns its
// codes into the A fragments of warp-level MMAs (m16n8k16, bf16 in, fp32
// accumulate) whose B fragments are the activation rows, so the only waits
// are on the code stream itself, which a producer warp keeps four to six
// stages (about 200 KB) deep per SM with bulk copies.  The MMAs do a few percent of the work of a
// tensor-core-bound kernel; the kernel is bound by HBM and by the integer
// instructions that unpack the codes (7 per 8 weights).
//
// Orientation: D[f][n] = sum_k W[f][k] X[n][k], weight rows f as the M = 16
// operand, activation rows n as the N = 8 operand.  The first projection's
// eight columns are eight activation rows; the second projection's are four
// rows of the hidden activation's hi plane and the same four rows of its lo
// plane (summed in the epilogue), so one token costs one MMA per 256 weights.
//
// K order inside a k-block: the MMA sums over its 16 k positions in any
// order as long as A and B agree.  Thread t of a quad takes words 2t and
// 2t + 1 of each weight row (elements 16t .. 16t + 15 of the k-block) and
// feeds pairs 2s, 2s + 1 of them to k step s; its B fragments are the same
// sixteen elements of the activation rows.  Each thread thus reads 8
// contiguous bytes per row and a warp reads 256 contiguous bytes.
//
// Scales: one bf16 per row and 128 elements.  The MMAs of one scale group
// (two k-blocks) accumulate (code - 8) * x, exact products of bf16 values,
// into fp32 registers that are then scaled and added to the totals.
// Unpacking 8 codes takes 3 shifts, 4 logic ops and 4 bf16x2 subtractions.
//
// Outputs are fp32 partial rows per K range: the first projection writes
// W1 x (and W3 x) for the activation kernel after it; the second writes
// gate * W2 h for the combine.
//
// Warp roles (544 threads, one CTA per SM): warps 0..15 compute, 16 weight
// rows each (one m16 tile) of one of the unit's two 128-row slots (four warps
// per scheduler hide the latency of the dependent unpack-and-MMA chains);
// warp 16 lane 0 produces.  A unit is (expert group, pair of slots, K range):
// W1 and W3 rows of one m-tile for SwiGLU, two m-tiles of the single matrix
// otherwise.  A stage holds two scale groups (four k-blocks) of the unit: both
// slots' codes (16 KB each) and scales (512 B each) and the same 256 columns
// of the group's activation rows (one bulk copy per row and plane), so each
// warp unpacks 16 words per pipeline handshake and a unit's activations are
// read once, stage by stage, whatever the length of its K range.  Every wait
// is bounded as in the other pipelined kernels.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr int SB = 128;                            // weight rows per slot (one code tile)
constexpr int GROUP_CODES = SB * W4_GROUP / 2;     // codes of one slot and scale group: 8 KB
constexpr int GROUP_SCALES = SB * 2;               // scales of one slot and scale group: 256 B
constexpr int SPS = 2;                             // scale groups per stage
constexpr int SLOT_CODES = SPS * GROUP_CODES;
constexpr int SLOT_SCALES = SPS * GROUP_SCALES;
constexpr int X_OFF = 2 * (SLOT_CODES + SLOT_SCALES);  // activation rows within a stage
constexpr int XROW = SPS * W4_GROUP * 2 + 16;      // bytes per activation row in a stage (padded)
constexpr int MAX_STAGE = 8;
constexpr int SMEM_BUDGET = 224 * 1024;
constexpr int CWARPS = 16;
constexpr int SM_THREADS = 32 * (CWARPS + 1);
constexpr int MAX_G = 256;

struct SmCtl {
  uint64_t full[MAX_STAGE];
  uint64_t empty[MAX_STAGE];
  volatile int abort;
  int nprefix[MAX_G + 1];  // prefix over groups of their row chunks
  int offsets[MAX_G + 1];
  uint4 zero[XROW / 16];   // a zero activation row: B fragments of rows past the group's
};

struct SmItem {
  int e, b, ks, g0, g1;  // group, row block, K range, scale groups [g0, g1)
  int row0, rows;        // the unit's activation rows (one chunk of the group's)
};

// Unit u -> (group e, row block b, chunk c of at most rows_cap rows, K range
// ks), K ranges innermost, then chunks (the chunks of one code tile run side
// by side, so the later ones find its codes in L2).
__device__ __forceinline__ bool sm_item(const SmCtl* c, const W4SmallParams& p, int u, SmItem& w) {
  const int units = c->nprefix[p.G] * p.row_blocks * p.ksplit;
  if (u >= units) return false;
  const int tile = u / p.ksplit;
  w.ks = u - tile * p.ksplit;
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (c->nprefix[mid] * p.row_blocks <= tile) lo = mid; else hi = mid;
  }
  w.e = lo;  // the largest lo with nprefix[lo] <= tile / row_blocks: a group with rows
  const int local = tile - c->nprefix[lo] * p.row_blocks;
  const int chunks = c->nprefix[lo + 1] - c->nprefix[lo];
  w.b = local / chunks;
  const int ch = local - w.b * chunks;
  w.row0 = c->offsets[lo] + ch * p.rows_cap;
  w.rows = min(p.rows_cap, c->offsets[lo + 1] - w.row0);
  w.g0 = w.ks * p.gp;
  w.g1 = min(p.num_g, w.g0 + p.gp);
  return true;
}

// Code tile (slot) of a unit: SwiGLU takes m-tile b of W1 (slot 0) and W3
// (slot 1); otherwise m-tiles 2b and 2b + 1 of the one matrix.
__device__ __forceinline__ int slot_mtile(const W4SmallParams& p, int b, int slot) {
  return p.two_mats ? b : 2 * b + slot;
}

__device__ __forceinline__ bool sm_wait(SmCtl* c, uint64_t* bar, uint32_t parity, const W4SmallParams& p) {
  return mbar_wait_or_abort(bar, parity, &c->abort, p.err, p.limit_ns);
}

// bf16 pair (code - 8) of the codes in bits 4j.. and 4j + 16.. of w: exact.
// (w >> 4j) & 0x000F000F | 0x43004300 is the bf16 pair 128 + code (one lop3),
// minus the pair 136 (bits 0x4308).
template <int J>
__device__ __forceinline__ uint32_t code_pair(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b32 t;\n\t"
      "lop3.b32 t, %1, 0x000F000F, 0x43004300, 0xEA;\n\t"
      "sub.rn.bf16x2 %0, t, %2;\n\t}"
      : "=r"(r)
      : "r"(w >> (4 * J)), "r"(0x43084308u));
  return r;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The same with a zero accumulator in: d = A B.
__device__ __forceinline__ void mma_bf16_first(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Shared-memory loads at 32-bit shared addresses (constant offsets fold
// into the instruction).
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_bf16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// A fragments of k step s for rows g (word w) and g + 8 (word v) of an m16
// tile: pairs 2s' and 2s' + 1 of the thread's sixteen elements, s' = s % 2
// within the word of step s.
template <int S>
__device__ __forceinline__ void a_frag(uint32_t w, uint32_t v, uint32_t (&a)[4]) {
  constexpr int J = 2 * (S & 1);
  a[0] = code_pair<J>(w);
  a[1] = code_pair<J>(v);
  a[2] = code_pair<J + 1>(w);
  a[3] = code_pair<J + 1>(v);
}

// NG scale groups (2 NG k-blocks) of one stage for one m16 tile against NTA
// n-tiles: codes at shared address q (group gi, k-block kbl, rows g and g + 8
// at q + gi 8 KB + kbl 4 KB + {0, 256}), this lane's activation rows at
// xa[j] (+ gi 256 + kbl 128 bytes), scales at sadr (+ gi 256; row g + 8 at
// + 16).  Every load of the stage is issued first; the body is straight-line.
template <int NT, int NTA, int NG>
__device__ __forceinline__ void stage_mma(uint32_t q, const uint32_t (&xa)[NT], uint32_t sadr, float (&acc)[NT][4]) {
  if constexpr (NG == 2 && NTA > 2) {  // registers are short: one scale group at a time
    uint32_t xa2[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) xa2[j] = xa[j] + W4_GROUP * 2;
    stage_mma<NT, NTA, 1>(q, xa, sadr, acc);
    stage_mma<NT, NTA, 1>(q + GROUP_CODES, xa2, sadr + GROUP_SCALES, acc);
    return;
  }
  constexpr int PAR = NTA >= 3 ? 1 : 2;  // accumulator chains per n-tile (one when registers are short)
  uint2 cw[NG][2][2];
  float sc[NG][2];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
#pragma unroll
    for (int kbl = 0; kbl < 2; ++kbl) {
      cw[gi][kbl][0] = lds64(q + gi * GROUP_CODES + kbl * 4096);
      cw[gi][kbl][1] = lds64(q + gi * GROUP_CODES + kbl * 4096 + 8 * 32);
    }
    sc[gi][0] = lds_bf16(sadr + gi * GROUP_SCALES);
    sc[gi][1] = lds_bf16(sadr + gi * GROUP_SCALES + 16);
  }
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    float tmp[PAR][NTA][4];
#pragma unroll
    for (int kbl = 0; kbl < 2; ++kbl) {
      const uint2 c0 = cw[gi][kbl][0], c1 = cw[gi][kbl][1];
      uint32_t a[4][4];  // [k step][fragment]
      a_frag<0>(c0.x, c1.x, a[0]);
      a_frag<1>(c0.x, c1.x, a[1]);
      a_frag<2>(c0.y, c1.y, a[2]);
      a_frag<3>(c0.y, c1.y, a[3]);
#pragma unroll
      for (int j = 0; j < NTA; ++j) {
        const uint32_t xb = xa[j] + gi * W4_GROUP * 2 + kbl * 128;
        const uint4 b0 = lds128(xb);
        const uint4 b1 = lds128(xb + 16);
        if (kbl == 0) mma_bf16_first(tmp[0][j], a[0], b0.x, b0.y);
        else mma_bf16(tmp[0][j], a[0], b0.x, b0.y);
        if (kbl == 0 && PAR == 2) mma_bf16_first(tmp[PAR - 1][j], a[1], b0.z, b0.w);
        else mma_bf16(tmp[PAR - 1][j], a[1], b0.z, b0.w);
        mma_bf16(tmp[0][j], a[2], b1.x, b1.y);
        mma_bf16(tmp[PAR - 1][j], a[3], b1.z, b1.w);
      }
    }
#pragma unroll
    for (int j = 0; j < NTA; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float v = PAR == 2 ? tmp[0][j][c] + tmp[PAR - 1][j][c] : tmp[0][j][c];
        acc[j][c] = fmaf(sc[gi][c >> 1], v, acc[j][c]);
      }
  }
}

// The K range of one unit for a warp whose group has NTA active n-tiles:
// wait for each stage, run its scale groups, release it.  Returns false if a
// wait gave up.
template <int NT, int NTA>
__device__ __forceinline__ bool unit_range(SmCtl* ctl, const W4SmallParams& p, const SmItem& w, bool active,
                                           uint32_t ring_a, uint32_t q_off, uint32_t s_off, const int (&x_off)[NT],
                                           uint32_t zero_a, int lane, int& stage, uint32_t& phase,
                                           float (&acc)[NT][4]) {
  for (int grp = w.g0; grp < w.g1; grp += SPS) {
    if (!__all_sync(0xffffffffu, sm_wait(ctl, &ctl->full[stage], phase, p))) return false;
    const uint32_t st = ring_a + static_cast<uint32_t>(stage * p.stage_bytes);
    if (active) {
      uint32_t xa[NT];
#pragma unroll
      for (int j = 0; j < NT; ++j) xa[j] = x_off[j] >= 0 ? st + static_cast<uint32_t>(x_off[j]) : zero_a;
      if (grp + 1 < w.g1) stage_mma<NT, NTA, 2>(st + q_off, xa, st + s_off, acc);
      else stage_mma<NT, NTA, 1>(st + q_off, xa, st + s_off, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->empty[stage]);
    if (++stage == p.nstage) { stage = 0; phase ^= 1u; }
  }
  return true;
}

static_assert(SPS == 2, "stage_mma takes one or two scale groups");

// PLANES 1: first projection (bf16 activation rows, 8 rows per n-tile);
// PLANES 2: second projection (hidden hi + lo planes, 4 rows per n-tile).
template <int PLANES, int NT>
__global__ void __launch_bounds__(SM_THREADS, 1) w4_small_kernel(const W4SmallParams p) {
  constexpr int RPT = 8 / PLANES;  // activation rows per n-tile
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* ring = smem;
  SmCtl* ctl = reinterpret_cast<SmCtl*>(ring + p.nstage * p.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstage; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], CWARPS); }
    ctl->abort = 0;
    for (int i = 0; i < XROW / 16; ++i) ctl->zero[i] = make_uint4(0, 0, 0, 0);
    fence_mbarrier_init();
  }
  pdl_wait();  // group offsets and the activation rows come from the kernels before
  pdl_trigger();
  if (threadIdx.x == 0) {
    ctl->nprefix[0] = 0;
    for (int g = 0; g < p.G; ++g) {
      const int o0 = p.offsets[g], o1 = p.offsets[g + 1];
      ctl->offsets[g] = o0;
      ctl->nprefix[g + 1] = ctl->nprefix[g] + (o1 - o0 + p.rows_cap - 1) / p.rows_cap;
    }
    ctl->offsets[p.G] = p.offsets[p.G];
  }
  __syncthreads();

  if (warp == CWARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_phase = 0;
      bool ok = true;
      SmItem w;
      for (int u = blockIdx.x; ok && sm_item(ctl, p, u, w); u += gridDim.x) {
        const int row0 = w.row0, rows = w.rows;
        const int mt0 = slot_mtile(p, w.b, 0), mt1 = slot_mtile(p, w.b, 1);
        const bool has1 = p.two_mats || mt1 < p.m_tiles;
        const int64_t t0 = static_cast<int64_t>(w.e) * p.m_tiles + mt0;
        const int64_t t1 = static_cast<int64_t>(w.e) * p.m_tiles + mt1;
        for (int g = w.g0; g < w.g1; g += SPS) {
          const int ng = min(SPS, w.g1 - g);
          if (!sm_wait(ctl, &ctl->empty[stage], phase ^ 1u, p)) { ok = false; break; }
          uint8_t* st = ring + stage * p.stage_bytes;
          uint64_t* bar = &ctl->full[stage];
          const uint32_t qb = static_cast<uint32_t>(ng * GROUP_CODES), sb = static_cast<uint32_t>(ng * GROUP_SCALES);
          const uint32_t xb = static_cast<uint32_t>(ng * W4_GROUP * 2);
          mbar_arrive_expect_tx(bar, (has1 ? 2u : 1u) * (qb + sb) + static_cast<uint32_t>(PLANES * rows) * xb);
          bulk_load(st, p.Q0 + (t0 * p.num_g + g) * GROUP_CODES, qb, bar);
          bulk_load(st + 2 * SLOT_CODES, p.S0 + (t0 * p.num_g + g) * SB, sb, bar);
          if (has1) {
            bulk_load(st + SLOT_CODES, p.Q1 + (t1 * p.num_g + g) * GROUP_CODES, qb, bar);
            bulk_load(st + 2 * SLOT_CODES + SLOT_SCALES, p.S1 + (t1 * p.num_g + g) * SB, sb, bar);
          }
          // the same columns of the group's activation rows (hi and lo planes for the second projection)
          for (int pl = 0; pl < PLANES; ++pl) {
            const __nv_bfloat16* src = (pl == 0 ? p.X : p.X_lo) + static_cast<int64_t>(row0) * p.K + g * W4_GROUP;
            for (int n = 0; n < rows; ++n)
              bulk_load(st + X_OFF + (pl * p.rows_cap + n) * XROW, src + static_cast<int64_t>(n) * p.K, xb, bar);
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == p.nstage) { stage = 0; phase ^= 1u; }
        }
      }
      // copies still in flight complete before the CTA exits
      for (int s = 0; s < p.nstage; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (issued_phase >> s) & 1u, p.limit_ns);
    }
    return;
  }

  // -------------------------------------------------------------- compute
  const int slot = warp >> 3;
  const int g = lane >> 2, t = lane & 3;
  const int rbase = (warp & 7) * 16 + g;  // rows rbase and rbase + 8 of the slot
  // B fragment source of this lane: plane and row within an n-tile
  const int bplane = PLANES == 2 ? (g >> 2) : 0;
  const int brow = PLANES == 2 ? (g & 3) : g;
  const uint32_t ring_a = smem_u32(ring);
  const uint32_t zero_a = smem_u32(ctl->zero) + 32 * t;
  // this lane's addresses within a stage: codes of row rbase, scales of row rbase
  const uint32_t q_off = static_cast<uint32_t>(slot * SLOT_CODES + rbase * 32 + t * 8);
  const uint32_t s_off = static_cast<uint32_t>(2 * SLOT_CODES + slot * SLOT_SCALES + rbase * 2);
  int stage = 0;
  uint32_t phase = 0;
  SmItem w;
  bool ok = true;
  for (int u = blockIdx.x; ok && sm_item(ctl, p, u, w); u += gridDim.x) {
    const int row0 = w.row0, rows = w.rows;
    const int nt = (rows + RPT - 1) / RPT;
    const int mt = slot_mtile(p, w.b, slot);
    const bool active = p.two_mats || mt < p.m_tiles;
    // B rows of this lane, as offsets within a stage, or -1 for a row past the group's
    int x_off[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int n = j * RPT + brow;
      x_off[j] = n < rows ? X_OFF + (bplane * p.rows_cap + n) * XROW + 32 * t : -1;
    }
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[j][c] = 0.f;
    // the group's active n-tiles select a guard-free body (uniform per unit)
    if (nt <= 1) {
      ok = unit_range<NT, 1>(ctl, p, w, active, ring_a, q_off, s_off, x_off, zero_a, lane, stage, phase, acc);
    } else if (NT >= 2 && nt == 2) {
      ok = unit_range<NT, (NT >= 2 ? 2 : 1)>(ctl, p, w, active, ring_a, q_off, s_off, x_off, zero_a, lane, stage,
                                             phase, acc);
    } else if (NT >= 4 && nt == 3) {
      ok = unit_range<NT, (NT >= 4 ? 3 : 1)>(ctl, p, w, active, ring_a, q_off, s_off, x_off, zero_a, lane, stage,
                                             phase, acc);
    } else {
      ok = unit_range<NT, NT>(ctl, p, w, active, ring_a, q_off, s_off, x_off, zero_a, lane, stage, phase, acc);
    }
    if (!ok) break;
    // ---------------------------------------------------------- epilogue
    float* out = (slot == 1 && p.two_mats ? p.out3 : p.out) + static_cast<int64_t>(w.ks) * p.split_stride;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      float v[4] = {acc[j][0], acc[j][1], acc[j][2], acc[j][3]};
      if (PLANES == 2) {  // columns 4..7 (lanes t = 2, 3) are the lo plane of columns 0..3
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] += __shfl_xor_sync(0xffffffffu, v[c], 2);
      }
      if (!active || j >= nt || (PLANES == 2 && t >= 2)) continue;
      const int f = mt * SB + rbase;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = j * RPT + 2 * t + (c & 1);
        if (n >= rows) continue;
        const int64_t row = row0 + n;
        const float val = p.row_gate != nullptr ? v[c] * p.row_gate[row] : v[c];
        out[row * p.N + f + (c >> 1) * 8] = val;
      }
    }
  }
}

// Hidden rows from the first projection's partials: h = act(sum of the K
// ranges of W1 x) (* sum of W3 x), the ranges summed in order, as the bf16
// pair hi + lo that the second projection reads.
template <int ACT>
__global__ void __launch_bounds__(256) w4_hidden_kernel(const float* __restrict__ P1, const float* __restrict__ P3,
                                                        int ksplit, int64_t split_stride, const int32_t* total_rows,
                                                        int N, __nv_bfloat16* H, __nv_bfloat16* H_lo) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = static_cast<int64_t>(*total_rows) * N;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float a = 0.f, b = 0.f;
    for (int k = 0; k < ksplit; ++k) {
      a += P1[k * split_stride + i];
      if (ACT == MOE_ACT_SWIGLU) b += P3[k * split_stride + i];
    }
    const float h = ACT == MOE_ACT_SWIGLU ? __fdividef(a, 1.f + __expf(-a)) * b : fmaxf(a, 0.f);
    const __nv_bfloat16 hi = __float2bfloat16_rn(h);
    H[i] = hi;
    H_lo[i] = __float2bfloat16_rn(h - __bfloat162float(hi));
  }
}

size_t small_smem_bytes(int nstage, int stage_bytes) {
  return static_cast<size_t>(nstage) * stage_bytes + sizeof(SmCtl);
}

template <int PLANES, int NT>
cudaError_t launch_small_t(const W4SmallParams& p, int num_sms, cudaStream_t s) {
  const size_t bytes = small_smem_bytes(p.nstage, p.stage_bytes);
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(&w4_small_kernel<PLANES, NT>),
                                      static_cast<int>(SMEM_BUDGET + sizeof(SmCtl)));
  if (e != cudaSuccess) return e;
  return launch_pdl(w4_small_kernel<PLANES, NT>, dim3(num_sms), dim3(SM_THREADS), bytes, s, p);
}

// Scale groups per K range for `tiles` units of `num_g` scale groups on
// `ctas` CTAs: the cut whose longest CTA (its groups of codes plus its share
// of the fp32 partial rows written and read back) is shortest; more ranges
// only for a gain above 3 %.
int small_groups_per_range(int64_t tiles, int num_g, int64_t rows, int ctas) {
  if (tiles <= 0) return num_g;
  int best_gp = 0;
  double best = 0.0;
  for (int r = 1; r <= num_g; ++r) {
    const int gp = (num_g + r - 1) / r;
    const int64_t ranges = (num_g + gp - 1) / gp;
    const double groups = static_cast<double>((tiles * ranges + ctas - 1) / ctas) * gp;
    // a group streams 16 KB of codes; a unit writes and reads back rows x 256 fp32 partials
    const double partial = static_cast<double>(tiles * ranges) * static_cast<double>(rows) * 256 * 4 * 2 /
                           ctas / 16384.0;
    const double cost = groups + partial;
    if (best_gp == 0 || cost * 1.03 < best) { best = cost; best_gp = gp; }
  }
  return best_gp == 0 ? 1 : best_gp;
}

}  // namespace

// Activation rows of one unit: four n-tiles (32 rows of the first
// projection, 16 of the second's two planes); a larger group is cut into
// chunks of that many rows, each its own unit.
int small_chunk_rows(int mode) { return mode == W4_GATE ? 16 : 32; }

W4SmallSplit w4_small_split(int mode, int G, int64_t x_rows, int64_t max_group_rows, int N, int K, int ctas) {
  W4SmallSplit sp;
  const int m_tiles = N / SB;
  sp.row_blocks = mode == W4_SWIGLU ? m_tiles : (m_tiles + 1) / 2;
  const int num_g = K / W4_GROUP;
  int64_t rc = max_group_rows < small_chunk_rows(mode) ? max_group_rows : small_chunk_rows(mode);
  if (rc < 1) rc = 1;
  sp.rows_cap = static_cast<int>(rc);
  // (group, chunk) pairs: at most min(G, x_rows) groups with rows, ceil(rows / rc) chunks each
  const int64_t groups = x_rows < G ? x_rows : G;
  const int64_t chunks = (x_rows + groups * (rc - 1)) / rc;
  sp.gp = small_groups_per_range(chunks * sp.row_blocks, num_g, rc, ctas);
  sp.ksplit = (num_g + sp.gp - 1) / sp.gp;
  return sp;
}

cudaError_t plan_w4_small(const W4Args& g, int ctas, W4SmallPlan* pl, const char** why) {
  *why = nullptr;
  if (g.G > MAX_G) { *why = "4-bit products support at most 256 expert groups"; return cudaErrorInvalidValue; }
  if (g.K % W4_GROUP != 0 || g.N % SB != 0) {
    *why = "4-bit weights need d and d_ff to be multiples of 128";
    return cudaErrorInvalidValue;
  }
  const bool two = g.mode == W4_SWIGLU;
  const uintptr_t al = reinterpret_cast<uintptr_t>(g.Q0) | reinterpret_cast<uintptr_t>(g.S0) |
                       reinterpret_cast<uintptr_t>(g.X) |
                       (two ? (reinterpret_cast<uintptr_t>(g.Q1) | reinterpret_cast<uintptr_t>(g.S1)) : 0) |
                       (g.mode == W4_GATE ? reinterpret_cast<uintptr_t>(g.X_lo) : 0);
  if ((al & 15) != 0) {
    *why = "4-bit few-row products need 16-byte aligned codes and scales";
    return cudaErrorInvalidValue;
  }
  const W4SmallSplit sp = w4_small_split(g.mode, g.G, g.x_rows, g.max_group_rows, g.N, g.K, ctas);
  W4SmallParams& p = pl->p;
  memset(&p, 0, sizeof(p));
  p.G = g.G;
  p.N = g.N;
  p.K = g.K;
  p.m_tiles = g.N / SB;
  p.row_blocks = sp.row_blocks;
  p.num_g = g.K / W4_GROUP;
  p.gp = sp.gp;
  p.ksplit = sp.ksplit;
  p.two_mats = two ? 1 : 0;
  p.rows_cap = sp.rows_cap;
  const int planes = g.mode == W4_GATE ? 2 : 1;
  p.stage_bytes = X_OFF + planes * p.rows_cap * XROW;
  p.nstage = static_cast<int>((SMEM_BUDGET - sizeof(SmCtl)) / static_cast<size_t>(p.stage_bytes));
  if (p.nstage > MAX_STAGE) p.nstage = MAX_STAGE;
  p.Q0 = static_cast<const uint8_t*>(g.Q0);
  p.Q1 = static_cast<const uint8_t*>(two ? g.Q1 : g.Q0);
  p.S0 = static_cast<const __nv_bfloat16*>(g.S0);
  p.S1 = static_cast<const __nv_bfloat16*>(two ? g.S1 : g.S0);
  p.X = static_cast<const __nv_bfloat16*>(g.X);
  p.X_lo = static_cast<const __nv_bfloat16*>(g.mode == W4_GATE ? g.X_lo : g.X);
  p.out = static_cast<float*>(g.out);
  p.out3 = static_cast<float*>(two ? g.out_lo : g.out);
  p.split_stride = g.split_stride;
  p.offsets = g.offsets;
  p.row_gate = g.mode == W4_GATE ? g.row_gate : nullptr;
  p.err = g.err;
  p.limit_ns = kWaitLimitNs;
  pl->planes = planes;
  pl->nt = (p.rows_cap + 8 / planes - 1) / (8 / planes);
  if (p.nstage < 3) {
    *why = "4-bit few-row products: shared memory";
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_w4_small(const W4SmallPlan& pl, int num_sms, cudaStream_t s) {
  if (pl.planes == 1) {
    if (pl.nt <= 1) return launch_small_t<1, 1>(pl.p, num_sms, s);
    if (pl.nt <= 2) return launch_small_t<1, 2>(pl.p, num_sms, s);
    return launch_small_t<1, 4>(pl.p, num_sms, s);
  }
  if (pl.nt <= 1) return launch_small_t<2, 1>(pl.p, num_sms, s);
  if (pl.nt <= 2) return launch_small_t<2, 2>(pl.p, num_sms, s);
  return launch_small_t<2, 4>(pl.p, num_sms, s);
}

cudaError_t launch_w4_hidden(int act, const float* P1, const float* P3, int ksplit, int64_t split_stride,
                             const int32_t* total_rows, int64_t max_rows, int N, void* H, void* H_lo, int num_sms,
                             cudaStream_t s) {
  const int64_t n = max_rows * N;
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4LL * num_sms) blocks = 4LL * num_sms;
  __nv_bfloat16* h = static_cast<__nv_bfloat16*>(H);
  __nv_bfloat16* hl = static_cast<__nv_bfloat16*>(H_lo);
  if (act == MOE_ACT_SWIGLU)
    return launch_pdl(w4_hidden_kernel<MOE_ACT_SWIGLU>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, P1, P3,
                      ksplit, split_stride, total_rows, N, h, hl);
  return launch_pdl(w4_hidden_kernel<MOE_ACT_RELU>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, P1, P3,
                    ksplit, split_stride, total_rows, N, h, hl);
}

}  // namespace moe

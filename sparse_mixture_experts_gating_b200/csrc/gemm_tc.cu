// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA, for the expert FFNs of the MoE layer ("Mixture of experts",
// rayaq.ca, section "Implementation": each expert runs once on the sub-batch of
// its tokens; production code sorts tokens by expert and runs one grouped
// matrix multiply).
//
// C_e[m][n] = sum_k A[offsets[e] + m][k] * B_e[n][k] for every expert e, where
// A holds the expert-sorted rows (ragged groups, offsets on the device) and
// B_e is the expert's nn.Linear weight [N][K].  Tiles are 128 rows x 256 MMA
// columns; the tile list is expert-major, then n-tile, then m-tile, so tiles
// sharing a weight slab run at the same time and the slab is read from HBM once.
//
// Warp roles (192 threads, one CTA per SM):
//   warp 0       TMA producer: A box [AR x 64] (both planes of a split A in one
//                3D copy) + the B box(es) [256 x 64] per stage
//   warp 1       TMEM allocator; lane 0 issues tcgen05.mma (M=128, N=256, K=16)
//   warps 2..5   epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane per
//                row), activation or gate, masked stores
// Pipelines: STAGES-deep smem ring (full/empty mbarriers) and two TMEM
// accumulators of 256 columns (tmem_full/tmem_empty), so the epilogue of tile i
// overlaps the MMAs of tile i+1.  Every wait is bounded; a wait that runs out
// records MOE_ERR_TIMEOUT, raises the CTA's abort flag, drains its in-flight
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = kTileM;               // rows per tile
constexpr int BK = 64;                   // bf16 per 128-byte smem row
constexpr int MMA_N = 256;               // columns per MMA / accumulator
constexpr int MAX_STAGES = 5;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int B_HALF = 128 * BK * 2;     // 16 KB per B box
constexpr int NUM_THREADS = 192;

// Pipeline geometry.  SPLIT: the A operand is held as two bf16 planes
// (hi + lo, about 16 significant bits) and every k-block issues the MMAs of
// both planes against the same B tile, so one stage holds two A boxes.
// AR: A rows a stage holds (32, 64 or 128).  No expert group has more rows
// than the batch has tokens, so small batches stage only AR rows of A and fit
// more stages (more weight bytes in flight per SM) in the same shared memory;
// the M = 128 MMA still reads 128 rows from the A base, and rows past AR (the
// next bytes of the stage) only feed accumulator rows that are never stored.
template <bool SPLIT, int AR>
struct Geo {
  static constexpr int kA = SPLIT ? 2 : 1;
  static constexpr int A_ST = AR * BK * 2;  // one plane of A in a stage
  static constexpr int STAGE_BYTES = kA * A_ST + 2 * B_HALF;
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < MAX_STAGES ? (200 * 1024 / STAGE_BYTES) : MAX_STAGES;
};
constexpr uint32_t TMEM_COLS = 2 * MMA_N;
constexpr int MAX_E = 256;

using Params = TcParams;

struct Ctl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  volatile int abort;
  int mprefix[MAX_E + 1];
  int offsets[MAX_E + 1];
  // epilogue staging, per epilogue warp: 32 rows x 128 B (+16 B pad)
  alignas(16) uint8_t stage_out[4][32 * 144];
};

template <bool SPLIT, int AR>
constexpr size_t smem_bytes() {
  return Geo<SPLIT, AR>::STAGES * Geo<SPLIT, AR>::STAGE_BYTES + sizeof(Ctl) + 1024;
}

// Tile t -> (expert, m-tile, n-tile); tiles are expert-major, then n, then m.
__device__ __forceinline__ void decode_tile(int t, const Ctl* c, int E, int n_tiles, int& e, int& mt, int& nt) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (c->mprefix[mid] * n_tiles <= t) lo = mid; else hi = mid;
  }
  e = lo;
  const int local = t - c->mprefix[e] * n_tiles;
  const int mtiles = c->mprefix[e + 1] - c->mprefix[e];
  nt = local / mtiles;
  mt = local - nt * mtiles;
}

// Work of one CTA, identical in every role: units u = blockIdx.x + j * gridDim.x
// below the unit count.  With ksplit > 1 (the gated fp32 epilogue only, whose
// partial outputs the combine kernel sums in order) unit u is tile u / ksplit,
// K range u % ksplit.  Otherwise, when the tiles leave a last wave at most
// half full (p.split_tail: not SwiGLU, whose tile pairs W1 and W3 columns),
// each tile of that last wave becomes two units of half its columns (N 128),
// so the last wave takes half as long.  With a per-group K (p.k_rows, the
// weight gradients over each expert's rows) a tile runs only its group's
// k-blocks, none for an empty group (whose output the epilogue writes as 0).
struct Item {
  int tile, ks;    // tile and K-range index
  int kb0, kb1;    // k-blocks [kb0, kb1)
  int half;        // -1: all of the tile's columns; 0 / 1: that half of them
};
struct ItemIter {
  int u, units, whole;  // whole: units that are whole tiles (the rest are halves)
};
__device__ __forceinline__ ItemIter iter_begin(const Ctl* c, const Params& p) {
  ItemIter it;
  it.u = static_cast<int>(blockIdx.x);
  const int tiles = c->mprefix[p.E] * p.n_tiles;
  if (p.ksplit == 1 && p.split_tail) {
    const int ctas = static_cast<int>(gridDim.x);
    const int r = tiles % ctas;
    it.whole = (r > 0 && 2 * r <= ctas) ? tiles - r : tiles;
    it.units = it.whole + 2 * (tiles - it.whole);
  } else {
    it.whole = it.units = tiles * p.ksplit;
  }
  return it;
}
__device__ __forceinline__ bool iter_next(ItemIter& it, const Params& p, const Ctl* ctl, Item& w) {
  if (it.u >= it.units) return false;
  if (it.u < it.whole) {
    w.tile = it.u / p.ksplit;
    w.ks = it.u - w.tile * p.ksplit;
    w.half = -1;
  } else {
    const int v = it.u - it.whole;
    w.tile = it.whole + (v >> 1);
    w.ks = 0;
    w.half = v & 1;
  }
  w.kb0 = w.ks * p.kb_per;
  w.kb1 = min(p.num_kb, w.kb0 + p.kb_per);
  if (p.k_rows != nullptr) {  // this group's own K (no K ranges): its k-blocks only, possibly none
    int e, mt, nt;
    decode_tile(w.tile, ctl, p.E, p.n_tiles, e, mt, nt);
    w.kb1 = min(w.kb1, (p.k_rows[e + 1] - p.k_rows[e] + BK - 1) / BK);
  }
  it.u += static_cast<int>(gridDim.x);
  return true;
}

__device__ __forceinline__ bool wait_or_abort(Ctl* c, uint64_t* bar, uint32_t parity, const Params& p) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (c->abort) return false;
    if (globaltimer_ns() - t0 > p.limit_ns) {
      record_error(p.err, DEV_ERR_TIMEOUT);
      c->abort = 1;
      return false;
    }
  }
}

// silu(a) * b with the fast divide (2 ulp; 0 once 1 + e^-a overflows, the limit of silu).
__device__ __forceinline__ float silu_mul(float a, float b) { return __fdividef(a, 1.f + __expf(-a)) * b; }

// fp16 pair of (v0, v1); `valid`: the pair is a stored element of the hidden
// activation (rows past an expert's group and columns past N hold whatever
// the tile's stale operands gave and are never stored), and only then can it
// raise *bad when out of the fp16 range.
__device__ __forceinline__ uint32_t pack_f16x2_in_range(float v0, float v1, bool valid, bool& bad) {
  bool b = false;
  const uint32_t r = pack_f16x2_checked(v0, v1, b);
  bad |= b && valid;
  return r;
}

// bf16 pair (hi, lo) with hi = RNE(v) and lo = RNE(v - hi): hi + lo carries
// about 16 significant bits of v.
__device__ __forceinline__ void split_bf16(float v0, float v1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
  const float2 hf = __bfloat1622float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_bf16x2(v0 - hf.x, v1 - hf.y);
}

// EPI: epilogue (internal.h GemmEpi).  HID (internal.h HiddenKind): how the
// hidden activation is held.  HID_BF16X2: the first projection's epilogue
// writes it as hi/lo bf16 planes, the second reads its A operand as hi (tmA)
// + lo (tmA2) planes.  HID_F16: the first projection writes it as fp16 (and
// flags values beyond the fp16 range), the second multiplies fp16 A by an
// fp16 image of its weights.
template <int EPI, int HID, int AR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                        const Params p) {
  constexpr bool GATE = EPI == EPI_GATE_F32 || EPI == EPI_GATE_SCATTER_BF16;
  constexpr bool A_SPLIT = HID == HID_BF16X2 && GATE;
  constexpr bool OUT_SPLIT = HID == HID_BF16X2 && !GATE;
  constexpr bool OUT_F16 = HID == HID_F16 && !GATE;
  constexpr uint32_t IDESC = (HID == HID_F16 && GATE) ? idesc_f16_f32(BM, MMA_N) : idesc_bf16_f32(BM, MMA_N);
  constexpr uint32_t IDESC_HALF =
      (HID == HID_F16 && GATE) ? idesc_f16_f32(BM, MMA_N / 2) : idesc_bf16_f32(BM, MMA_N / 2);
  using G = Geo<A_SPLIT, AR>;
  constexpr int STAGES = G::STAGES;
  constexpr int STAGE_BYTES = G::STAGE_BYTES;
  constexpr int A_ST = G::A_ST;
  constexpr int B_OFF = G::kA * A_ST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* stages = smem_raw + pad;
  Ctl* ctl = reinterpret_cast<Ctl*>(stages + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&ctl->tfull[a], 1); mbar_init(&ctl->tempty[a], 128); }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    if (A_SPLIT) tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) tmem_alloc(&ctl->tmem_slot, TMEM_COLS);
  pdl_wait();  // tile offsets and the A rows come from the kernels before
  pdl_trigger();
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) {
    ctl->mprefix[i] = p.mprefix[i];
    ctl->offsets[i] = p.offsets[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_phase = 0;  // per-stage bits: a copy was issued / its phase
      bool ok = true;
      ItemIter it = iter_begin(ctl, p);
      Item w;
      while (ok && iter_next(it, p, ctl, w)) {
        int e, mt, nt;
        decode_tile(w.tile, ctl, p.E, p.n_tiles, e, mt, nt);
        const int row0 = ctl->offsets[e] + mt * BM;
        const int brow = e * p.N + nt * p.bn + (w.half > 0 ? 128 : 0);
        const int kb0 = w.kb0, kb1 = w.kb1;
        const uint32_t tx = (A_SPLIT ? 2u : 1u) * A_ST + (w.half >= 0 ? 1u : 2u) * B_HALF;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(ctl, &ctl->empty[stage], phase ^ 1u, p)) { ok = false; break; }
          uint8_t* sa = stages + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl->full[stage], tx);
          if (A_SPLIT) tma_load_3d(sa, &tmA, &ctl->full[stage], kb * BK, row0, 0);  // hi and lo planes
          else tma_load_2d(sa, &tmA, &ctl->full[stage], kb * BK, row0);
          if (EPI == EPI_SWIGLU_BF16 || EPI == EPI_GATE_F32_B2) {  // W1 / W3, or B's hi / lo planes
            tma_load_2d(sa + B_OFF, &tmB0, &ctl->full[stage], kb * BK, brow);
            tma_load_2d(sa + B_OFF + B_HALF, &tmB1, &ctl->full[stage], kb * BK, brow);
          } else if (w.half >= 0) {
            tma_load_2d(sa + B_OFF, &tmB1, &ctl->full[stage], kb * BK, brow);  // 128-row box
          } else {
            tma_load_2d(sa + B_OFF, &tmB0, &ctl->full[stage], kb * BK, brow);  // 256-row box
          }
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl->full[s], (issued_phase >> s) & 1u, p.limit_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      ItemIter it = iter_begin(ctl, p);
      Item w;
      while (ok && iter_next(it, p, ctl, w)) {
        if (!wait_or_abort(ctl, &ctl->tempty[acc], acc_phase ^ 1u, p)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * MMA_N);
        const int kb0 = w.kb0, kb1 = w.kb1;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(ctl, &ctl->full[stage], phase, p)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + stage * STAGE_BYTES);
          const uint32_t sb = sa + B_OFF;
          const uint32_t idesc = w.half >= 0 ? IDESC_HALF : IDESC;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d_tmem, sdesc_k_sw128(sa + k * 32), sdesc_k_sw128(sb + k * 32), idesc,
                      (kb != kb0 || k != 0) ? 1u : 0u);
          if (A_SPLIT) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_bf16(d_tmem, sdesc_k_sw128(sa + A_ST + k * 32), sdesc_k_sw128(sb + k * 32), idesc, 1u);
          }
          umma_commit(&ctl->empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&ctl->tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // Drain: all MMAs of this CTA complete before TMEM is freed.
      umma_commit(&ctl->drain);
      mbar_wait(&ctl->drain, 0, p.limit_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns 32 rows of the tile (its TMEM lane quarter).  Per chunk of
    // 32 columns a lane computes its row's values, stages them in shared
    // memory, and the warp then stores the 32 x 32 block with whole-row
    // coalescing (8 rows x 64 B, or 4 rows x 128 B, per instruction).
    const int q = warp & 3;
    const int r_in_tile = q * 32 + lane;
    uint8_t* stg = reinterpret_cast<uint8_t*>(ctl->stage_out[q]);
    int acc = 0;
    uint32_t acc_phase = 0;
    ItemIter it = iter_begin(ctl, p);
    Item w;
    while (iter_next(it, p, ctl, w)) {
      int e, mt, nt;
      decode_tile(w.tile, ctl, p.E, p.n_tiles, e, mt, nt);
      const int ks = w.ks;
      const bool ok = __all_sync(0xffffffffu, wait_or_abort(ctl, &ctl->tfull[acc], acc_phase, p));
      if (!ok) break;  // warp-uniform: tcgen05.ld below is .sync.aligned
      tc_fence_after();
      const int m_local = mt * BM + r_in_tile;
      const bool vrow = m_local < ctl->offsets[e + 1] - ctl->offsets[e];
      if (!__any_sync(0xffffffffu, vrow)) {  // all 32 rows of this warp lie past the expert's group
        tc_fence_before();
        mbar_arrive(&ctl->tempty[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        continue;
      }
      const int row = ctl->offsets[e] + m_local;  // expert-sorted row of this lane
      const int n0 = nt * p.bn + (w.half > 0 ? 128 : 0);
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * MMA_N);
      // destination row of each 32-row block row this lane stores (for bf16: rows lane/4 + 8i)
      int drow[4];
      bool dval[4];
      const float g =
          (EPI == EPI_GATE_F32 || EPI == EPI_GATE_SCATTER_BF16 || EPI == EPI_GATE_F32_B2) && vrow ? p.row_gate[row] : 0.f;
      const int my_dst = (EPI == EPI_GATE_SCATTER_BF16) ? (vrow ? p.row_token[row] : 0) : row;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int src = (lane >> 2) + 8 * i;
        drow[i] = __shfl_sync(0xffffffffu, my_dst, src);
        dval[i] = __shfl_sync(0xffffffffu, vrow ? 1 : 0, src) != 0;
      }

      if (EPI == EPI_SWIGLU_BF16 || EPI == EPI_RELU_BF16 || EPI == EPI_GATE_SCATTER_BF16) {
        const int NCH = (EPI == EPI_SWIGLU_BF16 || w.half >= 0) ? 4 : 8;
        bool out_of_range = false;  // OUT_F16: a hidden value beyond the fp16 range
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        __nv_bfloat16* out_lo = static_cast<__nv_bfloat16*>(p.out_lo);
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          uint32_t ra[32];
          uint32_t hi[16], lo[16];
          if (EPI == EPI_SWIGLU_BF16) {
            uint32_t rb[32];
            tmem_ld32(tb + c * 32, ra);
            tmem_ld32(tb + 128 + c * 32, rb);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_mul(__uint_as_float(ra[2 * i]), __uint_as_float(rb[2 * i]));
              const float h1 = silu_mul(__uint_as_float(ra[2 * i + 1]), __uint_as_float(rb[2 * i + 1]));
              if (OUT_SPLIT) split_bf16(h0, h1, hi[i], lo[i]);
              else if (OUT_F16) hi[i] = pack_f16x2_in_range(h0, h1, vrow && n0 + c * 32 + 2 * i < p.N, out_of_range);
              else hi[i] = pack_bf16x2(h0, h1);
            }
          } else {
            tmem_ld32(tb + c * 32, ra);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float h0 = __uint_as_float(ra[2 * i]), h1 = __uint_as_float(ra[2 * i + 1]);
              if (EPI == EPI_RELU_BF16) {
                h0 = fmaxf(h0, 0.f);
                h1 = fmaxf(h1, 0.f);
              } else {
                h0 *= g;
                h1 *= g;
              }
              if (OUT_SPLIT) split_bf16(h0, h1, hi[i], lo[i]);
              else if (OUT_F16) hi[i] = pack_f16x2_in_range(h0, h1, vrow && n0 + c * 32 + 2 * i < p.N, out_of_range);
              else hi[i] = pack_bf16x2(h0, h1);
            }
            if (EPI == EPI_GATE_SCATTER_BF16 && p.out_f32 != nullptr && vrow) {  // debug copy
              float* of = p.out_f32 + static_cast<int64_t>(my_dst) * p.N + n0 + c * 32;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + c * 32 + i < p.N) of[i] = __uint_as_float(ra[i]) * g;
            }
          }
          const int col = n0 + c * 32;
#pragma unroll
          for (int plane = 0; plane < (OUT_SPLIT ? 2 : 1); ++plane) {
            const uint32_t* src = plane == 0 ? hi : lo;
            uint4* srow = reinterpret_cast<uint4*>(stg + lane * 80);
#pragma unroll
            for (int v = 0; v < 4; ++v) srow[v] = make_uint4(src[4 * v], src[4 * v + 1], src[4 * v + 2], src[4 * v + 3]);
            __syncwarp();
            __nv_bfloat16* dst = plane == 0 ? out : out_lo;
            const int seg = lane & 3;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rr = (lane >> 2) + 8 * i;
              if (dval[i] && col + seg * 8 < p.N)
                *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(drow[i]) * p.N + col + seg * 8) =
                    *reinterpret_cast<const uint4*>(stg + rr * 80 + seg * 16);
            }
            __syncwarp();
          }
        }
        if (OUT_F16 && __any_sync(0xffffffffu, out_of_range) && lane == 0) record_error(p.err, DEV_ERR_RANGE);
      } else {  // EPI_GATE_F32(_B2): gated fp32 rows of the expert-sorted buffer (partial ks)
        float* out = static_cast<float*>(p.out) + static_cast<int64_t>(ks) * p.split_stride;
        const int nch = (w.half >= 0 || EPI == EPI_GATE_F32_B2) ? 4 : 8;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t ra[32];
          if (w.kb1 > w.kb0 && EPI == EPI_GATE_F32_B2) {  // hi-plane and lo-plane products summed
            uint32_t rb[32];
            tmem_ld32(tb + c * 32, ra);
            tmem_ld32(tb + 128 + c * 32, rb);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) ra[i] = __float_as_uint(__uint_as_float(ra[i]) + __uint_as_float(rb[i]));
          } else if (w.kb1 > w.kb0) {
            tmem_ld32(tb + c * 32, ra);
            tmem_ld_wait();
          } else {  // a group with no k-blocks (per-group K of 0): the product is zero
#pragma unroll
            for (int i = 0; i < 32; ++i) ra[i] = 0u;
          }
          float4* srow = reinterpret_cast<float4*>(stg + lane * 144);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            srow[v] = make_float4(__uint_as_float(ra[4 * v]) * g, __uint_as_float(ra[4 * v + 1]) * g,
                                  __uint_as_float(ra[4 * v + 2]) * g, __uint_as_float(ra[4 * v + 3]) * g);
          __syncwarp();
          const int col = n0 + c * 32;
          const int seg = lane & 7;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rr = (lane >> 3) + 4 * i;
            const int dr = __shfl_sync(0xffffffffu, row, rr);
            const bool dv = __shfl_sync(0xffffffffu, vrow ? 1 : 0, rr) != 0;
            if (dv && col + seg * 4 < p.N)
              *reinterpret_cast<float4*>(out + static_cast<int64_t>(dr) * p.N + col + seg * 4) =
                  *reinterpret_cast<const float4*>(stg + rr * 144 + seg * 16);
          }
          __syncwarp();
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
// Host: tensor maps through the driver entry point (no libcuda link needed).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// Row-major bf16 matrix [rows][cols] -> map with box [128 rows][64 cols], 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return make_map_bf16(m, base, rows, cols, 128);
}

// Row-major 16-bit matrix [rows][cols] of the given type -> map with box
// [box_rows][64 cols], 128-byte swizzle.
bool make_map_16(CUtensorMap* m, CUtensorMapDataType type, const void* base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_map_planes_bf16(CUtensorMap* m, const void* base, uint64_t plane_stride, uint64_t rows, uint64_t cols,
                          uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[3] = {cols, rows, 2};
  const cuuint64_t strides[2] = {cols * 2, plane_stride};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType type, const void* base, uint64_t rows, uint64_t cols,
                 uint32_t elem_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int EPI, int HID, int AR>
cudaError_t launch_t(const TcGemmPlan& pl, int num_sms, cudaStream_t s) {
  constexpr bool A_SPLIT = HID == HID_BF16X2 && (EPI == EPI_GATE_F32 || EPI == EPI_GATE_SCATTER_BF16);
  constexpr size_t bytes = smem_bytes<A_SPLIT, AR>();
  static_assert(bytes <= 227 * 1024, "grouped GEMM shared memory");
  cudaError_t e = set_smem_limit_once(reinterpret_cast<const void*>(&grouped_gemm_kernel<EPI, HID, AR>),
                                      static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  return launch_pdl(grouped_gemm_kernel<EPI, HID, AR>, dim3(num_sms), dim3(NUM_THREADS), bytes, s, pl.a, pl.a2,
                    pl.b0, pl.b1, pl.p);
}

template <int EPI, int HID>
cudaError_t launch_ar(const TcGemmPlan& pl, int num_sms, cudaStream_t s) {
  if (pl.ar == 32) return launch_t<EPI, HID, 32>(pl, num_sms, s);
  if (pl.ar == 64) return launch_t<EPI, HID, 64>(pl, num_sms, s);
  return launch_t<EPI, HID, 128>(pl, num_sms, s);
}

template <int HID>
cudaError_t launch_epi(const TcGemmPlan& pl, int num_sms, cudaStream_t s) {
  switch (pl.epi) {
    case EPI_RELU_BF16: return launch_ar<EPI_RELU_BF16, HID>(pl, num_sms, s);
    case EPI_SWIGLU_BF16: return launch_ar<EPI_SWIGLU_BF16, HID>(pl, num_sms, s);
    case EPI_GATE_F32: return launch_ar<EPI_GATE_F32, HID>(pl, num_sms, s);
    case EPI_GATE_F32_B2:
      if constexpr (HID == HID_BF16) return launch_ar<EPI_GATE_F32_B2, HID>(pl, num_sms, s);
      return cudaErrorInvalidValue;
    default: return launch_ar<EPI_GATE_SCATTER_BF16, HID>(pl, num_sms, s);
  }
}

// bf16 -> fp16, eight values per 16-byte access, four accesses in flight per
// thread; see launch_convert_f16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 v, bool& bad) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
    w[i] = pack_f16x2_checked(lo, hi, bad);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void __launch_bounds__(256) convert_f16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          int64_t n8, unsigned int* err) {
  pdl_trigger();  // the second projection may be scheduled at once
  bool bad = false;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n8; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = __ldcs(src + i + j * stride);
#pragma unroll
    for (int j = 0; j < 4; ++j) dst[i + j * stride] = bf16x8_to_f16x8(v[j], bad);
  }
  for (; i < n8; i += stride) dst[i] = bf16x8_to_f16x8(__ldcs(src + i), bad);
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) record_error(err, DEV_ERR_RANGE);
  // complete only after the kernel before (the first projection): the kernel
  // after this one waits for this one alone
  pdl_wait();
}

}  // namespace

cudaError_t plan_gemm_tc(const GemmArgs& g, TcGemmPlan* pl, const char** why) {
  *why = nullptr;
  if (g.E > MAX_E) { *why = "grouped GEMM supports at most 256 experts"; return cudaErrorInvalidValue; }
  const bool gate = g.epi == EPI_GATE_F32 || g.epi == EPI_GATE_SCATTER_BF16;
  if (g.f16 && g.split) { *why = "grouped GEMM: fp16 and split hidden modes exclude each other"; return cudaErrorInvalidValue; }
  const bool a_split = g.split && g.A2 != nullptr;
  const bool ops_f16 = g.f16 && gate;  // A and B of the second projection in fp16
  const bool swiglu = g.epi == EPI_SWIGLU_BF16;
  const bool b2 = g.epi == EPI_GATE_F32_B2;  // B as hi + lo planes, like W1 / W3: two 128-row boxes
  if (b2 && (g.split || g.f16 || g.B1 == nullptr)) {
    *why = "grouped GEMM: a split B operand takes a single-plane bf16 A and both B planes";
    return cudaErrorInvalidValue;
  }
  // A rows per stage: every expert group has at most max_group_rows rows
  pl->ar = g.max_group_rows <= 32 ? 32 : g.max_group_rows <= 64 ? 64 : 128;
  const uint32_t ar = static_cast<uint32_t>(pl->ar);
  const uint64_t a_rows = static_cast<uint64_t>(g.a_rows), K = static_cast<uint64_t>(g.K);
  const uint64_t b_rows = static_cast<uint64_t>(g.E) * g.N;
  // a split A is read through one 3D map over both planes (the lo plane must
  // follow the hi plane at a 16-byte multiple)
  const intptr_t plane_stride = static_cast<const uint8_t*>(g.A2) - static_cast<const uint8_t*>(g.A);
  if (a_split && (plane_stride <= 0 || plane_stride % 16 != 0 ||
                  static_cast<uint64_t>(plane_stride) < a_rows * K * 2)) {
    *why = "grouped GEMM: the lo plane of the A operand must follow the hi plane";
    return cudaErrorInvalidValue;
  }
  const bool maps_ok =
      ops_f16
          ? (make_map_16(&pl->a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.A, a_rows, K, ar) &&
             make_map_16(&pl->a2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.A, a_rows, K, 128) &&
             make_map_16(&pl->b0, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.B0, b_rows, K, 256) &&
             make_map_16(&pl->b1, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, g.B0, b_rows, K, 128))
          : ((a_split ? make_map_planes_bf16(&pl->a, g.A, static_cast<uint64_t>(plane_stride), a_rows, K, ar)
                      : make_map_bf16(&pl->a, g.A, a_rows, K, ar)) &&
             make_map(&pl->a2, a_split ? g.A2 : g.A, a_rows, K) &&
             // B: two 128-row boxes (W1 and W3) for SwiGLU, else one 256-row box
             make_map_bf16(&pl->b0, g.B0, b_rows, K, swiglu || b2 ? 128 : 256) &&
             make_map(&pl->b1, swiglu || b2 ? g.B1 : g.B0, b_rows, K));
  if (!maps_ok) {
    *why = "cuTensorMapEncodeTiled failed (alignment or driver entry point)";
    return cudaErrorInvalidValue;
  }
  Params& p = pl->p;
  p.E = g.E;
  p.N = g.N;
  p.K = g.K;
  p.bn = (swiglu || b2) ? 128 : 256;
  p.n_tiles = (g.N + p.bn - 1) / p.bn;
  p.num_kb = (g.K + BK - 1) / BK;
  p.ksplit = g.epi == EPI_GATE_F32 ? (g.ksplit < 1 ? 1 : (g.ksplit > p.num_kb ? p.num_kb : g.ksplit)) : 1;
  p.kb_per = (p.num_kb + p.ksplit - 1) / p.ksplit;
  p.split_stride = g.split_stride;
  p.split_tail = (swiglu || b2) ? 0 : 1;
  p.out = g.out;
  p.out_lo = g.out2;
  p.out_f32 = g.out_f32;
  p.offsets = g.offsets;
  p.mprefix = g.mprefix;
  p.row_gate = g.row_gate;
  p.row_token = g.row_token;
  p.err = g.err;
  p.limit_ns = kWaitLimitNs;
  p.k_rows = g.k_rows;
  if (g.k_rows != nullptr && ((g.epi != EPI_GATE_F32 && !b2) || p.ksplit != 1)) {
    *why = "grouped GEMM: a per-group K needs the gated fp32 epilogue without K ranges";
    return cudaErrorInvalidValue;
  }
  pl->epi = g.epi;
  pl->hid = g.f16 ? HID_F16 : g.split ? HID_BF16X2 : HID_BF16;
  if (g.epi < EPI_RELU_BF16 || g.epi > EPI_GATE_F32_B2) {
    *why = "unknown epilogue";
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_tc(const TcGemmPlan& pl, int num_sms, cudaStream_t s) {
  if (pl.hid == HID_F16) return launch_epi<HID_F16>(pl, num_sms, s);
  if (pl.hid == HID_BF16X2) return launch_epi<HID_BF16X2>(pl, num_sms, s);
  return launch_epi<HID_BF16>(pl, num_sms, s);
}

cudaError_t launch_convert_f16(const void* src, void* dst, int64_t n, unsigned int* err, int num_sms,
                               cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  // one block per SM: it runs beside the first projection's CTA on each SM
  // and should take few of its issue slots (four 16-byte loads in flight per
  // thread keep ~1 MB in flight across the GPU, enough for the ~1 TB/s it needs)
  const int64_t n8 = n / 8;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > num_sms) blocks = num_sms;
  return launch_pdl(convert_f16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<const uint4*>(src), static_cast<uint4*>(dst), n8, err);
}

}  // namespace moe

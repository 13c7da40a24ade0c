// Host-side interface between the translation units of the MoE library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Tokens per router / dispatch block; the per-block partial counts use it.
constexpr int kRouterTokens = 32;
// Rows per tensor-core tile (M of one tcgen05.mma).
constexpr int kTileM = 128;

struct RoutingArgs {
  int64_t T;
  int E, k, d, gate_mode;
  int64_t capacity;  // -1: dropless
  int nblk;          // ceil(T / kRouterTokens)
  int x_is_bf16;
  const void* x;
  const float* W_r;
  const float* b_r;
  const float* logits_in;
  // workspace
  int32_t* topk_idx;   // [T][k]
  float* topk_gate;    // [T][k]
  int32_t* dest_row;   // [T][k]
  int32_t* part_hist;  // [E][nblk]
  int32_t* part_cnt1;  // [E][nblk]
  float* part_psum;    // [E][nblk]
  float* part_lse2;    // [nblk]
  int32_t* blockoff;   // [E][nblk]
  int32_t* counts;     // [E]   (may alias the user output)
  int32_t* offsets;    // [E+1]
  int32_t* mprefix;    // [E+1] prefix of ceil(kept_e / kTileM)
  int32_t* tot_cnt1;   // [E]   first-choice count of each expert (scan)
  float* tot_psum;     // [E]   probability sum of each expert (scan)
  float* balance_out;    // [3] aux over all choices, CV of counts, cv^2 of P (scan)
  int n_shared;          // shared experts: groups E .. E + n_shared - 1 of T rows each
  int32_t* row_token;  // [S_max]
  float* row_gate;     // [S_max]
  void* Xp;            // [S_max][d]
  // outputs
  int32_t* dropped;
  float* aux;
  float* z;
  // debug
  float* logits_out;
  float* lse_out;
  uint8_t* drop_mask;
  int32_t* offsets_out;
  // k == 1 tensor-core path: the dispatch zeroes y rows of dropped tokens
  void* y_zero_dropped;
  float* yf_zero_dropped;  // and the fp32 debug copy of them
};

cudaError_t launch_router(const RoutingArgs& a, cudaStream_t s);

// Tensor-core router for bf16 layers with E <= 128: W_r is first split exactly
// into three bf16 planes [3][E_pad][d] (E_pad = E rounded up to 16) in `wsplit`.
constexpr int kRouterTcMaxE = 128;
inline int router_pad_e(int E) { return (E + 15) / 16 * 16; }
// K ranges of the tensor-core router (split when the 128-token tiles alone
// cannot occupy the GPU); the split CTAs exchange fp32 partial logits through
// `partials` ([tiles][ksplit][128][E_pad]) and per-tile tickets.
int router_ksplit(int64_t T, int d);
size_t router_partials_bytes(int64_t T, int E, int d);
cudaError_t launch_router_tc(const RoutingArgs& a, void* wsplit, void* partials, int num_sms, unsigned int* err,
                             cudaStream_t s, const char** why);

// bf16 [rows][cols] tensor map, box [box_rows][64], 128-byte swizzle.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Two bf16 planes [2][rows][cols], plane_stride bytes apart -> 3D map with box
// [2 planes][box_rows][64 cols], 128-byte swizzle: one copy lands plane 0's
// [box_rows x 64] tile followed by plane 1's.
bool make_map_planes_bf16(CUtensorMap* m, const void* base, uint64_t plane_stride, uint64_t rows, uint64_t cols,
                          uint32_t box_rows);
cudaError_t launch_scan(const RoutingArgs& a, cudaStream_t s);
// Batches of at most 32 tokens (one router block): router, scan and dispatch
// in two launches (fp32 partial logits over d-chunks, then one block for the
// rest).  `partials` holds route_small_partials_bytes(E).
constexpr int kRouteSmallMaxT = 32;
size_t route_small_partials_bytes(int E);
cudaError_t launch_route_small(const RoutingArgs& a, void* partials, cudaStream_t s);
cudaError_t launch_dispatch(const RoutingArgs& a, cudaStream_t s);
// y_t = sum over kept choices j (in order j) of sum over the ksplit partials
// (in order) of Yp[partial][dest_row[t][j]], then (in order s) of the rows
// *shared_base + s * T + t of the n_shared shared experts.
cudaError_t launch_combine(int64_t T, int k, int d, int y_is_bf16, const int32_t* dest_row, int n_shared,
                           const int32_t* shared_base, const float* Yp,
                           int ksplit, int64_t split_stride, void* y, float* y_f32, cudaStream_t s);

// K ranges of the second projection: split K when the tiles alone cannot
// occupy the GPU (small token counts), for a 148-SM B200.
constexpr int kSplitTargetCtas = 148;
int gemm2_ksplit(int64_t s_max, int E, int d, int d_ff);

// Grouped GEMM epilogues
// EPI_GATE_F32_B2: the gated fp32 epilogue with B given as hi + lo bf16 planes
// (B0, B1): one N 256 MMA per step over a 128-row box of each, the two
// halves of the accumulator summed per output column (128 columns per tile).
enum GemmEpi { EPI_RELU_BF16 = 0, EPI_SWIGLU_BF16 = 1, EPI_GATE_F32 = 2, EPI_GATE_SCATTER_BF16 = 3, EPI_GATE_F32_B2 = 4 };

struct GemmArgs {
  int epi;
  int E;
  int N;  // output columns per expert
  int K;  // reduction length
  int64_t a_rows;  // rows of the A buffer (S_max)
  int64_t max_group_rows;  // no expert group has more rows (the batch's T)
  const void* A;   // [a_rows][K]  (the hi plane when split)
  const void* A2;  // [a_rows][K]  lo plane of a split A operand, else NULL
  int split;       // first projection: write hi/lo planes; second: read them
  int f16;         // first projection: write the hidden activation as fp16; second:
                   // A (that activation) and B (an fp16 image of W2) are fp16
  const void* B0;  // [E][N][K]  (W1, or W2)
  const void* B1;  // [E][N][K]  (W3 for SwiGLU, else unused)
  void* out;       // Hp [S][N] | Yp [S][N] fp32 | y [T][N]
  void* out2;      // lo plane of a split Hp, else NULL
  int ksplit;      // EPI_GATE_F32: K is cut into ksplit ranges, partial j written at out + j * split_stride
  int64_t split_stride;
  float* out_f32;  // scatter epilogue only: optional fp32 copy of y
  const int32_t* offsets;
  const int32_t* mprefix;
  const float* row_gate;
  const int32_t* row_token;
  unsigned int* err;
  const int32_t* k_rows;  // gated fp32 epilogue: group e's K is k_rows[e + 1] - k_rows[e] (NULL: K)
};

// Kernel parameters of the tensor-core grouped GEMM.
struct TcParams {
  int E, N, K, n_tiles, bn, num_kb;
  int ksplit, kb_per;      // K ranges per (expert, m-tile, n-tile) and k-blocks in each
  int split_tail;          // a last wave at most half full runs as half-width (N 128) units
  int64_t split_stride;    // elements between the partial outputs of consecutive K ranges
  void* out;
  void* out_lo;     // first projection with a split hidden activation: the lo plane
  float* out_f32;   // scatter epilogue only: optional fp32 copy of y
  const int32_t* offsets;
  const int32_t* mprefix;
  const float* row_gate;
  const int32_t* row_token;
  unsigned int* err;
  uint64_t limit_ns;
  const int32_t* k_rows;  // per-group K (k-blocks ceil(K_e / 64)), NULL: K for every group
};

// How the hidden activation between the projections is held.
enum HiddenKind { HID_BF16 = 0, HID_BF16X2 = 1, HID_F16 = 2 };

// Everything a tensor-core GEMM launch needs, prepared on the host up front.
struct TcGemmPlan {
  CUtensorMap a, a2, b0, b1;
  TcParams p;
  int epi;
  int hid;  // HiddenKind
  int ar;   // A rows per pipeline stage: 32, 64 or 128
};

// fp16 image of n bf16 values (n a multiple of 8, both pointers 16-byte
// aligned), for the second projection's B operand in the fp16 hidden mode.
// Launched right after the first projection: it starts while that kernel
// runs, and waits for it to complete before it ends itself, so the kernel
// launched after it sees both complete.  A value beyond the fp16 range
// records DEV_ERR_RANGE in *err.
cudaError_t launch_convert_f16(const void* src, void* dst, int64_t n, unsigned int* err, int num_sms,
                               cudaStream_t s);

cudaError_t plan_gemm_tc(const GemmArgs& g, TcGemmPlan* plan, const char** why);
cudaError_t launch_gemm_tc(const TcGemmPlan& plan, int num_sms, cudaStream_t s);

// Any row-major 2D tensor [rows][cols] of elements of elem_bytes bytes -> map
// with box [box_rows][box_cols] and the given swizzle.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType type, const void* base, uint64_t rows, uint64_t cols,
                 uint32_t elem_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// ---------------------------------------------------------------- 4-bit weights
// Codes in tiles of 128 rows x 64 elements, each tile 4 KB contiguous (row r
// of the tile at 32 r bytes): uint32 [rows / 128][K / 64][128][8]; in a word,
// element 2j of its 8 in bits 4j.., element 2j + 1 in bits 4j + 16.., code =
// q + 8.  Scales: bf16 [rows / 128][K / W4_GROUP][128].  rows and K multiples
// of 128.
constexpr int W4_GROUP = 128;
enum W4Mode { W4_RELU = 0, W4_SWIGLU = 1, W4_GATE = 2 };

struct W4Params {
  int G, N, K, m_tiles, num_kb, ksplit, kb_per;
  const uint8_t* Q0;                 // codes of W1 (or W2), tiled
  const uint8_t* Q1;                 // codes of W3 (SwiGLU)
  int64_t split_stride;              // W4_GATE: elements between K-range partials of the output
  const __nv_bfloat16* S0;           // scales of W1 (or W2)
  const __nv_bfloat16* S1;           // scales of W3 (SwiGLU)
  void* out;                         // first projection: hidden hi plane [S][N] bf16; second: Yp fp32
  void* out_lo;                      // first projection: hidden lo plane
  const int32_t* offsets;            // [G + 1] rows of each expert group in the sorted buffers
  const float* row_gate;             // [S] gate of each sorted row (second projection)
  unsigned int* err;
  uint64_t limit_ns;
};

struct W4Args {
  int mode, G, N, K;
  int64_t x_rows, max_group_rows;
  const void* Q0;  // codes of W1 (or W2) [G * N][K / 8]
  const void* Q1;  // codes of W3 (SwiGLU)
  const void* S0;
  const void* S1;
  const void* X;     // activation rows [x_rows][K] bf16 (sorted x, or the hidden hi plane)
  const void* X_lo;  // second projection: the hidden lo plane
  int ksplit;
  int64_t split_stride;
  void* out;
  void* out_lo;
  const int32_t* offsets;
  const float* row_gate;
  unsigned int* err;
};

struct W4Plan {
  CUtensorMap x;
  W4Params p;
  int mode, nb;
};

int w4_rows_per_tile(int64_t max_group_rows);
cudaError_t plan_w4_gemm(const W4Args& g, W4Plan* plan, const char** why);
cudaError_t launch_w4_gemm(const W4Plan& plan, int num_sms, cudaStream_t s);

// Few-row 4-bit products (register-fed warp MMAs) for batches of at most
// kW4SmallMaxT tokens (groups of more than 32 / 16 rows run as several
// units); they write fp32 partial rows per K range.
constexpr int kW4SmallMaxT = 64;

struct W4SmallParams {
  int G, N, K, m_tiles, row_blocks, num_g, gp, ksplit;  // gp: scale groups (128 elements) per K range
  int two_mats;                       // SwiGLU: W1 and W3 rows of one m-tile per unit
  int rows_cap;                       // activation rows of one group at most
  int stage_bytes, nstage;            // pipeline stages (codes, scales and activation columns)
  const uint8_t* Q0;
  const uint8_t* Q1;
  const __nv_bfloat16* S0;
  const __nv_bfloat16* S1;
  const __nv_bfloat16* X;     // activation rows [x_rows][K] (sorted x, or the hidden hi plane)
  const __nv_bfloat16* X_lo;  // second projection: the hidden lo plane
  float* out;                 // partials [ksplit][split_stride] of W1 x, or of gate * W2 h
  float* out3;                // partials of W3 x (SwiGLU)
  int64_t split_stride;
  const int32_t* offsets;
  const float* row_gate;      // second projection only
  unsigned int* err;
  uint64_t limit_ns;
};

struct W4SmallPlan {
  W4SmallParams p;
  int planes, nt;
};

struct W4SmallSplit {
  int row_blocks, gp, ksplit, rows_cap;
};

// Units and K ranges of a few-row product (mode W4Mode; x_rows activation
// rows in all; max_group_rows the rows of the largest group) spread over
// `ctas` CTAs.
W4SmallSplit w4_small_split(int mode, int G, int64_t x_rows, int64_t max_group_rows, int N, int K, int ctas);
cudaError_t plan_w4_small(const W4Args& g, int ctas, W4SmallPlan* plan, const char** why);
cudaError_t launch_w4_small(const W4SmallPlan& plan, int num_sms, cudaStream_t s);
// Hidden bf16 hi + lo planes [rows][N] from the first projection's partials
// (rows = *total_rows <= max_rows, read on the device).
cudaError_t launch_w4_hidden(int act, const float* P1, const float* P3, int ksplit, int64_t split_stride,
                             const int32_t* total_rows, int64_t max_rows, int N, void* H, void* H_lo, int num_sms,
                             cudaStream_t s);
cudaError_t launch_quantize_int4(const void* W, int64_t rows, int K, void* codes, void* scales, cudaStream_t s);

// Raise a kernel's dynamic shared memory limit, once per (kernel, device, size).
cudaError_t set_smem_limit_once(const void* kernel, int bytes);
cudaError_t launch_gemm_simt(const GemmArgs& g, int64_t s_max, cudaStream_t s);

cudaError_t launch_selftest_timeout(unsigned int* err, int64_t limit_ns, cudaStream_t s);

void count_launch();

// Launch `kernel` with programmatic dependent launch (the kernel calls
// pdl_wait() before it touches what the previous kernel of the stream
// wrote).  Every kernel of a forward pass except the first is launched so.
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<A&&>(args)...);
  count_launch();
  return e;
}

// Set the calling thread's moe_last_error() message.
void set_error_message(const char* msg);

}  // namespace moe

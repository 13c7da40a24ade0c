// C ABI of the MoE layer forward pass: handle, validation, workspace layout and
// the launch sequence router -> scan -> dispatch -> GEMM1 -> GEMM2 -> combine,
// all on the caller's stream with no host synchronisation.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <set>
#include <string>
#include <tuple>

#include "moe.h"
#include "common.cuh"
#include "internal.h"
#include "scan_dispatch.h"
#include "backward.h"

struct moe_layer {
  int E, k, d, d_ff, act, gate_mode, dtype;
  double capacity_factor;
  int hidden;    // MOE_HIDDEN_*
  int n_shared;  // shared experts every token visits (weights E .. E + n_shared - 1)
};

// Sticky device error word (one per device that loads the library).
__device__ unsigned int g_moe_error_word = 0;

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

thread_local std::string t_err;

int fail(int code, const std::string& msg) {
  t_err = msg;
  return code;
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int num_sms = 0;
  unsigned int* err = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device set-up, done once per device with that device current.
cudaError_t device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.err == nullptr) {
    e = cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_moe_error_word);
    if (e != cudaSuccess) return e;
    di.err = static_cast<unsigned int*>(p);
  }
  *out = &di;
  return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The second projection writes fp32 rows for the combine (k > 1, shared
// experts, or fp32 layers) instead of scattering bf16 rows straight into y.
// (A k = 1 layer keeps the scatter: splitting its K range would add a combine
// pass over y that costs more than the split saves.)
// The second projection splits its K range for at most this many tiles.
constexpr int kSplitMaxTiles = 4 * kSplitTargetCtas;

// (4-bit weights always go through the fp32 rows and the combine.)
bool need_yp_of(const moe_layer& L, bool w4) {
  return w4 || !(L.dtype == MOE_BF16 && L.k == 1 && L.n_shared == 0);
}

// K ranges of the 4-bit second projection: its tiles are (group, n-tile of
// at most NB rows, 128 output columns); cut K until about two waves of
// (tile, range) units cover the SMs.
int w4_ksplit(int64_t s, int groups, int d, int d_ff) {
  const int64_t nb = w4_rows_per_tile(s);
  const int64_t g = std::min<int64_t>(groups, s);
  const int64_t tiles = (g + (s - g) / nb) * ((d + 127) / 128);
  const int64_t num_kb = d_ff / 64;
  if (tiles <= 0 || tiles >= 4 * kSplitTargetCtas) return 1;
  // the cut whose longest CTA (ceil(units / SMs) ranges of `per` k-blocks) is
  // shortest; more ranges only for a gain above 3 % (each adds fp32 partial rows)
  int64_t best = 1, best_len = (tiles + kSplitTargetCtas - 1) / kSplitTargetCtas * num_kb;
  for (int64_t ks = 2; ks <= num_kb / 4; ++ks) {
    const int64_t per = (num_kb + ks - 1) / ks;
    const int64_t ranges = (num_kb + per - 1) / per;
    const int64_t len = (tiles * ranges + kSplitTargetCtas - 1) / kSplitTargetCtas * per;
    if (len * 32 < best_len * 31) { best = ranges; best_len = len; }
  }
  return static_cast<int>(best);
}

int ksplit_of(const moe_layer& L, int64_t s_max, bool w4) {
  if (w4) return w4_ksplit(s_max, L.E + L.n_shared, L.d, L.d_ff);
  return (L.dtype == MOE_BF16 && need_yp_of(L, false)) ? gemm2_ksplit(s_max, L.E + L.n_shared, L.d, L.d_ff) : 1;
}

// Yp rows a batch of s rows needs (0: none, the bf16 rows go straight into y).
int64_t yp_rows_of(const moe_layer& L, int64_t s, bool w4) {
  return need_yp_of(L, w4) ? ksplit_of(L, s, w4) * s : 0;
}

// The automatic hidden mode holds the hidden activation in fp16 when the
// batch averages at least this many rows per expert group: there the second
// projection is bound by the tensor cores, and one fp16 plane halves its MMAs
// against the hi + lo bf16 pair, which more than pays for the fp16 image of
// W2 (made while the first projection runs).  Smaller batches are bound by
// the weight stream, where the pair costs no time.
constexpr int64_t kAutoF16RowsPerGroup = 1024;

bool f16_hidden_of(const moe_layer& L, int64_t s_max) {
  if (L.dtype != MOE_BF16) return false;
  if (L.hidden == MOE_HIDDEN_F16) return true;
  return L.hidden == MOE_HIDDEN_AUTO && s_max >= kAutoF16RowsPerGroup * (L.E + L.n_shared);
}

int64_t capacity_of(const moe_layer& L, int64_t T) {
  if (!(L.capacity_factor > 0.0)) return -1;
  const double c = ceil(L.capacity_factor * static_cast<double>(T) * static_cast<double>(L.k) /
                        static_cast<double>(L.E));
  if (c > 2147483647.0) return 2147483647;
  return static_cast<int64_t>(c);
}

struct Layout {
  int64_t T, s_max, capacity;
  int nblk;
  bool need_yp;
  bool split;  // hidden activation as a hi + lo bf16 pair
  bool f16;    // hidden activation (and the second projection's operands) in fp16
  bool small;  // 4-bit weights, at most kW4SmallMaxT tokens: the few-row products
  int ksplit;
  int ks1;     // few-row products: K ranges of the first projection
  size_t idx, gate, dest, row_token, row_gate, part_hist, part_cnt1, part_psum, part_lse2, blockoff, counts,
      offsets, mprefix, scal, wsplit, rpart, spart, Xp, Hp, Hp_lo, Yp, W2h, P, total;
};

// Batches of 4-bit layers up to kW4SmallMaxT tokens take the few-row products.

int64_t s_max_of(const moe_layer& L, int64_t T) {
  const int64_t cap = capacity_of(L, T);
  int64_t s = T * L.k;
  if (cap >= 0) s = std::min<int64_t>(s, static_cast<int64_t>(L.E) * cap);
  return s + static_cast<int64_t>(L.n_shared) * T;
}

// The K ranges of both few-row products for a batch of T tokens.
struct SmallSplits {
  W4SmallSplit g1, g2;
  int64_t s_max;
};

SmallSplits small_splits_of(const moe_layer& L, int64_t T) {
  SmallSplits r;
  r.s_max = s_max_of(L, T);
  const int G = L.E + L.n_shared;
  const int mode1 = L.act == MOE_ACT_SWIGLU ? W4_SWIGLU : W4_RELU;
  r.g1 = w4_small_split(mode1, G, r.s_max, T, L.d_ff, L.d, kSplitTargetCtas);
  r.g2 = w4_small_split(W4_GATE, G, r.s_max, T, L.d, L.d_ff, kSplitTargetCtas);
  return r;
}

// w4: the layout of moe_forward_w4 (4-bit weights: hidden as a hi + lo pair,
// fp32 rows for the combine, no fp16 image of W2).
Layout make_layout(const moe_layer& L, int64_t T, bool w4 = false) {
  Layout w;
  w.T = T;
  w.capacity = capacity_of(L, T);
  const int64_t Tk = T * L.k;
  w.s_max = Tk;
  if (w.capacity >= 0) w.s_max = std::min<int64_t>(Tk, static_cast<int64_t>(L.E) * w.capacity);
  w.s_max += static_cast<int64_t>(L.n_shared) * T;  // every token's rows of the shared experts
  w.nblk = static_cast<int>((T + kRouterTokens - 1) / kRouterTokens);
  const size_t elt = L.dtype == MOE_BF16 ? 2 : 4;
  w.f16 = !w4 && f16_hidden_of(L, w.s_max);
  w.split = L.dtype == MOE_BF16 &&
            (w4 || (!w.f16 && (L.hidden == MOE_HIDDEN_BF16X2 || L.hidden == MOE_HIDDEN_AUTO)));
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  w.idx = take(sizeof(int32_t) * Tk);
  w.gate = take(sizeof(float) * Tk);
  w.dest = take(sizeof(int32_t) * Tk);
  w.row_token = take(sizeof(int32_t) * w.s_max);
  w.row_gate = take(sizeof(float) * w.s_max);
  w.part_hist = take(sizeof(int32_t) * L.E * static_cast<size_t>(w.nblk));
  w.part_cnt1 = take(sizeof(int32_t) * L.E * static_cast<size_t>(w.nblk));
  w.part_psum = take(sizeof(float) * L.E * static_cast<size_t>(w.nblk));
  w.part_lse2 = take(sizeof(float) * w.nblk);
  w.blockoff = take(sizeof(int32_t) * L.E * static_cast<size_t>(w.nblk));
  w.counts = take(sizeof(int32_t) * L.E);
  // [groups + 1]: the routed experts' groups, then one per shared expert
  w.offsets = take(sizeof(int32_t) * (L.E + L.n_shared + 1));
  w.mprefix = take(sizeof(int32_t) * (L.E + L.n_shared + 1));
  // scan totals [E] + [E], 16 spare bytes, the three balance statistics
  w.scal = take(sizeof(int32_t) * L.E + sizeof(float) * L.E + 64);
  const bool tc_router = L.dtype == MOE_BF16 && L.E <= kRouterTcMaxE;
  w.wsplit = take(tc_router ? 3 * sizeof(uint16_t) * router_pad_e(L.E) * static_cast<size_t>(L.d) : 0);
  w.rpart = take(tc_router ? router_partials_bytes(T, L.E, L.d) : 0);
  w.spart = take(route_small_partials_bytes(L.E));  // batches of <= 32 tokens (constant: sizes stay monotone)
  w.Xp = take(elt * static_cast<size_t>(w.s_max) * L.d);
  w.Hp = take(elt * static_cast<size_t>(w.s_max) * L.d_ff);
  // The automatic mode keeps the lo plane's room once it switches to fp16
  // (the largest pair any smaller batch uses), so sizes never shrink as T grows.
  int64_t lo_rows = w.split ? w.s_max : 0;
  if (!w4 && L.dtype == MOE_BF16 && L.hidden == MOE_HIDDEN_AUTO && w.f16)
    lo_rows = kAutoF16RowsPerGroup * (L.E + L.n_shared) - 1;
  w.Hp_lo = take(elt * static_cast<size_t>(lo_rows) * L.d_ff);
  w.ksplit = ksplit_of(L, w.s_max, w4);
  w.need_yp = need_yp_of(L, w4);
  // Yp holds ksplit partials of s_max rows; reserve the most any smaller batch
  // needs as well, so a workspace sized for some T serves every smaller batch.
  // ksplit(s) depends on s through the m-tile bound min(G, s) + floor((s - min(G, s)) / 128)
  // (G groups), which changes at every s up to G and then every 128 rows, and
  // ksplit(s) = 1 once the bound reaches kSplitMaxTiles; the product ksplit(s) * s
  // peaks at the last s before each change.
  int64_t yp_rows = yp_rows_of(L, w.s_max, w4);
  const int64_t groups = L.E + L.n_shared;
  for (int64_t s = 1; s < w.s_max && s <= groups; ++s) yp_rows = std::max<int64_t>(yp_rows, yp_rows_of(L, s, w4));
  for (int64_t s = groups + 127; s < w.s_max && s <= groups + int64_t{kSplitMaxTiles} * 128; s += 128)
    yp_rows = std::max<int64_t>(yp_rows, yp_rows_of(L, s, w4));
  if (w4) {  // the 4-bit split also changes at every 16 / 32 / 64 rows (n-tile sizes) up to two waves of tiles
    for (int64_t s = groups + 1; s < w.s_max && s <= groups + int64_t{2 * kSplitTargetCtas} * 64; ++s)
      yp_rows = std::max<int64_t>(yp_rows, yp_rows_of(L, s, w4));
  }
  // fp16 image of W2 (every expert, shared ones included) for the fp16 mode
  w.W2h = take(w.f16 ? sizeof(uint16_t) * static_cast<size_t>(L.E + L.n_shared) * L.d * L.d_ff : 0);
  // Few-row products: fp32 partials of the first projection [nq][ks1][s_max][d_ff],
  // and the second projection's partials in Yp; sized for every batch up to
  // kW4SmallMaxT tokens, so sizes stay monotone in T.
  w.small = w4 && T <= kW4SmallMaxT;
  w.ks1 = 1;
  size_t p_bytes = 0;
  if (w4) {
    const size_t nq = L.act == MOE_ACT_SWIGLU ? 2 : 1;
    for (int64_t t = 1; t <= std::min<int64_t>(T, kW4SmallMaxT); ++t) {
      const SmallSplits sp = small_splits_of(L, t);
      p_bytes = std::max(p_bytes, nq * sizeof(float) * static_cast<size_t>(sp.g1.ksplit) *
                                      static_cast<size_t>(sp.s_max) * L.d_ff);
      yp_rows = std::max<int64_t>(yp_rows, static_cast<int64_t>(sp.g2.ksplit) * sp.s_max);
    }
    if (w.small) {
      const SmallSplits sp = small_splits_of(L, T);
      w.ks1 = sp.g1.ksplit;
      w.ksplit = sp.g2.ksplit;
    }
  }
  w.Yp = take(yp_rows > 0 ? sizeof(float) * static_cast<size_t>(yp_rows) * L.d : 0);
  w.P = take(p_bytes);
  w.total = o;
  return w;
}

// Scratch of the backward pass: fp32 A1, U [S][d_ff] (and A3 for SwiGLU),
// dg [S], dXp [S][d], dh [T][E], cnt1 [E]; for bf16 layers (tensor-core
// products) also gate 1 [S], bf16 dy rows [S][d], the transposed weights
// [G][d][d_ff] / [G][d_ff][d], the hi + lo planes of da1 (and da3)
// [2][S][d_ff], and a second dXp part for SwiGLU.
struct BwLayout {
  size_t A1, A3, U, dg, dXp, dh, cnt1, ones, dYs, W1t, W3t, W2t, dA1p, dA3p, P1, P3, PH, XT, DT, woff, wpre, woff_d, wpre_d,
      wr_part, total;
  // the forward's router kernel run again for its logits (bf16, E <= kRouterTcMaxE)
  bool rt;
  size_t rt_idx, rt_gate, rt_hist, rt_cnt1, rt_psum, rt_lse2, rt_logits, rt_wsplit, rt_rpart;
  int max_group_rows, k_pad, wr_chunks;
};

// No group has more rows: a token takes an expert at most once, and a shared
// expert's group has T rows.
int64_t max_group_rows_of(const moe_layer& L, const Layout& w) {
  int64_t mg = w.T;
  if (L.n_shared == 0 && w.capacity >= 0 && w.capacity < mg) mg = w.capacity;
  return mg;
}

BwLayout make_bw_layout(const moe_layer& L, const Layout& w) {
  BwLayout b;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  const bool swiglu = L.act == MOE_ACT_SWIGLU, tc = L.dtype == MOE_BF16;
  const size_t S = static_cast<size_t>(w.s_max), G = static_cast<size_t>(L.E + L.n_shared);
  const size_t hid = sizeof(float) * S * L.d_ff;
  b.A1 = take(hid);
  b.A3 = take(swiglu ? hid : 0);
  b.U = take(hid);
  b.dg = take(sizeof(float) * S);
  b.dXp = take(sizeof(float) * S * L.d * (tc && swiglu ? 2 : 1));
  b.dh = take(sizeof(float) * static_cast<size_t>(w.T) * L.E);
  b.cnt1 = take(sizeof(int32_t) * L.E);
  const size_t wsz = tc ? 2 * G * L.d * static_cast<size_t>(L.d_ff) : 0;
  b.max_group_rows = static_cast<int>(max_group_rows_of(L, w));
  b.k_pad = (b.max_group_rows + 7) / 8 * 8;
  const size_t kp = static_cast<size_t>(b.k_pad);
  // gate 1 for every row of the products: the sorted rows, and G groups of d_ff or d rows
  b.ones = take(tc ? sizeof(float) * std::max(S, G * static_cast<size_t>(std::max(L.d_ff, L.d))) : 0);
  b.dYs = take(tc ? 2 * S * L.d : 0);
  b.W1t = take(wsz);
  b.W3t = take(swiglu ? wsz : 0);
  b.W2t = take(wsz);
  b.dA1p = take(tc ? 2 * 2 * S * L.d_ff : 0);
  b.dA3p = take(tc && swiglu ? 2 * 2 * S * L.d_ff : 0);
  // the weight gradients' per-expert operands (rows zero-padded to k_pad)
  const size_t plane2 = tc ? 2 * 2 * G * L.d_ff * kp : 0;
  b.P1 = take(plane2);
  b.P3 = take(swiglu ? plane2 : 0);
  b.PH = take(plane2);
  b.XT = take(tc ? 2 * G * L.d * kp : 0);
  b.DT = take(tc ? 2 * G * L.d * kp : 0);
  b.woff = take(tc ? sizeof(int32_t) * (G + 1) : 0);
  b.wpre = take(tc ? sizeof(int32_t) * (G + 1) : 0);
  b.woff_d = take(tc ? sizeof(int32_t) * (G + 1) : 0);
  b.wpre_d = take(tc ? sizeof(int32_t) * (G + 1) : 0);
  // dW_r's partials: chunks of at least 256 tokens, at most 64 of them
  const int64_t ch = (w.T + 255) / 256;
  b.wr_chunks = static_cast<int>(ch < 1 ? 1 : (ch > 64 ? 64 : ch));
  b.wr_part = take(sizeof(float) * b.wr_chunks * static_cast<size_t>(L.E) * L.d);
  b.rt = tc && L.E <= kRouterTcMaxE;
  const size_t Tk = static_cast<size_t>(w.T) * L.k, EB = static_cast<size_t>(L.E) * w.nblk;
  b.rt_idx = take(b.rt ? sizeof(int32_t) * Tk : 0);
  b.rt_gate = take(b.rt ? sizeof(float) * Tk : 0);
  b.rt_hist = take(b.rt ? sizeof(int32_t) * EB : 0);
  b.rt_cnt1 = take(b.rt ? sizeof(int32_t) * EB : 0);
  b.rt_psum = take(b.rt ? sizeof(float) * EB : 0);
  b.rt_lse2 = take(b.rt ? sizeof(float) * w.nblk : 0);
  b.rt_logits = take(b.rt ? sizeof(float) * static_cast<size_t>(w.T) * L.E : 0);
  b.rt_wsplit = take(b.rt ? 3 * sizeof(uint16_t) * router_pad_e(L.E) * static_cast<size_t>(L.d) : 0);
  b.rt_rpart = take(b.rt ? router_partials_bytes(w.T, L.E, L.d) : 0);
  b.total = o;
  return b;
}

void record(const moe_debug* dbg, int stage, int which, cudaStream_t s) {
  if (dbg == nullptr) return;
  void* ev = dbg->events[2 * stage + which];
  if (ev != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(ev), s);
}

}  // namespace

void set_error_message(const char* msg) { t_err = msg; }

int gemm2_ksplit(int64_t s_max, int E, int d, int d_ff) {
  // Most m-tiles the second projection can have: a group of c rows takes
  // 1 + floor((c - 1) / 128) tiles, so S rows over at most min(E, S) groups
  // take at most min(E, S) + floor((S - min(E, S)) / 128).
  const int64_t g = std::min<int64_t>(E, s_max);
  const int64_t mtiles = g + (s_max - g) / kTileM;
  const int64_t base = mtiles * ((d + 255) / 256);
  if (base <= 0 || base > kSplitMaxTiles) return 1;
  // A few waves of tiles or less: cut K into ranges so that the last wave
  // fills the SMs.  Each persistent CTA takes every num_sms-th (tile, range)
  // unit, so the longest CTA runs ceil(units / num_sms) ranges of `per`
  // k-blocks; take the cut that shortens it, a cut with more ranges only when
  // it saves over 3 % (each range adds an fp32 partial of the tile's rows).
  const int64_t num_kb = (d_ff + 63) / 64;
  int64_t best = 1, best_len = (base + kSplitTargetCtas - 1) / kSplitTargetCtas * num_kb;
  for (int64_t ks = 2; ks <= num_kb / 4; ++ks) {
    const int64_t per = (num_kb + ks - 1) / ks;
    const int64_t ranges = (num_kb + per - 1) / per;  // no empty K range
    const int64_t len = (base * ranges + kSplitTargetCtas - 1) / kSplitTargetCtas * per;
    if (len * 32 < best_len * 31) { best = ranges; best_len = len; }
  }
  return static_cast<int>(best);
}

cudaError_t set_smem_limit_once(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::tuple<const void*, int, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_tuple(kernel, dev, bytes);
  std::lock_guard<std::mutex> lk(mu);
  if (done.count(key)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_create(int num_experts, int k, int d, int d_ff, int act, int gate_mode, double capacity_factor, int dtype,
               moe_handle* out) {
  if (out == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_create: out is NULL");
  if (num_experts < 1 || num_experts > 256) return fail(MOE_ERR_INVALID_ARG, "moe_create: num_experts must be in [1, 256]");
  if (k < 1 || k > num_experts || k > 8) return fail(MOE_ERR_INVALID_ARG, "moe_create: need 1 <= k <= min(E, 8)");
  if (d < 1 || d_ff < 1) return fail(MOE_ERR_INVALID_ARG, "moe_create: d and d_ff must be positive");
  if (act != MOE_ACT_RELU && act != MOE_ACT_SWIGLU) return fail(MOE_ERR_INVALID_ARG, "moe_create: unknown act");
  if (gate_mode != MOE_GATE_SWITCH && gate_mode != MOE_GATE_RENORM)
    return fail(MOE_ERR_INVALID_ARG, "moe_create: unknown gate_mode");
  if (dtype != MOE_F32 && dtype != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "moe_create: unknown dtype");
  if (!(capacity_factor == capacity_factor)) return fail(MOE_ERR_INVALID_ARG, "moe_create: capacity_factor is NaN");
  if (dtype == MOE_BF16 && (d % 8 != 0 || d_ff % 8 != 0))
    return fail(MOE_ERR_UNSUPPORTED, "moe_create: bf16 layers need d and d_ff to be multiples of 8");
  moe_layer* L =
      new moe_layer{num_experts, k, d, d_ff, act, gate_mode, dtype, capacity_factor, MOE_HIDDEN_AUTO, 0};
  *out = L;
  t_err.clear();
  return MOE_OK;
}

int moe_set_hidden_precision(moe_handle h, int mode) {
  if (h == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_set_hidden_precision: handle is NULL");
  if (mode != MOE_HIDDEN_BF16X2 && mode != MOE_HIDDEN_BF16 && mode != MOE_HIDDEN_F16 && mode != MOE_HIDDEN_AUTO)
    return fail(MOE_ERR_INVALID_ARG, "moe_set_hidden_precision: unknown mode");
  h->hidden = mode;
  return MOE_OK;
}

int moe_set_shared_experts(moe_handle h, int n_shared) {
  if (h == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_set_shared_experts: handle is NULL");
  if (n_shared < 0 || n_shared > 8 || h->E + n_shared > 256)
    return fail(MOE_ERR_INVALID_ARG, "moe_set_shared_experts: need 0 <= n_shared <= 8 and E + n_shared <= 256");
  h->n_shared = n_shared;
  return MOE_OK;
}

int moe_balance_losses(moe_handle h, int64_t T, const void* workspace, float* out, void* stream) {
  if (h == nullptr || T < 0 || out == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_balance_losses: NULL handle or output, or T < 0");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (T == 0) {
    e = cudaMemsetAsync(out, 0, 3 * sizeof(float), s);
  } else {
    if (workspace == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_balance_losses: workspace is NULL");
    const Layout w = make_layout(*h, T);
    const uint8_t* src = static_cast<const uint8_t*>(workspace) + w.scal +
                         (sizeof(int32_t) + sizeof(float)) * h->E + 16;
    e = cudaMemcpyAsync(out, src, 3 * sizeof(float), cudaMemcpyDeviceToDevice, s);
  }
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_balance_losses: ") + cudaGetErrorString(e));
  t_err.clear();
  return MOE_OK;
}

int moe_destroy(moe_handle h) {
  delete h;
  return MOE_OK;
}

int64_t moe_capacity(moe_handle h, int64_t T) {
  if (h == nullptr || T < 0) return -1;
  return capacity_of(*h, T);
}

size_t moe_workspace_bytes(moe_handle h, int64_t T) {
  if (h == nullptr || T < 0) return 0;
  return make_layout(*h, T).total;
}

}  // extern "C"

namespace {

// The expert weights of one forward call: bf16 / fp32 tensors, or 4-bit codes
// with their scales (moe_forward_w4).
struct ExpertWeights {
  bool w4;
  const void *W1, *W3, *W2;   // bf16 / fp32
  const void *Q1, *Q3, *Q2;   // 4-bit codes
  const void *S1, *S3, *S2;   // their scales
};

int forward_impl(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r, const ExpertWeights& ew,
                 void* y, int32_t* expert_counts, int32_t* dropped, float* aux_loss, float* z_loss, void* workspace,
                 size_t workspace_bytes, const moe_debug* dbg, void* stream, const char* fn) {
  const std::string F = std::string(fn) + ": ";
  if (h == nullptr) return fail(MOE_ERR_INVALID_ARG, F + "handle is NULL");
  const moe_layer& L = *h;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, F + "T < 0");
  if (T * L.k > 2147483647LL / 2) return fail(MOE_ERR_UNSUPPORTED, F + "T * k too large");
  if (T * static_cast<int64_t>(L.d) >= 4294967296LL) return fail(MOE_ERR_UNSUPPORTED, F + "T * d too large");
  if (expert_counts == nullptr || dropped == nullptr || aux_loss == nullptr || z_loss == nullptr)
    return fail(MOE_ERR_INVALID_ARG, F + "a statistics output pointer is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * L.E, s) != cudaSuccess ||
        cudaMemsetAsync(dropped, 0, sizeof(int32_t), s) != cudaSuccess ||
        cudaMemsetAsync(aux_loss, 0, sizeof(float), s) != cudaSuccess ||
        cudaMemsetAsync(z_loss, 0, sizeof(float), s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, std::string(F + "") + cudaGetErrorString(cudaGetLastError()));
    t_err.clear();
    return MOE_OK;
  }
  const void* W1 = ew.w4 ? ew.Q1 : ew.W1;
  const void* W3 = ew.w4 ? ew.Q3 : ew.W3;
  const void* W2 = ew.w4 ? ew.Q2 : ew.W2;
  if (x == nullptr || W_r == nullptr || W1 == nullptr || W2 == nullptr || y == nullptr)
    return fail(MOE_ERR_INVALID_ARG, F + "x, W_r, W1, W2 and y must be non-NULL");
  if ((L.act == MOE_ACT_SWIGLU) != (W3 != nullptr))
    return fail(MOE_ERR_INVALID_ARG, F + "W3 must be given for SwiGLU and NULL for ReLU");
  if (ew.w4) {
    if (ew.S1 == nullptr || ew.S2 == nullptr || (W3 != nullptr && ew.S3 == nullptr))
      return fail(MOE_ERR_INVALID_ARG, F + "every 4-bit weight needs its scales");
    if (L.dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, F + "4-bit weights serve bf16 layers only");
    if (L.d % W4_GROUP != 0 || L.d_ff % W4_GROUP != 0)
      return fail(MOE_ERR_UNSUPPORTED, F + "4-bit weights need d and d_ff to be multiples of 128");
    const uintptr_t sal = reinterpret_cast<uintptr_t>(ew.S1) | reinterpret_cast<uintptr_t>(ew.S2) |
                          reinterpret_cast<uintptr_t>(ew.S3);
    if ((sal & 15) != 0) return fail(MOE_ERR_INVALID_ARG, F + "scales must be 16-byte aligned");
  }
  const Layout w = make_layout(L, T, ew.w4);
  if (workspace == nullptr || workspace_bytes < w.total)
    return fail(MOE_ERR_INVALID_ARG, F + "workspace missing or smaller than moe_workspace_bytes()");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return fail(MOE_ERR_INVALID_ARG, F + "workspace must be 256-byte aligned");
  const uintptr_t al = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y) |
                       reinterpret_cast<uintptr_t>(W1) | reinterpret_cast<uintptr_t>(W2) |
                       reinterpret_cast<uintptr_t>(W3);
  if ((al & 15) != 0) return fail(MOE_ERR_INVALID_ARG, F + "x, y and weights must be 16-byte aligned");
  if (L.dtype == MOE_F32 && (w.s_max + 7) / 8 > 65535)
    return fail(MOE_ERR_UNSUPPORTED, F + "fp32 layers are limited to 524280 assignments");

  DeviceInfo* di = nullptr;
  cudaError_t ce = device_info(&di);
  if (ce != cudaSuccess) return fail(MOE_ERR_CUDA, std::string(F + "") + cudaGetErrorString(ce));

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  RoutingArgs r;
  memset(&r, 0, sizeof(r));
  r.T = T;
  r.E = L.E;
  r.k = L.k;
  r.d = L.d;
  r.gate_mode = L.gate_mode;
  r.capacity = w.capacity;
  r.nblk = w.nblk;
  r.x_is_bf16 = L.dtype == MOE_BF16;
  r.x = x;
  r.W_r = W_r;
  r.b_r = b_r;
  r.logits_in = dbg ? dbg->logits_in : nullptr;
  r.topk_idx = reinterpret_cast<int32_t*>(ws + w.idx);
  r.topk_gate = reinterpret_cast<float*>(ws + w.gate);
  r.dest_row = reinterpret_cast<int32_t*>(ws + w.dest);
  r.part_hist = reinterpret_cast<int32_t*>(ws + w.part_hist);
  r.part_cnt1 = reinterpret_cast<int32_t*>(ws + w.part_cnt1);
  r.part_psum = reinterpret_cast<float*>(ws + w.part_psum);
  r.part_lse2 = reinterpret_cast<float*>(ws + w.part_lse2);
  r.blockoff = reinterpret_cast<int32_t*>(ws + w.blockoff);
  r.counts = expert_counts;
  r.offsets = reinterpret_cast<int32_t*>(ws + w.offsets);
  r.mprefix = reinterpret_cast<int32_t*>(ws + w.mprefix);
  r.row_token = reinterpret_cast<int32_t*>(ws + w.row_token);
  r.tot_cnt1 = reinterpret_cast<int32_t*>(ws + w.scal);
  r.tot_psum = reinterpret_cast<float*>(ws + w.scal + sizeof(int32_t) * L.E);
  r.balance_out = reinterpret_cast<float*>(ws + w.scal + (sizeof(int32_t) + sizeof(float)) * L.E + 16);
  r.n_shared = L.n_shared;
  r.row_gate = reinterpret_cast<float*>(ws + w.row_gate);
  r.Xp = ws + w.Xp;
  r.dropped = dropped;
  r.aux = aux_loss;
  r.z = z_loss;
  r.logits_out = dbg ? dbg->logits_out : nullptr;
  r.lse_out = dbg ? dbg->lse_out : nullptr;
  r.drop_mask = dbg ? dbg->drop_mask : nullptr;
  r.offsets_out = dbg ? dbg->expert_offsets : nullptr;
  r.y_zero_dropped = w.need_yp ? nullptr : y;
  r.yf_zero_dropped = (w.need_yp || dbg == nullptr) ? nullptr : dbg->y_f32;

  GemmArgs g1;
  memset(&g1, 0, sizeof(g1));
  g1.epi = L.act == MOE_ACT_SWIGLU ? EPI_SWIGLU_BF16 : EPI_RELU_BF16;
  g1.E = L.E + L.n_shared;  // routed groups, then one group of T rows per shared expert
  g1.N = L.d_ff;
  g1.K = L.d;
  g1.a_rows = w.s_max;
  g1.max_group_rows = T;  // a token takes each expert at most once; a shared expert's group has T rows
  g1.A = ws + w.Xp;
  g1.B0 = W1;
  g1.B1 = W3;
  g1.out = ws + w.Hp;
  g1.split = w.split;
  g1.f16 = w.f16;
  g1.out2 = w.split ? static_cast<void*>(ws + w.Hp_lo) : nullptr;
  g1.offsets = r.offsets;
  g1.mprefix = r.mprefix;
  g1.row_gate = r.row_gate;
  g1.row_token = r.row_token;
  g1.err = di->err;

  GemmArgs g2 = g1;
  g2.epi = w.need_yp ? EPI_GATE_F32 : EPI_GATE_SCATTER_BF16;
  g2.N = L.d;
  g2.K = L.d_ff;
  g2.A = ws + w.Hp;
  g2.A2 = w.split ? static_cast<const void*>(ws + w.Hp_lo) : nullptr;
  g2.out2 = nullptr;
  g2.B0 = w.f16 ? static_cast<const void*>(ws + w.W2h) : W2;
  g2.B1 = nullptr;
  g2.out = w.need_yp ? static_cast<void*>(ws + w.Yp) : y;
  g2.out_f32 = (w.need_yp || dbg == nullptr) ? nullptr : dbg->y_f32;
  g2.ksplit = w.ksplit;
  g2.split_stride = static_cast<int64_t>(w.s_max) * L.d;
  g1.ksplit = 1;

  // Host-side preparation of both GEMM launches happens before the first launch.
  TcGemmPlan plan1, plan2;
  W4Plan wplan1, wplan2;
  W4SmallPlan splan1, splan2;
  if (ew.w4) {
    W4Args a1;
    memset(&a1, 0, sizeof(a1));
    a1.mode = L.act == MOE_ACT_SWIGLU ? W4_SWIGLU : W4_RELU;
    a1.G = L.E + L.n_shared;
    a1.N = L.d_ff;
    a1.K = L.d;
    a1.x_rows = w.s_max;
    a1.max_group_rows = T;
    a1.Q0 = ew.Q1;
    a1.Q1 = ew.Q3;
    a1.S0 = ew.S1;
    a1.S1 = ew.S3;
    a1.X = ws + w.Xp;
    a1.out = ws + w.Hp;
    a1.out_lo = ws + w.Hp_lo;
    a1.offsets = r.offsets;
    a1.row_gate = r.row_gate;
    a1.err = di->err;
    W4Args a2 = a1;
    a2.mode = W4_GATE;
    a2.N = L.d;
    a2.K = L.d_ff;
    a2.Q0 = ew.Q2;
    a2.Q1 = nullptr;
    a2.S0 = ew.S2;
    a2.S1 = nullptr;
    a2.X = ws + w.Hp;
    a2.X_lo = ws + w.Hp_lo;
    a2.out = ws + w.Yp;
    a2.out_lo = nullptr;
    a2.ksplit = w.ksplit;
    a2.split_stride = static_cast<int64_t>(w.s_max) * L.d;
    const char* why = nullptr;
    if (w.small) {
      // few-row products: fp32 partials of W1 x (and W3 x), then the hidden
      // planes, then gated partials of W2 h in Yp
      const size_t p1 = static_cast<size_t>(w.ks1) * static_cast<size_t>(w.s_max) * L.d_ff;
      a1.out = ws + w.P;
      a1.out_lo = reinterpret_cast<float*>(ws + w.P) + p1;
      a1.split_stride = static_cast<int64_t>(w.s_max) * L.d_ff;
      if (plan_w4_small(a1, kSplitTargetCtas, &splan1, &why) != cudaSuccess ||
          plan_w4_small(a2, kSplitTargetCtas, &splan2, &why) != cudaSuccess)
        return fail(MOE_ERR_UNSUPPORTED, F + (why ? why : "4-bit few-row plan failed"));
      if (splan1.p.ksplit != w.ks1 || splan2.p.ksplit != w.ksplit)
        return fail(MOE_ERR_UNSUPPORTED, F + "4-bit few-row plan disagrees with the workspace layout");
    } else if (plan_w4_gemm(a1, &wplan1, &why) != cudaSuccess || plan_w4_gemm(a2, &wplan2, &why) != cudaSuccess) {
      return fail(MOE_ERR_UNSUPPORTED, F + (why ? why : "4-bit GEMM plan failed"));
    }
  } else if (L.dtype == MOE_BF16) {
    const char* why = nullptr;
    if (plan_gemm_tc(g1, &plan1, &why) != cudaSuccess || plan_gemm_tc(g2, &plan2, &why) != cudaSuccess)
      return fail(MOE_ERR_UNSUPPORTED, std::string(F + "") + (why ? why : "GEMM plan failed"));
  }

  const bool tc = L.dtype == MOE_BF16 && !ew.w4;  // bf16 expert products on the tensor-core grouped GEMM
  const bool tc_router = L.dtype == MOE_BF16;     // every bf16 layer routes on the tensor cores (E <= 128)
  auto check = [&](cudaError_t e, const char* what) -> int {
    if (e == cudaSuccess) return MOE_OK;
    return fail(MOE_ERR_CUDA, std::string(F + "") + what + ": " + cudaGetErrorString(e));
  };
  int rc;
  record(dbg, MOE_STAGE_ROUTER, 0, s);
  if (T <= kRouteSmallMaxT) {
    // one router block: router, scan and dispatch in two launches (the scan
    // and dispatch stages of the debug events stay empty)
    if ((rc = check(launch_route_small(r, ws + w.spart, s), "router")) != MOE_OK) return rc;
    record(dbg, MOE_STAGE_ROUTER, 1, s);
    record(dbg, MOE_STAGE_SCAN, 0, s);
    record(dbg, MOE_STAGE_SCAN, 1, s);
    record(dbg, MOE_STAGE_DISPATCH, 0, s);
    record(dbg, MOE_STAGE_DISPATCH, 1, s);
  } else {
    if (tc_router && L.E <= kRouterTcMaxE && r.logits_in == nullptr) {
      const char* why = nullptr;
      ce = launch_router_tc(r, ws + w.wsplit, ws + w.rpart, di->num_sms, di->err, s, &why);
      if (why != nullptr) return fail(MOE_ERR_UNSUPPORTED, std::string(F + "") + why);
      if ((rc = check(ce, "router")) != MOE_OK) return rc;
    } else if ((rc = check(launch_router(r, s), "router")) != MOE_OK) {
      return rc;
    }
    record(dbg, MOE_STAGE_ROUTER, 1, s);
    if (scan_dispatch_fits(r)) {  // one launch (the scan stage of the debug events stays empty)
      record(dbg, MOE_STAGE_SCAN, 0, s);
      record(dbg, MOE_STAGE_SCAN, 1, s);
      record(dbg, MOE_STAGE_DISPATCH, 0, s);
      if ((rc = check(launch_scan_dispatch(r, s), "dispatch")) != MOE_OK) return rc;
      record(dbg, MOE_STAGE_DISPATCH, 1, s);
    } else {
      record(dbg, MOE_STAGE_SCAN, 0, s);
      if ((rc = check(launch_scan(r, s), "scan")) != MOE_OK) return rc;
      record(dbg, MOE_STAGE_SCAN, 1, s);
      record(dbg, MOE_STAGE_DISPATCH, 0, s);
      if ((rc = check(launch_dispatch(r, s), "dispatch")) != MOE_OK) return rc;
      record(dbg, MOE_STAGE_DISPATCH, 1, s);
    }
  }

  record(dbg, MOE_STAGE_GEMM1, 0, s);
  if (w.small) {
    ce = launch_w4_small(splan1, di->num_sms, s);
    if ((rc = check(ce, "gemm1")) != MOE_OK) return rc;
    const float* P1 = reinterpret_cast<const float*>(ws + w.P);
    ce = launch_w4_hidden(L.act, P1, P1 + static_cast<size_t>(w.ks1) * static_cast<size_t>(w.s_max) * L.d_ff, w.ks1,
                          static_cast<int64_t>(w.s_max) * L.d_ff, r.offsets + (L.E + L.n_shared), w.s_max, L.d_ff,
                          ws + w.Hp, ws + w.Hp_lo, di->num_sms, s);
  } else {
    ce = ew.w4 ? launch_w4_gemm(wplan1, di->num_sms, s)
               : tc ? launch_gemm_tc(plan1, di->num_sms, s) : launch_gemm_simt(g1, w.s_max, s);
  }
  if ((rc = check(ce, "gemm1")) != MOE_OK) return rc;
  if (w.f16) {  // the fp16 image of W2, made while the first projection runs
    ce = launch_convert_f16(W2, ws + w.W2h, static_cast<int64_t>(L.E + L.n_shared) * L.d * L.d_ff, di->err,
                            di->num_sms, s);
    if ((rc = check(ce, "fp16 image of W2")) != MOE_OK) return rc;
  }
  record(dbg, MOE_STAGE_GEMM1, 1, s);
  record(dbg, MOE_STAGE_GEMM2, 0, s);
  ce = w.small ? launch_w4_small(splan2, di->num_sms, s)
       : ew.w4  ? launch_w4_gemm(wplan2, di->num_sms, s)
       : tc     ? launch_gemm_tc(plan2, di->num_sms, s)
                : launch_gemm_simt(g2, w.s_max, s);
  if ((rc = check(ce, "gemm2")) != MOE_OK) return rc;
  record(dbg, MOE_STAGE_GEMM2, 1, s);
  if (w.need_yp) {
    record(dbg, MOE_STAGE_COMBINE, 0, s);
    if ((rc = check(launch_combine(T, L.k, L.d, L.dtype == MOE_BF16, r.dest_row, L.n_shared, r.offsets + L.E,
                                   reinterpret_cast<const float*>(ws + w.Yp), w.ksplit,
                                   static_cast<int64_t>(w.s_max) * L.d, y, dbg ? dbg->y_f32 : nullptr, s),
                    "combine")) != MOE_OK)
      return rc;
    record(dbg, MOE_STAGE_COMBINE, 1, s);
  }
  if (dbg != nullptr) {
    const size_t tk = static_cast<size_t>(T) * L.k;
    if (dbg->topk_idx && cudaMemcpyAsync(dbg->topk_idx, r.topk_idx, 4 * tk, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, F + "debug copy failed");
    if (dbg->topk_gate && cudaMemcpyAsync(dbg->topk_gate, r.topk_gate, 4 * tk, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, F + "debug copy failed");
    if (dbg->dest_row && cudaMemcpyAsync(dbg->dest_row, r.dest_row, 4 * tk, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, F + "debug copy failed");
  }
  t_err.clear();
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_forward(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r, const void* W1,
                const void* W3, const void* W2, void* y, int32_t* expert_counts, int32_t* dropped, float* aux_loss,
                float* z_loss, void* workspace, size_t workspace_bytes, const moe_debug* dbg, void* stream) {
  ExpertWeights ew;
  memset(&ew, 0, sizeof(ew));
  ew.W1 = W1;
  ew.W3 = W3;
  ew.W2 = W2;
  return forward_impl(h, T, x, W_r, b_r, ew, y, expert_counts, dropped, aux_loss, z_loss, workspace,
                      workspace_bytes, dbg, stream, "moe_forward");
}

size_t moe_workspace_bytes_w4(moe_handle h, int64_t T) {
  if (h == nullptr || T < 0) return 0;
  return make_layout(*h, T, true).total;
}

int moe_forward_w4(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r,
                   const uint32_t* W1_codes, const void* W1_scales, const uint32_t* W3_codes, const void* W3_scales,
                   const uint32_t* W2_codes, const void* W2_scales, void* y, int32_t* expert_counts,
                   int32_t* dropped, float* aux_loss, float* z_loss, void* workspace, size_t workspace_bytes,
                   const moe_debug* dbg, void* stream) {
  ExpertWeights ew;
  memset(&ew, 0, sizeof(ew));
  ew.w4 = true;
  ew.Q1 = W1_codes;
  ew.Q3 = W3_codes;
  ew.Q2 = W2_codes;
  ew.S1 = W1_scales;
  ew.S3 = W3_scales;
  ew.S2 = W2_scales;
  return forward_impl(h, T, x, W_r, b_r, ew, y, expert_counts, dropped, aux_loss, z_loss, workspace,
                      workspace_bytes, dbg, stream, "moe_forward_w4");
}

int moe_quantize_int4(const void* W, int64_t rows, int64_t K, uint32_t* codes, void* scales, void* stream) {
  if (rows < 0 || K < 0) return fail(MOE_ERR_INVALID_ARG, "moe_quantize_int4: rows < 0 or K < 0");
  if (K % W4_GROUP != 0 || rows % 128 != 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_quantize_int4: rows and K must be multiples of 128");
  if (K > 2147483647LL) return fail(MOE_ERR_UNSUPPORTED, "moe_quantize_int4: K too large");
  if (rows == 0 || K == 0) {
    t_err.clear();
    return MOE_OK;
  }
  if (W == nullptr || codes == nullptr || scales == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_quantize_int4: NULL pointer");
  if (((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(codes)) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(scales) & 1) != 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_quantize_int4: W and codes must be 16-byte aligned, scales 2-byte");
  const cudaError_t e = launch_quantize_int4(W, rows, static_cast<int>(K), codes, scales,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_quantize_int4: ") + cudaGetErrorString(e));
  t_err.clear();
  return MOE_OK;
}

int moe_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_status: ") + cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_moe_error_word, sizeof(word));
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_status: ") + cudaGetErrorString(e));
  if (word == DEV_ERR_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "moe_status: a device-side bounded wait ran out");
  if (word == DEV_ERR_RANGE)
    return fail(MOE_ERR_RANGE, "moe_status: a value of the fp16 hidden mode was beyond the fp16 range");
  if (word != 0) return fail(MOE_ERR_CUDA, "moe_status: unknown device error word");
  return MOE_OK;
}

int moe_clear_status(void) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyToSymbol(g_moe_error_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_clear_status: ") + cudaGetErrorString(e));
  return MOE_OK;
}

const char* moe_last_error(void) { return t_err.c_str(); }

uint64_t moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_selftest_timeout(int64_t limit_ns, void* stream) {
  DeviceInfo* di = nullptr;
  cudaError_t ce = device_info(&di);
  if (ce != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_selftest_timeout: ") + cudaGetErrorString(ce));
  const int64_t lim = std::min<int64_t>(std::max<int64_t>(limit_ns, 1000), 2000000000LL);
  ce = launch_selftest_timeout(di->err, lim, static_cast<cudaStream_t>(stream));
  if (ce != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_selftest_timeout: ") + cudaGetErrorString(ce));
  return MOE_OK;
}

size_t moe_backward_workspace_bytes(moe_handle h, int64_t T) {
  if (h == nullptr || T < 0) return 0;
  return make_bw_layout(*h, make_layout(*h, T)).total;
}

int moe_backward(moe_handle h, int64_t T, const void* x, const float* W_r, const float* b_r, const void* W1,
                 const void* W3, const void* W2, const void* dy, float aux_coef, float z_coef, float* dx,
                 float* dW_r, float* db_r, float* dW1, float* dW3, float* dW2, const void* workspace,
                 size_t workspace_bytes, void* bw_workspace, size_t bw_workspace_bytes, void* stream) {
  if (h == nullptr) return fail(MOE_ERR_INVALID_ARG, "moe_backward: handle is NULL");
  const moe_layer& L = *h;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_backward: T < 0");
  if (T * L.k > 2147483647LL / 2) return fail(MOE_ERR_UNSUPPORTED, "moe_backward: T * k too large");
  if (W_r == nullptr || W1 == nullptr || W2 == nullptr || dW_r == nullptr || dW1 == nullptr || dW2 == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: W_r, W1, W2, dW_r, dW1 and dW2 must be non-NULL");
  const bool swiglu = L.act == MOE_ACT_SWIGLU;
  if (swiglu != (W3 != nullptr) || swiglu != (dW3 != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: W3 and dW3 must be given for SwiGLU and NULL for ReLU");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int groups = L.E + L.n_shared;
  const size_t wexp = sizeof(float) * static_cast<size_t>(groups) * L.d_ff * L.d;
  if (T == 0) {  // L = 0: every gradient is zero
    if (cudaMemsetAsync(dW_r, 0, sizeof(float) * L.E * static_cast<size_t>(L.d), s) != cudaSuccess ||
        (db_r != nullptr && cudaMemsetAsync(db_r, 0, sizeof(float) * L.E, s) != cudaSuccess) ||
        cudaMemsetAsync(dW1, 0, wexp, s) != cudaSuccess || cudaMemsetAsync(dW2, 0, wexp, s) != cudaSuccess ||
        (swiglu && cudaMemsetAsync(dW3, 0, wexp, s) != cudaSuccess))
      return fail(MOE_ERR_CUDA, std::string("moe_backward: ") + cudaGetErrorString(cudaGetLastError()));
    t_err.clear();
    return MOE_OK;
  }
  if (x == nullptr || dy == nullptr || dx == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: x, dy and dx must be non-NULL");
  const Layout w = make_layout(L, T);
  const BwLayout b = make_bw_layout(L, w);
  if (workspace == nullptr || workspace_bytes < w.total)
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: forward workspace missing or smaller than moe_workspace_bytes()");
  if (bw_workspace == nullptr || bw_workspace_bytes < b.total)
    return fail(MOE_ERR_INVALID_ARG,
                "moe_backward: backward workspace missing or smaller than moe_backward_workspace_bytes()");
  if (((reinterpret_cast<uintptr_t>(workspace) | reinterpret_cast<uintptr_t>(bw_workspace)) & 255) != 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: workspaces must be 256-byte aligned");
  const uintptr_t al = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy) |
                       reinterpret_cast<uintptr_t>(W1) | reinterpret_cast<uintptr_t>(W2) |
                       reinterpret_cast<uintptr_t>(W3) | reinterpret_cast<uintptr_t>(dx) |
                       reinterpret_cast<uintptr_t>(dW1) | reinterpret_cast<uintptr_t>(dW2) |
                       reinterpret_cast<uintptr_t>(dW3);
  if ((al & 15) != 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_backward: x, dy, weights, dx and the expert-weight gradients must be 16-byte aligned");
  DeviceInfo* di = nullptr;
  cudaError_t de = device_info(&di);
  if (de != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_backward: ") + cudaGetErrorString(de));

  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  uint8_t* bw = static_cast<uint8_t*>(bw_workspace);
  BackwardArgs a;
  memset(&a, 0, sizeof(a));
  a.T = T;
  a.E = L.E;
  a.k = L.k;
  a.d = L.d;
  a.d_ff = L.d_ff;
  a.act = L.act;
  a.gate_mode = L.gate_mode;
  a.n_shared = L.n_shared;
  a.x_is_bf16 = L.dtype == MOE_BF16;
  a.max_group_rows = b.max_group_rows;
  a.k_pad = b.k_pad;
  a.wr_chunks = b.wr_chunks;
  a.wr_part = reinterpret_cast<float*>(bw + b.wr_part);
  a.s_max = w.s_max;
  a.x = x;
  a.W_r = W_r;
  a.b_r = b_r;
  a.W1 = W1;
  a.W3 = W3;
  a.W2 = W2;
  a.dy = dy;
  a.aux_coef = aux_coef;
  a.z_coef = z_coef;
  a.topk_idx = reinterpret_cast<const int32_t*>(ws + w.idx);
  a.topk_gate = reinterpret_cast<const float*>(ws + w.gate);
  a.dest_row = reinterpret_cast<const int32_t*>(ws + w.dest);
  a.offsets = reinterpret_cast<const int32_t*>(ws + w.offsets);
  a.row_token = reinterpret_cast<const int32_t*>(ws + w.row_token);
  a.row_gate = reinterpret_cast<const float*>(ws + w.row_gate);
  a.Xp = ws + w.Xp;
  a.A1 = reinterpret_cast<float*>(bw + b.A1);
  a.A3 = swiglu ? reinterpret_cast<float*>(bw + b.A3) : nullptr;
  a.U = reinterpret_cast<float*>(bw + b.U);
  a.dg = reinterpret_cast<float*>(bw + b.dg);
  a.dXp = reinterpret_cast<float*>(bw + b.dXp);
  a.dh = reinterpret_cast<float*>(bw + b.dh);
  a.cnt1 = reinterpret_cast<int32_t*>(bw + b.cnt1);
  a.num_sms = di->num_sms;
  a.err = di->err;
  a.mprefix = reinterpret_cast<const int32_t*>(ws + w.mprefix);
  if (L.dtype == MOE_BF16) {
    a.ones = reinterpret_cast<float*>(bw + b.ones);
    a.dYs = bw + b.dYs;
    a.W1t = bw + b.W1t;
    a.W3t = swiglu ? bw + b.W3t : nullptr;
    a.W2t = bw + b.W2t;
    a.dA1p = bw + b.dA1p;
    a.dA3p = swiglu ? bw + b.dA3p : nullptr;
    a.P1 = bw + b.P1;
    a.P3 = swiglu ? bw + b.P3 : nullptr;
    a.PH = bw + b.PH;
    a.XT = bw + b.XT;
    a.DT = bw + b.DT;
    a.woff = reinterpret_cast<int32_t*>(bw + b.woff);
    a.wpre = reinterpret_cast<int32_t*>(bw + b.wpre);
    a.woff_d = reinterpret_cast<int32_t*>(bw + b.woff_d);
    a.wpre_d = reinterpret_cast<int32_t*>(bw + b.wpre_d);
  }
  a.dx = dx;
  a.dW_r = dW_r;
  a.db_r = db_r;
  a.dW1 = dW1;
  a.dW3 = dW3;
  a.dW2 = dW2;
  cudaError_t ce = cudaSuccess;
  if (b.rt) {  // the router logits, as the forward computed them (its top-k and tables go to scratch)
    RoutingArgs r;
    memset(&r, 0, sizeof(r));
    r.T = T;
    r.E = L.E;
    r.k = L.k;
    r.d = L.d;
    r.gate_mode = L.gate_mode;
    r.capacity = w.capacity;
    r.nblk = w.nblk;
    r.x_is_bf16 = 1;
    r.x = x;
    r.W_r = W_r;
    r.b_r = b_r;
    r.topk_idx = reinterpret_cast<int32_t*>(bw + b.rt_idx);
    r.topk_gate = reinterpret_cast<float*>(bw + b.rt_gate);
    r.part_hist = reinterpret_cast<int32_t*>(bw + b.rt_hist);
    r.part_cnt1 = reinterpret_cast<int32_t*>(bw + b.rt_cnt1);
    r.part_psum = reinterpret_cast<float*>(bw + b.rt_psum);
    r.part_lse2 = reinterpret_cast<float*>(bw + b.rt_lse2);
    r.logits_out = reinterpret_cast<float*>(bw + b.rt_logits);
    const char* why = nullptr;
    ce = launch_router_tc(r, bw + b.rt_wsplit, bw + b.rt_rpart, di->num_sms, di->err, s, &why);
    if (why != nullptr) return fail(MOE_ERR_UNSUPPORTED, std::string("moe_backward: ") + why);
    a.logits = r.logits_out;
  }
  if (ce == cudaSuccess) ce = launch_backward(a, s);
  if (ce != cudaSuccess) return fail(MOE_ERR_CUDA, std::string("moe_backward: ") + cudaGetErrorString(ce));
  t_err.clear();
  return MOE_OK;
}

}  // extern "C"

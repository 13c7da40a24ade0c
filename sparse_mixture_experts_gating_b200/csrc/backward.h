// Backward pass of the MoE layer (backward.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Everything the backward launches need.  The routing tables and the
// expert-sorted rows come from the forward pass's workspace; the scratch
// buffers from the caller's backward workspace.
struct BackwardArgs {
  int64_t T;
  int E, k, d, d_ff, act, gate_mode, n_shared, x_is_bf16;
  int max_group_rows;  // no group has more rows
  int64_t s_max;       // rows of the expert-sorted buffers
  const void* x;       // [T][d]
  const float* W_r;    // [E][d]
  const float* logits;  // [T][E] the forward's router logits (bias added), or NULL: recomputed here
  const float* b_r;    // [E] or NULL
  const void* W1;      // [E + n_shared][d_ff][d]
  const void* W3;      // same, SwiGLU only
  const void* W2;      // [E + n_shared][d][d_ff]
  const void* dy;      // [T][d]
  float aux_coef, z_coef;
  // forward workspace
  const int32_t* topk_idx;   // [T][k]
  const float* topk_gate;    // [T][k]
  const int32_t* dest_row;   // [T][k]
  const int32_t* offsets;    // [E + n_shared + 1]
  const int32_t* row_token;  // [s_max]
  const float* row_gate;     // [s_max]
  const void* Xp;            // [s_max][d]
  // backward scratch
  float* A1;    // [s_max][d_ff]: w1 x, then the hidden activation
  float* A3;    // [s_max][d_ff]: w3 x, then its gradient (SwiGLU)
  float* U;     // [s_max][d_ff]: W2^T dy, then the gradient of w1 x
  float* dg;    // [s_max]: gradient reaching each row's gate
  float* dXp;   // [s_max][d] (bf16 SwiGLU layers: [2][s_max][d], the W1 and W3 parts)
  float* dh;    // [T][E]: gradient reaching the router logits
  int32_t* cnt1;  // [E]: first-choice counts
  // bf16 layers: the row-grouped products run on the tensor cores
  int num_sms;
  unsigned int* err;       // device error word (bounded waits of the tensor-core GEMM)
  const int32_t* mprefix;  // [E + n_shared + 1] m-tile prefix of the forward's scan
  float* ones;             // [max(s_max, G d_ff)] gate 1 for the fp32 epilogue
  void* dYs;               // [s_max][d] bf16: dy rows in expert-sorted order
  void* W1t;               // [E + n_shared][d][d_ff] bf16: W1 transposed per expert
  void* W3t;               // same for W3 (SwiGLU)
  void* W2t;               // [E + n_shared][d_ff][d] bf16: W2 transposed per expert
  void* dA1p;              // [2][s_max][d_ff] bf16: hi and lo planes of the gradient of w1 x
  void* dA3p;              // same for w3 x (SwiGLU)
  // bf16 layers: the weight gradients as per-expert products over K_pad
  // (every expert's rows, zero-padded to the same count) on the tensor cores
  int k_pad;               // max_group_rows rounded up to 8
  void* P1;                // [2][G][d_ff][k_pad] bf16 planes: da1 per expert, transposed
  void* P3;                // same for da3 (SwiGLU)
  void* PH;                // same for g * hid
  void* XT;                // [G][d][k_pad] bf16: Xp per expert, transposed
  void* DT;                // [G][d][k_pad] bf16: dy (sorted rows) per expert, transposed
  int32_t* woff;           // [G + 1] rows of the per-expert products: e * d_ff
  int32_t* wpre;           // [G + 1] their m-tile prefix: e * ceil(d_ff / 128)
  int32_t* woff_d;         // [G + 1] the same for products of d rows (dW2): e * d
  int32_t* wpre_d;         // [G + 1] e * ceil(d / 128)
  // dW_r: the sum over tokens cut into wr_chunks chunks of partials
  int wr_chunks;
  float* wr_part;          // [wr_chunks][E][d]
  // outputs (fp32)
  float* dx;    // [T][d]
  float* dW_r;  // [E][d]
  float* db_r;  // [E] or NULL
  float* dW1;   // [E + n_shared][d_ff][d]
  float* dW3;   // same or NULL
  float* dW2;   // [E + n_shared][d][d_ff]
};

// Launches the backward kernels on s (no host synchronisation).
cudaError_t launch_backward(const BackwardArgs& a, cudaStream_t s);

}  // namespace moe

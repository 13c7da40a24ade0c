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
  float* dXp;   // [s_max][d]
  float* dh;    // [T][E]: gradient reaching the router logits
  int32_t* cnt1;  // [E]: first-choice counts
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

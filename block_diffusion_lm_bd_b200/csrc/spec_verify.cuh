// Commit rule of self-speculative verification ("Nemotron-Labs Diffusion",
// self-speculation: a block drafted bidirectionally is checked causally and
// its matching prefix commits; at temperature 0 the result is that of
// autoregressive decoding). Given every block position's autoregressive token
// a_i (the argmax of its verification logits, computed by the unmask reduce
// over all rows), block b accepts its longest prefix with a_i == draft_i; those
// positions commit, and so does the first mismatching position with a_i.
#pragma once

#include "bd_common.cuh"

namespace bd {

constexpr int kVerifyThreads = 64;  // one thread per block position (S <= 64)

struct VerifyParams {
  const int32_t *ar_tokens;  // [rows] argmax of each row
  const int32_t *draft;      // [rows]
  uint8_t *commit_out;       // [rows]
  int32_t *n_accept;         // [rows / S]
  int S;
};

__global__ void __launch_bounds__(kVerifyThreads) spec_verify_kernel(VerifyParams p) {
  __shared__ int s_n;
  const int b = blockIdx.x, i = threadIdx.x;
  if (i == 0) s_n = p.S;
  __syncthreads();
  const int64_t r = int64_t(b) * p.S + i;
  if (i < p.S && p.ar_tokens[r] != p.draft[r]) atomicMin(&s_n, i);
  __syncthreads();
  const int n = s_n;
  if (i < p.S) p.commit_out[r] = (i <= n) ? 1 : 0;  // matching prefix + the first mismatch
  if (i == 0) p.n_accept[b] = n;
}

}  // namespace bd

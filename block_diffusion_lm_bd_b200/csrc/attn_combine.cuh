// Log-sum-exp merge of the partial results of (b, kv) pairs whose work units
// were split over several CTAs. For parts s with normalised outputs o_s and
// log-normalisers lse_s: M = max_s lse_s, w_s = exp(lse_s - M),
// o = sum_s w_s o_s / sum_s w_s, lse = M + log(sum_s w_s) - the identity that
// lets a long prefix be split into chunks that are attended independently.
#pragma once

#include "attn_common.cuh"

namespace bd {

constexpr int kCombineThreads = 256;
constexpr int kCombineMaxParts = 1024;

__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(AttnParams p) {
  __shared__ int s_part[kCombineMaxParts];
  __shared__ float s_max[kMaxRows];
  __shared__ float s_den[kMaxRows];
  __shared__ int s_np;
  pdl_wait_previous();
  if (*p.ws.flag) return;
  const int pair = blockIdx.x;
  const int b = pair / p.H_kv, kv = pair % p.H_kv;
  const int n = attn_units(p.prefix_len[b]);
  const int64_t G = p.G;
  const int64_t W = int64_t(p.H_kv) * p.ws.cum[p.B];
  const int64_t base = int64_t(p.H_kv) * p.ws.cum[b] + int64_t(kv) * n;
  const int64_t c0 = part_owner(base, W, G), c1 = part_owner(base + n - 1, W, G);
  if (c0 == c1) return;  // finished inside one CTA, already written
  if (threadIdx.x == 0) {
    int np = 0;
    s_part[np++] = int(2 * c0 + (part_start(c0, W, G) == base ? 0 : 1));
    for (int64_t c = c0 + 1; c <= c1 && np < kCombineMaxParts; ++c)
      if (part_start(c, W, G) < part_start(c + 1, W, G)) s_part[np++] = int(2 * c);
    s_np = np;
  }
  __syncthreads();
  const int np = s_np, M = p.M, d = p.d, g = p.g;
  for (int m = threadIdx.x; m < M; m += blockDim.x) {
    float mx = -INFINITY;
    for (int i = 0; i < np; ++i) mx = fmaxf(mx, p.ws.slot_lse[int64_t(s_part[i]) * M + m]);
    float den = 0.f;
    for (int i = 0; i < np; ++i) den += expf(p.ws.slot_lse[int64_t(s_part[i]) * M + m] - mx);
    s_max[m] = mx;
    s_den[m] = den;
    if (p.lse) {
      const int s = m / g, j = m % g;
      p.lse[(int64_t(b) * p.H_q + kv * g + j) * p.S + s] = mx + logf(den);
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < M * d; idx += blockDim.x) {
    const int m = idx / d, k = idx % d;
    float acc = 0.f;
    for (int i = 0; i < np; ++i) {
      const int64_t sl = s_part[i];
      acc += expf(p.ws.slot_lse[sl * M + m] - s_max[m]) * p.ws.slot[(sl * M + m) * d + k];
    }
    const int s = m / g, j = m % g;
    p.o[((int64_t(b) * p.S + s) * p.H_q + kv * g + j) * d + k] = acc / s_den[m];
  }
}

}  // namespace bd

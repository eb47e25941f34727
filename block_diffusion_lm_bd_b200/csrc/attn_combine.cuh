// Log-sum-exp merge of the partial results of (b, kv) pairs whose work units
// were split over several CTAs. For parts s with normalised outputs o_s and
// log-normalisers lse_s: M = max_s lse_s, w_s = exp(lse_s - M),
// o = sum_s w_s o_s / sum_s w_s, lse = M + log(sum_s w_s) - the identity that
// lets a long prefix be split into chunks that are attended independently.
#pragma once

#include "attn_common.cuh"

namespace bd {

constexpr int kCombineThreads = 256;
constexpr int kCombineSplit = 4;       // CTAs per (b, kv) pair, each a quarter of the rows
constexpr int kCombineMaxParts = 1024;
constexpr int kCombineWParts = 48;     // parts whose weights are kept in shared memory

// grid (B * H_kv, kCombineSplit)
__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(AttnParams p) {
  __shared__ int s_part[kCombineMaxParts];
  __shared__ float s_w[kCombineWParts][kMaxRows / kCombineSplit];
  __shared__ float s_max[kMaxRows / kCombineSplit];
  __shared__ float s_den[kMaxRows / kCombineSplit];
  __shared__ int s_np;
  pdl_launch_dependents();
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
  const int M = p.M, d = p.d, g = p.g;
  const int rows = (M + kCombineSplit - 1) / kCombineSplit;
  const int r0 = blockIdx.y * rows, r1 = min(M, r0 + rows);
  if (r0 >= r1) return;
  if (threadIdx.x == 0) {
    int np = 0;
    s_part[np++] = int(2 * c0 + (part_start(c0, W, G) == base ? 0 : 1));
    for (int64_t c = c0 + 1; c <= c1 && np < kCombineMaxParts; ++c)
      if (part_start(c, W, G) < part_start(c + 1, W, G)) s_part[np++] = int(2 * c);
    s_np = np;
  }
  __syncthreads();
  const int np = s_np;
  for (int m = r0 + threadIdx.x; m < r1; m += blockDim.x) {
    float mx = -INFINITY;
    for (int i = 0; i < np; ++i) mx = fmaxf(mx, p.ws.slot_lse[int64_t(s_part[i]) * M + m]);
    float den = 0.f;
    for (int i = 0; i < np; ++i) {
      const float w = expf(p.ws.slot_lse[int64_t(s_part[i]) * M + m] - mx);
      if (i < kCombineWParts) s_w[i][m - r0] = w;
      den += w;
    }
    s_max[m - r0] = mx;
    s_den[m - r0] = den;
    if (p.lse) {
      const int s = m / g, j = m % g;
      p.lse[(int64_t(b) * p.H_q + kv * g + j) * p.S + s] = mx + logf(den);
    }
  }
  __syncthreads();
  const int d4 = d / 4;
  for (int idx = threadIdx.x; idx < (r1 - r0) * d4; idx += blockDim.x) {
    const int m = r0 + idx / d4, k4 = idx % d4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int i = 0; i < np; ++i) {
      const int64_t sl = s_part[i];
      const float w = i < kCombineWParts ? s_w[i][m - r0]
                                         : expf(p.ws.slot_lse[sl * M + m] - s_max[m - r0]);
      const float4 v = reinterpret_cast<const float4 *>(p.ws.slot + (sl * M + m) * d)[k4];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = 1.f / s_den[m - r0];
    const int s = m / g, j = m % g;
    reinterpret_cast<float4 *>(p.o + ((int64_t(b) * p.S + s) * p.H_q + kv * g + j) * d)[k4] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
}

}  // namespace bd

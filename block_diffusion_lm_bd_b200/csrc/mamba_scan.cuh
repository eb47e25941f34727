// Block-local bidirectional Mamba scan ("Training Hybrid Block Diffusion
// Language Models with Partial Bidirectionality", Methodology: the finished
// prefix keeps only a forward boundary state of each Mamba layer, and the
// reverse scan is confined to the active block, so the cached state depends on
// the clean prefix alone). Mamba-2 recurrence, per head h (scalar decay A < 0,
// grouped B / C, head h in group h / (H / G)):
//   forward from the cached boundary state h0:
//     s[t] = exp(dt[t] A) s[t-1] + dt[t] x[t] B[t]^T,  y_fwd[t] = s[t] C[t] + D x[t]
//   reverse inside the block, from zero after its last token:
//     r[t] = exp(dt_r[t] A_r) r[t+1] + dt_r[t] x[t] B_r[t]^T,  y_rev[t] = r[t] C_r[t]
//   y = y_fwd + y_rev.
// The boundary state is read, never written.
//
// Two kernels compute it. Blocks of at most 16 tokens take mamba_ssd_kernel
// (the unrolled, chunked form, further below). Longer blocks take
// mamba_scan_kernel, the recurrence itself:
// one CTA per (head, sequence); thread (c, q) owns state row q, columns
// 32c .. 32c+31 of both directions in registers, a warp holding 32 rows of one
// column chunk. The block's x, dt, B, C of the head's group are staged in
// shared memory by asynchronous copies. A step is 32 FMAs of update and 32 of
// output per thread (B / C read as warp-wide broadcasts, four independent
// partial sums); the state is carried scaled by the running product of decays
// so that an update is a single FMA. Bound by fp32 FMA throughput:
// 4 * S * P * N FMAs per head and sequence against P * N * 4 bytes of boundary
// state (read once, streaming loads).
#pragma once

#include "bd_common.cuh"

namespace bd {

struct MambaParams {
  const float *x;       // [B, S, H, P]
  const float *dt;      // [B, S, H]
  const float *Bf;      // [B, S, G, N]
  const float *Cf;      // [B, S, G, N]
  const float *dt_r;    // [B, S, H]
  const float *Br;      // [B, S, G, N]
  const float *Cr;      // [B, S, G, N]
  const float *Af;      // [H]
  const float *Ar;      // [H]
  const float *Dskip;   // [H]
  const float *h0;      // [B, H, P, N]
  float *y;             // [B, S, H, P]
  int B, S, H, P, N, G;
};

constexpr int kMambaMaxS = 64;

constexpr float kMambaMinScale = 0x1p-30f;  // fold the decay product into u below this

// shared floats: x [S][P]; per-chunk output partials [NC][S][P]; B and C of
// both directions [S][N]; per-step a, 1/a, a_r, 1/a_r and dt, dt_r [S]
__host__ __device__ inline size_t mamba_smem_bytes(int S, int P, int N) {
  const int NC = N / 32;
  return sizeof(float) * (size_t(1 + NC) * S * P + size_t(4) * S * N + size_t(6) * S);
}

// The state is kept scaled: s[t] = pi[t] * u[t] with pi[t] the product of the
// decays since u was last renormalised, so a step is
//     u += (dt x / pi) b     (one FMA per column)
//     y  = pi * (u . c)      (one FMA per column, one multiply)
// Whenever the product would fall below kMambaMinScale the decay is folded
// into u instead (u *= pi, pi = 1), so 1/pi never exceeds 2^30 and nothing
// overflows; the branch depends only on (sequence, head, step), so a whole CTA
// takes it together. A thread carries RB rows of one 32-column chunk, so each
// of the step's B / C values it loads feeds RB updates and RB output terms.
// acc[r] receives row r's 32-column part of u . c.
template <int RB>
__device__ __forceinline__ void mamba_step(float (&u)[RB][32], const float (&w)[RB],
                                           const float *bv, const float *cv, float (&acc)[RB]) {
  float part[RB][2];
#pragma unroll
  for (int r = 0; r < RB; ++r) part[r][0] = part[r][1] = 0.f;
  // the step's 64 B / C values are all requested before the first FMA; every
  // lane of the warp reads the same addresses (one broadcast per load)
  float4 bb[8], cc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    bb[k] = reinterpret_cast<const float4 *>(bv)[k];
    cc[k] = reinterpret_cast<const float4 *>(cv)[k];
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float bk[4] = {bb[k].x, bb[k].y, bb[k].z, bb[k].w};
    const float ck[4] = {cc[k].x, cc[k].y, cc[k].z, cc[k].w};
#pragma unroll
    for (int r = 0; r < RB; ++r) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        u[r][4 * k + j] = fmaf(w[r], bk[j], u[r][4 * k + j]);
        part[r][j & 1] = fmaf(u[r][4 * k + j], ck[j], part[r][j & 1]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < RB; ++r) acc[r] = part[r][0] + part[r][1];
}

__device__ __forceinline__ void cp_async16(float *smem, const float *gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}

// Thread (c, q) = (tid / (P/RB), tid % (P/RB)): state rows q + j * P/RB
// (j < RB), columns 32c .. 32c+31. A warp covers 32 row slots of one column
// chunk, so its B / C loads are broadcasts; each thread writes its chunk's
// part of y[t][row] to its own partial slot and the chunks are summed once at
// the end.
template <int NC, int RB>
__global__ void __launch_bounds__(512, 1) mamba_scan_kernel(MambaParams p) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, b = blockIdx.y;
  const int S = p.S, P = p.P, N = p.N, H = p.H, G = p.G;
  const int PR = P / RB;          // row slots per column chunk
  float *sx = sm;                 // x[t]            [S][P]
  float *syp = sx + S * P;        // partials        [NC][S][P]
  float *sBf = syp + NC * S * P;  // [S][N] each
  float *sCf = sBf + S * N;
  float *sBr = sCf + S * N;
  float *sCr = sBr + S * N;
  float *sa = sCr + S * N;        // exp(dt A), exp(-dt A), exp(dt_r A_r), exp(-dt_r A_r), dt, dt_r
  float *sai = sa + S;
  float *sar = sai + S;
  float *sari = sar + S;
  float *sdt = sari + S;
  float *sdtr = sdt + S;
  const int g = h / (H / G);
  const int tid = threadIdx.x, nth = blockDim.x;
  const float A = p.Af[h], Arv = p.Ar[h], Dk = p.Dskip[h];

  // stage the block's inputs with 16-byte asynchronous copies, all in flight at once
  const int pv = P / 4, nv = N / 4;
  for (int v = tid; v < S * pv; v += nth) {
    const int t = v / pv, q4 = v % pv;
    cp_async16(sx + t * P + 4 * q4, p.x + ((int64_t(b) * S + t) * H + h) * P + 4 * q4);
  }
  for (int v = tid; v < S * nv; v += nth) {
    const int t = v / nv, n = 4 * (v % nv);
    const int64_t o = ((int64_t(b) * S + t) * G + g) * N + n;
    const int s = t * N + n;
    cp_async16(sBf + s, p.Bf + o);
    cp_async16(sCf + s, p.Cf + o);
    cp_async16(sBr + s, p.Br + o);
    cp_async16(sCr + s, p.Cr + o);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  for (int t = tid; t < S; t += nth) {
    const float d = p.dt[(int64_t(b) * S + t) * H + h], dr = p.dt_r[(int64_t(b) * S + t) * H + h];
    sdt[t] = d;
    sdtr[t] = dr;
    sa[t] = expf(d * A);
    sai[t] = expf(-d * A);
    sar[t] = expf(dr * Arv);
    sari[t] = expf(-dr * Arv);
  }
  const int c = tid / PR, q0 = tid % PR;
  float u[RB][32];
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    const float4 *src = reinterpret_cast<const float4 *>(
        p.h0 + ((int64_t(b) * H + h) * P + q0 + r * PR) * N + c * 32);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 v = __ldcs(src + k);
      u[r][4 * k] = v.x;
      u[r][4 * k + 1] = v.y;
      u[r][4 * k + 2] = v.z;
      u[r][4 * k + 3] = v.w;
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();

  float *yp = syp + c * S * P + q0;
  float w[RB], acc[RB];
  // forward from the boundary state
  float pi = 1.f, ipi = 1.f;
  for (int t = 0; t < S; ++t) {
    pi *= sa[t];
    ipi *= sai[t];
    if (pi < kMambaMinScale) {
#pragma unroll
      for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int i = 0; i < 32; ++i) u[r][i] *= pi;
      pi = 1.f;
      ipi = 1.f;
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) w[r] = sdt[t] * sx[t * P + q0 + r * PR] * ipi;
    mamba_step<RB>(u, w, sBf + t * N + c * 32, sCf + t * N + c * 32, acc);
#pragma unroll
    for (int r = 0; r < RB; ++r) yp[t * P + r * PR] = pi * acc[r];
  }
  // reverse inside the block, from zero
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int i = 0; i < 32; ++i) u[r][i] = 0.f;
  pi = 1.f;
  ipi = 1.f;
  for (int t = S - 1; t >= 0; --t) {
    pi *= sar[t];
    ipi *= sari[t];
    if (pi < kMambaMinScale) {
#pragma unroll
      for (int r = 0; r < RB; ++r)
#pragma unroll
        for (int i = 0; i < 32; ++i) u[r][i] *= pi;
      pi = 1.f;
      ipi = 1.f;
    }
#pragma unroll
    for (int r = 0; r < RB; ++r) w[r] = sdtr[t] * sx[t * P + q0 + r * PR] * ipi;
    mamba_step<RB>(u, w, sBr + t * N + c * 32, sCr + t * N + c * 32, acc);
#pragma unroll
    for (int r = 0; r < RB; ++r) yp[t * P + r * PR] += pi * acc[r];
  }
  __syncthreads();
  for (int i = tid; i < S * P; i += nth) {
    const int t = i / P, qq = i % P;
    float v = Dk * sx[i];
#pragma unroll
    for (int k = 0; k < NC; ++k) v += syp[k * S * P + i];
    p.y[((int64_t(b) * S + t) * H + h) * P + qq] = v;
  }
}

// ---------------------------------------------------------------------------
// Blocks of at most 16 tokens: the chunked ("state-space dual") form of the
// same two scans. Unrolling the recurrences gives, per head,
//   y[t] = e^{F(0,t)} (h0 C[t])
//        + sum_{s<=t} e^{F(s+1,t)} dt[s] (C[t].B[s]) x[s]
//        + sum_{s>=t} e^{R(t,s-1)} dt_r[s] (C_r[t].B_r[s]) x[s] + D x[t]
// with F(i,j) = sum_{u=i..j} dt[u] A and R(i,j) = sum_{u=i..j} dt_r[u] A_r.
// Only y is needed (the boundary state is not advanced), so the per-token
// states are never formed: one GEMM contracts C (and C_r) over the state
// dimension with the boundary state's rows and with B (and B_r) at once,
// S * (P + 2 S) * N multiply-adds instead of the recurrence's 4 S P N; the
// decays and dt fold into a 16 x 16 mixing matrix M, and y = e^F (h0 C) + M x
// + D x.
// ---------------------------------------------------------------------------
constexpr int kSsdMaxS = 16;

template <int P, int N>
struct SsdShape {
  static constexpr int kCols = P + 2 * kSsdMaxS;  // GEMM columns: h0 rows, B rows, B_r rows
  static constexpr int kSlabs = kCols / 32;       // 32 columns per warp
  static constexpr int kWarps = 2 * kSlabs;       // the state dimension split in two halves
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kFStride = kCols + 8;      // GEMM result rows (padded: no bank conflicts)
  // shared-memory floats
  static constexpr int kR = 0;                        // [kCols][N] GEMM right operand, swizzled
  static constexpr int kCf = kR + kCols * N;          // [16][N] C, swizzled
  static constexpr int kCr = kCf + kSsdMaxS * N;      // [16][N] C_r, swizzled
  static constexpr int kX = kCr + kSsdMaxS * N;       // [16][P] x
  static constexpr int kM = kX + kSsdMaxS * P;        // [16][16] mixing matrix
  static constexpr int kVec = kM + kSsdMaxS * kSsdMaxS;  // dt A, dt_r A_r, dt, dt_r, e^{F(0,t)}
  static constexpr int kFloats = kVec + 5 * kSsdMaxS;
  static constexpr size_t kSmemBytes = sizeof(float) * kFloats;
  static_assert(P % 32 == 0 && N % 32 == 0, "whole warps of columns, whole swizzle rows");
  static_assert(kSsdMaxS * kFStride <= kX, "the GEMM result reuses the operand space");
};

// Row r of a [rows][N] operand keeps its 16-byte chunk j at j ^ (r & 7), so
// that 16-byte loads of one chunk index from 8 rows hit distinct banks.
template <int N>
__device__ __forceinline__ int ssd_swz(int r, int j) {
  return r * N + 4 * (j ^ (r & 7));
}

// acc[i][k] += sum over chunks [j0, j1) of A[t_i] . R[c_k], t_i = tq + 4i,
// c_k = 32 * slab + cq + 8k; A = C, except for k >= 2 of the slab holding
// the B and B_r columns (MIXED), where A = C_r.
template <int N, bool MIXED>
__device__ __forceinline__ void ssd_gemm_tile(float (&acc)[4][4], const float *sCf, const float *sCr,
                                              const float *sR, int slab, int tq, int cq, int j0,
                                              int j1) {
#pragma unroll 2
  for (int j = j0; j < j1; ++j) {
    float4 a[4], ar[4], r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4 *>(sCf + ssd_swz<N>(tq + 4 * i, j));
    if (MIXED) {
#pragma unroll
      for (int i = 0; i < 4; ++i) ar[i] = *reinterpret_cast<const float4 *>(sCr + ssd_swz<N>(tq + 4 * i, j));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      r[k] = *reinterpret_cast<const float4 *>(sR + ssd_swz<N>(32 * slab + cq + 8 * k, j));
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 av = (MIXED && k >= 2) ? ar[i] : a[i];
        float v = acc[i][k];
        v = fmaf(av.x, r[k].x, v);
        v = fmaf(av.y, r[k].y, v);
        v = fmaf(av.z, r[k].z, v);
        v = fmaf(av.w, r[k].w, v);
        acc[i][k] = v;
      }
  }
}

template <int P, int N>
__global__ void __launch_bounds__(SsdShape<P, N>::kThreads, (P >= 128 ? 2 : 3))
    mamba_ssd_kernel(MambaParams p) {
  using L = SsdShape<P, N>;
  extern __shared__ __align__(16) float sm[];
  float *sR = sm + L::kR, *sCf = sm + L::kCf, *sCr = sm + L::kCr, *sX = sm + L::kX;
  float *sM = sm + L::kM, *sla = sm + L::kVec, *slr = sla + kSsdMaxS, *sdt = slr + kSsdMaxS;
  float *sdtr = sdt + kSsdMaxS, *sef = sdtr + kSsdMaxS;
  const int h = blockIdx.x, b = blockIdx.y;
  const int S = p.S, H = p.H, G = p.G;
  const int g = h / (H / G);
  const int tid = threadIdx.x;
  constexpr int NT = L::kThreads, N4 = N / 4, P4 = P / 4;

  // 1. Stage the operands with 16-byte asynchronous copies; rows of tokens
  //    past the block are zero. The GEMM's right operand rows are h0 (P rows),
  //    then B and B_r (16 rows each); C and C_r (16 rows each) follow them, so
  //    all of it is one swizzled [P + 64][N] array.
  {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const float *h0b = p.h0 + (int64_t(b) * H + h) * (P * N);  // contiguous [P][N]
#pragma unroll 4
    for (int q = tid; q < P * N4; q += NT) cp_async16(sR + ssd_swz<N>(q / N4, q % N4), h0b + 4 * q);
    for (int q = tid; q < 4 * kSsdMaxS * N4; q += NT) {
      const int mat = q / (kSsdMaxS * N4), t = (q / N4) % kSsdMaxS, j = q % N4;
      float *dst = sR + ssd_swz<N>(P + kSsdMaxS * mat + t, j);
      if (t < S) {
        const float *src = mat == 0 ? p.Bf : mat == 1 ? p.Br : mat == 2 ? p.Cf : p.Cr;
        cp_async16(dst, src + ((int64_t(b) * S + t) * G + g) * N + 4 * j);
      } else {
        *reinterpret_cast<float4 *>(dst) = z;
      }
    }
    for (int q = tid; q < kSsdMaxS * P4; q += NT) {
      const int t = q / P4, j = q % P4;
      float *dst = sX + t * P + 4 * j;
      if (t < S)
        cp_async16(dst, p.x + ((int64_t(b) * S + t) * H + h) * P + 4 * j);
      else
        *reinterpret_cast<float4 *>(dst) = z;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    if (tid < kSsdMaxS) {
      const bool in = tid < S;
      const float d = in ? p.dt[(int64_t(b) * S + tid) * H + h] : 0.f;
      const float dr = in ? p.dt_r[(int64_t(b) * S + tid) * H + h] : 0.f;
      sdt[tid] = d;
      sdtr[tid] = dr;
      sla[tid] = d * p.Af[h];
      slr[tid] = dr * p.Ar[h];
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }

  // 2. GEMM: acc[i][k] = sum_n A[t_i][n] R[c_k][n] over this warp's half of
  //    the state dimension, A = C for the h0 and B columns, C_r for the B_r
  //    columns. Thread tile 4 tokens x 4 columns: t_i = tq + 4i,
  //    c_k = 32 * slab + cq + 8k.
  const int warp = tid >> 5, lane = tid & 31;
  const int slab = warp % L::kSlabs, kh = warp / L::kSlabs;
  const int tq = lane & 3, cq = lane >> 2;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[i][k] = 0.f;
  if (slab == L::kSlabs - 1)
    ssd_gemm_tile<N, true>(acc, sCf, sCr, sR, slab, tq, cq, kh * (N4 / 2), (kh + 1) * (N4 / 2));
  else
    ssd_gemm_tile<N, false>(acc, sCf, sCr, sR, slab, tq, cq, kh * (N4 / 2), (kh + 1) * (N4 / 2));
  // the two halves meet in shared memory (the operands are dead by now)
  float *sF = sm;  // [16][kFStride]
  __syncthreads();
  if (kh == 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) sF[(tq + 4 * i) * L::kFStride + 32 * slab + cq + 8 * k] = acc[i][k];
  }
  __syncthreads();
  if (kh == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float *f = sF + (tq + 4 * i) * L::kFStride + 32 * slab + cq + 8 * k;
        *f = *f + acc[i][k];
      }
  }
  __syncthreads();

  // 3. Mixing matrix M[t][s] (decays and step sizes folded in) and the
  //    boundary decay e^{F(0,t)}.
  for (int e = tid; e < kSsdMaxS * kSsdMaxS; e += NT) {
    const int t = e / kSsdMaxS, s = e % kSsdMaxS;
    float m = 0.f;
    if (t < S && s < S) {
      if (s <= t) {
        float f = 0.f;
        for (int u = s + 1; u <= t; ++u) f += sla[u];
        m += expf(f) * sdt[s] * sF[t * L::kFStride + P + s];
      }
      if (s >= t) {
        float f = 0.f;
        for (int u = t; u < s; ++u) f += slr[u];
        m += expf(f) * sdtr[s] * sF[t * L::kFStride + P + kSsdMaxS + s];
      }
    }
    sM[e] = m;
  }
  if (tid < kSsdMaxS) {
    float f = 0.f;
    for (int u = 0; u <= tid; ++u) f += sla[u];
    sef[tid] = expf(f);
  }
  __syncthreads();

  // 4. y[t][p] = e^{F(0,t)} (h0 C[t])[p] + sum_s M[t][s] x[s][p] + D x[t][p];
  //    thread tile 2 tokens x 4 channels.
  const float Dk = p.Dskip[h];
  const bool y16 = (reinterpret_cast<uintptr_t>(p.y) & 15u) == 0;
  for (int q = tid; q < (kSsdMaxS / 2) * P4; q += NT) {
    const int t0 = 2 * (q / P4), p0 = 4 * (q % P4);
    float4 o[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float ef = sef[t0 + i];
      const float4 f = *reinterpret_cast<const float4 *>(sF + (t0 + i) * L::kFStride + p0);
      const float4 xv = *reinterpret_cast<const float4 *>(sX + (t0 + i) * P + p0);
      o[i] = make_float4(fmaf(ef, f.x, Dk * xv.x), fmaf(ef, f.y, Dk * xv.y), fmaf(ef, f.z, Dk * xv.z),
                         fmaf(ef, f.w, Dk * xv.w));
    }
#pragma unroll
    for (int s = 0; s < kSsdMaxS; ++s) {
      const float4 xv = *reinterpret_cast<const float4 *>(sX + s * P + p0);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float m = sM[(t0 + i) * kSsdMaxS + s];
        o[i].x = fmaf(m, xv.x, o[i].x);
        o[i].y = fmaf(m, xv.y, o[i].y);
        o[i].z = fmaf(m, xv.z, o[i].z);
        o[i].w = fmaf(m, xv.w, o[i].w);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (t0 + i >= S) continue;
      float *yo = p.y + ((int64_t(b) * S + t0 + i) * H + h) * P + p0;
      if (y16) {
        *reinterpret_cast<float4 *>(yo) = o[i];
      } else {
        yo[0] = o[i].x;
        yo[1] = o[i].y;
        yo[2] = o[i].z;
        yo[3] = o[i].w;
      }
    }
  }
}

}  // namespace bd

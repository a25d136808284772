// gate_kernels.cuh -- K1: the low-rank forget-gate projection
//   g[n, j] = logsigmoid(sum_r (x[n,:] . W_down[:, r]) W_up[r, j] + b[j]) / tau
// (GTR article, 方法详解 §1: the gate is produced from the input by a light
// low-rank projection with a temperature).  One block handles kGateTok tokens:
// the x tile is staged through shared memory in column slabs, the rank-r
// intermediate stays in shared memory, and every output row of H*dk gates is
// written with consecutive threads on consecutive columns.
#pragma once
#include "common.cuh"

namespace gtr {

constexpr int kGateTok = 32;
constexpr int kGateThreads = 256;
constexpr int kGateSlab = 128;     // x columns staged per pass
constexpr int kGateMaxRank = 64;

template <typename TX>
__global__ void __launch_bounds__(kGateThreads)
gate_proj_kernel(const TX* __restrict__ x, const float* __restrict__ w_down,
                 const float* __restrict__ w_up, const float* __restrict__ bias,
                 float* __restrict__ g, long long N, int dm, int rank, int HD, float tau) {
  __shared__ float xs[kGateTok][kGateSlab + 1];
  __shared__ float low[kGateTok][kGateMaxRank];
  const long long tok0 = (long long)blockIdx.x * kGateTok;
  const int ntok = (int)min((long long)kGateTok, N - tok0);
  const int tid = threadIdx.x;

  // stage 1: low[t][r] = x[t, :] . w_down[:, r], accumulated slab by slab
  const int nout = kGateTok * rank;
  float acc[(kGateTok * kGateMaxRank) / kGateThreads];
#pragma unroll
  for (int u = 0; u < (kGateTok * kGateMaxRank) / kGateThreads; ++u) acc[u] = 0.f;
  for (int c0 = 0; c0 < dm; c0 += kGateSlab) {
    const int nc = min(kGateSlab, dm - c0);
    __syncthreads();
    for (int idx = tid; idx < kGateTok * kGateSlab; idx += kGateThreads) {
      const int t = idx / kGateSlab, c = idx - t * kGateSlab;
      float val = 0.f;
      if (t < ntok && c < nc) val = Elem<TX>::to_f(x[(tok0 + t) * dm + c0 + c]);
      xs[t][c] = val;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < (kGateTok * kGateMaxRank) / kGateThreads; ++u) {
      const int idx = tid + u * kGateThreads;
      if (idx < nout) {
        const int t = idx / rank, r = idx - t * rank;
        float a = acc[u];
        for (int c = 0; c < nc; ++c) a = fmaf(xs[t][c], __ldg(w_down + (size_t)(c0 + c) * rank + r), a);
        acc[u] = a;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < (kGateTok * kGateMaxRank) / kGateThreads; ++u) {
    const int idx = tid + u * kGateThreads;
    if (idx < nout) low[idx / rank][idx % rank] = acc[u];
  }
  __syncthreads();

  // stage 2: u = low . w_up + b, g = logsigmoid(u) / tau
  for (int idx = tid; idx < ntok * HD; idx += kGateThreads) {
    const int t = idx / HD, j = idx - t * HD;
    float u = bias ? __ldg(bias + j) : 0.f;
    for (int r = 0; r < rank; ++r) u = fmaf(low[t][r], __ldg(w_up + (size_t)r * HD + j), u);
    g[(tok0 + t) * HD + j] = logsigmoid_f(u) / tau;
  }
}

// ---------------------------------------------------------------------------
// Register-tiled variant for rank <= 16 and H*dk a multiple of 4 (<= 1024):
// one block of 384 threads per 64 tokens.
//   stage 1 (threads 0..255): thread = (token t, ranks r..r+3), 16 FMAs per
//           5 shared-memory loads, x and W_down staged in 128-column slabs;
//   stage 2 (all threads): item = (token t, columns j..j+3), 64 FMAs per
//           item against W_up held in shared memory, a 16-byte store of 4 gates.
// logsigmoid(u) = min(u, 0) - log1p(e), e = exp(-|u|): log1p(e) from the
// series e - e^2/2 below e = 1e-3 (truncation error < e^3/3) and from
// log(1 + e) above it.
constexpr int kGate2Tok = 64;
constexpr int kGate2Threads = 384;
constexpr int kGate2Slab = 128;
constexpr int kGate2MaxHD = 1024;

__device__ __forceinline__ float logsigmoid_fast(float u) {
  const float e = __expf(-fabsf(u));
  const float l = e < 1e-3f ? e * (1.0f - 0.5f * e) : __logf(1.0f + e);
  return fminf(u, 0.0f) - l;
}

template <typename TX>
__global__ void __launch_bounds__(kGate2Threads)
gate_proj_tiled(const TX* __restrict__ x, const float* __restrict__ w_down,
                const float* __restrict__ w_up, const float* __restrict__ bias,
                float* __restrict__ g, long long N, int dm, int rank, int HD, float inv_tau) {
  extern __shared__ float sh[];
  float* xs = sh;                                   // [64][kGate2Slab + 4]
  float* wd = xs + kGate2Tok * (kGate2Slab + 4);    // [kGate2Slab][16]
  float* low = wd + kGate2Slab * 16;                // [64][16]
  float* wu = low + kGate2Tok * 16;                 // [16][HD]
  const long long tok0 = (long long)blockIdx.x * kGate2Tok;
  const int ntok = (int)min((long long)kGate2Tok, N - tok0);
  const int tid = threadIdx.x;
  for (int i = tid; i < 16 * HD; i += kGate2Threads) {
    const int r = i / HD;
    wu[i] = r < rank ? w_up[i] : 0.f;
  }
  const int t1 = tid >> 2, r1 = (tid & 3) * 4;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  for (int c0 = 0; c0 < dm; c0 += kGate2Slab) {
    const int nc = min(kGate2Slab, dm - c0);
    __syncthreads();
    for (int i = tid; i < kGate2Tok * kGate2Slab; i += kGate2Threads) {
      const int t = i / kGate2Slab, c = i - t * kGate2Slab;
      xs[t * (kGate2Slab + 4) + c] =
          (t < ntok && c < nc) ? Elem<TX>::to_f(x[(tok0 + t) * dm + c0 + c]) : 0.f;
    }
    for (int i = tid; i < kGate2Slab * 16; i += kGate2Threads) {
      const int c = i >> 4, r = i & 15;
      wd[i] = (c < nc && r < rank) ? __ldg(w_down + (size_t)(c0 + c) * rank + r) : 0.f;
    }
    __syncthreads();
    if (tid < 256) {
      const float* xr = xs + t1 * (kGate2Slab + 4);
#pragma unroll 4
      for (int c = 0; c < kGate2Slab; c += 4) {
        const float4 xv = *reinterpret_cast<const float4*>(xr + c);
        const float xe[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 w = *reinterpret_cast<const float4*>(wd + (c + e) * 16 + r1);
          acc0 = fmaf(xe[e], w.x, acc0);
          acc1 = fmaf(xe[e], w.y, acc1);
          acc2 = fmaf(xe[e], w.z, acc2);
          acc3 = fmaf(xe[e], w.w, acc3);
        }
      }
    }
  }
  if (tid < 256) *reinterpret_cast<float4*>(low + t1 * 16 + r1) = make_float4(acc0, acc1, acc2, acc3);
  __syncthreads();
  const int nq = HD >> 2;
  for (int item = tid; item < ntok * nq; item += kGate2Threads) {
    const int t = item / nq, j = (item - t * nq) * 4;
    float4 u = bias ? *reinterpret_cast<const float4*>(bias + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float* lr = low + t * 16;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float l = lr[r];
      const float4 w = *reinterpret_cast<const float4*>(wu + r * HD + j);
      u.x = fmaf(l, w.x, u.x);
      u.y = fmaf(l, w.y, u.y);
      u.z = fmaf(l, w.z, u.z);
      u.w = fmaf(l, w.w, u.w);
    }
    *reinterpret_cast<float4*>(g + (tok0 + t) * HD + j) =
        make_float4(logsigmoid_fast(u.x) * inv_tau, logsigmoid_fast(u.y) * inv_tau,
                    logsigmoid_fast(u.z) * inv_tau, logsigmoid_fast(u.w) * inv_tau);
  }
}

inline size_t gate_tiled_smem(int HD) {
  return sizeof(float) * ((size_t)kGate2Tok * (kGate2Slab + 4) + kGate2Slab * 16 + kGate2Tok * 16 +
                          16 * (size_t)HD);
}

}  // namespace gtr

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

}  // namespace gtr

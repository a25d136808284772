// scan_kernel.cuh -- K3: the light sequential pass over segment-boundary
// states (GTR article, 方法详解 §4: "the chunk-boundary state carried from
// chunk to chunk is tiny and is passed forward sequentially with contiguous,
// coalesced accesses").
//
// One thread per state element (b, h, i, j); consecutive threads own
// consecutive j, so every load and store is a coalesced 128-byte line.  For
// each (b, h) the segments are visited in scan order:
//     S_in[0] = 0,   S_in[s+1] = A_s[i] * S_in[s] + dS_s[i][j]
// where dS_s is the state segment s produces from a zero start and
// A_s = exp(L_s) its decay factor (L_s = the segment's summed log-gate), both
// written by the summary stage.  The result overwrites dS in place (exclusive form: the
// state each segment starts from) or, with `inclusive`, the state each segment
// ends with.  The loads of a group of up to 32 segments are all issued before
// any store, so one memory latency covers the whole group and the dependent
// chain is only the FMA; blocks of 128 threads spread the pass over the SMs.
#pragma once
#include "common.cuh"

namespace gtr {

constexpr int kScanThreads = 128;
constexpr int kScanGroup = 32;

__global__ void __launch_bounds__(kScanThreads)
gla_state_scan(float* __restrict__ wsS, const float* __restrict__ wsA, long long total, int nseg,
               int dk, int dv, int inclusive) {
  pdl_wait();                             // the summaries are complete
  pdl_trigger();
  const long long e = (long long)blockIdx.x * kScanThreads + threadIdx.x;
  if (e >= total) return;
  const int dkdv = dk * dv;
  const long long bh = e / dkdv;
  const int rem = (int)(e - bh * dkdv);
  const int i = rem / dv;
  float* p = wsS + (size_t)bh * nseg * dkdv + rem;
  const float* A = wsA + (size_t)bh * nseg * dk + i;
  float S = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += kScanGroup) {
    const int n = min(kScanGroup, nseg - s0);
    float dS[kScanGroup], a[kScanGroup];
#pragma unroll
    for (int u = 0; u < kScanGroup; ++u) {
      if (u < n) {
        dS[u] = p[(size_t)(s0 + u) * dkdv];
        a[u] = A[(size_t)(s0 + u) * dk];
      }
    }
#pragma unroll
    for (int u = 0; u < kScanGroup; ++u) {
      if (u < n) {
        if (!inclusive) p[(size_t)(s0 + u) * dkdv] = S;
        S = fmaf(a[u], S, dS[u]);
        if (inclusive) p[(size_t)(s0 + u) * dkdv] = S;
      }
    }
  }
}

}  // namespace gtr

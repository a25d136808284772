// scan_kernel.cuh -- K3: the light pass over segment-boundary states (GTR
// article, 方法详解 §4: the state carried across chunk boundaries is small
// and moves forward in scan order with coalesced accesses).
//
// Each state element (b, h, i, j) follows the affine recurrence
//     S_in[0] = 0,   S_in[s+1] = A_s[i] * S_in[s] + dS_s[i][j]
// over the segments in scan order, where dS_s is the state segment s produces
// from a zero start and A_s = exp(L_s) its decay factor (L_s = the segment's
// summed log-gate), both written by the summary stage.  The result overwrites
// dS in place (exclusive form: the state each segment starts from) or, with
// `inclusive`, the state each segment ends with.
//
// A block takes 32 consecutive elements (one coalesced 128-byte line per
// segment) and splits their segments into kScanParts consecutive ranges, one
// per warp.  Each warp first reduces its range to one affine map
// S -> P S + R (P the product of the range's A, R its scan from zero), the
// warps exchange the maps through shared memory, and each range then replays
// its recurrence from the state composed of the maps before it.  A range of
// up to kScanReg segments stays in registers between the two passes, so the
// whole pass costs one load latency, not one per segment.
#pragma once
#include "common.cuh"

namespace gtr {

constexpr int kScanParts = 4;
constexpr int kScanThreads = 32 * kScanParts;
constexpr int kScanReg = 12;

// at most 64 registers: eight blocks per SM, so a 16k-token, 6-head problem
// (768 blocks) is resident in one wave
__global__ void __launch_bounds__(kScanThreads, 8)
gla_state_scan(float* __restrict__ wsS, const float* __restrict__ wsA, long long total, int nseg,
               int dk, int dv, int inclusive) {
  __shared__ float mapP[kScanParts][32], mapR[kScanParts][32];
  pdl_wait();                             // the summaries are complete
  pdl_trigger();
  const int lane = threadIdx.x & 31, part = threadIdx.x >> 5;
  const long long e = (long long)blockIdx.x * 32 + lane;
  const bool live = e < total;
  const int dkdv = dk * dv;
  const long long bh = live ? e / dkdv : 0;
  const int rem = live ? (int)(e - bh * dkdv) : 0;
  const int i = rem / dv;
  float* p = wsS + (size_t)bh * nseg * dkdv + rem;
  const float* A = wsA + (size_t)bh * nseg * dk + i;
  const int len = (nseg + kScanParts - 1) / kScanParts;
  const int sa = min(nseg, part * len), sb = min(nseg, sa + len);

  // pass 1: this range as one map S -> P S + R
  float dS[kScanReg], a[kScanReg];
  float P = 1.f, R = 0.f;
  for (int s0 = sa; s0 < sb; s0 += kScanReg) {
    const int n = min(kScanReg, sb - s0);
#pragma unroll
    for (int u = 0; u < kScanReg; ++u) {
      if (u < n && live) {
        dS[u] = p[(size_t)(s0 + u) * dkdv];
        a[u] = A[(size_t)(s0 + u) * dk];
      }
    }
#pragma unroll
    for (int u = 0; u < kScanReg; ++u) {
      if (u < n && live) {
        R = fmaf(a[u], R, dS[u]);
        P *= a[u];
      }
    }
  }
  mapP[part][lane] = P;
  mapR[part][lane] = R;
  __syncthreads();
  // the state entering this range
  float S = 0.f;
  for (int r = 0; r < part; ++r) S = fmaf(mapP[r][lane], S, mapR[r][lane]);
  if (!live) return;

  // pass 2: the states, from registers when the range is one group
  for (int s0 = sa; s0 < sb; s0 += kScanReg) {
    const int n = min(kScanReg, sb - s0);
    if (sb - sa > kScanReg) {
#pragma unroll
      for (int u = 0; u < kScanReg; ++u) {
        if (u < n) {
          dS[u] = p[(size_t)(s0 + u) * dkdv];
          a[u] = A[(size_t)(s0 + u) * dk];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kScanReg; ++u) {
      if (u < n) {
        if (!inclusive) p[(size_t)(s0 + u) * dkdv] = S;
        S = fmaf(a[u], S, dS[u]);
        if (inclusive) p[(size_t)(s0 + u) * dkdv] = S;
      }
    }
  }
}

}  // namespace gtr

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
// A group of 32 consecutive elements (one coalesced 128-byte line per
// segment) has its segments split into consecutive ranges, one per warp.
// Each warp first reduces its range to one affine map S -> P S + R (P the product of the range's A, R its scan from zero), the
// warps exchange the maps through shared memory, and each range then replays
// its recurrence from the state composed of the maps before it.  A range of
// up to one register window of segments stays in registers between the two
// passes, so the whole pass costs one load latency, not one per segment.
#pragma once
#include "common.cuh"

namespace gtr {

constexpr int kScanParts = 4;             // ranges per group
constexpr int kScanPartsWide = 16;        // ranges per group for very long scans
constexpr int kScanReg = 12;              // segments per register window
constexpr int kScanRegLong = 24;          // the window of four ranges of up to 96 segments

// Pass 1 / pass 2 over `n` segments held in registers (n <= kReg); the
// full-window case is unrolled without predicates.
template <bool kFull, int kReg>
__device__ __forceinline__ void scan_window(const float* pd, const float* pa, int n, int dkdv, int dk, float (&dS)[kReg],
                                            float (&a)[kReg]) {
#pragma unroll
  for (int u = 0; u < kReg; ++u) {
    if (kFull || u < n) {
      dS[u] = pd[u * dkdv];
      a[u] = pa[u * dk];
    }
  }
}

// at most 64 registers, 1024 threads per SM (128 registers and 512 threads
// with the long window).  A block holds kGroups groups of
// 32 elements, each group's segments split into kParts ranges (one warp
// each): four ranges of one group per block, so a 16k-token, 6-head problem
// (768 blocks) is resident in one wave; sixteen ranges per group when the
// segments are many, so that each range stays short; one range for each of
// four groups when the segments fit one register window, so that problems of
// many short sequences need a quarter of the blocks
template <int kParts, int kGroups, int kReg = kScanReg>
__global__ void __launch_bounds__(32 * kParts * kGroups, 32 / (kParts * kGroups) * kScanReg / kReg)
gla_state_scan(float* __restrict__ wsS, const float* __restrict__ wsA, long long total, int nseg,
               int dk, int dv, int inclusive) {
  constexpr int kScanParts = kParts;
  __shared__ float mapP[kGroups][kScanParts][32], mapR[kGroups][kScanParts][32];
  pdl_wait();                             // the summaries are complete
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = warp / kScanParts, part = warp - grp * kScanParts;
  // 32 elements per group; dk * dv is a multiple of 32, so a group stays in one (b, h)
  const int dkdv = dk * dv;
  const int per_bh = dkdv >> 5;
  const long long gi = (long long)blockIdx.x * kGroups + grp;
  const long long bh = gi / per_bh;
  const int rem = (int)(gi - bh * per_bh) * 32 + lane;
  const bool live = gi * 32 + lane < total;
  const int i = rem / dv;
  const int len = (nseg + kScanParts - 1) / kScanParts;
  const int sa = min(nseg, part * len), sb = min(nseg, sa + len);
  const int n = sb - sa;
  // this range's first segment; offsets within a (b, h) fit in 32 bits (nseg dk dv < 2^31)
  float* p = wsS + (size_t)bh * nseg * dkdv + (size_t)sa * dkdv + rem;
  const float* A = wsA + (size_t)bh * nseg * dk + (size_t)sa * dk + i;

  // pass 1: this range as one map S -> P S + R
  float dS[kReg], a[kReg];
  float P = 1.f, R = 0.f;
  if (live) {
    for (int s0 = 0; s0 < n; s0 += kReg) {
      const int m = min(kReg, n - s0);
      if (m == kReg) scan_window<true, kReg>(p + s0 * dkdv, A + s0 * dk, m, dkdv, dk, dS, a);
      else scan_window<false, kReg>(p + s0 * dkdv, A + s0 * dk, m, dkdv, dk, dS, a);
#pragma unroll
      for (int u = 0; u < kReg; ++u) {
        if (u < m) {
          R = fmaf(a[u], R, dS[u]);
          P *= a[u];
        }
      }
    }
  }
  mapP[grp][part][lane] = P;
  mapR[grp][part][lane] = R;
  __syncthreads();
  if (!live) return;
  // the state entering this range
  float S = 0.f;
  for (int r = 0; r < part; ++r) S = fmaf(mapP[grp][r][lane], S, mapR[grp][r][lane]);

  // pass 2: the states, from registers when the range is one window
  for (int s0 = 0; s0 < n; s0 += kReg) {
    const int m = min(kReg, n - s0);
    if (n > kReg) scan_window<false, kReg>(p + s0 * dkdv, A + s0 * dk, m, dkdv, dk, dS, a);
    float* q = p + s0 * dkdv;
    if (inclusive) {
#pragma unroll
      for (int u = 0; u < kReg; ++u)
        if (u < m) {
          S = fmaf(a[u], S, dS[u]);
          q[u * dkdv] = S;
        }
    } else {
#pragma unroll
      for (int u = 0; u < kReg; ++u)
        if (u < m) {
          q[u * dkdv] = S;
          S = fmaf(a[u], S, dS[u]);
        }
    }
  }
}

}  // namespace gtr

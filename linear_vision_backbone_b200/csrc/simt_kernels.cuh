// simt_kernels.cuh -- the exact fp32 CUDA-core path of the Key-only GLA.
//
// Stage layout follows the chunkwise operator of the GTR article (方法详解 §4):
//   K2 summary : for every segment (a run of consecutive chunks) of one
//                (batch, head), the state the segment produces from a zero
//                start, dS_seg, and its total log-decay L_seg = sum of g;
//   K3 scan    : the light sequential pass over segment-boundary states
//                (scan_kernel.cuh);
//   K4 output  : every segment restarts from its incoming state and emits
//                o_s = q_s S_s, then RMSNorm x SiLU(z) in the epilogue.
// Inside a segment this path applies the recurrence of 方法详解 §1 token by
// token, S = diag(exp g_s) S + k_s^T v_s, with the dk x dv state spread over
// the 256 threads of the block (thread -> column j = tid % dv and the ROWS
// consecutive rows i = (tid / dv) * ROWS + r, so that a warp reads the staged
// per-row values of a token as 16-byte broadcasts).  Every product is an fp32
// FMA: no factorisation of the decay, so no overflow whatever the gate values.
#pragma once
#include "common.cuh"

namespace gtr {

constexpr int kSimtThreads = 256;
constexpr int kSimtBatch = 16;    // tokens staged in shared memory per pass

// Shared-memory floats used by the SIMT kernels for head dims dk, dv.
__host__ __device__ inline int simt_summary_smem_floats(int dk, int dv) {
  return kSimtBatch * (3 * dk + dv);
}
__host__ __device__ inline int simt_output_smem_floats(int dk, int dv) {
  return kSimtBatch * (3 * dk + 2 * dv + (kSimtThreads / dv) * dv);
}

template <typename T>
__device__ __forceinline__ size_t token_row(int b, int t, int T_, int H, int h) {
  return ((size_t)b * T_ + t) * H + h;
}

// Four consecutive staged floats (16-byte aligned) when ROWS is a multiple of
// four, else one at a time.
template <int ROWS>
__device__ __forceinline__ void rows4(const float* p, int r, float (&x)[4]) {
  if constexpr (ROWS % 4 == 0) {
    const float4 f = *reinterpret_cast<const float4*>(p + r);
    x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = (r + e < ROWS) ? p[r + e] : 0.f;
  }
}

template <typename T, int ROWS>
__global__ void __launch_bounds__(kSimtThreads)
gla_summary_simt(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ g,
                 float* __restrict__ wsS, float* __restrict__ wsA, int H, int T_, int gh, int gw,
                 int dk, int dv, int dir, int chunk, int nseg) {
  extern __shared__ float sm[];
  float* ks = sm;                            // [batch][dk]
  float* as = ks + kSimtBatch * dk;          // [batch][dk]  exp(g)
  float* gs = as + kSimtBatch * dk;          // [batch][dk]  g
  float* vs = gs + kSimtBatch * dk;          // [batch][dv]
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int d = dir_of_batch(dir, b);
  if (d < 0 || d > 3) { if (threadIdx.x == 0) gtr_flag(kStatusBadDir); return; }
  const int tid = threadIdx.x;
  const int j = tid % dv, rg = tid / dv;
  const int nc = (T_ + chunk - 1) / chunk;
  const int s0 = seg_first_chunk(seg, nc, nseg) * chunk;
  const int s1 = min(T_, seg_first_chunk(seg + 1, nc, nseg) * chunk);
  float S[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) S[r] = 0.f;
  float lsum = 0.f;
  for (int sb = s0; sb < s1; sb += kSimtBatch) {
    const int nb = min(kSimtBatch, s1 - sb);
    __syncthreads();
    for (int idx = tid; idx < nb * dk; idx += kSimtThreads) {
      const int u = idx / dk, i = idx - u * dk;
      const size_t row = token_row<T>(b, scan_to_grid(d, sb + u, T_, gh, gw), T_, H, h);
      const float gg = g[row * dk + i];
      ks[u * dk + i] = ld_f(k + row * dk + i);
      gs[u * dk + i] = gg;
      as[u * dk + i] = expf(gg);
    }
    for (int idx = tid; idx < nb * dv; idx += kSimtThreads) {
      const int u = idx / dv, jj = idx - u * dv;
      const size_t row = token_row<T>(b, scan_to_grid(d, sb + u, T_, gh, gw), T_, H, h);
      vs[u * dv + jj] = ld_f(v + row * dv + jj);
    }
    __syncthreads();
    for (int u = 0; u < nb; ++u) {
      const float vj = vs[u * dv + j];
      const float* ar = as + u * dk + rg * ROWS;
      const float* kr = ks + u * dk + rg * ROWS;
#pragma unroll
      for (int r = 0; r < ROWS; r += 4) {
        float a4[4], k4[4];
        rows4<ROWS>(ar, r, a4);
        rows4<ROWS>(kr, r, k4);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (r + e < ROWS) S[r + e] = fmaf(a4[e], S[r + e], k4[e] * vj);
      }
    }
    if (tid < dk)
      for (int u = 0; u < nb; ++u) lsum += gs[u * dk + tid];
  }
  float* outS = wsS + ((size_t)bh * nseg + seg) * dk * dv;
#pragma unroll
  for (int r = 0; r < ROWS; ++r) outS[(size_t)(rg * ROWS + r) * dv + j] = S[r];
  if (tid < dk) wsA[((size_t)bh * nseg + seg) * dk + tid] = expf(lsum);   // segment decay factor
}

template <typename T, int ROWS>
__global__ void __launch_bounds__(kSimtThreads)
gla_output_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ g, const T* __restrict__ z, const float* __restrict__ w,
                const float* __restrict__ wsS, T* __restrict__ out, int H, int T_, int gh, int gw,
                int dk, int dv, int dir, int chunk, int nseg) {
  extern __shared__ float sm[];
  const int nrg = kSimtThreads / dv;
  float* qs = sm;                            // [batch][dk]
  float* ks = qs + kSimtBatch * dk;          // [batch][dk]
  float* as = ks + kSimtBatch * dk;          // [batch][dk]
  float* vs = as + kSimtBatch * dk;          // [batch][dv]
  float* zs = vs + kSimtBatch * dv;          // [batch][dv]
  float* po = zs + kSimtBatch * dv;          // [batch][nrg][dv] partial outputs
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / H, h = bh - b * H;
  const int d = dir_of_batch(dir, b);
  if (d < 0 || d > 3) { if (threadIdx.x == 0) gtr_flag(kStatusBadDir); return; }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = tid % dv, rg = tid / dv;
  const int nc = (T_ + chunk - 1) / chunk;
  const int s0 = seg_first_chunk(seg, nc, nseg) * chunk;
  const int s1 = min(T_, seg_first_chunk(seg + 1, nc, nseg) * chunk);
  const float* inS = wsS + ((size_t)bh * nseg + seg) * dk * dv;
  float S[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) S[r] = inS[(size_t)(rg * ROWS + r) * dv + j];
  for (int sb = s0; sb < s1; sb += kSimtBatch) {
    const int nb = min(kSimtBatch, s1 - sb);
    __syncthreads();
    for (int idx = tid; idx < nb * dk; idx += kSimtThreads) {
      const int u = idx / dk, i = idx - u * dk;
      const size_t row = token_row<T>(b, scan_to_grid(d, sb + u, T_, gh, gw), T_, H, h);
      qs[u * dk + i] = ld_f(q + row * dk + i);
      ks[u * dk + i] = ld_f(k + row * dk + i);
      as[u * dk + i] = expf(g[row * dk + i]);
    }
    for (int idx = tid; idx < nb * dv; idx += kSimtThreads) {
      const int u = idx / dv, jj = idx - u * dv;
      const size_t row = token_row<T>(b, scan_to_grid(d, sb + u, T_, gh, gw), T_, H, h);
      vs[u * dv + jj] = ld_f(v + row * dv + jj);
      zs[u * dv + jj] = ld_f(z + row * dv + jj);
    }
    __syncthreads();
    for (int u = 0; u < nb; ++u) {
      const float vj = vs[u * dv + j];
      const float* ar = as + u * dk + rg * ROWS;
      const float* kr = ks + u * dk + rg * ROWS;
      const float* qr = qs + u * dk + rg * ROWS;
      float part = 0.f;
#pragma unroll
      for (int r = 0; r < ROWS; r += 4) {
        float a4[4], k4[4], q4[4];
        rows4<ROWS>(ar, r, a4);
        rows4<ROWS>(kr, r, k4);
        rows4<ROWS>(qr, r, q4);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (r + e < ROWS) {
            S[r + e] = fmaf(a4[e], S[r + e], k4[e] * vj);
            part = fmaf(q4[e], S[r + e], part);
          }
      }
      po[(u * nrg + rg) * dv + j] = part;
    }
    __syncthreads();
    // epilogue: one warp per token -- reduce partials, RMSNorm over dv, x w x SiLU(z)
    for (int u = warp; u < nb; u += kSimtThreads / 32) {
      float o[4];
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jx = lane + 32 * c;
        float acc = 0.f;
        if (jx < dv)
          for (int r = 0; r < nrg; ++r) acc += po[(u * nrg + r) * dv + jx];
        o[c] = acc;
        ss = fmaf(acc, acc, ss);
      }
      ss = warp_sum(ss);
      const float inv = 1.0f / sqrtf(ss / (float)dv + kRmsEps);
      const size_t row = token_row<T>(b, scan_to_grid(d, sb + u, T_, gh, gw), T_, H, h);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jx = lane + 32 * c;
        if (jx < dv) {
          const float wj = w ? __ldg(w + jx) : 1.0f;
          out[row * dv + jx] = Elem<T>::from_f(o[c] * inv * wj * silu_f(zs[u * dv + jx]));
        }
      }
    }
  }
}

}  // namespace gtr

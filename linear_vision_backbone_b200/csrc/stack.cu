// stack.cu -- a stack of GTR blocks on one stream (GTR article, 方法详解 §1:
// a single-scale topology of 12 blocks, each built around the Key-only GLA,
// the scan direction cycling LR, RL, TB, BT from one block to the next; 方法详解
// §2: the Spatial SwiGLU feed-forward half).  The pages leave a block's wiring
// blank; it is taken as pre-normalised with a residual around each half:
//     a = RMSNorm(x) * gamma_mixer            (16-bit)
//     q, k, v, z = a W_in;  g = gate(a)        (one GEMM with four outputs; K1)
//     x += GLA(q, k, v, g, z) W_o              (K2 -> K3 -> K4, then a GEMM)
//     c = RMSNorm(x) * gamma_ffn
//     x += S-SwiGLU(c)                         (GEMM, mixing kernel, GEMM)
// with the residual stream x in fp32 and every other activation in the
// stack's 16-bit type.  The one kernel of this file adds a projection's
// output to the residual stream and normalises the sum for the next half in
// the same pass; every other step is a library entry point (gtr_gla.cu,
// sswiglu.cu).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gtr_gla.h"
#include "gemm_tc.cuh"

namespace {

constexpr int kNormThreads = 256;                 // 8 rows (one per warp) per block
constexpr int kNormRows = kNormThreads / 32;
constexpr float kNormEps = 1e-5f;

__device__ __forceinline__ float4 load4(const __half* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&a);
  r.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = r;
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&a);
  r.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = r;
}

// One warp per token row of width dm (a multiple of 4, at most 32 * 4 * kMaxUnits):
//   x[row] += y[row]                      (when y is given; fp32 sum)
//   out[row] = x[row] / sqrt(mean(x[row]^2) + eps) * gamma   (when out is given)
// The row stays in registers between the two steps, so x is read and
// written once and y read once: 12 bytes per element at 16-bit y and out.
template <typename T, int kMaxUnits>
__global__ void __launch_bounds__(kNormThreads) add_rmsnorm_kernel(float* __restrict__ x,
                                                                   const T* __restrict__ y,
                                                                   const float* __restrict__ gamma,
                                                                   T* __restrict__ out, int N, int dm) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kNormRows + (threadIdx.x >> 5);
  if (row >= N) return;
  const int units = dm >> 2;
  float4* xr = reinterpret_cast<float4*>(x + row * dm);
  float4 r[kMaxUnits];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxUnits; ++j) {
    const int u = lane + 32 * j;
    if (u < units) {
      float4 v = xr[u];
      if (y) {
        const float4 a = load4(y + row * dm + 4 * u);
        v.x += a.x; v.y += a.y; v.z += a.z; v.w += a.w;
        xr[u] = v;
      }
      r[j] = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  }
  if (!out) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / (float)dm + kNormEps);
  const float4* gr = reinterpret_cast<const float4*>(gamma);
#pragma unroll
  for (int j = 0; j < kMaxUnits; ++j) {
    const int u = lane + 32 * j;
    if (u < units) {
      const float4 w = gr[u];
      const float4 v = r[j];
      store4(out + row * dm + 4 * u, make_float4(v.x * inv * w.x, v.y * inv * w.y, v.z * inv * w.z,
                                                 v.w * inv * w.w));
    }
  }
}

constexpr int kMaxUnits = 8;                       // dm <= 1024
constexpr int kMaxStackDm = 32 * 4 * kMaxUnits;

int add_rmsnorm(int dtype, float* x, const void* y, const float* gamma, void* out, int N, int dm,
                cudaStream_t st) {
  const unsigned blocks = (unsigned)((N + kNormRows - 1) / kNormRows);
  if (dtype == GTR_F16)
    add_rmsnorm_kernel<__half, kMaxUnits><<<blocks, kNormThreads, 0, st>>>(x, (const __half*)y, gamma,
                                                                          (__half*)out, N, dm);
  else
    add_rmsnorm_kernel<__nv_bfloat16, kMaxUnits><<<blocks, kNormThreads, 0, st>>>(
        x, (const __nv_bfloat16*)y, gamma, (__nv_bfloat16*)out, N, dm);
  return cudaGetLastError() == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Workspace carve-up: the normalised input (shared by both halves), q, k, v,
// z, g, the GLA output, a projection output, the S-SwiGLU expansion and
// hidden activation.
struct Carve {
  size_t a, q, k, v, z, g, y, p, u, h, total;
};

Carve carve(long long N, int dm, int H, int dk, int dv, int C) {
  Carve c{};
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t at = off; off += align256(bytes); return at; };
  c.a = take((size_t)N * dm * 2);
  c.q = take((size_t)N * H * dk * 2);
  c.k = take((size_t)N * H * dk * 2);
  c.v = take((size_t)N * H * dv * 2);
  c.z = take((size_t)N * H * dv * 2);
  c.g = take((size_t)N * H * dk * 4);
  c.y = take((size_t)N * H * dv * 2);
  c.p = take((size_t)N * dm * 2);
  c.u = take((size_t)N * 2 * C * 2);
  c.h = take((size_t)N * C * 2);
  c.total = off;
  return c;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

GTR_API size_t gtr_stack_workspace_bytes(int B, int grid_h, int grid_w, int d_model, int H, int dk, int dv,
                                         int hidden) {
  if (B < 0 || grid_h < 0 || grid_w < 0 || d_model < 0 || H < 0 || dk < 0 || dv < 0 || hidden < 0) return 0;
  return carve((long long)B * grid_h * grid_w, d_model, H, dk, dv, hidden).total;
}

GTR_API gtr_status_t gtr_stack_fwd(float* x, const gtr_block_weights* blocks, int nblocks, const int* dirs,
                                   int B, int grid_h, int grid_w, int d_model, int H, int dk, int dv,
                                   int hidden, float tau, int chunk, int dtype, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (nblocks < 0 || B < 0 || grid_h < 0 || grid_w < 0 || d_model < 0 || H < 0 || dk < 0 || dv < 0 ||
      hidden < 0)
    return GTR_ERR_INVALID_ARG;
  if (dtype != GTR_F16 && dtype != GTR_BF16) return dtype == GTR_F32 ? GTR_ERR_UNSUPPORTED : GTR_ERR_INVALID_ARG;
  if (!(tau > 0.0f) || !(tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  const long long N = (long long)B * grid_h * grid_w;
  if (N >= (1LL << 31)) return GTR_ERR_INVALID_ARG;
  if (nblocks == 0 || N == 0) return GTR_OK;
  if (d_model % 8 != 0 || d_model > kMaxStackDm || H == 0 || dk == 0 || dv == 0) return GTR_ERR_UNSUPPORTED;
  // every stage's own shape checks, run first on empty problems (they launch
  // nothing), so that an unsupported shape is refused before any block runs
  int rc;
  if ((rc = gtr_gate_fwd_packed(nullptr, dtype, nullptr, nullptr, nullptr, 0, 0, d_model, 16, H, dk, tau,
                                stream)))
    return (gtr_status_t)rc;
  if ((rc = gtr_gla_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, H, grid_h, grid_w,
                        dk, dv, 0, chunk, dtype, stream)))
    return (gtr_status_t)rc;
  if ((rc = gtr_sswiglu_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, 0, grid_h,
                            grid_w, d_model, hidden, 3, dtype, stream)))
    return (gtr_status_t)rc;
  if (!x || !blocks || !workspace) return GTR_ERR_INVALID_ARG;
  const Carve c = carve(N, d_model, H, dk, dv, hidden);
  if (workspace_bytes < c.total) return GTR_ERR_NO_MEMORY;
  if (!aligned16(x) || !aligned16(workspace)) return GTR_ERR_ALIGNMENT;
  for (int i = 0; i < nblocks; ++i) {
    const gtr_block_weights& w = blocks[i];
    if (!w.norm_mixer || !w.w_in || !w.gate_packed || !w.w_o || !w.norm_ffn || !w.w_e || !w.conv_w || !w.w_p)
      return GTR_ERR_INVALID_ARG;
    if (!aligned16(w.norm_mixer) || !aligned16(w.w_in) || !aligned16(w.gate_packed) ||
        (w.gate_bias && !aligned16(w.gate_bias)) || (w.gla_norm && !aligned16(w.gla_norm)) ||
        !aligned16(w.w_o) || !aligned16(w.norm_ffn) || !aligned16(w.w_e) || !aligned16(w.conv_w) ||
        (w.conv_b && !aligned16(w.conv_b)) || !aligned16(w.w_p))
      return GTR_ERR_ALIGNMENT;
    if (dirs && (dirs[i] < GTR_LR || dirs[i] > GTR_BT)) return GTR_ERR_INVALID_ARG;
  }
  char* ws = (char*)workspace;
  void *a = ws + c.a, *q = ws + c.q, *k = ws + c.k, *v = ws + c.v, *z = ws + c.z, *y = ws + c.y, *p = ws + c.p;
  void *u = ws + c.u, *h = ws + c.h;
  float* g = (float*)(ws + c.g);
  const cudaStream_t st = (cudaStream_t)stream;
  const int n = (int)N;
  if ((rc = add_rmsnorm(dtype, x, nullptr, blocks[0].norm_mixer, a, n, d_model, st))) return (gtr_status_t)rc;
  for (int i = 0; i < nblocks; ++i) {
    const gtr_block_weights& w = blocks[i];
    const int dir = dirs ? dirs[i] : i % 4;
    if ((rc = gtr_mixer_in_proj(a, w.w_in, q, k, v, z, B, grid_h * grid_w, d_model, H, dk, dv, dtype, stream)))
      return (gtr_status_t)rc;
    if ((rc = gtr_gate_fwd_packed(a, dtype, w.gate_packed, w.gate_bias, g, B, grid_h * grid_w, d_model, 16, H,
                                  dk, tau, stream)))
      return (gtr_status_t)rc;
    if ((rc = gtr_gla_fwd(q, k, v, g, z, w.gla_norm, y, B, H, grid_h, grid_w, dk, dv, dir, chunk, dtype,
                          stream)))
      return (gtr_status_t)rc;
    if ((rc = gtr_mixer_out_proj(y, w.w_o, p, N, H * dv, d_model, dtype, stream))) return (gtr_status_t)rc;
    if ((rc = add_rmsnorm(dtype, x, p, w.norm_ffn, a, n, d_model, st))) return (gtr_status_t)rc;
    if ((rc = gtr_sswiglu_fwd(a, w.w_e, w.conv_w, w.conv_b, w.w_p, u, h, p, B, grid_h, grid_w, d_model, hidden,
                              3, dtype, stream)))
      return (gtr_status_t)rc;
    const bool last = i + 1 == nblocks;
    if ((rc = add_rmsnorm(dtype, x, p, last ? nullptr : blocks[i + 1].norm_mixer, last ? nullptr : a, n,
                          d_model, st)))
      return (gtr_status_t)rc;
  }
  return GTR_OK;
}

}  // extern "C"

// sswiglu.cu -- the Spatial SwiGLU feed-forward block of a GTR layer (GTR
// article, 方法详解 §2): the channel expansion u = x W_in gives a gate branch and
// a value branch; the value branch, laid out as the 2-D token grid, is mixed by
// a depthwise convolution, multiplied by SiLU of the gate branch, and the
// product is projected back to the model width:
//     h = SiLU(u_gate) * (DWConv_kxk(u_value) + b),     y = h W_out.
// The pages leave the kernel size blank; this library takes k = 3 with zero
// padding (output grid = input grid), the smallest kernel that mixes every
// token with its eight neighbours.
//
// The mixing step is one HBM-bound kernel (it reads u once and writes h once;
// the halo columns and rows are re-read from L2);
// the two projections are dense GEMMs on the library's tensor-core GEMM
// (gemm_tc.cuh), cuBLAS only for shapes outside its tensor maps.
//
// Layout: u [B, gh*gw, 2C] (gate channels [0, C), value channels [C, 2C)),
// h [B, gh*gw, C], token t = row * gw + column, all rows of one 16-bit type;
// weights [3, 3, C] and bias [C] fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gtr_gla.h"
#include "gemm_tc.cuh"
#include "mixer_proj.cuh"

namespace {

constexpr int kMixThreads = 128;

// Eight consecutive channels (16 bytes of storage) rounded from fp32.
__device__ __forceinline__ uint4 narrow8(const float (&f)[8], const __half*) {
  uint4 r;
  __half2* p = reinterpret_cast<__half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return r;
}
__device__ __forceinline__ uint4 narrow8(const float (&f)[8], const __nv_bfloat16*) {
  uint4 r;
  __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return r;
}

// Two fp32 lanes per instruction (sm_100 fma.rn.f32x2): a pair of
// floats in one 64-bit register, the first in the low half.
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t pk2(float a, float b) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 up2(f2_t r) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
  return make_float2(a, b);
}
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// Eight consecutive channels as four fp32 pairs.
__device__ __forceinline__ void widen8x2(const uint4& r, const __half*, f2_t (&f)[4]) {
  const __half2* p = reinterpret_cast<const __half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(p[i]);
    f[i] = pk2(t.x, t.y);
  }
}
__device__ __forceinline__ void widen8x2(const uint4& r, const __nv_bfloat16*, f2_t (&f)[4]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[i] = pk2(t.x, t.y);
  }
}
// SiLU(g) x a for a pair: g / (1 + 2^{-g log2 e}) x a, the exponential and
// the reciprocal by the hardware approximations (relative error near 1e-7).
__device__ __forceinline__ float2 silu_times2(float2 g, float2 a) {
  const float ea = __expf(-g.x), eb = __expf(-g.y);
  return make_float2(__fdividef(g.x, 1.f + ea) * a.x, __fdividef(g.y, 1.f + eb) * a.y);
}

// A block owns a tile of kTileCols grid columns x 64 channels over a strip of
// rows [y0, y1) of one image; thread (column, octet) owns eight channels of
// one column.  The value rows (the tile's columns plus one halo column on each
// side) and the gate rows are staged in shared memory by 16-byte cp.async
// copies through a ring of kStages row slots, kStages - 1 rows ahead of the
// arithmetic, so the copies in flight cost no registers.  Slot of input row r:
// value row r and gate row r - 1.  Row r's three taps (columns x-1, x, x+1)
// feed the partial sums of output rows r+1 (kernel row 0), r (kernel row 1)
// and r-1 (kernel row 2); after row r the output row r-1 is complete and is
// gated and stored.  Rows and columns outside the grid are copied as zeros
// (a copy of source size 0 reads nothing).
constexpr int kTileCols = 16;
constexpr int kOcts = 8;                                      // 8 x 8 = 64 channels per tile
constexpr int kStages = 16;
constexpr int kValBytes = (kTileCols + 2) * kOcts * 16;       // 2304
constexpr int kGateBytes = kTileCols * kOcts * 16;            // 2048
constexpr int kSlotBytes = kValBytes + kGateBytes;            // 4352
static_assert(kTileCols * kOcts == kMixThreads, "one thread per (column, octet)");

__device__ __forceinline__ void cp16(unsigned char* dst, const void* src, bool valid) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <typename E>
__global__ void __launch_bounds__(kMixThreads, 3) sswiglu_mix_kernel(const E* __restrict__ u, E* __restrict__ h,
                                                                     const float* __restrict__ cw,
                                                                     const float* __restrict__ cb, int gh, int gw,
                                                                     int C, int rows, int nstrip, int ncx, int ncg) {
  extern __shared__ __align__(128) unsigned char ring[];   // kStages * kSlotBytes
  long long bid = blockIdx.x;
  const int cgi = (int)(bid % ncg);
  bid /= ncg;
  const int cxi = (int)(bid % ncx);
  bid /= ncx;
  const int s = (int)(bid % nstrip);
  const long long b = bid / nstrip;
  const int col = threadIdx.x / kOcts, oct = threadIdx.x % kOcts;
  const int x0 = cxi * kTileCols;
  const int x = x0 + col;
  const int c = cgi * (kOcts * 8) + oct * 8;
  const bool ok = c < C && x < gw;
  const int y0 = s * rows;
  const int y1 = min(y0 + rows, gh);
  const size_t ldu = 2 * (size_t)C;
  const E* ub = u + (size_t)b * gh * gw * ldu;
  E* hb = h + (size_t)b * gh * gw * C;
  const bool cok = c < C;
  const int cl = cok ? c : 0;

  // Row-0 addresses of the pieces this thread copies and stores (clamped to a
  // valid piece where the copy reads nothing); a row adds rs (input) or hrs
  // (output) elements.
  const size_t rs = (size_t)gw * ldu, hrs = (size_t)gw * C;
  const int xc = ok ? x : 0;
  const E* vcol = ub + C + cl + (size_t)xc * ldu;
  const E* vleft = ub + C + cl + (size_t)(x0 > 0 ? x0 - 1 : 0) * ldu;
  const E* vright = ub + C + cl + (size_t)(x0 + kTileCols < gw ? x0 + kTileCols : 0) * ldu;
  const E* gcol = ub + cl + (size_t)xc * ldu;
  E* hcol = hb + (size_t)xc * C + cl;

  // stage input row r (value) and output row r - 1 (gate) into slot `si`
  auto issue = [&](int r, int si) {
    unsigned char* slot = ring + si * kSlotBytes;
    const bool rok = r >= 0 && r < gh;
    const size_t ro = (size_t)(rok ? r : 0) * rs;
    cp16(slot + ((col + 1) * kOcts + oct) * 16, vcol + ro, ok && rok);
    if (col == 0) cp16(slot + oct * 16, vleft + ro, cok && rok && x0 > 0);
    if (col == kTileCols - 1)
      cp16(slot + ((kTileCols + 1) * kOcts + oct) * 16, vright + ro, cok && rok && x0 + kTileCols < gw);
    const int yg = r - 1;
    const bool gv = ok && yg >= y0 && yg < y1;
    cp16(slot + kValBytes + threadIdx.x * 16, gcol + (size_t)(gv ? yg : 0) * rs, gv);
  };

  // taps and bias of the thread's eight channels, as four channel pairs
  f2_t w[3][3][4], bias[4];
#pragma unroll
  for (int i = 0; i < 3; ++i)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const float4* p = reinterpret_cast<const float4*>(cw + (size_t)(i * 3 + j) * C + cl);
      const float4 a = __ldg(p), q = __ldg(p + 1);
      w[i][j][0] = pk2(a.x, a.y); w[i][j][1] = pk2(a.z, a.w);
      w[i][j][2] = pk2(q.x, q.y); w[i][j][3] = pk2(q.z, q.w);
    }
  if (cb) {
    const float4* p = reinterpret_cast<const float4*>(cb + cl);
    const float4 a = __ldg(p), q = __ldg(p + 1);
    bias[0] = pk2(a.x, a.y); bias[1] = pk2(a.z, a.w); bias[2] = pk2(q.x, q.y); bias[3] = pk2(q.z, q.w);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) bias[k] = pk2(0.f, 0.f);
  }

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (y0 - 1 + i <= y1) issue(y0 - 1 + i, i);
    cp_commit();
  }
  f2_t acc_prev[4], acc_cur[4];    // partial sums of output rows r-1 and r (channel pairs)
#pragma unroll
  for (int k = 0; k < 4; ++k) acc_prev[k] = acc_cur[k] = bias[k];
  static_assert((kStages & (kStages - 1)) == 0, "ring index by mask");
  for (int r = y0 - 1, si = 0; r <= y1; ++r, si = (si + 1) & (kStages - 1)) {
    cp_wait<kStages - 2>();
    __syncthreads();
    const unsigned char* slot = ring + si * kSlotBytes;
    f2_t vl[4], vm[4], vr[4];
    widen8x2(*reinterpret_cast<const uint4*>(slot + (col * kOcts + oct) * 16), (const E*)nullptr, vl);
    widen8x2(*reinterpret_cast<const uint4*>(slot + ((col + 1) * kOcts + oct) * 16), (const E*)nullptr, vm);
    widen8x2(*reinterpret_cast<const uint4*>(slot + ((col + 2) * kOcts + oct) * 16), (const E*)nullptr, vr);
    f2_t acc_next[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc_next[k] = fma2(w[0][2][k], vr[k], fma2(w[0][1][k], vm[k], fma2(w[0][0][k], vl[k], bias[k])));
      acc_cur[k] = fma2(w[1][2][k], vr[k], fma2(w[1][1][k], vm[k], fma2(w[1][0][k], vl[k], acc_cur[k])));
      acc_prev[k] = fma2(w[2][2][k], vr[k], fma2(w[2][1][k], vm[k], fma2(w[2][0][k], vl[k], acc_prev[k])));
    }
    const int y = r - 1;   // output row completed by input row r
    if (ok && y >= y0) {
      f2_t gt[4];
      widen8x2(*reinterpret_cast<const uint4*>(slot + kValBytes + threadIdx.x * 16), (const E*)nullptr, gt);
      float o[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 v = silu_times2(up2(gt[k]), up2(acc_prev[k]));
        o[2 * k] = v.x;
        o[2 * k + 1] = v.y;
      }
      *reinterpret_cast<uint4*>(hcol + (size_t)y * hrs) = narrow8(o, (const E*)nullptr);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc_prev[k] = acc_cur[k];
      acc_cur[k] = acc_next[k];
    }
    // the slot of row r - 1, read by every thread before this iteration's barrier
    if (r + kStages - 1 <= y1) issue(r + kStages - 1, (si + kStages - 1) & (kStages - 1));
    cp_commit();
  }
  cp_wait<0>();
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int sswiglu_check(int B, int gh, int gw, int C, int ksize, int dtype) {
  if (B < 0 || gh < 0 || gw < 0 || C < 0) return GTR_ERR_INVALID_ARG;
  if (dtype < 0 || dtype > 2) return GTR_ERR_INVALID_ARG;
  if (ksize <= 0 || ksize % 2 == 0) return GTR_ERR_INVALID_ARG;
  if ((long long)gh * gw >= (1LL << 31) || (long long)B * gh * gw >= (1LL << 31)) return GTR_ERR_INVALID_ARG;
  if (ksize != 3) return GTR_ERR_UNSUPPORTED;
  if (dtype == GTR_F32) return GTR_ERR_UNSUPPORTED;
  if (C % 8 != 0) return GTR_ERR_UNSUPPORTED;
  return GTR_OK;
}

// Strips per image: as many as keep every block of the launch resident at
// once (one wave, at the kernel's occupancy), at least one; each strip
// re-reads two halo rows.
template <typename E>
int mix_launch(const void* u, const float* cw, const float* cb, void* h, int B, int gh, int gw, int C,
               cudaStream_t st) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GTR_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  constexpr int smem = kStages * kSlotBytes;
  static bool attr_done[64];
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(sswiglu_mix_kernel<E>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return GTR_ERR_CUDA;
    attr_done[dev] = true;
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sswiglu_mix_kernel<E>, kMixThreads, smem) !=
          cudaSuccess ||
      per_sm <= 0)
    per_sm = 1;
  const int ncx = (gw + kTileCols - 1) / kTileCols;
  const int ncg = (C + kOcts * 8 - 1) / (kOcts * 8);
  const long long tiles = (long long)B * ncx * ncg;
  const long long slots = (long long)sms * per_sm;
  long long nstrip = slots / tiles;
  nstrip = nstrip < 1 ? 1 : (nstrip > gh ? gh : nstrip);
  const int rows = (int)((gh + nstrip - 1) / nstrip);
  const int ns = (gh + rows - 1) / rows;
  const long long blocks = tiles * ns;
  if (blocks > 0x7fffffffLL) return GTR_ERR_INVALID_ARG;
  sswiglu_mix_kernel<E><<<(unsigned)blocks, kMixThreads, smem, st>>>((const E*)u, (E*)h, cw, cb, gh, gw, C, rows,
                                                                 ns, ncx, ncg);
  return cudaGetLastError() == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

}  // namespace

extern "C" {

GTR_API gtr_status_t gtr_sswiglu_mix(const void* u, const float* conv_w, const float* conv_b, void* h, int B,
                                     int grid_h, int grid_w, int C, int ksize, int dtype, void* stream) {
  int rc = sswiglu_check(B, grid_h, grid_w, C, ksize, dtype);
  if (rc) return (gtr_status_t)rc;
  if (B == 0 || grid_h == 0 || grid_w == 0 || C == 0) return GTR_OK;
  if (!u || !conv_w || !h) return GTR_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(conv_w) || !aligned16(h) || (conv_b && !aligned16(conv_b)))
    return GTR_ERR_ALIGNMENT;
  {  // h is written while u is still being read by other blocks: the two must not overlap
    const uintptr_t u0 = (uintptr_t)u, h0 = (uintptr_t)h;
    const uintptr_t tok = (uintptr_t)B * grid_h * grid_w;
    const uintptr_t u1 = u0 + tok * 2 * C * 2, h1 = h0 + tok * C * 2;
    if (u0 < h1 && h0 < u1) return GTR_ERR_INVALID_ARG;
  }
  const cudaStream_t st = (cudaStream_t)stream;
  rc = dtype == GTR_F16 ? mix_launch<__half>(u, conv_w, conv_b, h, B, grid_h, grid_w, C, st)
                        : mix_launch<__nv_bfloat16>(u, conv_w, conv_b, h, B, grid_h, grid_w, C, st);
  return (gtr_status_t)rc;
}

GTR_API gtr_status_t gtr_sswiglu_fwd(const void* x, const void* w_in, const float* conv_w, const float* conv_b,
                                     const void* w_out, void* u, void* h, void* y, int B, int grid_h, int grid_w,
                                     int d_model, int C, int ksize, int dtype, void* stream) {
  int rc = sswiglu_check(B, grid_h, grid_w, C, ksize, dtype);
  if (rc) return (gtr_status_t)rc;
  if (d_model < 0) return GTR_ERR_INVALID_ARG;
  if (B == 0 || grid_h == 0 || grid_w == 0 || d_model == 0) return GTR_OK;
  if (!x || !w_in || !conv_w || !w_out || !u || !h || !y) return GTR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_in) || !aligned16(conv_w) || !aligned16(w_out) || !aligned16(u) ||
      !aligned16(h) || !aligned16(y) || (conv_b && !aligned16(conv_b)))
    return GTR_ERR_ALIGNMENT;
  if (2LL * C >= (1LL << 31)) return GTR_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GTR_ERR_CUDA;
  const cudaStream_t st = (cudaStream_t)stream;
  const cudaDataType dt = dtype == GTR_F16 ? CUDA_R_16F : CUDA_R_16BF;
  const int N = B * grid_h * grid_w;
  if (C == 0) return cudaMemsetAsync(y, 0, (size_t)N * d_model * 2, st) == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
  // the expansion and the projection on our tensor-core GEMM; cuBLAS for the
  // shapes its tensor maps cannot address
  void* ou[1] = {u};
  rc = gtr::gemm_tc(dtype, x, d_model, w_in, 2 * C, ou, 1, 2 * C, 2 * C, N, 2 * C, d_model, st);
  if (rc == GTR_ERR_UNSUPPORTED)
    rc = gtr::blas_gemm_rowmajor(dev, st, dt, x, d_model, w_in, 2 * C, u, 2 * C, N, d_model, 2 * C);
  if (rc) return (gtr_status_t)rc;
  if ((rc = gtr_sswiglu_mix(u, conv_w, conv_b, h, B, grid_h, grid_w, C, ksize, dtype, stream)))
    return (gtr_status_t)rc;
  void* oy[1] = {y};
  rc = gtr::gemm_tc(dtype, h, C, w_out, d_model, oy, 1, d_model, d_model, N, d_model, C, st);
  if (rc == GTR_ERR_UNSUPPORTED)
    rc = gtr::blas_gemm_rowmajor(dev, st, dt, h, C, w_out, d_model, y, d_model, N, C, d_model);
  return (gtr_status_t)rc;
}

}  // extern "C"

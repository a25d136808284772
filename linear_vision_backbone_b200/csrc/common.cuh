// common.cuh -- element types, scan-order index maps and device status shared
// by the kernels of the Key-only GLA library.  Every kernel that uses them is
// in one translation unit (gtr_gla.cu), so device globals need no relocatable
// device code.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

namespace gtr {

enum DtypeId { kF32 = 0, kF16 = 1, kBF16 = 2 };
enum DirId { kLR = 0, kRL = 1, kTB = 2, kBT = 3, kRotate = 4 };

// RMSNorm epsilon of the output normalisation (the page leaves it unstated).
constexpr float kRmsEps = 1e-5f;

// Bits of the device status word.
enum StatusBits : unsigned {
  kStatusBadDir = 1u,        // a kernel met a direction outside LR/RL/TB/BT
  kStatusBadShape = 2u,      // a kernel met a shape its launch did not allow
  kStatusTmemAlloc = 4u,     // tensor-memory allocation returned an unusable address
  kStatusMbarTimeout = 8u,   // a bounded mbarrier wait ran out
};

// Segment s of nseg covers chunks [first(s), first(s + 1)) of a sequence of
// nc chunks: an even split, lengths differing by at most one chunk.
__host__ __device__ __forceinline__ int seg_first_chunk(int s, int nc, int nseg) {
  return (int)(((long long)s * nc) / nseg);
}

// Direction of batch entry b (GTR_ROTATE_BATCH cycles LR, RL, TB, BT).
__device__ __forceinline__ int dir_of_batch(int dir, int b) { return dir == kRotate ? (b & 3) : dir; }

// Scan position s -> grid index (row-major t = row*gw + col).  GTR article
// 方法详解 §1: LR raster, RL its reverse, TB column-major, BT its reverse.
__device__ __forceinline__ int scan_to_grid(int dir, int s, int T, int gh, int gw) {
  switch (dir) {
    case kLR: return s;
    case kRL: return T - 1 - s;
    case kTB: return (s % gh) * gw + s / gh;
    case kBT: { int r = T - 1 - s; return (r % gh) * gw + r / gh; }
    default: return -1;
  }
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
  static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

template <typename T> __device__ __forceinline__ float ld_f(const T* p) { return Elem<T>::to_f(*p); }

// logsigmoid in the overflow-free form min(u,0) - log1p(exp(-|u|)).
__device__ __forceinline__ float logsigmoid_f(float u) {
  return fminf(u, 0.0f) - log1pf(expf(-fabsf(u)));
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running; pdl_wait() returns once that kernel has completed and its memory
// is visible (at once for a kernel launched without the attribute).
// pdl_trigger() lets the next kernel be scheduled early; every kernel here
// calls it only after its own pdl_wait(), so a kernel that starts early can
// rely on everything before its predecessor being complete.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Launch with programmatic stream serialization (see pdl_wait); 0 on success.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? 0 : -5;
}

}  // namespace gtr

// Device status word and debug counters of this library (one per device that
// loads it).  Read and cleared by gtr_last_device_status.
static __device__ unsigned int g_gtr_status;
static __device__ unsigned long long g_gtr_exact_chunks;

__device__ __forceinline__ void gtr_flag(unsigned bits) { atomicOr(&g_gtr_status, bits); }

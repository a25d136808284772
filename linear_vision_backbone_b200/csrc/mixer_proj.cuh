// mixer_proj.cuh -- the token mixer's input and output projections, the steps
// on either side of the GLA (GTR article, 方法详解 §1: q, k, v and the output
// gate z are linear maps of the block input x; the mixer's output is mapped
// back to the model width).  Both are plain dense GEMMs,
//     C[N, n] = X[N, K] W[K, n]        (X, W, C row-major, one 16-bit type),
// run by cuBLAS with fp32 accumulation.  cuBLAS is loaded with dlopen at the
// first call, so the rest of the library neither links nor needs it.
#pragma once
#include <dlfcn.h>

#include <mutex>

#include <cublas_v2.h>

namespace gtr {

using BlasCreateFn = cublasStatus_t (*)(cublasHandle_t*);
using BlasSetStreamFn = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
using BlasGemmExFn = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                        const void*, const void*, cudaDataType, int, const void*, cudaDataType,
                                        int, const void*, void*, cudaDataType, int, cublasComputeType_t,
                                        cublasGemmAlgo_t);
using BlasGemmBatchFn = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                            const void*, const void*, cudaDataType, int, long long, const void*,
                                            cudaDataType, int, long long, const void*, void*, cudaDataType, int,
                                            long long, int, cublasComputeType_t, cublasGemmAlgo_t);
// One cuBLAS handle per device, created at its first projection call and kept
// for the life of the process (the library has no teardown entry point).
struct BlasApi {
  bool tried = false;
  void* lib = nullptr;
  BlasCreateFn create = nullptr;
  BlasSetStreamFn set_stream = nullptr;
  BlasGemmExFn gemm = nullptr;
  BlasGemmBatchFn gemm_batch = nullptr;
  cublasHandle_t handle[64] = {};
};

inline BlasApi& blas_api() {
  static BlasApi api;
  return api;
}
inline std::mutex& blas_mutex() {
  static std::mutex mu;
  return mu;
}

// The cuBLAS entry points, loaded once; false when the library is missing.
inline bool blas_load(BlasApi& a) {
  if (a.tried) return a.gemm != nullptr;
  a.tried = true;
  for (const char* name : {"libcublas.so.12", "libcublas.so"}) {
    a.lib = dlopen(name, RTLD_NOW | RTLD_LOCAL);
    if (a.lib) break;
  }
  if (!a.lib) return false;
  a.create = (BlasCreateFn)dlsym(a.lib, "cublasCreate_v2");
  a.set_stream = (BlasSetStreamFn)dlsym(a.lib, "cublasSetStream_v2");
  a.gemm = (BlasGemmExFn)dlsym(a.lib, "cublasGemmEx");
  a.gemm_batch = (BlasGemmBatchFn)dlsym(a.lib, "cublasGemmStridedBatchedEx");
  if (!a.create || !a.set_stream || !a.gemm || !a.gemm_batch) a.gemm = nullptr;
  return a.gemm != nullptr;
}

// C[N, n] = X[N, K] W[K, n] on `st`: X with row stride ldx, W with row stride
// ldw (a column block of a wider weight matrix), C with row stride ldc, all
// 16-bit of type `dt` (CUDA_R_16F / CUDA_R_16BF), fp32 accumulation.  In
// cuBLAS's column-major terms this is C^T = W^T X^T.  With batch > 1, `batch`
// such products with the same X, W and C advanced by w_step and c_step
// elements (one strided-batched call).  Returns a gtr status.
inline int blas_gemm_rowmajor(int dev, cudaStream_t st, cudaDataType dt, const void* X, int ldx, const void* W,
                              int ldw, void* C, int ldc, int N, int K, int n, int batch = 1, long long w_step = 0,
                              long long c_step = 0) {
  std::lock_guard<std::mutex> lk(blas_mutex());
  BlasApi& a = blas_api();
  if (!blas_load(a)) return -2;   // GTR_ERR_UNSUPPORTED
  if (dev < 0 || dev >= 64) return -2;
  if (!a.handle[dev] && a.create(&a.handle[dev]) != CUBLAS_STATUS_SUCCESS) {
    a.handle[dev] = nullptr;
    return -5;                    // GTR_ERR_CUDA
  }
  if (a.set_stream(a.handle[dev], st) != CUBLAS_STATUS_SUCCESS) return -5;
  const float one = 1.0f, zero = 0.0f;
  const cublasStatus_t r =
      batch == 1 ? a.gemm(a.handle[dev], CUBLAS_OP_N, CUBLAS_OP_N, n, N, K, &one, W, dt, ldw, X, dt, ldx, &zero, C,
                          dt, ldc, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT)
                 : a.gemm_batch(a.handle[dev], CUBLAS_OP_N, CUBLAS_OP_N, n, N, K, &one, W, dt, ldw, w_step, X, dt,
                                ldx, 0, &zero, C, dt, ldc, c_step, batch, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return r == CUBLAS_STATUS_SUCCESS ? 0 : -5;
}

}  // namespace gtr

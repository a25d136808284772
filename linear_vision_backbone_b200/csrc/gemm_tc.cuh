// gemm_tc.cuh -- the dense projections of a GTR layer on tcgen05 tensor cores
// (sm_100a): C = A B with A [M, K] and B [K, N] row-major, one 16-bit type,
// fp32 accumulation, C rounded to the same type.  The token mixer's input
// projection (x -> q, k, v, z), its output projection, and the Spatial SwiGLU
// expansion and projection (GTR article, 方法详解 §1 and §2) are all of this
// form.  Defined in gemm_tc.cu.
#pragma once
#include <cuda_runtime.h>

namespace gtr {

// C[o] (o < nout) receives columns [o * ncols, (o + 1) * ncols) of A B, each
// output row-major with row pitch ldc elements (nout = 1, ncols = N: one
// output).  dtype 1 = fp16, 2 = bf16.  Returns 0 on success, -2 when the shape
// is outside what the kernel's tensor maps address (row pitches and column
// blocks not multiples of 8 elements, base addresses not 16-byte aligned, a
// column block not a multiple of the 128-column tile when nout > 1), -5 on a
// CUDA error.  Launches one persistent kernel on `st`.
int gemm_tc(int dtype, const void* A, int lda, const void* B, int ldb, void* const* C, int nout, int ncols,
            int ldc, int M, int N, int K, cudaStream_t st);

}  // namespace gtr

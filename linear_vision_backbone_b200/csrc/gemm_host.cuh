// gemm_host.cuh -- host side of the projections' GEMM (gemm_tc.cuh):
// argument checks, tensor maps, the tile width and the persistent launch.
// Included once, by gtr_gla.cu, after its launch and tensor-map helpers; the
// kernel is in gemm_kernel.cuh.
#pragma once
#include "gemm_kernel.cuh"

namespace gtr {

namespace {

template <bool kBF16, int kBN>
int gemm_launch(const gemm::Params& p, const gemm::Maps& mp, unsigned grid, cudaStream_t st, int dev) {
  static bool done[kMaxDevices];
  auto kern = gemm::gemm_tc_kernel<kBF16, kBN>;
  if (int rc = ensure_smem(kern, gemm::Cfg<kBN>::kSmem, done, dev)) return rc;
  return launch_pdl(kern, dim3(grid), dim3(gemm::kThreads), gemm::Cfg<kBN>::kSmem, st, p, mp) ? GTR_ERR_CUDA
                                                                                            : GTR_OK;
}

// The CTA-pair kernel: clusters of two CTAs, as many pairs as fit on the
// device at once (asked of the occupancy calculator once per device), at most
// one per 256-row tile.  Returns GTR_ERR_UNSUPPORTED when no pair fits.
template <bool kBF16, int kBN>
int gemm_pair_launch(const gemm::Params& p, const gemm::Maps& mp, cudaStream_t st, int dev) {
  static bool done[kMaxDevices];
  static int pairs[kMaxDevices];
  auto kern = gemm::gemm_pair_kernel<kBF16, kBN>;
  constexpr int smem = gemm::PairCfg<kBN>::kSmem;
  if (int rc = ensure_smem(kern, smem, done, dev)) return rc;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pairs[dev] == 0) {
    cfg.gridDim = dim3(2 * sm_count(dev));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      (void)cudaGetLastError();
      n = -1;
    }
    pairs[dev] = n > 0 ? n : -1;
  }
  if (pairs[dev] < 0) return GTR_ERR_UNSUPPORTED;
  const long long tiles = (long long)p.mt * p.nt;
  cfg.gridDim = dim3((unsigned)(2 * (tiles < pairs[dev] ? tiles : pairs[dev])));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, p, mp) == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

}  // namespace

int gemm_tc(int dtype, const void* A, int lda, const void* B, int ldb, void* const* C, int nout, int ncols,
            int ldc, int M, int N, int K, cudaStream_t st) {
  if (dtype != GTR_F16 && dtype != GTR_BF16) return GTR_ERR_UNSUPPORTED;
  if (M <= 0 || N <= 0 || K <= 0) return GTR_OK;
  if (nout < 1 || nout > gemm::kMaxOut) return GTR_ERR_UNSUPPORTED;
  if (nout == 1) ncols = N;
  // with several outputs every 64-column store box lies in one of them
  if (nout > 1 && (ncols % 64 != 0 || (long long)nout * ncols != N)) return GTR_ERR_UNSUPPORTED;
  // tensor maps: 16-byte aligned bases and row pitches
  if (lda % 8 || ldb % 8 || ldc % 8 || ncols % 8 || !aligned16(A) || !aligned16(B)) return GTR_ERR_UNSUPPORTED;
  for (int o = 0; o < nout; ++o)
    if (!C[o] || !aligned16(C[o])) return GTR_ERR_UNSUPPORTED;
  int dev;
  if (int rc = current_device(&dev)) return rc;
  const CUtensorMapDataType dt = dtype == GTR_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  gemm::Maps mp{};
  if (int rc = tmap_2d(&mp.a, dt, A, (unsigned long long)M, (unsigned long long)K, (unsigned long long)lda * 2,
                       gemm::kBK, gemm::kBM))
    return rc;
  if (int rc = tmap_2d(&mp.b, dt, B, (unsigned long long)K, (unsigned long long)N, (unsigned long long)ldb * 2, 64,
                       gemm::kBK))
    return rc;
  for (int o = 0; o < nout; ++o)
    if (int rc = tmap_2d(&mp.c[o], dt, C[o], (unsigned long long)M, (unsigned long long)ncols,
                         (unsigned long long)ldc * 2, 64, 32))
      return rc;
  // Tile choice, as measured on the projections' shapes (16384 rows): CTA
  // pairs on 256 x 256 tiles only for deep products (K >= 1024, N whole tiles
  // of 256: 1.26 vs 1.17 PFLOP/s at K = 1024, N = 2048); at K = 384 the
  // single-CTA 128 x 256 tile is faster (27.0 vs 32.0 us at N = 2048), and
  // for N not a multiple of 256 the single-CTA 128 x 128 tile (11.0 us vs
  // 13.5 us for the 256 x 128 pair tile at N = K = 384).
  const int bn = N % 256 == 0 ? 256 : 128;
  if (bn == 256 && K >= 1024) {
    gemm::Params pp{M, N, K, nout, ncols, (M + 255) / 256, N / 256, (K + gemm::kBK - 1) / gemm::kBK};
    const int rc = dtype == GTR_BF16 ? gemm_pair_launch<true, 256>(pp, mp, st, dev)
                                     : gemm_pair_launch<false, 256>(pp, mp, st, dev);
    if (rc != GTR_ERR_UNSUPPORTED) return rc;
  }
  gemm::Params p{M, N, K, nout, ncols, (M + gemm::kBM - 1) / gemm::kBM, (N + bn - 1) / bn, (K + gemm::kBK - 1) / gemm::kBK};
  const long long tiles = (long long)p.mt * p.nt;
  const unsigned grid = (unsigned)(tiles < sm_count(dev) ? tiles : sm_count(dev));
  if (dtype == GTR_BF16)
    return bn == 256 ? gemm_launch<true, 256>(p, mp, grid, st, dev) : gemm_launch<true, 128>(p, mp, grid, st, dev);
  return bn == 256 ? gemm_launch<false, 256>(p, mp, grid, st, dev) : gemm_launch<false, 128>(p, mp, grid, st, dev);
}

}  // namespace gtr

// gemm_kernel.cuh -- the projections' GEMM C = A B on tcgen05 (see
// gemm_tc.cuh for the contract), in the gate / GLA translation unit so that
// its bounded waits report through the library's device status word.
//
// A persistent kernel: one CTA per SM walks output tiles of 128 x 128
// (tile t = blockIdx.x, + gridDim.x, ..., the N tiles of one M tile
// consecutive so that CTAs running at the same time share their A rows in L2).
// Warp 0 streams the K blocks (64 deep) of A (K-major, 128 x 64) and B
// (MN-major, 64 x 128 as two 64-column boxes) into a four-stage ring with
// tensor-map loads; warp 1's first thread issues, per K block, four
// tcgen05.mma kind::f16 (M = 128, N = 128, K = 16) into one of two TMEM
// accumulators; warps 2-5 (one TMEM lane quadrant each, thread = output row)
// read a finished accumulator 32 columns at a time, round it to the 16-bit
// type into a 128B-swizzled staging tile (two of them, so the next tile's
// epilogue overlaps this one's stores) and one thread writes it with two
// tensor-map stores.  Rows and columns past the matrix edges are zero on load
// and clipped on store.
#pragma once
#include "gate_tc.cuh"
#include "gemm_tc.cuh"
#include "tc_kernels.cuh"

namespace gtr {
namespace gemm {

using tc::saddr;
constexpr int kBM = 128, kBN = 128, kBK = 64;
constexpr int kStages = 4;
constexpr int kATile = kBM * kBK * 2;            // 16 KB
constexpr int kBTile = kBK * kBN * 2;            // 16 KB (two 64-column boxes, 8 KB apart)
constexpr int kStage = kATile + kBTile;
constexpr int kCTile = kBM * kBN * 2;            // 32 KB (two 64-column halves)
constexpr int kThreads = 6 * 32;
constexpr int kWarpEpi0 = 2;
constexpr int kMaxOut = 4;

struct Misc {
  uint64_t full[kStages], empty[kStages];        // ring: loaded / read by the MMAs
  uint64_t tfull[2], tempty[2];                  // accumulators: complete / read out
  uint32_t tmem;
  int abort;
};
constexpr int kSmem = kStages * kStage + 2 * kCTile + (int)sizeof(Misc) + 1024;
static_assert(kSmem <= 227 * 1024, "GEMM CTA must fit one SM");

struct Params {
  int M, N, K, nout, ncols;
  int mt, nt, kt;                                // tiles along M, N and K blocks
};
struct Maps {
  CUtensorMap a, b, c[kMaxOut];
};

// Instruction descriptor: kind::f16, fp32 accumulate, A K-major, B MN-major,
// M = 128, N = 128; bf16 or fp16 operands.
__host__ __device__ constexpr uint32_t idesc(bool bf16) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (0u << 15) | (1u << 16) |
         ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

// 32 lanes x 32 bit, 32 consecutive columns: thread t of warp w <- lane 32(w%4)+t.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                 "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                 "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ uint32_t pack2(float a, float b, bool bf16) {
  uint32_t u;
  if (bf16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    memcpy(&u, &h, 4);
  } else {
    const __half2 h = __floats2half2_rn(a, b);
    memcpy(&u, &h, 4);
  }
  return u;
}

template <bool kBF16>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p,
                                                              const __grid_constant__ Maps mp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ctile = sm + kStages * kStage;
  Misc& m = *reinterpret_cast<Misc*>(ctile + 2 * kCTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.mt * p.nt;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&m.full[s], 1);
      tc::mbar_init(&m.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&m.tfull[a], 1);
      tc::mbar_init(&m.tempty[a], 4);            // one arrival per epilogue warp
    }
    m.abort = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&m.tmem, 2 * kBN);
    tc::tmem_relinquish();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  const uint32_t tm = m.tmem;
  bool failed = false;
  // the operands may come from the previous kernel in the stream
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;                                // K blocks issued so far (ring position)
      for (int t = blockIdx.x; t < ntiles && !failed; t += gridDim.x) {
        const int m0 = (t / p.nt) * kBM, n0 = (t % p.nt) * kBN;
        for (int kb = 0; kb < p.kt; ++kb, ++it) {
          const int s = it % kStages, use = it / kStages;
          if (use > 0 && !tc::mbar_wait(&m.empty[s], (uint32_t)(use - 1) & 1u)) { failed = true; break; }
          uint8_t* st = sm + s * kStage;
          tc::mbar_arrive_tx(&m.full[s], kStage);
          gate_tc::tma_load_2d(st, &mp.a, kb * kBK, m0, &m.full[s]);
          gate_tc::tma_load_2d(st + kATile, &mp.b, n0, kb * kBK, &m.full[s]);
          gate_tc::tma_load_2d(st + kATile + kBTile / 2, &mp.b, n0 + 64, kb * kBK, &m.full[s]);
        }
      }
      // every load issued lands before the CTA leaves
      for (int x = it - kStages < 0 ? 0 : it - kStages; x < it; ++x)
        if (!tc::mbar_wait(&m.full[x % kStages], (uint32_t)(x / kStages) & 1u)) failed = true;
      if (failed) m.abort = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id = idesc(kBF16);
      int it = 0, n = 0;
      for (int t = blockIdx.x; t < ntiles && !failed; t += gridDim.x, ++n) {
        const int acc = n & 1, use = n >> 1;
        if (use > 0 && !tc::mbar_wait(&m.tempty[acc], (uint32_t)(use - 1) & 1u)) { failed = true; break; }
        tc::tc_after_sync();
        const uint32_t d = tm + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < p.kt; ++kb, ++it) {
          const int s = it % kStages;
          if (!tc::mbar_wait(&m.full[s], (uint32_t)(it / kStages) & 1u)) { failed = true; break; }
          tc::tc_after_sync();
          const uint8_t* st = sm + s * kStage;
          const uint64_t a = tc::desc_k(st), b = tc::desc_mn(st + kATile);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            tc::mma_f16(d, a + k * tc::kStepK, b + k * tc::kStepMN, id, (kb > 0 || k > 0) ? 1u : 0u);
          tc::mma_commit(&m.empty[s]);           // the stage is free once these have read it
        }
        if (failed) break;
        tc::mma_commit(&m.tfull[acc]);
      }
      // the last products complete before tensor memory is released
      if (n > 0 && !tc::mbar_wait(&m.tfull[(n - 1) & 1], (uint32_t)((n - 1) >> 1) & 1u)) failed = true;
      if (failed) m.abort = 1;
    }
  } else {
    // ---- epilogue: thread = output row (TMEM lane) of its quadrant
    const int qd = warp & 3, row = qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const bool is_issuer = warp == kWarpEpi0 && lane == 0;
    int n = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++n) {
      const int acc = n & 1, use = n >> 1;
      const int m0 = (t / p.nt) * kBM, n0 = (t % p.nt) * kBN;
      uint8_t* ct = ctile + acc * kCTile;
      failed |= !tc::mbar_wait(&m.tfull[acc], (uint32_t)use & 1u);
      // the staging tile's stores of two tiles ago have read it
      if (is_issuer) tc::bulk_wait_read<1>();
      if (tc::named_barrier_or(1, 128, failed || *reinterpret_cast<volatile int*>(&m.abort) != 0)) { failed = true; break; }
      tc::tc_after_sync();
#pragma unroll 1
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tm + lane_base + (uint32_t)(acc * kBN + c), r);
        tmem_ld32_wait(r);
        // 32 columns = 4 units of 8; half c / 64, units (c % 64) / 8 ..
        uint8_t* half = ct + (c >> 6) * (kCTile / 2);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = ((c & 63) >> 3) + u;
          uint4 w;
          w.x = pack2(__uint_as_float(r[8 * u + 0]), __uint_as_float(r[8 * u + 1]), kBF16);
          w.y = pack2(__uint_as_float(r[8 * u + 2]), __uint_as_float(r[8 * u + 3]), kBF16);
          w.z = pack2(__uint_as_float(r[8 * u + 4]), __uint_as_float(r[8 * u + 5]), kBF16);
          w.w = pack2(__uint_as_float(r[8 * u + 6]), __uint_as_float(r[8 * u + 7]), kBF16);
          *reinterpret_cast<uint4*>(half + row * 128 + ((unit ^ (row & 7)) << 4)) = w;
        }
      }
      tc::tc_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_one(&m.tempty[acc]);   // this warp has read the accumulator
      tc::fence_async_smem();
      tc::named_barrier(1, 128);
      if (is_issuer) {
        const int o = p.nout > 1 ? n0 / p.ncols : 0;
        const int col = p.nout > 1 ? n0 - o * p.ncols : n0;
        gate_tc::tma_store_2d(&mp.c[o], col, m0, ct);
        if (col + 64 < p.ncols) gate_tc::tma_store_2d(&mp.c[o], col + 64, m0, ct + kCTile / 2);
        tc::bulk_commit();
      }
    }
    if (is_issuer) tc::bulk_wait<0>();           // every store complete before the CTA leaves
    if (failed && threadIdx.x == 32 * kWarpEpi0) m.abort = 1;
  }
  if (failed) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tm, 2 * kBN);
}

}  // namespace gemm
}  // namespace gtr

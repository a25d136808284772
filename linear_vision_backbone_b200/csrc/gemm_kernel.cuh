// gemm_kernel.cuh -- the projections' GEMM C = A B on tcgen05 (see
// gemm_tc.cuh for the contract), in the gate / GLA translation unit so that
// its bounded waits report through the library's device status word.
//
// A persistent kernel: one CTA per SM walks output tiles of 128 x kBN, kBN =
// 128 or 256 (tile t = blockIdx.x, + gridDim.x, ..., the N tiles of one M tile
// consecutive so that CTAs running at the same time share their A rows in L2).
// Warp 0 streams the K blocks (64 deep) of A (K-major, 128 x 64) and B
// (MN-major, 64 x kBN as 64-column boxes) into a ring of kStages stages with
// tensor-map loads; warp 1's first thread issues, per K block, four
// tcgen05.mma kind::f16 (M = 128, N = kBN, K = 16) into one of two TMEM
// accumulators; warps 2-5 (one TMEM lane quadrant each, thread = output row)
// read a finished accumulator 64 columns at a time, round it to the 16-bit
// type into a 128B-swizzled staging box of the warp's own 32 rows (a ring of
// two per warp, so a box's store overlaps the next box's packing) and the
// warp's first thread writes it with a tensor-map store; the four warps never
// wait for one another.  Rows and columns past the matrix edges are zero on load
// and clipped on store.  The wide tile reads A once per 256 output columns
// instead of twice (25% fewer bytes through L2 per FLOP): 1.17 PFLOP/s at
// M = 16384, K = 1024, N = 2048 against 0.95 for 128 x 128 tiles.
#pragma once
#include "gate_tc.cuh"
#include "gemm_tc.cuh"
#include "tc_kernels.cuh"

namespace gtr {
namespace gemm {

using tc::saddr;
constexpr int kBM = 128, kBK = 64;
constexpr int kATile = kBM * kBK * 2;            // 16 KB
constexpr int kBox = 32 * 64 * 2;                // one warp's 32 rows x 64 columns output box: 4 KB
constexpr int kEpiBoxes = 2;                     // per epilogue warp (a ring of two)
constexpr int kThreads = 6 * 32;
constexpr int kMaxOut = 4;

template <int kBN>
struct Cfg {
  static constexpr int kStages = kBN == 128 ? 6 : 4;
  static constexpr int kBTile = kBK * kBN * 2;   // kBN / 64 boxes of 8 KB
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kSmem = kStages * kStage + 4 * kEpiBoxes * kBox + 256 + 1024;
  static_assert(kSmem <= 227 * 1024, "GEMM CTA must fit one SM");
};

struct Misc {
  uint64_t full[8], empty[8];                    // ring: loaded / read by the MMAs
  uint64_t tfull[2], tempty[2];                  // accumulators: complete / read out
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Misc) <= 256, "bookkeeping fits its reserve");

struct Params {
  int M, N, K, nout, ncols;
  int mt, nt, kt;                                // tiles along M, N and K blocks
};
struct Maps {
  CUtensorMap a, b, c[kMaxOut];
};

// Instruction descriptor: kind::f16, fp32 accumulate, A K-major, B MN-major,
// M = 128, N = n; bf16 or fp16 operands.
__host__ __device__ constexpr uint32_t idesc(bool bf16, int n) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (0u << 15) | (1u << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
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

template <bool kBF16, int kBN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p,
                                                              const __grid_constant__ Maps mp) {
  using C = Cfg<kBN>;
  constexpr int kStages = C::kStages, kStage = C::kStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* boxes = sm + kStages * kStage;
  Misc& m = *reinterpret_cast<Misc*>(boxes + 4 * kEpiBoxes * kBox);
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
#pragma unroll
          for (int g = 0; g < kBN / 64; ++g)
            gate_tc::tma_load_2d(st + kATile + g * (kBK * 128), &mp.b, n0 + 64 * g, kb * kBK, &m.full[s]);
        }
      }
      // every load issued lands before the CTA leaves
      for (int x = it - kStages < 0 ? 0 : it - kStages; x < it; ++x)
        if (!tc::mbar_wait(&m.full[x % kStages], (uint32_t)(x / kStages) & 1u)) failed = true;
      if (failed) m.abort = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id = idesc(kBF16, kBN);
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
    const int qd = warp & 3;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    uint8_t* mine = boxes + qd * (kEpiBoxes * kBox);   // this warp's staging ring
    int n = 0, nbox = 0;
    for (int t = blockIdx.x; t < ntiles && !failed; t += gridDim.x, ++n) {
      const int acc = n & 1, use = n >> 1;
      const int m0 = (t / p.nt) * kBM, n0 = (t % p.nt) * kBN;
      failed |= !tc::mbar_wait(&m.tfull[acc], (uint32_t)use & 1u);
      tc::tc_after_sync();
#pragma unroll 1
      for (int j = 0; j < kBN / 64; ++j, ++nbox) {
        const int gcol = n0 + 64 * j;
        uint8_t* box = mine + (nbox % kEpiBoxes) * kBox;
        // the store that last used this staging box has read it
        if (lane == 0) tc::bulk_wait_read<kEpiBoxes - 1>();
        if (__any_sync(0xffffffffu, failed || *reinterpret_cast<volatile int*>(&m.abort) != 0)) {
          failed = true;
          break;
        }
        uint32_t r0[32], r1[32];
        const uint32_t src = tm + lane_base + (uint32_t)(acc * kBN + 64 * j);
        tmem_ld32(src, r0);
        tmem_ld32(src + 32, r1);
        tmem_ld32_wait(r0);
        tmem_ld32_wait(r1);
        if (j == kBN / 64 - 1) {
          // this warp has read the whole accumulator
          tc::tc_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive_one(&m.tempty[acc]);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* r = u < 4 ? r0 + 8 * u : r1 + 8 * (u - 4);
          uint4 w;
          w.x = pack2(__uint_as_float(r[0]), __uint_as_float(r[1]), kBF16);
          w.y = pack2(__uint_as_float(r[2]), __uint_as_float(r[3]), kBF16);
          w.z = pack2(__uint_as_float(r[4]), __uint_as_float(r[5]), kBF16);
          w.w = pack2(__uint_as_float(r[6]), __uint_as_float(r[7]), kBF16);
          *reinterpret_cast<uint4*>(box + lane * 128 + ((u ^ (lane & 7)) << 4)) = w;
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0 && gcol < p.N && m0 + qd * 32 < p.M) {
          const int o = p.nout > 1 ? gcol / p.ncols : 0;
          gate_tc::tma_store_2d(&mp.c[o], gcol - o * p.ncols, m0 + qd * 32, box);
          tc::bulk_commit();
        }
      }
    }
    if (lane == 0) tc::bulk_wait<0>();           // every store complete before the CTA leaves
    if (failed && lane == 0) m.abort = 1;
  }
  if (failed) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tm, 2 * kBN);
}

// ---------------------------------------------------------------------------
// The CTA-pair form: a cluster of two CTAs on two SMs computes a 256 x kBN
// tile with tcgen05.mma.cta_group::2 (M = 256): each CTA stages its own 128
// rows of A and half of the tile's B columns, the pair's first CTA (rank 0)
// issues the MMAs, which read both CTAs' shared memory and write each CTA's
// 128 accumulator rows into that CTA's tensor memory.  Per SM and K block that
// is 16 KB of A and kBN/2 x 64 of B for 128 x kBN outputs: a third less L2
// traffic per FLOP than the single-CTA 128 x 256 tile, half of 128 x 128.
// Measured faster than the single-CTA tile only for deep products (K >= 1024,
// where the host selects it); at K = 384 it is slower.
//
// Synchronisation (all waits bounded): both CTAs' tensor-map loads complete on
// rank 0's full[s] (rank 0 expects both CTAs' bytes); rank 0's MMA thread
// commits each consumed stage to empty[s] and each finished accumulator to
// tfull[a] of both CTAs; the eight epilogue warps of the pair arrive on rank
// 0's tempty[a].  No load uses cluster multicast.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The shared::cluster address of `p`'s counterpart in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t mbar_try_cluster(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity), "r"(20000u)
      : "memory");
  return ok;
}
// A wait on a barrier that the other CTA of the pair signals; false after the
// library's bounded-wait limit.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* b, uint32_t parity) {
  if (mbar_try_cluster(b, parity)) return true;
  const unsigned long long t0 = tc::globaltimer();
  while (!mbar_try_cluster(b, parity))
    if (tc::globaltimer() - t0 > tc::kWaitNs) return false;
  return true;
}
__device__ __forceinline__ void mbar_arrive_at(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* map, int x, int y, uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(saddr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void mma_f16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit_pair(uint32_t cluster_bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(dst)), "r"(cols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

template <int kBN>
struct PairCfg {
  static constexpr int kStages = 6;
  static constexpr int kBHalf = kBK * (kBN / 2) * 2;   // this CTA's B columns: kBN / 128 boxes of 8 KB
  static constexpr int kStage = kATile + kBHalf;
  static constexpr int kSmem = kStages * kStage + 4 * kEpiBoxes * kBox + 256 + 1024;
  static_assert(kSmem <= 227 * 1024, "GEMM CTA must fit one SM");
  static_assert(kStages <= 8, "barrier arrays");
};

// Instruction descriptor of the pair's product: M = 256, N = n.
__host__ __device__ constexpr uint32_t idesc_pair(bool bf16, int n) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (0u << 15) | (1u << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

template <bool kBF16, int kBN>
__global__ void __launch_bounds__(kThreads, 1) gemm_pair_kernel(const __grid_constant__ Params p,
                                                                const __grid_constant__ Maps mp) {
  using C = PairCfg<kBN>;
  constexpr int kStages = C::kStages, kStage = C::kStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* boxes = sm + kStages * kStage;
  Misc& m = *reinterpret_cast<Misc*>(boxes + 4 * kEpiBoxes * kBox);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  const int ntiles = p.mt * p.nt;                // tiles of 256 x kBN
  const int first = (int)cluster_id(), step = (int)cluster_count();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&m.full[s], 1);
      tc::mbar_init(&m.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&m.tfull[a], 1);
      tc::mbar_init(&m.tempty[a], 8);            // every epilogue warp of the pair
    }
    m.abort = 0;
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&m.tmem, 2 * kBN);
    tmem_relinquish_pair();
  }
  tc::tc_before_sync();
  __syncthreads();
  cluster_sync_all();                            // both CTAs' barriers exist before any signal
  tc::tc_after_sync();
  const uint32_t tm = m.tmem;
  bool failed = false;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = first; t < ntiles && !failed; t += step) {
        const int m0 = (t / p.nt) * 256 + (int)rank * kBM, n0 = (t % p.nt) * kBN + (int)rank * (kBN / 2);
        for (int kb = 0; kb < p.kt; ++kb, ++it) {
          const int s = it % kStages, use = it / kStages;
          if (use > 0 && !mbar_wait_cluster(&m.empty[s], (uint32_t)(use - 1) & 1u)) { failed = true; break; }
          uint8_t* st = sm + s * kStage;
          if (lead) tc::mbar_arrive_tx(&m.full[s], 2 * kStage);
          const uint32_t bar = peer_addr(&m.full[s], 0);
          tma_load_2d_pair(st, &mp.a, kb * kBK, m0, bar);
#pragma unroll
          for (int g = 0; g < kBN / 128; ++g)
            tma_load_2d_pair(st + kATile + g * (kBK * 128), &mp.b, n0 + 64 * g, kb * kBK, bar);
        }
      }
      if (failed) m.abort = 1;
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      constexpr uint32_t id = idesc_pair(kBF16, kBN);
      int it = 0, n = 0;
      for (int t = first; t < ntiles && !failed; t += step, ++n) {
        const int acc = n & 1, use = n >> 1;
        if (use > 0 && !mbar_wait_cluster(&m.tempty[acc], (uint32_t)(use - 1) & 1u)) { failed = true; break; }
        tc::tc_after_sync();
        const uint32_t d = tm + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < p.kt; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait_cluster(&m.full[s], (uint32_t)(it / kStages) & 1u)) { failed = true; break; }
          tc::tc_after_sync();
          const uint8_t* st = sm + s * kStage;
          const uint64_t a = tc::desc_k(st), b = tc::desc_mn(st + kATile);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_f16_pair(d, a + k * tc::kStepK, b + k * tc::kStepMN, id, (kb > 0 || k > 0) ? 1u : 0u);
          // the stage is free in both CTAs once these have read it
          mma_commit_pair(peer_addr(&m.empty[s], 0));
          mma_commit_pair(peer_addr(&m.empty[s], 1));
        }
        if (failed) break;
        mma_commit_pair(peer_addr(&m.tfull[acc], 0));
        mma_commit_pair(peer_addr(&m.tfull[acc], 1));
      }
      // the last products complete before the pair may leave
      if (n > 0 && !mbar_wait_cluster(&m.tfull[(n - 1) & 1], (uint32_t)((n - 1) >> 1) & 1u)) failed = true;
      if (failed) m.abort = 1;
    }
  } else {
    // ---- epilogue: thread = output row (TMEM lane) of its quadrant of this CTA's 128 rows; each warp stores its own 32 rows
    const int qd = warp & 3;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    uint8_t* mine = boxes + qd * (kEpiBoxes * kBox);   // this warp's staging ring
    int n = 0, nbox = 0;
    for (int t = first; t < ntiles && !failed; t += step, ++n) {
      const int acc = n & 1, use = n >> 1;
      const int m0 = (t / p.nt) * 256 + (int)rank * kBM, n0 = (t % p.nt) * kBN;
      failed |= !mbar_wait_cluster(&m.tfull[acc], (uint32_t)use & 1u);
      tc::tc_after_sync();
#pragma unroll 1
      for (int j = 0; j < kBN / 64; ++j, ++nbox) {
        const int gcol = n0 + 64 * j;
        uint8_t* box = mine + (nbox % kEpiBoxes) * kBox;
        // the store that last used this staging box has read it
        if (lane == 0) tc::bulk_wait_read<kEpiBoxes - 1>();
        if (__any_sync(0xffffffffu, failed || *reinterpret_cast<volatile int*>(&m.abort) != 0)) {
          failed = true;
          break;
        }
        uint32_t r0[32], r1[32];
        const uint32_t src = tm + lane_base + (uint32_t)(acc * kBN + 64 * j);
        tmem_ld32(src, r0);
        tmem_ld32(src + 32, r1);
        tmem_ld32_wait(r0);
        tmem_ld32_wait(r1);
        if (j == kBN / 64 - 1) {
          tc::tc_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive_at(peer_addr(&m.tempty[acc], 0));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint32_t* r = u < 4 ? r0 + 8 * u : r1 + 8 * (u - 4);
          uint4 w;
          w.x = pack2(__uint_as_float(r[0]), __uint_as_float(r[1]), kBF16);
          w.y = pack2(__uint_as_float(r[2]), __uint_as_float(r[3]), kBF16);
          w.z = pack2(__uint_as_float(r[4]), __uint_as_float(r[5]), kBF16);
          w.w = pack2(__uint_as_float(r[6]), __uint_as_float(r[7]), kBF16);
          *reinterpret_cast<uint4*>(box + lane * 128 + ((u ^ (lane & 7)) << 4)) = w;
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0 && gcol < p.N && m0 + qd * 32 < p.M) {
          const int o = p.nout > 1 ? gcol / p.ncols : 0;
          gate_tc::tma_store_2d(&mp.c[o], gcol - o * p.ncols, m0 + qd * 32, box);
          tc::bulk_commit();
        }
      }
    }
    if (lane == 0) tc::bulk_wait<0>();           // every store complete before the CTA leaves
    if (failed && lane == 0) m.abort = 1;
  }
  if (failed) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  cluster_sync_all();                            // neither CTA leaves while the other may still signal it
  tc::tc_after_sync();
  if (warp == 0) tmem_dealloc_pair(tm, 2 * kBN);
}

}  // namespace gemm
}  // namespace gtr

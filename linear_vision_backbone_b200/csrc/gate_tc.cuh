// gate_tc.cuh -- K1 on tensor cores: the low-rank forget-gate projection
//   g[n, j] = logsigmoid(sum_r (x[n,:] . W_down[:, r]) W_up[r, j] + b[j]) / tau
// (GTR article, 方法详解 §1: a light low-rank projection with a temperature).
//
// Two kernels.
//   gate_pack_tc  -- once per weight set: splits W_down and W_up into the
//     operand tiles the forward kernel multiplies, in their shared-memory
//     byte layout ("packed weights"), with the power-of-two scales:
//       * W_down (rank 16) into terms of x's own type with a scale per rank
//         (fp16: hi + lo, bf16: hi + mid + lo), the terms side by side along
//         N, K-major: x W_down is exact up to ~22-24 significant bits;
//       * W_up into two fp16 terms (hi + lo) with a scale per column, MN-major.
//   gate_fwd_tc -- one CTA (512 threads) per tile of up to 128 tokens (about
//     one tile per SM):
//       * TMA (tensor map, 128B swizzle) loads the x tile straight into the
//         K-major operand layout (rows past the tensor read as zero), and bulk
//         copies bring the packed weights;
//       * stage 1: one tcgen05.mma kind::f16 per K step (M = 128, N = 16 x
//         terms) gives every x W_t; their sum, per-row scaled, becomes a
//         two-term fp16 operand `low`;
//       * stage 2: u = low W_up as hi*hi + hi*lo + lo*hi (N = 64 per
//         instruction), fp32 in TMEM;
//       * epilogue, one 64-column slab at a time: thread = token row (TMEM lane
//         quadrant warp % 4), warps w, w+4, w+8, w+12 on the slab's four
//         16-column quarters; logsigmoid(u + b)/tau goes into a 128B-swizzled
//         shared-memory slab (the x tile's space, free by then) that TMA
//         stores to g, so the stores cost the warps nothing.
// The scales are exact powers of two and are undone on the fp32 accumulators;
// they run along M or N only, so they factor out of every sum.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "gate_kernels.cuh"
#include "tc_kernels.cuh"

namespace gtr {
namespace gate_tc {

using tc::saddr;

using tc::logsigmoid_over_tau;
using tc::pow2i;
using tc::scale_exp;
using tc::bulk_g2s;
using tc::bulk_commit;
using tc::bulk_wait;
using tc::bulk_wait_read;

// Two-term fp16 operand: x = hi + lo, hi = fp16(x), lo = fp16(x - hi); four
// consecutive elements at byte offset `off` of the (hi, lo) tiles.
__device__ __forceinline__ void put2(uint8_t* hi, uint8_t* lo, uint32_t off, float a, float b, float c,
                                     float d) {
  const __half2 h0 = __floats2half2_rn(a, b), h1 = __floats2half2_rn(c, d);
  const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
  const __half2 l0 = __floats2half2_rn(a - f0.x, b - f0.y), l1 = __floats2half2_rn(c - f1.x, d - f1.y);
  uint2 H, L;
  memcpy(&H.x, &h0, 4);
  memcpy(&H.y, &h1, 4);
  memcpy(&L.x, &l0, 4);
  memcpy(&L.y, &l1, 4);
  *reinterpret_cast<uint2*>(hi + off) = H;
  *reinterpret_cast<uint2*>(lo + off) = L;
}
// 32 lanes x 32 bit, 16 consecutive columns: thread t of warp w <- lane 32(w%4)+t.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// TMA: tiled 2-D copies through a tensor map (coordinates: x = innermost
// element index, y = row), and their completion.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(saddr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(saddr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const void* map, int x, int y, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map),
               "r"(x), "r"(y), "r"(saddr(src))
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes)
               : "memory");
}
constexpr int kM = 128;               // rows of the MMA tile (tokens per CTA <= kM)
constexpr int kThreads = 512;         // stages and epilogue: 16 warps
constexpr int kThreadsAll = kThreads + 32;   // + a warp that issues the g stores
constexpr int kPackThreads = 256;
constexpr int kMaxDm = 384;           // d_model: multiple of 64, <= 384
constexpr int kMaxHD = 448;           // H*dk: multiple of 64, <= 448
constexpr int kRank = 16;             // the projection's N (rank 16)

struct Layout {
  static constexpr int kX = kM * kMaxDm * 2;               // x tile: 96 KB
  static constexpr int kWd = kRank * kMaxDm * 2;           // one W_down term: 12 KB
  static constexpr int kLow = kM * 128;                    // one low term (K = 16 of a 64-wide tile): 16 KB
  static constexpr int kWu = kRank * kMaxHD * 2;           // one W_up term: 14 KB
  static constexpr int kOffX = 0;
  static constexpr int kOffWd = kOffX + kX;                // 3 terms
  static constexpr int kOffLow = kOffWd + 3 * kWd;         // 2 terms
  static constexpr int kOffWu = kOffLow + 2 * kLow;        // 2 terms
  static constexpr int kOffMisc = kOffWu + 2 * kWu;
  static constexpr int kMiscBytes = 6144;
  static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;
  static constexpr int kHalfSlab = kM * 128;               // 32 fp32 columns x 128 rows, 128B-swizzled
};
// Packed weights in global memory: the W_down and W_up term regions in their
// shared-memory byte layout, then the inverse scales (W_down per rank, W_up
// per column).
struct Pack {
  static constexpr int kOffWd = 0;
  static constexpr int kWdBytes = 3 * Layout::kWd;
  static constexpr int kOffWu = kOffWd + kWdBytes;
  static constexpr int kWuBytes = 2 * Layout::kWu;
  static constexpr int kOffScale = kOffWu + kWuBytes;
  static constexpr int kScaleBytes = (kRank + kMaxHD) * 4;
  static constexpr int kBytes = kOffScale + kScaleBytes;
  static constexpr int kSmem = kBytes + 1024;                // the pack kernel's image + alignment slack
};
static_assert(Pack::kBytes % 16 == 0 && Pack::kScaleBytes % 16 == 0, "bulk copies move 16-byte multiples");

struct Misc {
  uint64_t mma[2];
  uint64_t sfull[3];                 // epilogue slab buffer b staged (one arrival per epilogue warp)
  uint64_t sfree[3];                 // its tensor-map stores have read it
  uint64_t ld;                       // the packed weights
  uint64_t ldx[kMaxDm / 64];         // the x tile, one 64-column atom each
  uint32_t tmem;
  int pad;
  alignas(16) float wd_i[kRank];     // inverse W_down rank scales; wu_i follows (one bulk copy)
  float wu_i[kMaxHD];                // inverse W_up column scales
  alignas(16) float low_i[kM];       // inverse row scales of low
  alignas(16) float bias[kMaxHD];
};
static_assert(sizeof(Misc) <= Layout::kMiscBytes, "Misc must fit its reserved bytes");
static_assert(offsetof(Misc, wu_i) == offsetof(Misc, wd_i) + kRank * 4, "scales are one block");
static_assert(6 * Layout::kHalfSlab <= Layout::kX, "three staged slabs must fit in the x tile");

// K-major 16-bit tile (rows x K), 128B-swizzled atoms of 8 rows x 64 elements;
// atom columns (64 K-elements) `rows`*128 bytes apart.
__device__ __forceinline__ uint32_t swk(int r, int c, int rows) {
  return (uint32_t)((c >> 6) * (rows * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                    ((((c & 63) >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}
// MN-major 16-bit tile (K rows x N), atoms of 8 K-rows x 64 N-elements; N atoms
// `krows`*128 bytes apart.
__device__ __forceinline__ uint32_t swmn(int k, int n, int krows) {
  return (uint32_t)((n >> 6) * (krows * 128) + (k >> 3) * 1024 + (k & 7) * 128 +
                    ((((n & 63) >> 3) ^ (k & 7)) << 4) + (n & 7) * 2);
}
__host__ __device__ constexpr uint32_t idesc16(int M, int N, int a_mn, int b_mn, int bf16) {
  return (1u << 4) | ((uint32_t)bf16 << 7) | ((uint32_t)bf16 << 10) | ((uint32_t)a_mn << 15) |
         ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <typename T> struct Store16;
template <> struct Store16<__half> {
  static __device__ __forceinline__ void put(uint8_t* p, float v) { *reinterpret_cast<__half*>(p) = __float2half_rn(v); }
  static __device__ __forceinline__ float back(float v) { return __half2float(__float2half_rn(v)); }
};
template <> struct Store16<__nv_bfloat16> {
  static __device__ __forceinline__ void put(uint8_t* p, float v) {
    *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
  }
  static __device__ __forceinline__ float back(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }
};

// ------------------------------------------------------------- weight pack
template <typename TX>
__global__ void __launch_bounds__(kPackThreads, 1)
gate_pack_tc(const float* __restrict__ w_down, const float* __restrict__ w_up, int dm, int HD,
             uint8_t* __restrict__ pack) {
  constexpr int kTerms = std::is_same<TX, __nv_bfloat16>::value ? 3 : 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* img = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);   // Pack::kBytes
  uint8_t* tWd = img + Pack::kOffWd;
  uint8_t* tWu = img + Pack::kOffWu;
  float* wd_i = reinterpret_cast<float*>(img + Pack::kOffScale);
  float* wu_i = wd_i + kRank;
  __shared__ float wd_part[kPackThreads / 32][kRank];
  __shared__ float wd_s[kRank];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();                                     // the weights may come from the previous kernel
  pdl_trigger();
  // zero the image (regions beyond d_model / H*dk are never read, but are copied)
  for (int o = tid; o < Pack::kBytes / 16; o += kPackThreads)
    reinterpret_cast<uint4*>(img)[o] = make_uint4(0u, 0u, 0u, 0u);
  // W_down [dm][16]: thread t holds float4s t, t + 256, ... (ranks 4(t%4)..+3 of rows (t+256i)/4)
  constexpr int kWdVec = kMaxDm * kRank / 4 / kPackThreads;
  const int nwd = dm * kRank / 4;
  float4 wd[kWdVec];
  float4 wmx = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kWdVec; ++i) {
    const int idx = tid + i * kPackThreads;
    wd[i] = idx < nwd ? __ldg(reinterpret_cast<const float4*>(w_down) + idx) : make_float4(0.f, 0.f, 0.f, 0.f);
    wmx = make_float4(fmaxf(wmx.x, fabsf(wd[i].x)), fmaxf(wmx.y, fabsf(wd[i].y)),
                      fmaxf(wmx.z, fabsf(wd[i].z)), fmaxf(wmx.w, fabsf(wd[i].w)));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    wmx.x = fmaxf(wmx.x, __shfl_xor_sync(0xffffffffu, wmx.x, o));
    wmx.y = fmaxf(wmx.y, __shfl_xor_sync(0xffffffffu, wmx.y, o));
    wmx.z = fmaxf(wmx.z, __shfl_xor_sync(0xffffffffu, wmx.z, o));
    wmx.w = fmaxf(wmx.w, __shfl_xor_sync(0xffffffffu, wmx.w, o));
  }
  if (lane < 4) *reinterpret_cast<float4*>(&wd_part[warp][lane * 4]) = wmx;
  __syncthreads();                                // also orders the zeroing before the writes below
  if (tid < kRank) {
    float mx = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kPackThreads / 32; ++w8) mx = fmaxf(mx, wd_part[w8][tid]);
    const int e = scale_exp(mx);
    wd_s[tid] = pow2i(e);
    wd_i[tid] = pow2i(-e);
  }
  // W_up [16][HD]: thread t < HD/4 handles column quad t of all 16 ranks; fp16 hi + lo,
  // per-column scales (B of stage 2, MN-major: rows = rank (K), columns = H*dk)
  for (int qd = tid; qd < HD / 4; qd += kPackThreads) {
    float4 wu[kRank];
#pragma unroll
    for (int k = 0; k < kRank; ++k) wu[k] = __ldg(reinterpret_cast<const float4*>(w_up + (size_t)k * HD) + qd);
    float4 cm = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kRank; ++k)
      cm = make_float4(fmaxf(cm.x, fabsf(wu[k].x)), fmaxf(cm.y, fabsf(wu[k].y)),
                       fmaxf(cm.z, fabsf(wu[k].z)), fmaxf(cm.w, fabsf(wu[k].w)));
    const int e0 = scale_exp(cm.x), e1 = scale_exp(cm.y), e2 = scale_exp(cm.z), e3 = scale_exp(cm.w);
    *reinterpret_cast<float4*>(&wu_i[4 * qd]) = make_float4(pow2i(-e0), pow2i(-e1), pow2i(-e2), pow2i(-e3));
    const float s0 = pow2i(e0), s1 = pow2i(e1), s2 = pow2i(e2), s3 = pow2i(e3);
#pragma unroll
    for (int k = 0; k < kRank; ++k)
      put2(tWu, tWu + Layout::kWu, swmn(k, 4 * qd, kRank), wu[k].x * s0, wu[k].y * s1, wu[k].z * s2,
           wu[k].w * s3);
  }
  __syncthreads();
  // W_down^T terms (B of stage 1, K-major: row t * 16 + rank for term t, columns = d_model)
  {
    const float4 sc = *reinterpret_cast<const float4*>(&wd_s[(tid & 3) * 4]);
#pragma unroll
    for (int i = 0; i < kWdVec; ++i) {
      const int idx = tid + i * kPackThreads;
      if (idx < nwd) {
        const int c = idx >> 2, n0 = (idx & 3) * 4;
        const float w4[4] = {wd[i].x * sc.x, wd[i].y * sc.y, wd[i].z * sc.z, wd[i].w * sc.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float w = w4[e];
#pragma unroll
          for (int t = 0; t < kTerms; ++t) {
            Store16<TX>::put(tWd + swk(t * kRank + n0 + e, c, kTerms * kRank), w);
            w -= Store16<TX>::back(w);
          }
        }
      }
    }
  }
  __syncthreads();
  for (int o = tid; o < Pack::kBytes / 16; o += kPackThreads)
    reinterpret_cast<uint4*>(pack)[o] = reinterpret_cast<const uint4*>(img)[o];
}

// --------------------------------------------------------------- forward
// tmx: x as [N rows][dm] 16-bit, box 64 x 128, 128B swizzle.  tmg: g as
// [N rows][HD] fp32, box 32 x tpc, 128B swizzle.
template <typename TX>
__global__ void __launch_bounds__(kThreadsAll, 1)
gate_fwd_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmg,
            const uint8_t* __restrict__ pack, const float* __restrict__ bias, int dm, int HD,
            float inv_tau, int tpc, int spb) {
  constexpr bool kBf16 = std::is_same<TX, __nv_bfloat16>::value;
  constexpr int kTerms = kBf16 ? 3 : 2;   // W_down terms in x's type
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* tX = sm + Layout::kOffX;
  uint8_t* tWd = sm + Layout::kOffWd;
  uint8_t* tLow = sm + Layout::kOffLow;
  uint8_t* tWu = sm + Layout::kOffWu;
  Misc& m = *reinterpret_cast<Misc*>(sm + Layout::kOffMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tok0 = blockIdx.x * tpc;
  // this block's 64-column slabs of g: [j0, j1) (blockIdx.y splits the
  // columns when there are few token tiles)
  const int j0 = blockIdx.y * spb, j1 = min(HD / 64, j0 + spb);

  if (tid == 0) {
    tc::mbar_init(&m.ld, 1);
    for (int a = 0; a < kMaxDm / 64; ++a) tc::mbar_init(&m.ldx[a], 1);
    tc::mbar_init(&m.mma[0], 1);
    tc::mbar_init(&m.mma[1], 1);
    for (int b = 0; b < 3; ++b) {
      tc::mbar_init(&m.sfull[b], kThreads / 32);
      tc::mbar_init(&m.sfree[b], 1);
    }
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&m.tmem, 512);
    tc::tmem_relinquish();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  pdl_wait();                                     // x and the packed weights may come from the previous kernel
  pdl_trigger();
  const int natoms = dm / 64;
  if (tid == 0) {
    // the weights first (shared by every block, mostly from L2), then the x
    // atoms, each on its own barrier so stage 1 starts with the first
    mbar_expect_tx(&m.ld, (uint32_t)(Pack::kWdBytes + Pack::kWuBytes + Pack::kScaleBytes));
    bulk_g2s(tWd, pack + Pack::kOffWd, Pack::kWdBytes, &m.ld);
    bulk_g2s(tWu, pack + Pack::kOffWu, Pack::kWuBytes, &m.ld);
    bulk_g2s(&m.wd_i[0], pack + Pack::kOffScale, Pack::kScaleBytes, &m.ld);
    for (int a = 0; a < natoms; ++a) {
      mbar_expect_tx(&m.ldx[a], (uint32_t)(kM * 128));
      tma_load_2d(tX + a * (kM * 128), &tmx, a * 64, tok0, &m.ldx[a]);
    }
  }
  for (int j = tid; j < HD; j += kThreads) m.bias[j] = bias ? __ldg(bias + j) : 0.f;
  __syncthreads();
  const uint32_t tm = m.tmem;
  bool ok = true;

  // ---- stage 1: x W_t for every term t at once (TMEM columns 16 t .. 16 t + 15),
  // each 64-column atom of x as soon as it has landed
  if (tid == 0) {
    constexpr int kN1 = kTerms * kRank;
    const uint32_t id = idesc16(kM, kN1, 0, 0, kBf16 ? 1 : 0);
    ok &= tc::mbar_wait(&m.ld, 0);
    for (int at = 0; at < natoms; ++at) {
      ok &= tc::mbar_wait(&m.ldx[at], 0);
      tc::tc_after_sync();
      for (int s = 4 * at; s < 4 * at + 4; ++s) {
        const uint64_t a = tc::sdesc(saddr(tX) + (s >> 2) * (kM * 128) + (s & 3) * 32, 16, 1024);
        const uint64_t b = tc::sdesc(saddr(tWd) + (s >> 2) * (kN1 * 128) + (s & 3) * 32, 16, 1024);
        tc::mma_f16(tm + 0, a, b, id, s > 0 ? 1u : 0u);
      }
    }
    tc::mma_commit(&m.mma[0]);
  }
  // every thread reads the weight scales below: the weights' barrier, then stage 1's
  ok &= tc::mbar_wait(&m.ld, 0);
  ok &= tc::mbar_wait(&m.mma[0], 0);
  tc::tc_after_sync();
  // low row r (warps 0-3, thread = row) -> per-row scaled two-term fp16 A tile (K = 16)
  if (warp < 4) {
    float lw[16], lt[16];
    tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + 0, lw);
    tc::tmem_ld_wait(lw);
#pragma unroll
    for (int t = 1; t < kTerms; ++t) {
      tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + t * kRank, lt);
      tc::tmem_ld_wait(lt);
#pragma unroll
      for (int c = 0; c < 16; ++c) lw[c] += lt[c];
    }
    const int r = warp * 32 + lane;
    float mx = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      lw[c] *= m.wd_i[c];
      mx = fmaxf(mx, fabsf(lw[c]));
    }
    const int e = scale_exp(mx);
    const float s = pow2i(e);
    m.low_i[r] = pow2i(-e);
#pragma unroll
    for (int c = 0; c < 16; c += 4)
      put2(tLow, tLow + Layout::kLow, swk(r, c, kM), lw[c] * s, lw[c + 1] * s, lw[c + 2] * s,
           lw[c + 3] * s);
  }
  tc::fence_async_smem();
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();

  // ---- stage 2: u = low W_up  (TMEM columns 64 .. 64 + HD), 64 columns per instruction
  if (tid == 0) {
    const uint32_t id = idesc16(kM, 64, 0, 1, 0);
    const uint64_t al = tc::sdesc(saddr(tLow), 16, 1024), all = tc::sdesc(saddr(tLow) + Layout::kLow, 16, 1024);
    for (int nb = j0; nb < j1; ++nb) {
      const uint32_t ub = saddr(tWu) + nb * (kRank * 128);
      const uint64_t bh = tc::sdesc(ub, kRank * 128, 1024), bl = tc::sdesc(ub + Layout::kWu, kRank * 128, 1024);
      tc::mma_f16(tm + 64 + nb * 64, al, bh, id, 0u);
      tc::mma_f16(tm + 64 + nb * 64, al, bl, id, 1u);
      tc::mma_f16(tm + 64 + nb * 64, all, bh, id, 1u);
    }
    tc::mma_commit(&m.mma[1]);
  }
  ok &= tc::mbar_wait(&m.mma[1], 0);
  tc::tc_after_sync();
  ok = __syncthreads_and(ok) != 0;                // block-uniform: the epilogue has barriers
  if (!ok && tid == 0) gtr_flag(kStatusMbarTimeout);

  // ---- epilogue, one 64-column slab of u at a time: thread = token row (TMEM
  // lane quadrant warp % 4), warp w on the slab's 16-column quarter w / 4.  Each
  // slab is staged as two 32-column halves (128-byte rows, 16-byte units XOR-ed
  // with row % 8: the TMA 128B swizzle) in one of three rotating buffers; each
  // warp signals its part on the buffer's `sfull` barrier, and a seventeenth
  // warp issues the two tensor-map stores of a full slab and signals `sfree`
  // once they have read the buffer, which the warps wait for before staging
  // the slab three later there.  No block barrier runs between slabs.
  if (ok) {
    const int nslab = j1 - j0;                    // slabs j0 + l, l < nslab
    if (warp < kThreads / 32) {
      const float ln2_tau = 0.6931471805599453f * inv_tau;
      const int q = warp & 3, qp = warp >> 2;
      const int r = q * 32 + lane;
      const float ri = m.low_i[r];
      const uint32_t tq = tm + ((uint32_t)(q * 32) << 16) + 64 + 16 * qp;
      auto emit = [&](int l, const float* u) {
        uint8_t* slab = tX + (l % 3) * (2 * Layout::kHalfSlab);
        if (l >= 3) ok &= tc::mbar_wait(&m.sfree[l % 3], (uint32_t)((l / 3) - 1) & 1u);
        const int cb = 64 * (j0 + l) + 16 * qp;
        uint8_t* half = slab + (qp >> 1) * Layout::kHalfSlab + r * 128;
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
          const float4 bb = *reinterpret_cast<const float4*>(&m.bias[cb + c]);
          const float4 ci = *reinterpret_cast<const float4*>(&m.wu_i[cb + c]);
          const int unit = (qp & 1) * 4 + (c >> 2);
          const float2 g01 = tc::logsigmoid_over_tau2(fmaf(u[c + 0] * ri, ci.x, bb.x),
                                                      fmaf(u[c + 1] * ri, ci.y, bb.y), inv_tau, ln2_tau);
          const float2 g23 = tc::logsigmoid_over_tau2(fmaf(u[c + 2] * ri, ci.z, bb.z),
                                                      fmaf(u[c + 3] * ri, ci.w, bb.w), inv_tau, ln2_tau);
          *reinterpret_cast<float4*>(half + ((unit ^ (r & 7)) << 4)) = make_float4(g01.x, g01.y, g23.x, g23.y);
        }
        tc::fence_async_smem();                   // these writes, then the TMA engine's reads
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_one(&m.sfull[l % 3]);
      };
      // the next slab's TMEM columns are requested before this one is formed
      float ua[16], ub[16];
      tmem_ld16(tq + 64 * j0, ua);
      for (int j = 0; j < nslab; j += 2) {
        tc::tmem_ld_wait(ua);                     // slab j in ua
        if (j + 1 < nslab) tmem_ld16(tq + 64 * (j0 + j + 1), ub);
        emit(j, ua);
        if (j + 1 < nslab) {
          tc::tmem_ld_wait(ub);                   // slab j + 1 in ub
          if (j + 2 < nslab) tmem_ld16(tq + 64 * (j0 + j + 2), ua);
          emit(j + 1, ub);
        }
      }
    } else if (lane == 0) {
      for (int l = 0; l < nslab; ++l) {
        uint8_t* slab = tX + (l % 3) * (2 * Layout::kHalfSlab);
        ok &= tc::mbar_wait(&m.sfull[l % 3], (uint32_t)(l / 3) & 1u);
        tma_store_2d(&tmg, 64 * (j0 + l), tok0, slab);
        tma_store_2d(&tmg, 64 * (j0 + l) + 32, tok0, slab + Layout::kHalfSlab);
        bulk_commit();
        bulk_wait_read<0>();
        tc::mbar_arrive_one(&m.sfree[l % 3]);
      }
      bulk_wait<0>();                             // every store done before the block ends
    }
  }
  if (__syncthreads_or(!ok) && tid == 0) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tm, 512);
}

// --------------------------------------------------- rank-16 rows only
// The gate's first half for a summary stage that forms g itself: low = x
// W_down [N, 16] fp32 (the stage-1 product of gate_fwd_tc, its terms summed
// and the rank scales undone), one tile of up to 128 tokens per CTA.  One
// thread per token row writes its 64 bytes.
constexpr int kLowThreads = 128;
struct LowLayout {
  static constexpr int kOffX = 0;
  static constexpr int kOffWd = kOffX + Layout::kX;
  static constexpr int kOffMisc = kOffWd + 3 * Layout::kWd;
  static constexpr int kSmem = kOffMisc + (int)sizeof(Misc) + 1024;
};
static_assert(LowLayout::kOffWd % 1024 == 0, "operand tiles must be 1024-byte aligned");

template <typename TX>
__global__ void __launch_bounds__(kLowThreads, 1)
gate_low_tc(const __grid_constant__ CUtensorMap tmx, const uint8_t* __restrict__ pack, int dm,
            float* __restrict__ low, long long N, int tpc) {
  constexpr bool kBf16 = std::is_same<TX, __nv_bfloat16>::value;
  constexpr int kTerms = kBf16 ? 3 : 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* tX = sm + LowLayout::kOffX;
  uint8_t* tWd = sm + LowLayout::kOffWd;
  Misc& m = *reinterpret_cast<Misc*>(sm + LowLayout::kOffMisc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long tok0 = (long long)blockIdx.x * tpc;

  if (tid == 0) {
    tc::mbar_init(&m.ld, 1);
    for (int a = 0; a < kMaxDm / 64; ++a) tc::mbar_init(&m.ldx[a], 1);
    tc::mbar_init(&m.mma[0], 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&m.tmem, 64);
    tc::tmem_relinquish();
  }
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  pdl_wait();                                     // x and the packed weights may come from the previous kernel
  pdl_trigger();
  const int natoms = dm / 64;
  if (tid == 0) {
    mbar_expect_tx(&m.ld, (uint32_t)(kTerms * Layout::kWd + kRank * 4));
    bulk_g2s(tWd, pack + Pack::kOffWd, kTerms * Layout::kWd, &m.ld);   // the terms' rows side by side
    bulk_g2s(&m.wd_i[0], pack + Pack::kOffScale, kRank * 4, &m.ld);
    for (int a = 0; a < natoms; ++a) {
      mbar_expect_tx(&m.ldx[a], (uint32_t)(kM * 128));
      tma_load_2d(tX + a * (kM * 128), &tmx, a * 64, (int)tok0, &m.ldx[a]);
    }
  }
  __syncthreads();
  const uint32_t tm = m.tmem;
  bool ok = true;
  if (tid == 0) {
    constexpr int kN1 = kTerms * kRank;
    const uint32_t id = idesc16(kM, kN1, 0, 0, kBf16 ? 1 : 0);
    ok &= tc::mbar_wait(&m.ld, 0);
    for (int at = 0; at < natoms; ++at) {
      ok &= tc::mbar_wait(&m.ldx[at], 0);
      tc::tc_after_sync();
      for (int s = 4 * at; s < 4 * at + 4; ++s) {
        const uint64_t a = tc::sdesc(saddr(tX) + (s >> 2) * (kM * 128) + (s & 3) * 32, 16, 1024);
        const uint64_t b = tc::sdesc(saddr(tWd) + (s >> 2) * (kN1 * 128) + (s & 3) * 32, 16, 1024);
        tc::mma_f16(tm + 0, a, b, id, s > 0 ? 1u : 0u);
      }
    }
    tc::mma_commit(&m.mma[0]);
  }
  ok &= tc::mbar_wait(&m.ld, 0);
  ok &= tc::mbar_wait(&m.mma[0], 0);
  tc::tc_after_sync();
  {
    float lw[16], lt[16];
    tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + 0, lw);
    tc::tmem_ld_wait(lw);
#pragma unroll
    for (int t = 1; t < kTerms; ++t) {
      tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + t * kRank, lt);
      tc::tmem_ld_wait(lt);
#pragma unroll
      for (int c = 0; c < 16; ++c) lw[c] += lt[c];
    }
    const int r = warp * 32 + lane;
    if (ok && r < tpc && tok0 + r < N) {
      float4* dst = reinterpret_cast<float4*>(low + (tok0 + r) * kRank);
#pragma unroll
      for (int c = 0; c < 16; c += 4)
        dst[c / 4] = make_float4(lw[c] * m.wd_i[c], lw[c + 1] * m.wd_i[c + 1], lw[c + 2] * m.wd_i[c + 2],
                                 lw[c + 3] * m.wd_i[c + 3]);
    }
  }
  ok = __syncthreads_and(ok) != 0;
  if (!ok && tid == 0) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  tc::tc_after_sync();
  if (warp == 0) tc::tmem_dealloc(tm, 64);
}

}  // namespace gate_tc

// Shapes the tensor-core gate kernels take: 16-bit x, d_model a multiple of 64
// up to 384, rank 16, H*dk a multiple of 64 up to 448.
inline bool gate_tc_supported(int x_dtype, int dm, int rank, int HD) {
  return (x_dtype == kF16 || x_dtype == kBF16) && dm % 64 == 0 && dm <= gate_tc::kMaxDm &&
         rank == gate_tc::kRank && HD % 64 == 0 && HD <= gate_tc::kMaxHD;
}
// Tokens per CTA: about N / #SMs rounded up to a multiple of 16, at most 128.
inline int gate_tc_tile(long long N, int sms) {
  long long t = (N + sms - 1) / (sms > 0 ? sms : 1);
  t = (t + 15) / 16 * 16;
  return (int)(t < 16 ? 16 : t > gate_tc::kM ? gate_tc::kM : t);
}
// The forward kernel's grid: (token tiles of *tpc tokens) x (column blocks of
// *spb 64-column slabs).  A block's epilogue time grows with its slabs, not
// with its tokens (its warps cover all 128 TMEM lanes), so when the token
// tiles of 128 times the slabs fit on the SMs, the columns are split too,
// one slab per block.
inline void gate_tc_grid(long long N, int HD, int sms, int* tpc, int* spb, long long* rows, int* cols) {
  const int nslab = HD / 64;
  if (sms > 0 && (N + gate_tc::kM - 1) / gate_tc::kM * nslab <= sms) {
    *tpc = gate_tc_tile(N * nslab, sms);        // about N nslab / #SMs tokens per block
    *spb = 1;
  } else {
    *tpc = gate_tc_tile(N, sms);
    *spb = nslab;
  }
  *rows = (N + *tpc - 1) / *tpc;
  *cols = (nslab + *spb - 1) / *spb;
}

}  // namespace gtr

// pipe_kernels.cuh -- the chunk-parallel tcgen05 path of the Key-only GLA
// (sm_100a): 16-bit q/k/v/z, fp32 gates, dk = dv = 64, chunk C = 64.
//
// The three stages of the GTR article's chunkwise operator (方法详解 §4
// "硬件感知分块推理算子": chunk summaries on tensor cores, a light sequential
// pass over the chunk-boundary states with coalesced accesses, chunk outputs
// with the scores kept on chip and the output gate fused into the epilogue),
// each a kernel over independent work items:
//
//   gla_sum_pipe   one item per (sequence, chunk): the chunk's own state
//                  increment dS_c^T = V^T k^ (k^_j = k_j e^{Gam - G_j}, the
//                  decay from token j to the chunk end, at most one) and its
//                  decay factor a_c = e^{Gam}.
//   gla_chunk_scan the sequential pass: S_c = a_c (.) S_{c-1} + dS_c over the
//                  chunks of each sequence, per state element, writing the
//                  state each chunk starts from as the two-term bf16 operand
//                  tiles the output kernel multiplies.
//   gla_out_pipe   one item per (sequence, chunk): o = q~ S + mask(q~ k~^T) V
//                  (q~ = q e^{G}, k~ = k e^{-G}, referenced to the chunk start),
//                  RMSNorm x w x SiLU(z), stored at the tokens' grid rows.
//
// Nothing is sequential inside the summary and output kernels, so each is a
// persistent warp-specialised pipeline: one CTA per SM walks its items
// (blockIdx.x, + gridDim.x, ...) with a loader warp (tensor-map box loads or
// cp.async gathers), an MMA warp (one thread issues every tcgen05.mma), eight
// builder warps (in-chunk cumsum and operand tiles) and four epilogue warps
// (tensor memory -> registers -> global), hand-offs on mbarriers, and two or
// four slots of shared and tensor memory so that consecutive items overlap.
//
// State tiles.  For chunk c of sequence bh the workspace holds 16 KB at
// ((bh * nc) + c) * 16384: two 8 KB halves in the SWIZZLE_128B K-major
// operand layout of a 64 x 64 16-bit tile whose rows are the value dims j and
// whose columns are the key dims i (S^T).  The summary kernel writes dS^T in
// fp32 into the same 16 KB: the 8 values (j, 8u .. 8u+7) of swizzle unit
// (j, u) go 4 to the first half's unit and 4 to the second half's, so the
// scan reads and rewrites each unit in place (the bf16 hi term of the 8
// values into the first half, the lo term into the second), one thread per
// unit, with no other thread touching it.
#pragma once
#include "tc_kernels.cuh"

namespace gtr {
namespace tc {

// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// The arrive-on of all this thread's earlier cp.async copies (counted among
// the barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* b) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(saddr(b)) : "memory");
}
// The CTA's abort flag (set by a role whose bounded wait ran out), re-read every time.
__device__ __forceinline__ bool aborted(const int* f) { return *reinterpret_cast<const volatile int*>(f) != 0; }
// 16-byte cp.async that reads `src_bytes` (16 or 0) and zero-fills the rest.
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

// Parameters of the pipelined kernels.  Items run over nbh sequences (bh0 ..
// bh0 + nbh - 1 of the B*H in the tensors) times nc chunks.
struct PipeParams {
  const void* q; const void* k; const void* v; const float* g; const void* z; const float* w;
  uint8_t* st;          // state tiles, 16 KB per (sequence, chunk)
  float* a;             // chunk decay factors e^{Gam}, 64 per (sequence, chunk)
  void* out;
  float* states;        // chunk scan, inclusive fp32 mode: [nbh, nc, 64, 64] (else null)
  int H, T, gh, gw, dir, nc, bh0, nbh;
  int tma;              // 1: chunks arrive by tensor-map box loads (Maps valid)
};

constexpr int kStateTile = 2 * kTile;     // 16 KB per chunk state
constexpr int kPipeThreads = 14 * 32;     // loader, MMA, 8 builder warps, 4 epilogue warps
constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpBuild0 = 2, kWarpEpi0 = 10;
constexpr int kBarBuild = 1, kBarEpi = 2;  // named barriers: builders (256), epilogue warps (128)

// One work item: chunk c of sequence bh (batch b, head h), scan direction d.
struct Item {
  int bhl, c, b, h, d, s0, ntok, rmask;
};
__device__ __forceinline__ Item pipe_item(const PipeParams& p, int idx) {
  Item it;
  it.bhl = idx / p.nc;
  it.c = idx - it.bhl * p.nc;
  const int bh = p.bh0 + it.bhl;
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  it.d = dir_of_batch(p.dir, it.b);
  it.s0 = it.c * kC;
  it.ntok = min(kC, p.T - it.s0);
  it.rmask = (p.tma && dir_reversed(it.d)) ? kC - 1 : 0;
  return it;
}
// Grid row of the token at scan offset j of the item (j < ntok).
__device__ __forceinline__ long long item_row(const PipeParams& p, const Item& it, int j) {
  return ((long long)it.b * p.T + scan_to_grid(it.d, it.s0 + j, p.T, p.gh, p.gw)) * p.H + it.h;
}
// Items of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
__device__ __forceinline__ int pipe_count(int total) {
  return total > (int)blockIdx.x ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
}
__device__ __forceinline__ int pipe_index(int n) { return (int)blockIdx.x + n * (int)gridDim.x; }

// Gathered chunk rows (no box layout): lane l copies scan offsets l and l + 32
// of the 16-bit tensors in `which` (bit 0 q, 1 k, 2 v) and of the gate, 16
// bytes per cp.async; offsets past ntok read zeros.  q, k land row-major, v in
// the SWIZZLE_128B operand layout; completes on `bar` (an arrive per lane).
__device__ __forceinline__ void gather_chunk(const PipeParams& p, const Item& it, int lane, unsigned which,
                                             uint8_t* qdst, uint8_t* kdst, uint8_t* vdst, uint8_t* gdst,
                                             uint64_t* bar) {
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int j = lane + 32 * r;
    const bool ok = j < it.ntok;
    const long long row = ok ? item_row(p, it, j) : 0;
    const uint32_t nb = ok ? 16u : 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (which & 1u) cp_async16_zfill(qdst + j * 128 + u * 16, (const uint8_t*)p.q + row * kRowBytes + u * 16, nb);
      if (which & 2u) cp_async16_zfill(kdst + j * 128 + u * 16, (const uint8_t*)p.k + row * kRowBytes + u * 16, nb);
      if (which & 4u) cp_async16_zfill(vdst + sw_unit(j, u), (const uint8_t*)p.v + row * kRowBytes + u * 16, nb);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u)
      cp_async16_zfill(gdst + j * 256 + u * 16, (const uint8_t*)p.g + row * (kD * 4) + u * 16, nb);
  }
  cp_async_arrive_noinc(bar);
}
// Box loads of the item's tensors (tensor maps), issued by one thread.
__device__ __forceinline__ void box_load(const PipeParams& p, const Maps& mp, int which, void* dst, uint64_t* bar,
                                         const Item& it) {
  const int t0 = dir_reversed(it.d) ? p.T - it.s0 - kC : it.s0;
  if (!dir_orient(it.d)) {
    tma_load_4d(dst, &mp.t[0][which], 0, it.h, t0, it.b, bar);
  } else {
    const int col = t0 / p.gh, r0 = t0 - col * p.gh;
    tma_load_5d(dst, &mp.t[1][which], 0, it.h, col, r0, it.b, bar);
  }
}

// In-chunk inclusive cumsum of the staged gate (scan order) for the builder
// thread's eight scan offsets tb .. tb+7 and dims dc, dc+1: gc[i] = G at
// offset tb + i; returns the chunk total Gam.  `part` holds the warps'
// partial sums; one builder barrier.
__device__ __forceinline__ float2 chunk_cumsum(const float* G, float2 (&gc)[8], float (*part)[kD], int bw,
                                               int tb, int dc, int rmask) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    gc[i] = *reinterpret_cast<const float2*>(G + ((tb + i) ^ rmask) * kD + dc);
    if (i) { gc[i].x += gc[i - 1].x; gc[i].y += gc[i - 1].y; }
  }
  *reinterpret_cast<float2*>(&part[bw][dc]) = gc[7];
  named_barrier(kBarBuild, kThreads);
  float2 off = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float2 pp = *reinterpret_cast<const float2*>(&part[w][dc]);
    if (w < bw) { off.x += pp.x; off.y += pp.y; }
    tot.x += pp.x; tot.y += pp.y;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) { gc[i].x += off.x; gc[i].y += off.y; }
  return tot;
}

// =========================================================== summary (K2)
struct SumPipeLayout {
  static constexpr int kSlots = 4;
  // per slot: k (row-major), v (operand layout), k^ hi, lo (operand layout), gate (fp32 rows)
  static constexpr int kOffK = 0, kOffV = kTile, kOffKH = 2 * kTile, kOffKL = 3 * kTile, kOffG = 4 * kTile;
  static constexpr int kSlot = 4 * kTile + kGTile;
  static constexpr int kMisc = kSlots * kSlot;
  static constexpr int kTmemCols = 256;   // 64 per slot
};
struct SumPipeMisc {
  uint64_t full[SumPipeLayout::kSlots];    // the item's k, v, g have landed
  uint64_t built[SumPipeLayout::kSlots];   // k^ tiles written
  uint64_t mma[SumPipeLayout::kSlots];     // dS^T product complete (slot's tiles free)
  uint64_t tfree[SumPipeLayout::kSlots];   // accumulator read out
  uint32_t tmem;
  int abort;
  alignas(16) float part[kWarps][kD];
};
constexpr int kSumPipeSmem = SumPipeLayout::kMisc + (int)sizeof(SumPipeMisc) + 1024;
static_assert(kSumPipeSmem <= 227 * 1024, "summary pipeline must fit one SM");

template <typename T>
__global__ void __launch_bounds__(kPipeThreads, 1)
gla_sum_pipe(const __grid_constant__ PipeParams p, const __grid_constant__ Maps mp) {
  using L = SumPipeLayout;
  constexpr int NS = L::kSlots;
  constexpr bool kH = std::is_same<T, __half>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  SumPipeMisc& m = *reinterpret_cast<SumPipeMisc*>(sm + L::kMisc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.nbh * p.nc;
  const int nit = pipe_count(total);
  const bool tma = p.tma != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&m.full[s], tma ? 1 : 32);
      mbar_init(&m.built[s], 1);
      mbar_init(&m.mma[s], 1);
      mbar_init(&m.tfree[s], 1);
    }
    m.abort = 0;
    mbar_fence_init();
  }
  if (warp == kWarpLoad) {
    tmem_alloc(&m.tmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = m.tmem;
  bool failed = false;

  if (warp == kWarpLoad) {
    // ---- loader: k and v are inputs, their first boxes go out before the
    // dependency wait; the gate comes from the previous kernel
    int issued = 0;
    const int pre = min(nit, NS);
    if (tma && lane == 0) {
      for (int n = 0; n < pre; ++n) {
        const Item it = pipe_item(p, pipe_index(n));
        uint8_t* sl = sm + n * L::kSlot;
        mbar_arrive_tx(&m.full[n], 2 * kTile + kGTile);
        box_load(p, mp, kMapK, sl + L::kOffK, &m.full[n], it);
        box_load(p, mp, kMapV, sl + L::kOffV, &m.full[n], it);
      }
    }
    pdl_wait();
    pdl_trigger();
    for (int n = 0; n < nit; ++n) {
      const int s = n % NS, use = n / NS;
      uint8_t* sl = sm + s * L::kSlot;
      const Item it = pipe_item(p, pipe_index(n));
      if (n >= NS) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&m.mma[s], (uint32_t)(use - 1) & 1u);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) { failed = true; break; }
      }
      if (tma) {
        if (lane == 0) {
          if (n >= pre) {
            mbar_arrive_tx(&m.full[s], 2 * kTile + kGTile);
            box_load(p, mp, kMapK, sl + L::kOffK, &m.full[s], it);
            box_load(p, mp, kMapV, sl + L::kOffV, &m.full[s], it);
          }
          box_load(p, mp, kMapG, sl + L::kOffG, &m.full[s], it);
        }
      } else {
        gather_chunk(p, it, lane, 6u, nullptr, sl + L::kOffK, sl + L::kOffV, sl + L::kOffG, &m.full[s]);
      }
      issued = n + 1;
      // (items before `pre` had their k, v boxes issued before the wait: their
      // gates go out too, so that every barrier they expect completes)
      if (issued >= pre && __shfl_sync(0xffffffffu, aborted(&m.abort), 0)) { failed = true; break; }
    }
    // every copy issued lands before the CTA leaves
    if (lane == 0)
      for (int n = max(0, issued - NS); n < issued; ++n)
        if (!mbar_wait(&m.full[n % NS], (uint32_t)(n / NS) & 1u)) failed = true;
    if (!tma) cp_async_wait<0>();
  } else if (warp == kWarpMma) {
    constexpr uint32_t kIdVK = kH ? idesc_f16(1, 1) : idesc_bf16(1, 1);   // both MN-major
    int issued = 0;
    if (lane == 0) {
      for (int n = 0; n < nit; ++n) {
        const int s = n % NS, use = n / NS;
        uint8_t* sl = sm + s * L::kSlot;
        if (!mbar_wait(&m.built[s], (uint32_t)use & 1u)) { failed = true; break; }
        if (use > 0 && !mbar_wait(&m.tfree[s], (uint32_t)(use - 1) & 1u)) { failed = true; break; }
        tc_after_sync();
        // dS^T = V^T k^ (rows dv, columns dk): A = V, B = k^ hi then lo, both MN-major
        const uint32_t d = tm + 64u * (uint32_t)s;
        mma_k64<kStepMN, kStepMN>(d, desc_mn(sl + L::kOffV), desc_mn(sl + L::kOffKH), kIdVK, false);
        mma_k64<kStepMN, kStepMN>(d, desc_mn(sl + L::kOffV), desc_mn(sl + L::kOffKL), kIdVK, true);
        mma_commit(&m.mma[s]);
        issued = n + 1;
      }
      if (issued > 0 && !mbar_wait(&m.mma[(issued - 1) % NS], (uint32_t)((issued - 1) / NS) & 1u)) failed = true;
    }
  } else if (warp < kWarpEpi0) {
    // ---- builders: cumsum, weights e^{Gam - G_j}, k^ two-term (rows in the
    // staging order, which V shares, so no reordering in any scan order)
    pdl_wait();
    pdl_trigger();
    const int bt = threadIdx.x - 32 * kWarpBuild0, bw = bt >> 5;
    const int dc = 2 * lane, tb = 8 * bw;
    for (int n = 0; n < nit; ++n) {
      const int s = n % NS, use = n / NS;
      uint8_t* sl = sm + s * L::kSlot;
      const Item it = pipe_item(p, pipe_index(n));
      failed |= !mbar_wait(&m.full[s], (uint32_t)use & 1u);
      if (named_barrier_or(kBarBuild, kThreads, failed || aborted(&m.abort))) { failed = true; break; }
      float2 gc[8];
      const float2 tot = chunk_cumsum(reinterpret_cast<const float*>(sl + L::kOffG), gc, m.part, bw, tb, dc,
                                      it.rmask);
      const T* kst = reinterpret_cast<const T*>(sl + L::kOffK);
      uint8_t* KH = sl + L::kOffKH;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rs = (tb + i) ^ it.rmask;
        const uint32_t o = sw16(rs, dc);
        const float2 kk = ld2(kst + rs * kD + dc);
        const float wa = ex2((tot.x - gc[i].x) * kLog2e), wb = ex2((tot.y - gc[i].y) * kLog2e);
        if (kH) put2h(KH, KH + kTile, o, kk.x * wa, kk.y * wb);
        else put2x(KH, KH + kTile, o, kk.x * wa, kk.y * wb);
      }
      if (bw == 0)
        *reinterpret_cast<float2*>(p.a + ((size_t)it.bhl * p.nc + it.c) * kD + dc) =
            make_float2(expf(tot.x), expf(tot.y));
      fence_async_smem();
      named_barrier(kBarBuild, kThreads);   // tiles written; partials read
      if (bt == 0) mbar_arrive_one(&m.built[s]);
    }
    if (failed && bt == 0) m.abort = 1;
  } else {
    // ---- epilogue warps: dS^T from tensor memory into the state tile
    pdl_wait();
    pdl_trigger();
    const int qd = warp & 3;
    const int row = qd * 16 + (lane & 15), ch = lane >> 4;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    for (int n = 0; n < nit; ++n) {
      const int s = n % NS, use = n / NS;
      const Item it = pipe_item(p, pipe_index(n));
      failed |= !mbar_wait(&m.mma[s], (uint32_t)use & 1u);
      if (named_barrier_or(kBarEpi, 128, failed || aborted(&m.abort))) { failed = true; break; }
      tc_after_sync();
      float v0[16], v1[16];
      tmem_ld16x2(tm + 64u * (uint32_t)s + lane_base, v0);
      tmem_ld16x2(tm + 64u * (uint32_t)s + lane_base + 32, v1);
      tmem_ld_wait(v0);
      tmem_ld_wait(v1);
      tc_before_sync();
      named_barrier(kBarEpi, 128);
      if (warp == kWarpEpi0 && lane == 0) mbar_arrive_one(&m.tfree[s]);
      // columns (key dims) ch*16 .. +15 from v0 and 32 + ch*16 .. +15 from v1:
      // units u = 2 ch, 2 ch + 1, 4 + 2 ch, 5 + 2 ch of row `row`
      uint8_t* dst = p.st + ((size_t)it.bhl * p.nc + it.c) * kStateTile;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* x = q < 2 ? v0 + 8 * q : v1 + 8 * (q - 2);
        const int u = (q < 2 ? 0 : 4) + 2 * ch + (q & 1);
        const uint32_t o = sw_unit(row, u);
        *reinterpret_cast<float4*>(dst + o) = make_float4(x[0], x[1], x[2], x[3]);
        *reinterpret_cast<float4*>(dst + kTile + o) = make_float4(x[4], x[5], x[6], x[7]);
      }
    }
    if (failed && threadIdx.x == 32 * kWarpEpi0) m.abort = 1;
  }
  if (failed) gtr_flag(kStatusMbarTimeout);
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  if (warp == kWarpLoad) tmem_dealloc(tm, L::kTmemCols);
}

// ======================================================= chunk scan (K3)
// Block = one (sequence, value dim j): 8 units u (key dims 8u .. 8u+7) x 32
// ranges of consecutive chunks.  Each thread reduces its range to an affine
// map S -> P (.) S + R, the ranges exchange maps through shared memory, and
// each replays its range from the composed entering state, writing the state
// each chunk starts from (two-term bf16, in place) or, in inclusive fp32 mode,
// the state each chunk ends with into p.states.
constexpr int kScanRanges = 32;
constexpr int kChunkScanThreads = 8 * kScanRanges;
constexpr int kScanWin = 4;

__global__ void __launch_bounds__(kChunkScanThreads)
gla_chunk_scan(const __grid_constant__ PipeParams p) {
  __shared__ float4 mapP[kScanRanges][8][2], mapR[kScanRanges][8][2];
  pdl_wait();
  pdl_trigger();
  const int u = threadIdx.x & 7, part = threadIdx.x >> 3;
  const int bhl = blockIdx.x >> 6, j = blockIdx.x & 63;
  const int len = (p.nc + kScanRanges - 1) / kScanRanges;
  const int ca = min(p.nc, part * len), cb = min(p.nc, ca + len);
  uint8_t* base = p.st + (size_t)bhl * p.nc * kStateTile;
  const float* abase = p.a + (size_t)bhl * p.nc * kD + 8 * u;
  const uint32_t o = sw_unit(j, u);

  float P[8], R[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) { P[e] = 1.f; R[e] = 0.f; }
  for (int c0 = ca; c0 < cb; c0 += kScanWin) {
    float4 d[kScanWin][2], a[kScanWin][2];
#pragma unroll
    for (int w = 0; w < kScanWin; ++w) {
      if (c0 + w < cb) {
        const uint8_t* t = base + (size_t)(c0 + w) * kStateTile;
        d[w][0] = *reinterpret_cast<const float4*>(t + o);
        d[w][1] = *reinterpret_cast<const float4*>(t + kTile + o);
        a[w][0] = *reinterpret_cast<const float4*>(abase + (size_t)(c0 + w) * kD);
        a[w][1] = *reinterpret_cast<const float4*>(abase + (size_t)(c0 + w) * kD + 4);
      }
    }
#pragma unroll
    for (int w = 0; w < kScanWin; ++w) {
      if (c0 + w < cb) {
        const float dd[8] = {d[w][0].x, d[w][0].y, d[w][0].z, d[w][0].w, d[w][1].x, d[w][1].y, d[w][1].z, d[w][1].w};
        const float aa[8] = {a[w][0].x, a[w][0].y, a[w][0].z, a[w][0].w, a[w][1].x, a[w][1].y, a[w][1].z, a[w][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) { R[e] = fmaf(aa[e], R[e], dd[e]); P[e] *= aa[e]; }
      }
    }
  }
  mapP[part][u][0] = make_float4(P[0], P[1], P[2], P[3]);
  mapP[part][u][1] = make_float4(P[4], P[5], P[6], P[7]);
  mapR[part][u][0] = make_float4(R[0], R[1], R[2], R[3]);
  mapR[part][u][1] = make_float4(R[4], R[5], R[6], R[7]);
  __syncthreads();
  float S[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) S[e] = 0.f;
  for (int r = 0; r < part; ++r) {
    const float4 p0 = mapP[r][u][0], p1 = mapP[r][u][1], r0 = mapR[r][u][0], r1 = mapR[r][u][1];
    const float pp[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    const float rr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) S[e] = fmaf(pp[e], S[e], rr[e]);
  }
  for (int c0 = ca; c0 < cb; c0 += kScanWin) {
    float4 d[kScanWin][2], a[kScanWin][2];
#pragma unroll
    for (int w = 0; w < kScanWin; ++w) {
      if (c0 + w < cb) {
        const uint8_t* t = base + (size_t)(c0 + w) * kStateTile;
        d[w][0] = *reinterpret_cast<const float4*>(t + o);
        d[w][1] = *reinterpret_cast<const float4*>(t + kTile + o);
        a[w][0] = *reinterpret_cast<const float4*>(abase + (size_t)(c0 + w) * kD);
        a[w][1] = *reinterpret_cast<const float4*>(abase + (size_t)(c0 + w) * kD + 4);
      }
    }
#pragma unroll
    for (int w = 0; w < kScanWin; ++w) {
      if (c0 + w < cb) {
        const int c = c0 + w;
        const float dd[8] = {d[w][0].x, d[w][0].y, d[w][0].z, d[w][0].w, d[w][1].x, d[w][1].y, d[w][1].z, d[w][1].w};
        const float aa[8] = {a[w][0].x, a[w][0].y, a[w][0].z, a[w][0].w, a[w][1].x, a[w][1].y, a[w][1].z, a[w][1].w};
        if (p.states) {
#pragma unroll
          for (int e = 0; e < 8; ++e) S[e] = fmaf(aa[e], S[e], dd[e]);
          float* dst = p.states + ((size_t)bhl * p.nc + c) * (kD * kD) + (size_t)(8 * u) * kD + j;
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e * kD] = S[e];
        } else {
          // the state the chunk starts from, as the bf16 terms hi + lo
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) split2(S[2 * e], S[2 * e + 1], hi[e], lo[e]);
          uint8_t* t = base + (size_t)c * kStateTile;
          *reinterpret_cast<uint4*>(t + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(t + kTile + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
#pragma unroll
          for (int e = 0; e < 8; ++e) S[e] = fmaf(aa[e], S[e], dd[e]);
        }
      }
    }
  }
}

// =========================================================== output (K4)
struct OutPipeLayout {
  // per slot, operand tiles (1024-aligned): S^T hi, k~ hi, S^T lo, k~ lo, q~
  // hi, lo, V hi, lo; [S^T; k~] hi and lo are each one 128-row K-major B
  static constexpr int kSH = 0, kKH = kTile, kSL = 2 * kTile, kKL = 3 * kTile, kQH = 4 * kTile,
                       kQL = 5 * kTile, kVH = 6 * kTile, kVL = 7 * kTile;
  static constexpr int kOp = 8 * kTile;
  // per slot, staging: q, k (row-major), v (operand layout), gate (fp32 rows)
  static constexpr int kRq = 0, kRk = kTile, kRv = 2 * kTile, kRg = 3 * kTile;
  static constexpr int kRaw = 3 * kTile + kGTile;
  static constexpr int kOffRaw = 2 * kOp;
  static constexpr int kMisc = 2 * kOp + 2 * kRaw;
  // tensor memory per slot (256 columns): o [0, 64), scores [64, 128), P hi [128, 160), P lo [160, 192)
  static constexpr int kTmemCols = 512;
};
struct OutPipeMisc {
  uint64_t full[2];     // staging landed
  uint64_t sfull[2];    // state tiles (and a direct v) landed
  uint64_t rawfree[2];  // builders done with the staging
  uint64_t built[2];    // q~, k~, V tiles written
  uint64_t mma1[2];     // q~ [S^T; k~]^T complete
  uint64_t pready[2];   // P written (tensor memory, or the q~ tiles for an exact chunk)
  uint64_t mma2[2];     // P V complete (the slot's operand tiles are free)
  uint64_t tfree[2];    // o read out (the slot's tensor memory is free)
  uint32_t tmem;
  int abort;
  int exact[2];
  alignas(16) float part[kWarps][kD];
  alignas(16) float wv[kD];
};
constexpr int kOutPipeSmem = OutPipeLayout::kMisc + (int)sizeof(OutPipeMisc) + 1024;
static_assert(kOutPipeSmem <= 227 * 1024, "output pipeline must fit one SM");

// A bf16 v read in scan order by a box load lands in the V operand tile itself.
__device__ __forceinline__ bool v_direct(bool two_term_v, bool tma, const Item& it) {
  return !two_term_v && tma && it.rmask == 0;
}

template <typename T>
__global__ void __launch_bounds__(kPipeThreads, 1)
gla_out_pipe(const __grid_constant__ PipeParams p, const __grid_constant__ Maps mp) {
  using L = OutPipeLayout;
  constexpr bool kV2 = std::is_same<T, __half>::value;   // fp16 V: two bf16 terms
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  OutPipeMisc& m = *reinterpret_cast<OutPipeMisc*>(sm + L::kMisc);
  auto op = [&](int s) -> uint8_t* { return sm + s * L::kOp; };
  auto raw = [&](int s) -> uint8_t* { return sm + L::kOffRaw + s * L::kRaw; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = p.nbh * p.nc;
  const int nit = pipe_count(total);
  const bool tma = p.tma != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&m.full[s], tma ? 1 : 32);
      mbar_init(&m.sfull[s], 1);
      mbar_init(&m.rawfree[s], 1);
      mbar_init(&m.built[s], 1);
      mbar_init(&m.mma1[s], 1);
      mbar_init(&m.pready[s], 1);
      mbar_init(&m.mma2[s], 1);
      mbar_init(&m.tfree[s], 1);
    }
    m.abort = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < kD) m.wv[threadIdx.x] = p.w ? p.w[threadIdx.x] : 1.0f;
  if (warp == kWarpLoad) {
    tmem_alloc(&m.tmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = m.tmem;
  bool failed = false;

  if (warp == kWarpLoad) {
    // ---- loader.  q, k, v, g are complete before the scan kernel lets this
    // one start, so staging loads need no wait; the state tiles do.
    int nr = 0, ns = 0;
    bool waited = false;
    unsigned long long t_idle = 0;
    while (ns < nit) {
      bool progressed = false;
      if (nr < nit) {
        const int s = nr & 1, use = nr >> 1;
        bool ok = use == 0 || (lane == 0 && mbar_test(&m.rawfree[s], (uint32_t)(use - 1) & 1u));
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
          const Item it = pipe_item(p, pipe_index(nr));
          uint8_t* r = raw(s);
          const bool vd = v_direct(kV2, tma, it);
          if (tma) {
            if (lane == 0) {
              mbar_arrive_tx(&m.full[s], 2 * kTile + kGTile + (vd ? 0 : kTile));
              box_load(p, mp, kMapQ, r + L::kRq, &m.full[s], it);
              box_load(p, mp, kMapK, r + L::kRk, &m.full[s], it);
              if (!vd) box_load(p, mp, kMapV, r + L::kRv, &m.full[s], it);
              box_load(p, mp, kMapG, r + L::kRg, &m.full[s], it);
            }
          } else {
            gather_chunk(p, it, lane, 7u, r + L::kRq, r + L::kRk, r + L::kRv, r + L::kRg, &m.full[s]);
          }
          ++nr;
          progressed = true;
        }
      }
      if (ns < nr) {
        const int s = ns & 1, use = ns >> 1;
        bool ok = use == 0 || (lane == 0 && mbar_test(&m.mma2[s], (uint32_t)(use - 1) & 1u));
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
          if (!waited) {
            pdl_wait();                   // the state tiles come from the scan kernel
            pdl_trigger();
            waited = true;
          }
          const Item it = pipe_item(p, pipe_index(ns));
          if (lane == 0) {
            const bool vd = v_direct(kV2, tma, it);
            const uint8_t* src = p.st + ((size_t)it.bhl * p.nc + it.c) * kStateTile;
            mbar_arrive_tx(&m.sfull[s], kStateTile + (vd ? kTile : 0));
            bulk_g2s(op(s) + L::kSH, src, kTile, &m.sfull[s]);
            bulk_g2s(op(s) + L::kSL, src + kTile, kTile, &m.sfull[s]);
            if (vd) box_load(p, mp, kMapV, op(s) + L::kVH, &m.sfull[s], it);
          }
          ++ns;
          progressed = true;
        }
      }
      if (progressed) {
        t_idle = 0;
      } else {
        if (__shfl_sync(0xffffffffu, aborted(&m.abort), 0)) { failed = true; break; }
        const unsigned long long now = globaltimer();
        if (t_idle == 0) t_idle = now;
        else if (now - t_idle > kWaitNs) { failed = true; break; }
      }
    }
    if (!waited) { pdl_wait(); pdl_trigger(); }
    // every copy issued lands before the CTA leaves
    if (lane == 0) {
      for (int n = max(0, nr - 2); n < nr; ++n)
        if (!mbar_wait(&m.full[n & 1], (uint32_t)(n >> 1) & 1u)) failed = true;
      for (int n = max(0, ns - 2); n < ns; ++n)
        if (!mbar_wait(&m.sfull[n & 1], (uint32_t)(n >> 1) & 1u)) failed = true;
    }
    if (!tma) cp_async_wait<0>();
    if (failed && lane == 0) m.abort = 1;
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t kIdQSK = idesc_bf16(0, 0, 128);   // both K-major, N = 128: q~ [S^T; k~]^T
      constexpr uint32_t kIdPV = idesc_bf16(0, 1);          // A K-major, B MN-major: P V
      int n1 = 0, n2 = 0;
      unsigned long long t_idle = 0;
      while (n2 < nit) {
        bool progressed = false;
        if (n1 < nit) {
          const int s = n1 & 1, use = n1 >> 1;
          if (mbar_test(&m.built[s], (uint32_t)use & 1u) && mbar_test(&m.sfull[s], (uint32_t)use & 1u) &&
              (use == 0 || mbar_test(&m.tfree[s], (uint32_t)(use - 1) & 1u))) {
            tc_after_sync();
            uint8_t* o = op(s);
            mma_terms<kStepK, kStepK>(tm + 256u * s, desc_k(o + L::kQH), desc_k(o + L::kQL),
                                      desc_k(o + L::kSH), desc_k(o + L::kSL), true, kIdQSK, false);
            mma_commit(&m.mma1[s]);
            ++n1;
            progressed = true;
          }
        }
        if (n2 < n1) {
          const int s = n2 & 1, use = n2 >> 1;
          if (mbar_test(&m.pready[s], (uint32_t)use & 1u)) {
            tc_after_sync();
            uint8_t* o = op(s);
            const uint32_t d = tm + 256u * s;
            const uint64_t vh = desc_mn(o + L::kVH), vl = desc_mn(o + L::kVL);
            if (!m.exact[s])
              mma_terms_ts<kStepMN>(d, d + 128, d + 160, vh, vl, kV2, kIdPV);
            else   // an exact chunk's P is in the q~ tiles
              mma_terms<kStepK, kStepMN>(d, desc_k(o + L::kQH), desc_k(o + L::kQL), vh, vl, kV2, kIdPV, true);
            mma_commit(&m.mma2[s]);
            ++n2;
            progressed = true;
          }
        }
        if (progressed) {
          t_idle = 0;
        } else {
          if (aborted(&m.abort)) { failed = true; break; }
          const unsigned long long now = globaltimer();
          if (t_idle == 0) t_idle = now;
          else if (now - t_idle > kWaitNs) { failed = true; break; }
        }
      }
      // the last products complete before tensor memory is released
      if (n1 > n2 && !mbar_wait(&m.mma1[(n1 - 1) & 1], (uint32_t)((n1 - 1) >> 1) & 1u)) failed = true;
      if (n2 > 0 && !mbar_wait(&m.mma2[(n2 - 1) & 1], (uint32_t)((n2 - 1) >> 1) & 1u)) failed = true;
      if (failed) m.abort = 1;
    }
  } else if (warp < kWarpEpi0) {
    // ---- builders: cumsum, exact-chunk test, q~ = q e^{G}, k~ = k e^{-G}
    // and V as two-term bf16 operand tiles in scan order
    const int bt = threadIdx.x - 32 * kWarpBuild0, bw = bt >> 5;
    const int dc = 2 * lane, tb = 8 * bw;
    bool prev_exact[2] = {false, false};
    for (int n = 0; n < nit; ++n) {
      const int s = n & 1, use = n >> 1;
      const Item it = pipe_item(p, pipe_index(n));
      const bool vd = v_direct(kV2, tma, it);
      uint8_t* r = raw(s);
      uint8_t* o = op(s);
      failed |= !mbar_wait(&m.full[s], (uint32_t)use & 1u);
      if (use > 0) {
        failed |= !mbar_wait(&m.mma2[s], (uint32_t)(use - 1) & 1u);   // the slot's tiles are free
        // after an exact chunk the epilogue warps read its flag before it is rewritten
        if (prev_exact[s]) failed |= !mbar_wait(&m.tfree[s], (uint32_t)(use - 1) & 1u);
      }
      if (named_barrier_or(kBarBuild, kThreads, failed || aborted(&m.abort))) { failed = true; break; }
      float* G = reinterpret_cast<float*>(r + L::kRg);
      float2 gc[8];
      chunk_cumsum(G, gc, m.part, bw, tb, dc, it.rmask);
      int bad = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        bad |= !(gc[i].x <= 0.f && gc[i].x >= -kSpanMax && gc[i].y <= 0.f && gc[i].y >= -kSpanMax);
      const T* qst = reinterpret_cast<const T*>(r + L::kRq);
      const T* kst = reinterpret_cast<const T*>(r + L::kRk);
      {
        uint32_t qr[8], kr[8], vr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rs = (tb + i) ^ it.rmask;
          qr[i] = *reinterpret_cast<const uint32_t*>(qst + rs * kD + dc);
          kr[i] = *reinterpret_cast<const uint32_t*>(kst + rs * kD + dc);
          vr[i] = vd ? 0u : *reinterpret_cast<const uint32_t*>(r + L::kRv + sw16(rs, dc));
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t off = sw16(tb + i, dc);
          const float2 qq = ld2(reinterpret_cast<const T*>(&qr[i])), kk = ld2(reinterpret_cast<const T*>(&kr[i]));
          const float x0 = gc[i].x * kLog2e, x1 = gc[i].y * kLog2e;
          put2x(o + L::kQH, o + L::kQL, off, qq.x * ex2(x0), qq.y * ex2(x1));
          put2x(o + L::kKH, o + L::kKL, off, kk.x * ex2(-x0), kk.y * ex2(-x1));
          if (!vd) {
            if (kV2) {
              const float2 vv = ld2(reinterpret_cast<const T*>(&vr[i]));
              put2x(o + L::kVH, o + L::kVL, off, vv.x, vv.y);
            } else {
              *reinterpret_cast<uint32_t*>(o + L::kVH + off) = vr[i];
            }
          }
        }
      }
      fence_async_smem();
      // with G in [-kSpanMax, 0] everywhere no factor leaves [e^{-kSpanMax}, e^{kSpanMax}]
      const bool exact = named_barrier_or(kBarBuild, kThreads, bad != 0);
      prev_exact[s] = exact;
      if (bt == 0) {
        m.exact[s] = exact ? 1 : 0;
        mbar_arrive_one(&m.built[s]);
        if (!exact) mbar_arrive_one(&m.rawfree[s]);
      }
      if (exact) {
        // scores on CUDA cores, P_ji = sum_d q_jd k_id e^{G_jd - G_id}, into
        // the q~ tiles once the first product has read them; G in scan order
#pragma unroll
        for (int i = 0; i < 8; ++i) *reinterpret_cast<float2*>(G + (tb + i) * kD + dc) = gc[i];
        named_barrier(kBarBuild, kThreads);
        failed |= !mbar_wait(&m.mma1[s], (uint32_t)use & 1u);
        const int j = bt >> 2, ib = (bt & 3) * 16;
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        if (j < it.ntok && !failed) {
          const T* qj_row = qst + (j ^ it.rmask) * kD;
          for (int x = 0; x < kD; ++x) {
            const float qj = Elem<T>::to_f(qj_row[x]);
            const float gj = G[j * kD + x];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i = ib + e;
              if (i <= j)
                acc[e] = fmaf(qj * Elem<T>::to_f(kst[(i ^ it.rmask) * kD + x]), expf(gj - G[i * kD + x]), acc[e]);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          put4(o + L::kQH, o + L::kQL, sw16(j, ib + e), acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        fence_async_smem();
        named_barrier(kBarBuild, kThreads);
        if (bt == 0) {
          atomicAdd(&g_gtr_exact_chunks, 1ull);
          mbar_arrive_one(&m.pready[s]);
          mbar_arrive_one(&m.rawfree[s]);
        }
      }
    }
    if (failed && bt == 0) m.abort = 1;
  } else {
    // ---- epilogue warps: P (masked two-term scores back into tensor memory),
    // then RMSNorm x w x SiLU(z) and the stores at the tokens' grid rows.
    // Thread: accumulator row `row` (TMEM lane quadrant warp % 4), columns
    // ch*16 .. +15 and 32 + ch*16 .. +15.
    const int qd = warp & 3;
    const int row = qd * 16 + (lane & 15), ch = lane >> 4;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const bool out32 = ((uintptr_t)p.out & 31) == 0;
    const int c0 = ch * 16, c1 = 32 + ch * 16;
    for (int n = 0; n < nit; ++n) {
      const int s = n & 1, use = n >> 1;
      const Item it = pipe_item(p, pipe_index(n));
      const uint32_t tms = tm + 256u * s + lane_base;
      const bool live = row < it.ntok;
      const long long grow = live ? item_row(p, it, row) : 0;
      // this row's z, requested before the products complete
      uint4 z0a = make_uint4(0u, 0u, 0u, 0u), z0b = z0a, z1a = z0a, z1b = z0a;
      if (live) {
        const uint4* zp = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.z) + grow * kD);
        z0a = __ldg(zp + c0 / 8);
        z0b = __ldg(zp + c0 / 8 + 1);
        z1a = __ldg(zp + c1 / 8);
        z1b = __ldg(zp + c1 / 8 + 1);
      }
      failed |= !mbar_wait(&m.mma1[s], (uint32_t)use & 1u);
      failed |= !mbar_wait(&m.built[s], (uint32_t)use & 1u);
      if (named_barrier_or(kBarEpi, 128, failed || aborted(&m.abort))) { failed = true; break; }
      tc_after_sync();
      if (!m.exact[s]) {
        float sa[16], sb[16];
        tmem_ld16x2(tms + 64, sa);
        tmem_ld16x2(tms + 96, sb);
        tmem_ld_wait(sa);
        tmem_ld_wait(sb);
        uint32_t ha[8], la[8], hb[8], lb[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a0 = c0 + 2 * e <= row ? sa[2 * e] : 0.f, a1 = c0 + 2 * e + 1 <= row ? sa[2 * e + 1] : 0.f;
          const float b0 = c1 + 2 * e <= row ? sb[2 * e] : 0.f, b1 = c1 + 2 * e + 1 <= row ? sb[2 * e + 1] : 0.f;
          split2(a0, a1, ha[e], la[e]);
          split2(b0, b1, hb[e], lb[e]);
        }
        tmem_st8x2(tms + 128, ha);
        tmem_st8x2(tms + 144, hb);
        tmem_st8x2(tms + 160, la);
        tmem_st8x2(tms + 176, lb);
        tmem_st_wait();
        tc_before_sync();
        named_barrier(kBarEpi, 128);
        if (warp == kWarpEpi0 && lane == 0) mbar_arrive_one(&m.pready[s]);
      }
      // the output gate w * SiLU(z) while P V runs
      float wz[32];
      {
        const uint4 zs[4] = {z0a, z0b, z1a, z1b};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cb = (q < 2 ? c0 : c1) + 8 * (q & 1);
          const float4 za = Vec4<T>::from_bits(make_uint2(zs[q].x, zs[q].y));
          const float4 zb = Vec4<T>::from_bits(make_uint2(zs[q].z, zs[q].w));
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) wz[8 * q + e] = m.wv[cb + e] * silu_fast(zz[e]);
        }
      }
      failed |= !mbar_wait(&m.mma2[s], (uint32_t)use & 1u);
      tc_after_sync();
      float oa[16], ob[16];
      tmem_ld16x2(tms, oa);
      tmem_ld16x2(tms + 32, ob);
      tmem_ld_wait(oa);
      tmem_ld_wait(ob);
      tc_before_sync();
      named_barrier(kBarEpi, 128);
      if (warp == kWarpEpi0 && lane == 0) mbar_arrive_one(&m.tfree[s]);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) ss = fmaf(oa[e], oa[e], fmaf(ob[e], ob[e], ss));
      ss += __shfl_xor_sync(0xffffffffu, ss, 16);
      if (live && !failed) {
        const float inv = rsqrtf(ss * (1.0f / kD) + kRmsEps);
        T* dst = reinterpret_cast<T*>(p.out) + grow * kD;
        uint4 y[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* x = q < 2 ? oa + 8 * (q & 1) : ob + 8 * (q & 1);
          const float* wq = wz + 8 * q;
          const uint2 lo = pack4<T>(x[0] * inv * wq[0], x[1] * inv * wq[1], x[2] * inv * wq[2], x[3] * inv * wq[3]);
          const uint2 hi = pack4<T>(x[4] * inv * wq[4], x[5] * inv * wq[5], x[6] * inv * wq[6], x[7] * inv * wq[7]);
          y[q] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        if (out32) {
          st_global_v8(dst + c0, y[0], y[1]);
          st_global_v8(dst + c1, y[2], y[3]);
        } else {
          reinterpret_cast<uint4*>(dst + c0)[0] = y[0];
          reinterpret_cast<uint4*>(dst + c0)[1] = y[1];
          reinterpret_cast<uint4*>(dst + c1)[0] = y[2];
          reinterpret_cast<uint4*>(dst + c1)[1] = y[3];
        }
      }
    }
    if (failed && threadIdx.x == 32 * kWarpEpi0) m.abort = 1;
  }
  if (failed) gtr_flag(kStatusMbarTimeout);
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  if (warp == kWarpLoad) tmem_dealloc(tm, L::kTmemCols);
}

}  // namespace tc
}  // namespace gtr

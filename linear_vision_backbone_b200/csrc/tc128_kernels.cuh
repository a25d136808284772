// tc128_kernels.cuh -- the tensor-core path of the Key-only GLA for head
// dimensions dk = dv = 128 (16-bit q/k/v/z, fp32 gates, 64-token chunks).
//
// The chunkwise operator of the GTR article (方法详解 §4: chunk summaries on
// tensor cores, a light pass over the segment-boundary states, chunk outputs
// with the scores kept on chip and the output gate fused into the epilogue),
// one block per segment (a run of consecutive chunks of one sequence):
//
//   gla_sum_tc128  per (sequence, segment): the state the segment produces
//                  from zero, dS = sum_t diag(e^{Gam - G_t}) k_t^T v_t (G_t
//                  the cumulative log-gate through token t, Gam the
//                  segment's total, so every weight is at most one), one
//                  tcgen05.mma product dS^T += V^T k^ per chunk (M = 128
//                  value dims, N = 128 key dims, K = 64 tokens) with k^ in
//                  two 16-bit terms, chunks taken last first; and the
//                  segment's decay factor e^{Gam}.
//   (the boundary scan over segments, scan_kernel.cuh, turns dS into the
//   state each segment starts from)
//   gla_out_tc128  per (sequence, segment), chunk by chunk:
//                  o = q~ S + mask(q~ k~^T) V with q~ = q e^{G} and
//                  k~ = k e^{-G} referenced to the chunk start, each operand
//                  in two bf16 terms (hi + lo) and the products hi hi +
//                  hi lo + lo hi accumulated in fp32 in tensor memory; then
//                  RMSNorm over the 128 value dims x w x SiLU(z), stored at
//                  the tokens' grid rows; then the state carried to the next
//                  chunk on chip.  Chunks whose log-gate span exceeds kSpan
//                  nats (where k~ would leave the terms' precision) take
//                  their scores from an exact CUDA-core sum instead.
//
// Tiles in shared memory use the 128-byte swizzle of the tensor cores'
// operand layout: a tile of R rows x 128 columns (16-bit) is two column
// halves of 64, each R rows of 128 bytes; element (r, c) of half c / 64 sits
// at r * 128 + ((c % 64 / 8) ^ (r % 8)) * 16 + (c % 8) * 2.  The same bytes
// are a K-major operand when the rows are M or N and a MN-major operand when
// the rows are K.
#pragma once
#include "tc_kernels.cuh"

namespace gtr {
namespace tc128 {

using tc::saddr;

constexpr int kC = 64;             // tokens per chunk
constexpr int kD = 128;            // dk = dv
constexpr int kThreads = 256;
constexpr float kSpan = 20.0f;     // the chunk's log-gate span (nats) beyond which its scores are exact
constexpr int kHalf64 = kC * 128;  // one 64-column half of a 64-row tile: 8 KB
constexpr int kTile64 = 2 * kHalf64;           // 64 rows x 128 columns, 16-bit: 16 KB
constexpr int kGBytes = kC * kD * 4;           // fp32 gate / cumulative log-gate: 32 KB

struct Params {
  const void* q; const void* k; const void* v; const float* g; const void* z; const float* w;
  float* wsS; float* wsA; void* out;
  int H, T, gh, gw, dir, nc, nseg;   // segment s walks chunks [s nc / nseg, (s + 1) nc / nseg)
};

// byte offset of the 16-byte unit holding columns [8u, 8u + 8) of row r in a
// swizzled tile of `rows` rows x 128 columns
__device__ __forceinline__ uint32_t sw_unit_off(int rows, int r, int u) {
  return (uint32_t)((u >> 3) * rows * 128 + r * 128 + (((u & 7) ^ (r & 7)) << 4));
}

// Instruction descriptor, kind::f16 with fp32 accumulation: bf16 or fp16 A and
// B, A / B K-major (0) or MN-major (1), M x N.
__host__ __device__ constexpr uint32_t idesc(bool bf16, int a_mn, int b_mn, int m, int n) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

template <typename T> struct Half2;
template <> struct Half2<__half> {
  using t2 = __half2;
  static __device__ __forceinline__ t2 from(float a, float b) { return __floats2half2_rn(a, b); }
  static __device__ __forceinline__ float2 to(t2 x) { return __half22float2(x); }
};
template <> struct Half2<__nv_bfloat16> {
  using t2 = __nv_bfloat162;
  static __device__ __forceinline__ t2 from(float a, float b) { return __floats2bfloat162_rn(a, b); }
  static __device__ __forceinline__ float2 to(t2 x) { return __bfloat1622float2(x); }
};

// Eight values as a 16-byte unit of type T, and the remainders x - T(x) as a
// second unit (the two-term split of an fp32 value).
template <typename T>
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  using H = Half2<T>;
  typename H::t2 h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    h[e] = H::from(x[2 * e], x[2 * e + 1]);
    const float2 f = H::to(h[e]);
    l[e] = H::from(x[2 * e] - f.x, x[2 * e + 1] - f.y);
  }
  memcpy(&hi, h, 16);
  memcpy(&lo, l, 16);
}
template <typename T>
__device__ __forceinline__ void widen8(const uint4& u, float (&x)[8]) {
  using H = Half2<T>;
  typename H::t2 h[4];
  memcpy(h, &u, 16);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = H::to(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

// 32 lanes x 32 bit, 32 consecutive columns (thread t of warp w <- lane 32 (w % 4) + t).
__device__ __forceinline__ void tmem_ld32x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}



// 16-byte copy global -> shared that reads `bytes` (16 or 0) and zero-fills the rest.
__device__ __forceinline__ void cp16(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr(dst)), "l"(src), "r"(bytes)
               : "memory");
}

// Token of the chunk whose copies thread tid makes, e = 0..3: half a warp per
// token, so that one copy instruction of a warp moves two whole 256-byte rows
// of a 16-bit tensor (or two halves of 512-byte gate rows).
__device__ __forceinline__ int gtok(int tid, int e) { return 2 * (tid >> 5) + ((tid >> 4) & 1) + 16 * e; }

// Grid index of token t of chunk c in scan order, or -1 past the sequence.
__device__ __forceinline__ int chunk_gidx(const Params& p, int d, int c, int t) {
  const int s = c * kC + t;
  return s < p.T ? scan_to_grid(d, s, p.T, p.gh, p.gw) : -1;
}
__device__ __forceinline__ long long row_of(const Params& p, int b, int h, int gi) {
  return gi < 0 ? -1 : ((long long)b * p.T + gi) * p.H + h;
}

// Copies one chunk whose token rows (or -1, zero-filled) are rows[e] for
// tokens gtok(tid, e): unit tid % 16 of each 16-bit tensor (into the swizzled
// 64-row tiles) and units tid % 16 and tid % 16 + 16 of the fp32 gate row
// (plain row-major).  A null tile is not copied.
template <typename T>
__device__ __forceinline__ void gather(const Params& p, const long long (&rows)[4], int tid, uint8_t* Q, uint8_t* K,
                                       uint8_t* V, float* G) {
  const int u = tid & 15;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int tt = gtok(tid, e);
    const uint32_t ok = rows[e] >= 0 ? 16u : 0u;
    const long long rr = rows[e] >= 0 ? rows[e] : 0;
    const uint32_t off = sw_unit_off(kC, tt, u);
    if (Q) cp16(Q + off, (const T*)p.q + rr * kD + u * 8, ok);
    if (K) cp16(K + off, (const T*)p.k + rr * kD + u * 8, ok);
    if (V) cp16(V + off, (const T*)p.v + rr * kD + u * 8, ok);
    if (G) {
      cp16(G + tt * kD + u * 4, p.g + rr * kD + u * 4, ok);
      cp16(G + tt * kD + (u + 16) * 4, p.g + rr * kD + (u + 16) * 4, ok);
    }
  }
}

// The token rows of chunk c for the copies of thread tid.
__device__ __forceinline__ void chunk_rows4(const Params& p, int b, int h, int d, int c, int tid, long long (&rows)[4]) {
#pragma unroll
  for (int e = 0; e < 4; ++e) rows[e] = row_of(p, b, h, chunk_gidx(p, d, c, gtok(tid, e)));
}

// Token row (b T + grid index) H + h of scan offset t of chunk c, or -1 past the sequence.
__device__ __forceinline__ long long chunk_row(const Params& p, int b, int h, int d, int c, int t) {
  return row_of(p, b, h, chunk_gidx(p, d, c, t));
}

// In-place inclusive cumulative sum of the gate over the chunk's 64 tokens:
// thread tid sums key dim tid % 128 over tokens [32 (tid / 128), + 32); the
// second half then adds the first half's total.  Ends with a block barrier.
__device__ __forceinline__ void cumsum(float* G, int tid) {
  const int i = tid & (kD - 1), t0 = (tid >> 7) * (kC / 2);
  float s = 0.f;
#pragma unroll 8
  for (int t = t0; t < t0 + kC / 2; ++t) {
    s += G[t * kD + i];
    G[t * kD + i] = s;
  }
  __syncthreads();
  if (t0 > 0) {
    const float base = G[(t0 - 1) * kD + i];
#pragma unroll 8
    for (int t = t0; t < t0 + kC / 2; ++t) G[t * kD + i] += base;
  }
  __syncthreads();
}

// Waits for an mbarrier phase, bounded; false on timeout.
__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity) { return tc::mbar_wait(bar, parity); }

// ---------------------------------------------------------------------------
// Summary of one segment (chunks c_lo .. c_hi - 1 of a sequence): the state it
// produces from zero, dS = sum_t diag(e^{Gam_seg - G_t}) k_t^T v_t with G_t
// the cumulative log-gate from the segment start, and its decay e^{Gam_seg}.
// The chunks are taken last first, so that the accumulator never needs
// rescaling: Lam holds the log-decay of the chunks already taken (those after
// the current one), and chunk c adds V^T k^ with k^_t = k_t e^{Lam + Gam_c -
// G_t} (Gam_c, G_t now within the chunk), every weight at most one.  Written
// as dS [dk][dv] fp32 and e^{Lam} at the end.
struct SumLayout {
  static constexpr int kK = 0;                     // k tiles (two buffers), then k^ hi in place
  static constexpr int kV = kK + 2 * kTile64;      // v tiles (two buffers; the MN-major A operand V^T)
  static constexpr int kKlo = kV + 2 * kTile64;    // k^ lo
  static constexpr int kG = kKlo + kTile64;        // gates, then cumulative
  static constexpr int kLam = kG + kGBytes;        // log-decay of the chunks after the current one
  static constexpr int kMisc = kLam + kD * 4;
  static constexpr int kSmem = kMisc + 256;
};
static_assert(2 * (SumLayout::kSmem + 1024) <= 228 * 1024,
              "two summary blocks (and the 1 KB each reserves) must fit one SM");

template <typename T>
__global__ void __launch_bounds__(kThreads, 2) gla_sum_tc128(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  uint8_t* Klo = sm + SumLayout::kKlo;
  float* G = reinterpret_cast<float*>(sm + SumLayout::kG);
  float* Lam = reinterpret_cast<float*>(sm + SumLayout::kLam);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + SumLayout::kMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + SumLayout::kMisc + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = dir_of_batch(p.dir, b);
  const int c_lo = seg_first_chunk(seg, p.nc, p.nseg), c_hi = seg_first_chunk(seg + 1, p.nc, p.nseg);
  if ((saddr(smem_raw) & 1023u) != 0u) {           // the swizzled tiles need 1024-byte alignment
    if (tid == 0) gtr_flag(kStatusBadShape);
    return;
  }
  if (d < 0 || d > 3) {
    if (tid == 0) gtr_flag(kStatusBadDir);
    return;
  }
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::mbar_fence_init();
  }
  if (tid < kD) Lam[tid] = 0.f;
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 128);
    tc::tmem_relinquish();
  }
  pdl_wait();                                      // the gates may come from the kernel before
  pdl_trigger();
  constexpr uint32_t id = idesc(std::is_same<T, __nv_bfloat16>::value, 1, 1, 128, 128);
  uint32_t tm = 0, phase = 0;
  bool ok = true;
  long long rows4[4];
  chunk_rows4(p, b, h, d, c_hi - 1, tid, rows4);
  gather<T>(p, rows4, tid, nullptr, sm + SumLayout::kK, sm + SumLayout::kV, G);
  tc::cp_async_commit();
  int bi = 0;                                      // this chunk's k, v buffer
  for (int c = c_hi - 1; c >= c_lo; --c, bi ^= 1) {
    const bool more = c > c_lo;
    uint8_t* K = sm + SumLayout::kK + bi * kTile64;
    uint8_t* V = sm + SumLayout::kV + bi * kTile64;
    tc::cp_async_wait<0>();                        // this chunk's copies made by this thread
    __syncthreads();
    if (more) {
      // the other buffer was read by the previous chunk's product: the next k, v into it
      chunk_rows4(p, b, h, d, c - 1, tid, rows4);
      gather<T>(p, rows4, tid, nullptr, sm + SumLayout::kK + (bi ^ 1) * kTile64,
                sm + SumLayout::kV + (bi ^ 1) * kTile64, nullptr);
      tc::cp_async_commit();
    }
    cumsum(G, tid);
    const float gam = tid < kD ? G[(kC - 1) * kD + tid] : 0.f;
    // k^ = k e^{Lam + Gam_c - G_t} in two terms of k's type: unit (t, u) per thread step
#pragma unroll
    for (int k4 = 0; k4 < kC * 16 / kThreads; ++k4) {
      const int it = tid + k4 * kThreads;
      const int r = it >> 4, u = it & 15;
      const uint32_t off = sw_unit_off(kC, r, u);
      float x[8];
      widen8<T>(*reinterpret_cast<const uint4*>(K + off), x);
      const float* gr = G + r * kD + u * 8;
      const float* gl = G + (kC - 1) * kD + u * 8;
      const float* lm = Lam + u * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= __expf(lm[e] + gl[e] - gr[e]);
      uint4 hi, lo;
      split8<T>(x, hi, lo);
      *reinterpret_cast<uint4*>(K + off) = hi;
      *reinterpret_cast<uint4*>(Klo + off) = lo;
    }
    tc::fence_async_smem();
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    if (more) {
      gather<T>(p, rows4, tid, nullptr, nullptr, nullptr, G);   // the gates are read: the next ones
      tc::cp_async_commit();
    }
    tm = *tmem_slot;
    if (tid == 0) {
      // D [dv][dk] += V^T (MN-major A, M = 128) x k^ (MN-major B, N = 128), K = 64 tokens
      const uint64_t a = tc::desc_mn(V), bh_ = tc::desc_mn(K), bl = tc::desc_mn(Klo);
      const uint32_t acc0 = c < c_hi - 1 ? 1u : 0u;
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks)
        tc::mma_f16(tm, a + ks * tc::kStepMN, bh_ + ks * tc::kStepMN, id, ks > 0 ? 1u : acc0);
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks) tc::mma_f16(tm, a + ks * tc::kStepMN, bl + ks * tc::kStepMN, id, 1u);
      tc::mma_commit(bar);
    }
    ok = wait_phase(bar, phase) && ok;
    phase ^= 1u;
    tc::tc_after_sync();
    if (tid < kD) Lam[tid] += gam;
    // k^ lo and this buffer are read; a timed-out wait ends the walk in every thread
    if (!__syncthreads_and(ok)) break;
  }
  tc::cp_async_wait<0>();                          // no copy may land after the block exits
  float* dS = p.wsS + ((size_t)bh * p.nseg + seg) * kD * kD;
  if (warp < 4 && ok) {
    // lane j of quadrant `warp` holds row j of dS^T, i.e. column j of dS
    const int j = warp * 32 + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < kD; c0 += 32) {
      float v[32];
      tmem_ld32x32(tm + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) dS[(size_t)(c0 + i) * kD + j] = v[i];
    }
  }
  if (tid < kD) p.wsA[((size_t)bh * p.nseg + seg) * kD + tid] = __expf(Lam[tid]);
  if (!ok && lane == 0) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(*tmem_slot, 128);
}

// ---------------------------------------------------------------------------
// Output of one segment, chunk by chunk from the state it starts from,
// computed transposed so that the state is an operand in tensor memory rather
// than shared memory:
//   o^T = S^T q~^T + V^T P^T      (M = 128 value dims, N = 64 tokens)
// with S^T [dv][dk] held in tensor memory as two bf16 terms (the A operand),
// q~ and P read from shared memory as K-major B operands and V as the
// MN-major A operand.  The scores q~ k~^T (M = 64) are as before.  Between
// chunks the state is carried on chip:
//   S' = diag(e^{Gam}) (S + k~^T V)    (k~ = k e^{-G}), or, for a chunk
//   S' = diag(e^{Gam}) S + k^^T V      (k^ = k e^{Gam - G}) whose span sent
//                                       its scores to the exact sum,
// the product V^T k~ (M = 128, N = 128) accumulated in fp32 in the columns
// of o^T and the scores once both are read, and S' split again into its two
// bf16 terms.  With bf16 inputs a block takes 112 KB of shared memory (two
// blocks and the 1 KB each reserves just fit an SM's 228 KB) and 256
// tensor-memory columns, so two blocks share an SM.  Once the first products
// have read the q tiles, P goes over q~ hi and z over q~ lo (16-byte copies);
// the output is formed over z and stored as 16-byte units of token rows.
// Each tile is refilled with the next chunk as soon as it is read.
template <typename T>
struct OutLayout {
  static constexpr bool kTwoV = !std::is_same<T, __nv_bfloat16>::value;   // fp16 v: bf16 hi + lo
  static constexpr int kQ = 0;                     // q tile, then q~ hi; then P hi, P lo; then the next q
  static constexpr int kQlo = kQ + kTile64;        // q~ lo; then z, and the output over it
  static constexpr int kK = kQlo + kTile64;        // k tile, then k~ (or k^) hi
  static constexpr int kKlo = kK + kTile64;
  static constexpr int kV = kKlo + kTile64;
  static constexpr int kVlo = kV + kTile64;        // fp16 v only
  static constexpr int kG = kVlo + (kTwoV ? kTile64 : 0);   // gates; then the row sums and e^{Gam}
  static constexpr int kMisc = kG + kGBytes;      // barrier, TMEM address
  static constexpr int kIdx = kMisc + 128;         // grid indices of the tokens of two chunks (by parity)
  static constexpr int kSmem = kIdx + 2 * kC * 4;
  static constexpr int kBlocksPerSM = kTwoV ? 1 : 2;
};
static_assert(2 * (OutLayout<__nv_bfloat16>::kSmem + 1024) <= 228 * 1024,
              "two bf16 output blocks (and the 1 KB each reserves) must fit one SM");

// 32 lanes x 32 bit, `N` consecutive columns from registers (thread t of warp w -> lane 32 (w % 4) + t).
__device__ __forceinline__ void tmem_st32x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// 32 lanes x 32 bit, 16 consecutive columns into registers (no wait).
__device__ __forceinline__ void tmem_ld32x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Waits for this thread's tensor-memory loads; the registers of two x16 loads
// are operands, so that no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]),
                 "+r"(a[7]), "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]),
                 "+r"(a[14]), "+r"(a[15]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]),
                 "+r"(b[5]), "+r"(b[6]), "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]),
                 "+r"(b[12]), "+r"(b[13]), "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}

// 32 fp32 values as two bf16 terms, two per 32-bit word (the even index in the low half).
__device__ __forceinline__ void split_bf16_words(const float (&x)[32], uint32_t (&hw)[16], uint32_t (&lw)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const __nv_bfloat162 hi = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
    const float2 f = __bfloat1622float2(hi);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x[2 * e] - f.x, x[2 * e + 1] - f.y);
    memcpy(&hw[e], &hi, 4);
    memcpy(&lw[e], &lo, 4);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads, OutLayout<T>::kBlocksPerSM) gla_out_tc128(const Params p) {
  using L = OutLayout<T>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw;
  uint8_t* Q = sm + L::kQ;
  uint8_t* Qlo = sm + L::kQlo;
  uint8_t* K = sm + L::kK;
  uint8_t* Klo = sm + L::kKlo;
  uint8_t* V = sm + L::kV;
  uint8_t* Vlo = sm + L::kVlo;
  float* G = reinterpret_cast<float*>(sm + L::kG);
  float* aG = G + (kC - 1) * kD;                   // after the scores: e^{Gam} over the gate total
  float* rowss = G;                                // after the scores: [4][64] partial sums over gate rows 0-1
  uint8_t* P = Q;                                  // after the first products: P hi, then P lo 8 KB on
  uint8_t* Zt = Qlo;                               // after the first products: z, then the output, [64][128]
  T* Ze = reinterpret_cast<T*>(Zt);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kMisc + 16);
  int* gidx = reinterpret_cast<int*>(sm + L::kIdx);   // [2][64]: chunk c at c % 2
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = dir_of_batch(p.dir, b);
  const int c_lo = seg_first_chunk(seg, p.nc, p.nseg), c_hi = seg_first_chunk(seg + 1, p.nc, p.nseg);
  if ((saddr(smem_raw) & 1023u) != 0u) {           // the swizzled tiles need 1024-byte alignment
    if (tid == 0) gtr_flag(kStatusBadShape);
    return;
  }
  if (d < 0 || d > 3) {
    if (tid == 0) gtr_flag(kStatusBadDir);
    return;
  }
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 256);
    tc::tmem_relinquish();
  }
  pdl_wait();                                      // the boundary states come from the scan
  pdl_trigger();
  // the first chunk's copies go out first
  if (tid < kC) gidx[(c_lo & 1) * kC + tid] = chunk_gidx(p, d, c_lo, tid);
  long long rows4[4];
  chunk_rows4(p, b, h, d, c_lo, tid, rows4);
  gather<T>(p, rows4, tid, Q, K, V, G);
  tc::cp_async_commit();
  tc::tc_before_sync();
  __syncthreads();                                 // the barrier, the TMEM address, the grid indices
  tc::tc_after_sync();
  // the rows of this thread's tokens of chunk cc, from the grid indices
  auto rows_of = [&](int cc, long long (&rows)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) rows[e] = row_of(p, b, h, gidx[(cc & 1) * kC + gtok(tid, e)]);
  };
  const uint32_t tm = *tmem_slot;
  // tensor memory: S^T hi [0, 64), S^T lo [64, 128), o^T [128, 192), scores
  // [192, 256); the state increment over [128, 256) after both are read
  const uint32_t tmSh = tm, tmSl = tm + 64, tmO = tm + 128, tmP = tm + 192, tmI = tm + 128;
  const int qd = warp & 3, hf = warp >> 2;
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  {
    // S^T row j = 32 qd + lane (a value dim), key dims 64 hf .. 64 hf + 63, from S [dk][dv]
    const float* Sg = p.wsS + ((size_t)bh * p.nseg + seg) * kD * kD + 32 * qd + lane;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int i0 = 64 * hf + 32 * part;
      float sv[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) sv[e] = Sg[(size_t)(i0 + e) * kD];
      uint32_t hw[16], lw[16];
      split_bf16_words(sv, hw, lw);
      // two key dims per 32-bit column, the even one in the low half
      tmem_st32x16(tmSh + lane_base + (uint32_t)(i0 >> 1), hw);
      tmem_st32x16(tmSl + lane_base + (uint32_t)(i0 >> 1), lw);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  constexpr uint32_t kIdOT = idesc(true, 0, 0, 128, 64);       // S^T (tensor memory) x q~^T (K-major)
  constexpr uint32_t kIdScores = idesc(true, 0, 0, 64, 64);    // q~ (K-major) x k~ (K-major)
  constexpr uint32_t kIdVP = idesc(true, 1, 0, 128, 64);       // V^T (MN-major) x P^T (K-major)
  constexpr uint32_t kIdInc = idesc(true, 1, 1, 128, 128);     // V^T (MN-major) x k~ (MN-major)
  // P: thread (quadrant qd, half hf) holds score row r = 16 qd + lane % 16,
  // columns s0 .. s0 + 15 with s0 = 32 hf + 16 (lane / 16)
  const int r = qd * 16 + (lane & 15);
  const int s0 = hf * 32 + (lane >> 4) * 16;
  // epilogue: lane j = 32 qd + lane holds o[t][j] for tokens t0 .. t0 + 31, t0 = 32 hf
  const int j = qd * 32 + lane, t0 = hf * 32;
  const float wj = p.w ? __ldg(p.w + j) : 1.0f;
  uint32_t phase = 0;
  bool ok = true;
  for (int c = c_lo; c < c_hi; ++c) {
    const bool carry = c + 1 < c_hi;               // the next chunk needs this one's end state
    tc::cp_async_wait<0>();                        // this chunk's copies made by this thread
    __syncthreads();
    // the next chunk's grid indices (that half was last read before the barrier)
    if (carry && tid < kC) gidx[((c + 1) & 1) * kC + tid] = chunk_gidx(p, d, c + 1, tid);
    cumsum(G, tid);
    // a chunk whose log-gate span leaves [-kSpan, 0] takes exact scores
    const bool exact = __syncthreads_or(tid < kD && G[(kC - 1) * kD + tid] < -kSpan) != 0;
    // q~ = q e^{G}; k~ = k e^{-G}, or k^ = k e^{Gam - G} for an exact chunk; v split for fp16; in place
#pragma unroll
    for (int k4 = 0; k4 < kC * 16 / kThreads; ++k4) {
      const int it = tid + k4 * kThreads;
      const int rr = it >> 4, u = it & 15;
      const uint32_t off = sw_unit_off(kC, rr, u);
      const float* gr = G + rr * kD + u * 8;
      const float* gl = G + (kC - 1) * kD + u * 8;
      float x[8];
      uint4 hi, lo;
      widen8<T>(*reinterpret_cast<const uint4*>(Q + off), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= __expf(gr[e]);
      split8<__nv_bfloat16>(x, hi, lo);
      *reinterpret_cast<uint4*>(Q + off) = hi;
      *reinterpret_cast<uint4*>(Qlo + off) = lo;
      if (!exact || carry) {
        widen8<T>(*reinterpret_cast<const uint4*>(K + off), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= __expf(exact ? gl[e] - gr[e] : -gr[e]);
        split8<__nv_bfloat16>(x, hi, lo);
        *reinterpret_cast<uint4*>(K + off) = hi;
        *reinterpret_cast<uint4*>(Klo + off) = lo;
      }
      if (L::kTwoV) {
        widen8<T>(*reinterpret_cast<const uint4*>(V + off), x);
        split8<__nv_bfloat16>(x, hi, lo);        // exact: an fp16 value is bf16 hi + bf16 lo
        *reinterpret_cast<uint4*>(V + off) = hi;
        *reinterpret_cast<uint4*>(Vlo + off) = lo;
      }
    }
    tc::fence_async_smem();
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    if (tid == 0) {
      const uint64_t qh = tc::desc_k(Q), ql = tc::desc_k(Qlo);
      // o^T = S^T q~^T: K = 128 key dims, 8 tensor-memory columns per step of 16
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint64_t bo = (uint64_t)((ks >> 2) * (kHalf64 >> 4) + (ks & 3) * tc::kStepK);
        const uint32_t ao = (uint32_t)(ks * 8);
        tc::mma_f16_ts(tmO, tmSh + ao, qh + bo, kIdOT, ks > 0);
        tc::mma_f16_ts(tmO, tmSh + ao, ql + bo, kIdOT, 1u);
        tc::mma_f16_ts(tmO, tmSl + ao, qh + bo, kIdOT, 1u);
      }
      if (!exact) {
        const uint64_t kh = tc::desc_k(K), kl = tc::desc_k(Klo);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t o = (uint64_t)((ks >> 2) * (kHalf64 >> 4) + (ks & 3) * tc::kStepK);
          tc::mma_f16(tmP, qh + o, kh + o, kIdScores, ks > 0);
          tc::mma_f16(tmP, qh + o, kl + o, kIdScores, 1u);
          tc::mma_f16(tmP, ql + o, kh + o, kIdScores, 1u);
        }
      }
      tc::mma_commit(bar);
    }
    ok = wait_phase(bar, phase) && ok;
    phase ^= 1u;
    tc::tc_after_sync();
    {
      // the q tiles are read: this chunk's z into the lo tile, row-major 256-byte rows
      long long zr[4];
      rows_of(c, zr);
      const int u = tid & 15;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        cp16(Zt + gtok(tid, e) * 256 + u * 16, (const T*)p.z + (zr[e] >= 0 ? zr[e] : 0) * kD + u * 8,
             zr[e] >= 0 ? 16u : 0u);
      tc::cp_async_commit();
    }
    const int ntok = min(kC, p.T - c * kC);
    {
      float sc[16];
      if (!exact) {
        float tv[16];
        tc::tmem_ld16x2(tmP + lane_base + (uint32_t)(hf * 32), tv);
        tc::tmem_ld_wait(tv);
#pragma unroll
        for (int e = 0; e < 16; ++e) sc[e] = tv[e];
      } else {
        // exact scores from the 16-bit q, k rows: sum_i q_r[i] k_s[i] e^{G_r[i] - G_s[i]}
        const long long rq = chunk_row(p, b, h, d, c, r);
#pragma unroll 1
        for (int e = 0; e < 16; ++e) {
          const int s = s0 + e;
          float acc = 0.f;
          if (s <= r && r < ntok) {
            const long long rk = chunk_row(p, b, h, d, c, s);
            const T* qr = (const T*)p.q + rq * kD;
            const T* kr = (const T*)p.k + rk * kD;
            for (int i = 0; i < kD; ++i)
              acc = fmaf(ld_f(qr + i) * ld_f(kr + i), __expf(G[r * kD + i] - G[s * kD + i]), acc);
          }
          sc[e] = acc;
        }
        if (tid == 0) atomicAdd(&g_gtr_exact_chunks, 1ull);
      }
      // causal mask (s <= r), two bf16 terms into the K-major P tiles over q~ hi
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = (s0 + hb * 8 + e <= r) ? sc[hb * 8 + e] : 0.f;
        uint4 hi, lo;
        split8<__nv_bfloat16>(x, hi, lo);
        const uint32_t off = (uint32_t)(r * 128 + ((((s0 >> 3) + hb) ^ (r & 7)) << 4));
        *reinterpret_cast<uint4*>(P + off) = hi;
        *reinterpret_cast<uint4*>(P + kHalf64 + off) = lo;
      }
    }
    tc::fence_async_smem();
    tc::tc_before_sync();
    __syncthreads();
    tc::tc_after_sync();
    const uint64_t vh = tc::desc_mn(V), vl = tc::desc_mn(Vlo);
    if (tid == 0) {
      // o^T += V^T P^T: K = 64 tokens
      const uint64_t ph = tc::desc_k(P), pl = tc::desc_k(P + kHalf64);
#pragma unroll
      for (int ks = 0; ks < kC / 16; ++ks) {
        const uint64_t ao = (uint64_t)(ks * tc::kStepMN), bo = (uint64_t)(ks * tc::kStepK);
        tc::mma_f16(tmO, vh + ao, ph + bo, kIdVP, 1u);
        tc::mma_f16(tmO, vh + ao, pl + bo, kIdVP, 1u);
        if (L::kTwoV) tc::mma_f16(tmO, vl + ao, ph + bo, kIdVP, 1u);
      }
      tc::mma_commit(bar);
    }
    ok = wait_phase(bar, phase) && ok;
    phase ^= 1u;
    tc::tc_after_sync();
    if (carry) {
      // P is read: the next chunk's q over it
      rows_of(c + 1, rows4);
      gather<T>(p, rows4, tid, Q, nullptr, nullptr, nullptr);
      tc::cp_async_commit();
    }
    float o[32];
    tmem_ld32x32(tmO + lane_base + (uint32_t)t0, o);
    if (carry) {
      // o^T and the scores are read: the increment V^T k~ goes over them
      tc::tc_before_sync();
      __syncthreads();
      tc::tc_after_sync();
      if (tid < kD) aG[tid] = __expf(aG[tid]);     // the exact scores have read G
      if (tid == 0) {
        const uint64_t kh = tc::desc_mn(K), kl = tc::desc_mn(Klo);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
          const uint64_t o2 = (uint64_t)(ks * tc::kStepMN);
          tc::mma_f16(tmI, vh + o2, kh + o2, kIdInc, ks > 0);
          tc::mma_f16(tmI, vh + o2, kl + o2, kIdInc, 1u);
          if (L::kTwoV) tc::mma_f16(tmI, vl + o2, kh + o2, kIdInc, 1u);
        }
        tc::mma_commit(bar);
      }
    }
    // sum over the value dims of o[t][.]^2 for the 32 tokens at once: a
    // transposing butterfly (each step a lane keeps half of its sums and adds
    // its partner's copy of that half; 31 shuffles) leaves lane l with this
    // warp's sum for token t0 + l; then the four quadrants through shared memory
    float sq[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) sq[e] = o[e] * o[e];
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int e = 0; e < m; ++e) {
        const float send = up ? sq[e] : sq[m + e];
        const float keep = up ? sq[m + e] : sq[e];
        sq[e] = keep + __shfl_xor_sync(0xffffffffu, send, m);
      }
    }
    rowss[qd * kC + t0 + lane] = sq[0];
    if (carry) tc::cp_async_wait<1>();             // z (the next q may still be in flight)
    else tc::cp_async_wait<0>();
    __syncthreads();
    // lane l: 1 / RMS of token t0 + l, handed to the other lanes by shuffles;
    // the output over z in place
    const float tot =
        rowss[t0 + lane] + rowss[kC + t0 + lane] + rowss[2 * kC + t0 + lane] + rowss[3 * kC + t0 + lane];
    const float inv_l = rsqrtf(tot / (float)kD + kRmsEps);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float inv = __shfl_sync(0xffffffffu, inv_l, e);
      T* ze = Ze + (t0 + e) * kD + j;
      *ze = Elem<T>::from_f(o[e] * inv * wj * tc::silu_fast(Elem<T>::to_f(*ze)));
    }
    if (carry) {
      ok = wait_phase(bar, phase) && ok;
      phase ^= 1u;
      tc::tc_after_sync();
      // S' = e^{Gam} (S + inc), or e^{Gam} S + inc for an exact chunk, as two bf16 terms again
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        const int i0 = 64 * hf + 32 * part;
        float inc[32], av[32];
        uint32_t hw[16], lw[16];
        tmem_ld32x16(tmSh + lane_base + (uint32_t)(i0 >> 1), hw);
        tmem_ld32x16(tmSl + lane_base + (uint32_t)(i0 >> 1), lw);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 a4 = reinterpret_cast<const float4*>(aG + i0)[e];
          av[4 * e] = a4.x; av[4 * e + 1] = a4.y; av[4 * e + 2] = a4.z; av[4 * e + 3] = a4.w;
        }
        tmem_wait_ld(hw, lw);
        tmem_ld32x32(tmI + lane_base + (uint32_t)i0, inc);
        float sv[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 hi, lo;
          memcpy(&hi, &hw[e], 4);
          memcpy(&lo, &lw[e], 4);
          const float2 fh = __bfloat1622float2(hi), fl = __bfloat1622float2(lo);
          const float a0 = av[2 * e], a1 = av[2 * e + 1];
          const float x0 = fh.x + fl.x, x1 = fh.y + fl.y;
          sv[2 * e] = exact ? fmaf(a0, x0, inc[2 * e]) : a0 * (x0 + inc[2 * e]);
          sv[2 * e + 1] = exact ? fmaf(a1, x1, inc[2 * e + 1]) : a1 * (x1 + inc[2 * e + 1]);
        }
        split_bf16_words(sv, hw, lw);
        tmem_st32x16(tmSh + lane_base + (uint32_t)(i0 >> 1), hw);
        tmem_st32x16(tmSl + lane_base + (uint32_t)(i0 >> 1), lw);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    // the output tile is complete and the gates, the tiles and the increment
    // are read; a timed-out wait ends the walk in every thread
    tc::tc_before_sync();
    if (!__syncthreads_and(ok)) break;
    tc::tc_after_sync();
    if (carry) {
      rows_of(c + 1, rows4);
      gather<T>(p, rows4, tid, nullptr, K, V, G);   // the next chunk's k, v and gates
      tc::cp_async_commit();
    }
    {
      // the output rows: half a warp per 256-byte row
      long long orow[4];
      rows_of(c, orow);
      const int u = tid & 15;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (orow[e] >= 0)
          *reinterpret_cast<uint4*>((T*)p.out + orow[e] * kD + u * 8) =
              *reinterpret_cast<const uint4*>(Zt + gtok(tid, e) * 256 + u * 16);
    }
  }
  tc::cp_async_wait<0>();                          // no copy may land after the block exits
  if (!ok && lane == 0) gtr_flag(kStatusMbarTimeout);
  tc::tc_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tm, 256);
}

}  // namespace tc128

// output blocks per SM (the summary runs two)
inline int tc128_blocks_per_sm(int dtype) {
  return dtype == kF16 ? tc128::OutLayout<__half>::kBlocksPerSM : tc128::OutLayout<__nv_bfloat16>::kBlocksPerSM;
}

inline bool tc128_shape_supported(int dk, int dv, int chunk, int dtype) {
  return dk == tc128::kD && dv == tc128::kD && chunk == tc128::kC && (dtype == kF16 || dtype == kBF16);
}

// stage 0: summaries of every segment; stage 1: outputs of every segment.
inline int launch_tc128(int dtype, int stage, const tc128::Params& p, int BH, cudaStream_t st, int dev) {
  static bool done[4][64];
  const dim3 grid((unsigned)p.nseg, (unsigned)BH);
  auto go = [&](auto kern, int smem, bool* flag) -> int {
    if (!flag[dev]) {
      // all of the SM's unified L1 / shared memory as shared memory, so that
      // two blocks of 112 KB (or of the summary's 81 KB) fit side by side
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
          cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return -5;
      flag[dev] = true;
    }
    return launch_pdl(kern, grid, dim3(tc128::kThreads), (size_t)smem, st, p);
  };
  if (stage == 0)
    return dtype == kF16 ? go(tc128::gla_sum_tc128<__half>, tc128::SumLayout::kSmem, done[0])
                         : go(tc128::gla_sum_tc128<__nv_bfloat16>, tc128::SumLayout::kSmem, done[1]);
  return dtype == kF16 ? go(tc128::gla_out_tc128<__half>, tc128::OutLayout<__half>::kSmem, done[2])
                       : go(tc128::gla_out_tc128<__nv_bfloat16>, tc128::OutLayout<__nv_bfloat16>::kSmem, done[3]);
}

}  // namespace gtr

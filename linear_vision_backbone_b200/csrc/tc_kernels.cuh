// tc_kernels.cuh -- the tcgen05 / TMEM path of the Key-only GLA (sm_100a).
//
// Chunkwise evaluation (GTR article, 方法详解 §4 "硬件感知分块推理算子": chunk
// summaries on tensor cores, a light sequential pass over boundary states,
// chunk outputs with the scores kept on chip and the output gate fused into
// the epilogue), for 16-bit q/k/v/z, fp32 gates, dk = dv = 64, chunk C = 64.
//
// One CTA (256 threads) walks a segment of consecutive chunks of one (batch,
// head) sequence and carries the dk x dv state S in fp32 registers.  For chunk
// c with in-chunk inclusive log-gate cumsum G_j (per key dim), G_m = G at the
// middle position and Gam = G at the last one:
//   q~_j = q_j e^{G_j - G_m},  k~_i = k_i e^{G_m - G_i},  k^_i = k_i e^{Gam - G_i}
//   S'   = e^{G_m} S                                        (rows = key dims)
//   o_j  = q~_j S' + sum_{i<=j} (q~_j . k~_i) v_i              -> RMSNorm x SiLU(z)
//   S   <- e^{Gam} S + k^^T V
// exp(G_j - G_i) = e^{G_j - G_m} e^{G_m - G_i} keeps both factors within
// e^{+-span} of one, span = the chunk's own decay range.  A chunk whose span
// exceeds kSpanMax nats, or whose gates rise above zero, evaluates its scores
// exactly on CUDA cores instead (q~ = q e^{G_j}, S' = S,
// P_ji = sum_d q_jd k_id e^{G_jd - G_id}).
//
// Data movement: every token's head vector is one contiguous 128-byte row (256
// bytes for the fp32 gate), so the scan order is applied per token as the
// source address of 16-byte cp.async copies issued by all threads into a
// staging area; no transpose kernel runs and reversed orders are just
// reversed addresses.  The next chunk's q, k, v, g are fetched as soon as the
// current chunk's operand tiles are built, and its z as soon as the current
// epilogue is done, so the copies overlap the tensor-core work.  Two CTAs of
// eight warps share an SM, which hides the latency of one CTA's serial phases
// behind the other's.
//
// Tensor cores: tcgen05.mma kind::f16, M = 64, N = 64, K = 16 per
// instruction, fp32 accumulators in tensor memory.  Every operand is a pair of
// fp16 tiles (hi, lo) of a power-of-two-scaled fp32 value, multiplied as
// hi*hi + hi*lo + lo*hi: products carry ~22 significant bits, the precision of
// an fp32 evaluation for this operator's tolerance.
//   cols [  0, 64)  q~ S'           A = q~ (K-major),  B = S' (MN-major)
//   cols [ 64,128)  scores q~ k~^T  A = q~ (K-major),  B = k~ (K-major)
//   cols [128,192)  P V             A = P  (K-major),  B = V  (MN-major)
//   cols [192,256)  k~^T V          A = k~ (MN-major), B = V  (MN-major)
// The state update uses k^ = diag(e^{Gam - G_m}) k~, a per-row factor of the
// k~^T V accumulator, so one key tile serves both products (read K-major for
// the scores and MN-major for the state).  An M = 64 accumulator puts row r in
// TMEM lane 32*(r/16) + r%16; warps w and w+4 read those 16 lanes of quadrant
// w%4 with the 16x32bx2 shape, each thread taking 16 of the 64 columns, so the
// row phases (S', P, epilogue, state) run four threads per row and combine the
// RMSNorm row sums with one shuffle and a two-warp named barrier.  The masked
// scores P go back to shared memory (K-major, two-term, a fixed 2^-22 shift)
// for P V.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace gtr {
namespace tc {

constexpr int kC = 64;                 // chunk length
constexpr int kD = 64;                 // head dim (dk = dv)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kSpanMax = 20.0f;      // nats of in-chunk decay the scaled operands take
constexpr int kPShift = 22;            // masked scores enter P V as raw scores * 2^-22
constexpr unsigned long long kWaitNs = 500ull * 1000 * 1000;   // bounded waits: 0.5 s

constexpr int kRaw16 = kC * kD * 2;    // one 16-bit staging tile: 8 KB
constexpr int kRawG = kC * kD * 4;     // the fp32 gate tile: 16 KB
constexpr int kTile = kC * kD * 2;     // one fp16 operand tile: 8 KB

template <bool OUT> struct Layout {
  // single staging area: k, v, g [, q, z]
  static constexpr int kOffK = 0, kOffV = kRaw16, kOffG = 2 * kRaw16;
  static constexpr int kOffQ = 2 * kRaw16 + kRawG, kOffZ = 3 * kRaw16 + kRawG;
  static constexpr int kStage = OUT ? (4 * kRaw16 + kRawG) : (2 * kRaw16 + kRawG);
  // fp16 tiles: V, key tile (hi, lo) [, q~ (hi, lo), S' (hi, lo)]
  static constexpr int kTiles = OUT ? 7 : 3;
  static constexpr int kMisc = kStage + kTiles * kTile;        // 1024-aligned
  static constexpr int kMiscBytes = 4608;
  static constexpr int kSmem = kMisc + kMiscBytes + 1024;      // + alignment slack
  static constexpr int kTmemCols = OUT ? 256 : 64;
  static constexpr int kColDS = OUT ? 192 : 0;
  static constexpr int kBlocksPerSM = 2;
};

// ------------------------------------------------------------------ PTX
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One bounded probe of a phase; the thread may sleep in hardware for up to
// 20 us while the phase is incomplete (fewer polling instructions).
__device__ __forceinline__ uint32_t mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(saddr(b)), "r"(parity), "r"(20000u)
      : "memory");
  return ok;
}
// Wait for the phase with the given parity to complete; false after kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!mbar_try(b, parity))
    if (globaltimer() - t0 > kWaitNs) return false;
  return true;
}
// 16-byte asynchronous global -> shared copy (L2 only), grouped by commit.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most `pending` of this thread's committed groups are in flight
__device__ __forceinline__ void cp_async_wait(int pending) {
  if (pending) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else asm volatile("cp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(dst)),
               "r"(cols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(bar))
      : "memory");
}
// 32 lanes x 32 bit, 16 consecutive columns: thread t of warp w <- lane 32w+t.
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
// 16 lanes x 32 bit in two halves: thread t of warp w reads lane 32(w%4) + t%16
// of the address's quadrant, columns [c, c+16) for t < 16 and [c+16, c+32) for
// t >= 16 (c = the address's column).
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// barrier over `count` threads (whole warps) on hardware barrier `id` (1..15)
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------- operand layouts
// 16-bit operand tiles of 64 rows x 64 elements (128 bytes per row), layout
// SWIZZLE_128B: atoms of 8 rows x 128 bytes, the 16-byte unit index XOR-ed
// with the row's position in its atom.  The same physical layout serves a
// K-major operand (rows = M or N, columns = K) and an MN-major one (rows = K,
// columns = M or N); only the descriptor differs.
__device__ __forceinline__ uint32_t sw16(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + (((c >> 3) ^ (r & 7)) << 4) + (c & 7) * 2);
}
// tcgen05 shared-memory matrix descriptor (version 1): start address, leading
// and stride byte offsets, layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major tile, K step s: 16 elements = 32 bytes into every row.
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int s) {
  return sdesc(base + (uint32_t)(s * 32), 16, 1024);
}
// MN-major tile, K step s: 16 rows = two 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int s) {
  return sdesc(base + (uint32_t)(s * 2048), 8192, 1024);
}
// Instruction descriptor: kind::f16 with fp16 A and B, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// One 64x64x64 product: four K steps, accumulating onto the target unless it
// starts the accumulator.
__device__ __forceinline__ void mma_64(uint32_t d, uint32_t a, bool a_mn, uint32_t b, bool b_mn,
                                       bool accumulate) {
  const uint32_t id = idesc_f16(64, 64, a_mn, b_mn);
#pragma unroll
  for (int s = 0; s < 4; ++s)
    mma_f16(d, a_mn ? mndesc(a, s) : kdesc(a, s), b_mn ? mndesc(b, s) : kdesc(b, s), id,
            (accumulate || s > 0) ? 1u : 0u);
}
// (ah + al)(bh + bl) ~ ah bh + ah bl + al bh into d (fresh unless accumulate)
__device__ __forceinline__ void mma_pair(uint32_t d, uint32_t ah, uint32_t al, bool a_mn,
                                         uint32_t bh, uint32_t bl, bool b_mn, bool accumulate) {
  mma_64(d, ah, a_mn, bh, b_mn, accumulate);
  mma_64(d, ah, a_mn, bl, b_mn, true);
  mma_64(d, al, a_mn, bh, b_mn, true);
}

// ------------------------------------------------- two-term fp16 operands
// Every tensor-core operand is a pair (hi, lo) of fp16 tiles with
// x * 2^e = hi + lo, hi = fp16(x 2^e), lo = fp16(x 2^e - hi): 22 significant
// bits.  The power-of-two scale 2^e puts the largest magnitude of a row (or
// column, or tile) in [2^14, 2^15), inside fp16's range; it is exact and is
// undone on the fp32 accumulator.  Scales run along M or N, never along K, so
// they factor out of every sum.
__device__ __forceinline__ int scale_exp(float m) {
  if (!(m > 0.f) || !(m <= 3.0e38f)) return 0;
  const int ex = ((__float_as_int(m) >> 23) & 0xFF) - 127;
  return max(-60, min(60, 14 - ex));
}
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }
__device__ __forceinline__ uint2 split4(float a, float b, float c, float d, uint2* lo) {
  const __half2 h0 = __floats2half2_rn(a, b), h1 = __floats2half2_rn(c, d);
  const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
  const __half2 l0 = __floats2half2_rn(a - f0.x, b - f0.y), l1 = __floats2half2_rn(c - f1.x, d - f1.y);
  uint2 hi;
  memcpy(&hi.x, &h0, 4);
  memcpy(&hi.y, &h1, 4);
  memcpy(&lo->x, &l0, 4);
  memcpy(&lo->y, &l1, 4);
  return hi;
}
__device__ __forceinline__ uint2 half4(float a, float b, float c, float d) {
  const __half2 h0 = __floats2half2_rn(a, b), h1 = __floats2half2_rn(c, d);
  uint2 u;
  memcpy(&u.x, &h0, 4);
  memcpy(&u.y, &h1, 4);
  return u;
}
// store one two-term group of 4 elements at byte offset `off` of (hi, lo) tiles
__device__ __forceinline__ void put2(uint8_t* hi, uint8_t* lo, uint32_t off, float a, float b, float c,
                                     float d) {
  uint2 l;
  const uint2 h = split4(a, b, c, d, &l);
  *reinterpret_cast<uint2*>(hi + off) = h;
  *reinterpret_cast<uint2*>(lo + off) = l;
}
// max over the 16 lanes of a half warp (one operand row in the builders)
__device__ __forceinline__ float half_warp_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float amax4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

template <typename T> struct Vec4;
template <> struct Vec4<__half> {
  static __device__ __forceinline__ float4 from_bits(uint2 u) {
    __half2 a, b;
    memcpy(&a, &u.x, 4);
    memcpy(&b, &u.y, 4);
    const float2 fa = __half22float2(a), fb = __half22float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
  static __device__ __forceinline__ float4 load(const void* p) {
    return from_bits(*reinterpret_cast<const uint2*>(p));
  }
};
template <> struct Vec4<__nv_bfloat16> {
  static __device__ __forceinline__ float4 from_bits(uint2 u) {
    __nv_bfloat162 a, b;
    memcpy(&a, &u.x, 4);
    memcpy(&b, &u.y, 4);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    return make_float4(fa.x, fa.y, fb.x, fb.y);
  }
  static __device__ __forceinline__ float4 load(const void* p) {
    return from_bits(*reinterpret_cast<const uint2*>(p));
  }
};
template <typename T> __device__ __forceinline__ uint2 pack4(float a, float b, float c, float d);
template <> __device__ __forceinline__ uint2 pack4<__half>(float a, float b, float c, float d) {
  return half4(a, b, c, d);
}
template <> __device__ __forceinline__ uint2 pack4<__nv_bfloat16>(float a, float b, float c, float d) {
  const __nv_bfloat162 x = __floats2bfloat162_rn(a, b), y = __floats2bfloat162_rn(c, d);
  uint2 u;
  memcpy(&u.x, &x, 4);
  memcpy(&u.y, &y, 4);
  return u;
}

struct Params {
  const void* q; const void* k; const void* v; const float* g; const void* z; const float* w;
  float* wsS; float* wsL; void* out;
  int H, T, gh, gw, dir, seg_chunks, nseg;
};

struct Misc {                   // per-CTA scalars in shared memory; every array that is read
                                // as float4 is 16-byte aligned
  uint64_t mma[2];              // [0] q~ S' and scores committed, [1] every product committed
  uint32_t tmem;                // tensor-memory base address
  int pad;
  alignas(16) float smax[kWarps];   // per-warp max |S| of the carried state
  alignas(16) float kbound[2][2];   // per-warp max of the k~ [0] and k^ [1] bounds over key dims
  alignas(16) float Gm[kD];
  alignas(16) float Gam[kD];
  alignas(16) float aG[kD];
  alignas(16) float eK[kD];
  alignas(16) float wv[kD];
  alignas(16) float sev[kD];    // V column scales 2^e and 2^-e
  alignas(16) float iev[kD];
  // column statistics of the chunk: maxima of |k| and |v|, min and max of G
  // (order-preserving int encodings, combined with shared-memory atomics)
  alignas(16) int kmx[kD];
  alignas(16) int vmx[kD];
  alignas(16) int gmin[kD];
  alignas(16) int gmax[kD];
  union {
    alignas(16) float part[4][kD];        // column pass: per-quarter gate sums
    struct {
      alignas(16) float ieq[kC];          // row phases: inverse row scales of q~ and P
      alignas(16) float iep[kC];
      alignas(16) float rowred[2][kC];    // row reductions across the two column halves
    } r;
  } u;
  alignas(16) long long rows[kC];   // token rows (b*T + t)*H + h of the chunk being fetched
};
static_assert(sizeof(Misc) <= Layout<true>::kMiscBytes, "Misc must fit its reserved bytes");
static_assert(offsetof(Misc, Gm) % 16 == 0 && offsetof(Misc, Gam) % 16 == 0 &&
                  offsetof(Misc, wv) % 16 == 0 && offsetof(Misc, sev) % 16 == 0 &&
                  offsetof(Misc, iev) % 16 == 0 && offsetof(Misc, eK) % 16 == 0,
              "float4 reads of Misc arrays need 16-byte alignment");

// Order-preserving map of a float onto an int (for atomicMin / atomicMax).
__device__ __forceinline__ int ord_enc(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float ord_dec(int e) { return __int_as_float(e >= 0 ? e : e ^ 0x7FFFFFFF); }

// Token rows of the chunk starting at scan position s0 (threads 0..ntok-1).
__device__ __forceinline__ void chunk_rows(const Params& p, Misc& m, int b, int h, int d, int s0,
                                           int ntok, int tid) {
  if (tid < ntok)
    m.rows[tid] = ((long long)b * p.T + scan_to_grid(d, s0 + tid, p.T, p.gh, p.gw)) * p.H + h;
}

// Fetch k, v, g (and q for the output kernel) of a chunk: 16-byte pieces, the
// 128-byte row of a token split over 8 consecutive threads.  One commit group.
template <typename T, bool OUT>
__device__ __forceinline__ void fetch_kvqg(const Params& p, uint8_t* stg, const Misc& m, int ntok,
                                           int tid) {
  using L = Layout<OUT>;
  for (int o = tid; o < ntok * 8; o += kThreads) {
    const int j = o >> 3, part = (o & 7) * 16;
    const size_t src = (size_t)m.rows[j] * (kD * 2) + part;
    cp_async16(stg + L::kOffK + j * 128 + part, (const uint8_t*)p.k + src);
    cp_async16(stg + L::kOffV + j * 128 + part, (const uint8_t*)p.v + src);
    if (OUT) cp_async16(stg + L::kOffQ + j * 128 + part, (const uint8_t*)p.q + src);
  }
  for (int o = tid; o < ntok * 16; o += kThreads) {
    const int j = o >> 4, part = (o & 15) * 16;
    cp_async16(stg + L::kOffG + j * 256 + part, (const uint8_t*)p.g + (size_t)m.rows[j] * (kD * 4) + part);
  }
  cp_async_commit();
}
// Fetch z of a chunk (output kernel).  One commit group.
__device__ __forceinline__ void fetch_z(const Params& p, uint8_t* stg, const Misc& m, int ntok,
                                        int tid) {
  using L = Layout<true>;
  for (int o = tid; o < ntok * 8; o += kThreads) {
    const int j = o >> 3, part = (o & 7) * 16;
    cp_async16(stg + L::kOffZ + j * 128 + part, (const uint8_t*)p.z + (size_t)m.rows[j] * (kD * 2) + part);
  }
  cp_async_commit();
}

// Column pass over the chunk (four threads per column, 16 tokens each): the
// in-place inclusive cumsum of the gate tile, and the column maxima of |k| and
// |v|.  Then per column d: G_m, Gam, e^{Gam}, e^{Gam-G_m}, the V scales and
// the bounds of the k~ and k^ columns.  Returns true (block-uniform) if the
// chunk needs the exact scores: its decay range exceeds kSpanMax or some gate
// sum rises above zero.  m.kmx/vmx/gmin/gmax must hold their neutral values
// (column_stats_reset) when it starts.
__device__ __forceinline__ void column_stats_reset(Misc& m, int tid) {
  if (tid < kD) {
    m.kmx[tid] = 0;
    m.vmx[tid] = 0;
    m.gmin[tid] = ord_enc(0.0f);       // the running sum starts at 0 before the chunk
    m.gmax[tid] = ord_enc(-3.0e38f);
  }
}
template <typename T>
__device__ __forceinline__ bool column_pass(float* G, const T* kst, const T* vst, Misc& m, int ntok,
                                            int tid) {
  const int dd = tid & 63, qt = tid >> 6;
  const int j0 = qt * 16, j1 = min(j0 + 16, ntok);
  float run = 0.f, lo = 3.0e38f, hi = -3.0e38f, km = 0.f, vm = 0.f;
#pragma unroll 4
  for (int j = j0; j < j1; ++j) {
    run += G[j * kD + dd];
    G[j * kD + dd] = run;
    lo = fminf(lo, run);
    hi = fmaxf(hi, run);
    km = fmaxf(km, fabsf(Elem<T>::to_f(kst[j * kD + dd])));
    if (!std::is_same<T, __half>::value) vm = fmaxf(vm, fabsf(Elem<T>::to_f(vst[j * kD + dd])));
  }
  m.u.part[qt][dd] = run;
  atomicMax(&m.kmx[dd], __float_as_int(km));        // non-negative floats order as ints
  atomicMax(&m.vmx[dd], __float_as_int(vm));
  __syncthreads();
  float off = 0.f;
  for (int q = 0; q < qt; ++q) off += m.u.part[q][dd];
  if (qt > 0 && j1 > j0) {
#pragma unroll 4
    for (int j = j0; j < j1; ++j) G[j * kD + dd] += off;
  }
  if (j1 > j0) {
    atomicMin(&m.gmin[dd], ord_enc(lo + off));
    atomicMax(&m.gmax[dd], ord_enc(hi + off));
  }
  __syncthreads();
  int irregular = 0;
  if (tid < kD) {
    const float gam = G[(ntok - 1) * kD + tid];
    const float gm = G[((ntok - 1) >> 1) * kD + tid];
    const float mn = ord_dec(m.gmin[tid]), mx = ord_dec(m.gmax[tid]);
    const float km4 = __int_as_float(m.kmx[tid]), vm4 = __int_as_float(m.vmx[tid]);
    m.Gam[tid] = gam;
    m.Gm[tid] = gm;
    m.aG[tid] = expf(gam);
    m.eK[tid] = expf(gam - gm);
    const int ev = std::is_same<T, __half>::value ? 0 : scale_exp(vm4);
    m.sev[tid] = pow2i(ev);
    m.iev[tid] = pow2i(-ev);
    // |k~_id| <= max_i |k_id| e^{G_m,d - min_i G_id};  |k^_id| <= max_i |k_id| e^{Gam_d - min_i G_id}
    float kb0 = km4 * expf(gm - mn), kb1 = km4 * expf(gam - mn);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kb0 = fmaxf(kb0, __shfl_xor_sync(0xffffffffu, kb0, o));
      kb1 = fmaxf(kb1, __shfl_xor_sync(0xffffffffu, kb1, o));
    }
    if ((tid & 31) == 0) {
      m.kbound[0][tid >> 5] = kb0;
      m.kbound[1][tid >> 5] = kb1;
    }
    const float span = fmaxf(mx, 0.f) - mn;
    irregular = !(span <= kSpanMax) || mx > 0.f;
  }
  return __syncthreads_or(irregular) != 0;
}

// Sum over the four threads that share an accumulator row: the other half of
// the warp (lane ^ 16) and the same lanes of the partner warp (warp ^ 4),
// through shared memory and a named barrier of those two warps.
__device__ __forceinline__ float row_combine_sum(float v, Misc& m, int row, int half, int qd, int lane) {
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  if (lane < 16) m.u.r.rowred[half][row] = v;
  named_barrier(1 + qd, 64);
  return v + m.u.r.rowred[half ^ 1][row];
}

__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

template <typename T, bool OUT>
__global__ void __launch_bounds__(kThreads, Layout<OUT>::kBlocksPerSM)
gla_tc(const Params p) {
  using L = Layout<OUT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stg = sm;
  uint8_t* tiles = sm + L::kStage;
  uint8_t* VV = tiles;                       // V (MN-major B), one fp16 term
  uint8_t* KTh = tiles + 1 * kTile;          // key tile: k~ or k^, hi / lo
  uint8_t* KTl = tiles + 2 * kTile;
  uint8_t* QTh = tiles + 3 * kTile;          // q~ hi / lo, then P (K-major A)   [OUT]
  uint8_t* QTl = tiles + 4 * kTile;
  uint8_t* SPh = tiles + 5 * kTile;          // S' hi / lo   (MN-major B)        [OUT]
  uint8_t* SPl = tiles + 6 * kTile;
  Misc& m = *reinterpret_cast<Misc*>(sm + L::kMisc);
  float* G = reinterpret_cast<float*>(stg + L::kOffG);
  const T* kst = reinterpret_cast<const T*>(stg + L::kOffK);
  const T* vst = reinterpret_cast<const T*>(stg + L::kOffV);
  const T* qst = reinterpret_cast<const T*>(stg + L::kOffQ);
  const T* zst = reinterpret_cast<const T*>(stg + L::kOffZ);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = dir_of_batch(p.dir, b);
  const int nc = (p.T + kC - 1) / kC;
  const int c0 = seg * p.seg_chunks;
  const int nch = min(nc, c0 + p.seg_chunks) - c0;
  if (d < 0 || d > 3 || nch <= 0) {
    if (tid == 0) gtr_flag(d < 0 || d > 3 ? kStatusBadDir : kStatusBadShape);
    return;
  }
  // Row phases: four threads per accumulator row.  Warp w reads TMEM lane
  // quadrant qd = w % 4 (rows 16 qd .. 16 qd + 15) and column half w / 4; with
  // the 16x32bx2 shape, lanes 0-15 take the first 16 columns of that half and
  // lanes 16-31 the next 16, for the same 16 rows.
  const int qd = warp & 3, half = warp >> 2;
  const int row = qd * 16 + (lane & 15);
  const int cbase = half * 32 + (lane >> 4) * 16;    // this thread's 16 columns
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;

  // first chunk's copies go out before anything else
  chunk_rows(p, m, b, h, d, c0 * kC, min(kC, p.T - c0 * kC), tid);
  __syncthreads();
  fetch_kvqg<T, OUT>(p, stg, m, min(kC, p.T - c0 * kC), tid);
  if (OUT) fetch_z(p, stg, m, min(kC, p.T - c0 * kC), tid);

  // carried state: S[row][cbase .. cbase + 15]
  float S[16];
  if (OUT) {
    const float4* src = reinterpret_cast<const float4*>(
        p.wsS + (((size_t)bh * p.nseg + seg) * kD + row) * kD + cbase);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float4 x = src[c];
      S[4 * c] = x.x; S[4 * c + 1] = x.y; S[4 * c + 2] = x.z; S[4 * c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) S[c] = 0.f;
  }
  auto state_max = [&]() {
    float mx = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) mx = fmaxf(mx, fabsf(S[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) m.smax[warp] = mx;
  };
  if (OUT) state_max();
  if (tid == 0) {
    mbar_init(&m.mma[0], 1);
    mbar_init(&m.mma[1], 1);
    mbar_fence_init();
  }
  if (tid < kD) m.wv[tid] = (OUT && p.w) ? p.w[tid] : 1.0f;
  if (warp == 0) {
    tmem_alloc(&m.tmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = m.tmem;

  float lsum = 0.f;
  uint32_t ph0 = 0, ph1 = 0;
  bool failed = false;

  for (int it = 0; it < nch; ++it) {
    const int s0 = (c0 + it) * kC;
    const int ntok = min(kC, p.T - s0);
    const bool more = it + 1 < nch;
    const int s1 = s0 + kC;
    const int ntok1 = more ? min(kC, p.T - s1) : 0;

    cp_async_wait(OUT ? 1 : 0);          // k, v, g (, q) of this chunk are in
    column_stats_reset(m, tid);
    __syncthreads();
    const bool exact = column_pass<T>(G, kst, vst, m, ntok, tid) && OUT;

    // ---- operand tiles; rows beyond ntok are zero.  Items: (row r, 4 columns
    // cg..cg+3); a half warp covers one row, which makes per-row maxima cheap.
    // The key tile holds k~ = k e^{G_m - G} for a regular output chunk, else
    // k^ = k e^{Gam - G}.
    const bool tilde = OUT && !exact;
    const int ekt = scale_exp(fmaxf(m.kbound[tilde ? 0 : 1][0], m.kbound[tilde ? 0 : 1][1]));
    const float skt = pow2i(ekt);
#pragma unroll 2
    for (int u = 0; u < (kC * kD / 4) / kThreads; ++u) {
      const int item = u * kThreads + tid;
      const int r = item >> 4, cg = (item & 15) * 4;
      const bool valid = r < ntok;
      float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk, qq = kk;
      if (valid) {
        kk = Vec4<T>::load(kst + r * kD + cg);
        vv = Vec4<T>::load(vst + r * kD + cg);
        if (OUT) qq = Vec4<T>::load(qst + r * kD + cg);
      }
      const float4 gg = *reinterpret_cast<const float4*>(G + r * kD + cg);
      const uint32_t off = sw16(r, cg);
      if (std::is_same<T, __half>::value) {   // V: fp16 input is already an exact operand
        *reinterpret_cast<uint2*>(VV + off) =
            valid ? *reinterpret_cast<const uint2*>(vst + r * kD + cg) : make_uint2(0u, 0u);
      } else {   // bf16 V, column-scaled into fp16 (exact for all but tiny values)
        const float4 sv = *reinterpret_cast<const float4*>(&m.sev[cg]);
        *reinterpret_cast<uint2*>(VV + off) = half4(vv.x * sv.x, vv.y * sv.y, vv.z * sv.z, vv.w * sv.w);
      }
      const float4 gr = *reinterpret_cast<const float4*>(tilde ? &m.Gm[cg] : &m.Gam[cg]);
      put2(KTh, KTl, off, kk.x * __expf(gr.x - gg.x) * skt, kk.y * __expf(gr.y - gg.y) * skt,
           kk.z * __expf(gr.z - gg.z) * skt, kk.w * __expf(gr.w - gg.w) * skt);
      if (OUT) {   // q~ = q e^{G - G_m} (exact chunk: q e^{G}), row-scaled
        float q0, q1, q2, q3;
        if (!exact) {
          q0 = qq.x * __expf(gg.x - gr.x); q1 = qq.y * __expf(gg.y - gr.y);
          q2 = qq.z * __expf(gg.z - gr.z); q3 = qq.w * __expf(gg.w - gr.w);
        } else {
          q0 = qq.x * __expf(gg.x); q1 = qq.y * __expf(gg.y);
          q2 = qq.z * __expf(gg.z); q3 = qq.w * __expf(gg.w);
        }
        const int eq = scale_exp(half_warp_max(amax4(q0, q1, q2, q3)));
        const float s = pow2i(eq);
        put2(QTh, QTl, off, q0 * s, q1 * s, q2 * s, q3 * s);
        if (cg == 0) m.u.r.ieq[r] = pow2i(-eq);
      }
    }
    // S' = e^{G_m} S (S itself for an exact chunk), tile-scaled from max |S|
    float inv_es = 1.f;
    if (OUT) {
      float smx = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < kWarps; ++w8) smx = fmaxf(smx, m.smax[w8]);
      const int es = scale_exp(smx);
      inv_es = pow2i(-es);
      const float sc = (exact ? 1.0f : __expf(m.Gm[row])) * pow2i(es);
#pragma unroll
      for (int c = 0; c < 16; c += 4)
        put2(SPh, SPl, sw16(row, cbase + c), sc * S[c], sc * S[c + 1], sc * S[c + 2], sc * S[c + 3]);
    }
    if (more && !exact) chunk_rows(p, m, b, h, d, s1, ntok1, tid);
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();

    // staging of this chunk is consumed (except z): fetch the next chunk now
    if (more && !exact) fetch_kvqg<T, OUT>(p, stg, m, ntok1, tid);

    if (tid == 0) {
      // q~ S' and the scores first: their commit frees the q~ tiles for P
      if (OUT) {
        mma_pair(tm + 0, saddr(QTh), saddr(QTl), false, saddr(SPh), saddr(SPl), true, false);
        if (!exact)
          mma_pair(tm + 64, saddr(QTh), saddr(QTl), false, saddr(KTh), saddr(KTl), false, false);
        mma_commit(&m.mma[0]);
      }
      mma_64(tm + L::kColDS, saddr(KTh), true, saddr(VV), true, false);
      mma_64(tm + L::kColDS, saddr(KTl), true, saddr(VV), true, true);
      if (!OUT) mma_commit(&m.mma[1]);
    }

    if (OUT) {
      failed |= !mbar_wait(&m.mma[0], ph0);
      ph0 ^= 1;
      tc_after_sync();
      if (!exact) {
        // ---- masked scores P (rows = queries j, columns = keys i), row-scaled, into QT
        float sc[16];
        tmem_ld16x2(tm + lane_base + 64 + half * 32, sc);
        tmem_ld_wait();
        // The raw scores carry the q~ row scale and the key-tile scale and stay below
        // 64 * 2^15 * 2^15 = 2^36, so a fixed 2^-22 puts every row inside fp16's range;
        // P V is decoded with the same factors.
        const float f = pow2i(-kPShift);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int i = cbase + c;
          sc[c] = (i <= row && row < ntok) ? sc[c] * f : 0.f;
        }
        if (lane < 16 && half == 0) m.u.r.iep[row] = m.u.r.ieq[row] * pow2i(kPShift - ekt);
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          put2(QTh, QTl, sw16(row, cbase + c), sc[c], sc[c + 1], sc[c + 2], sc[c + 3]);
      } else {
        // exact scores on CUDA cores: P_ji = sum_d q_jd k_id e^{G_jd - G_id}; four threads per row
        if (tid == 0) atomicAdd(&g_gtr_exact_chunks, 1ull);
        const int j = tid >> 2, ib = (tid & 3) * 16;
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.f;
        if (j < ntok) {
          for (int dd = 0; dd < kD; ++dd) {
            const float qj = Elem<T>::to_f(qst[j * kD + dd]);
            const float gj = G[j * kD + dd];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i = ib + e;
              if (i <= j)
                acc[e] = fmaf(qj * Elem<T>::to_f(kst[i * kD + dd]), expf(gj - G[i * kD + dd]), acc[e]);
            }
          }
        }
        float mx = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(acc[e]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const int ep = scale_exp(mx);
        const float s = pow2i(ep);
        if ((tid & 3) == 0) m.u.r.iep[j] = pow2i(-ep);
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          put2(QTh, QTl, sw16(j, ib + e), acc[e] * s, acc[e + 1] * s, acc[e + 2] * s, acc[e + 3] * s);
        if (more) chunk_rows(p, m, b, h, d, s1, ntok1, tid);
      }
      cp_async_wait((more && !exact) ? 1 : 0);     // z of this chunk is in
      fence_async_smem();
      tc_before_sync();
      if (__syncthreads_or(failed)) break;
      tc_after_sync();
      if (exact && more) fetch_kvqg<T, OUT>(p, stg, m, ntok1, tid);
      if (tid == 0) {
        mma_64(tm + 128, saddr(QTh), false, saddr(VV), true, false);
        mma_64(tm + 128, saddr(QTl), false, saddr(VV), true, true);
        mma_commit(&m.mma[1]);
      }
    }
    failed |= !mbar_wait(&m.mma[1], ph1);
    ph1 ^= 1;
    tc_after_sync();

    if (OUT) {
      // ---- epilogue: o_j = q~_j S' + P_j V, then o_j / sqrt(mean o_j^2 + eps) * w * SiLU(z_j)
      float o[16], pv[16];
      tmem_ld16x2(tm + lane_base + 0 + half * 32, o);
      tmem_ld16x2(tm + lane_base + 128 + half * 32, pv);
      tmem_ld_wait();
      const float a = m.u.r.ieq[row] * inv_es, bsc = m.u.r.iep[row];
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        o[c] = o[c] * a + pv[c] * bsc * m.iev[cbase + c];
        ss = fmaf(o[c], o[c], ss);
      }
      ss = row_combine_sum(ss, m, row, half, qd, lane);
      if (row < ntok) {
        const float inv = rsqrtf(ss * (1.0f / kD) + kRmsEps);
        const T* zr = zst + row * kD + cbase;
        const int t = scan_to_grid(d, s0 + row, p.T, p.gh, p.gw);
        T* dst = reinterpret_cast<T*>(p.out) + (((size_t)b * p.T + t) * p.H + h) * kD + cbase;
#pragma unroll
        for (int c = 0; c < 16; c += 8) {
          const uint4 zz = *reinterpret_cast<const uint4*>(zr + c);
          const float4 z0 = Vec4<T>::from_bits(make_uint2(zz.x, zz.y));
          const float4 z1 = Vec4<T>::from_bits(make_uint2(zz.z, zz.w));
          const float4 w0 = *reinterpret_cast<const float4*>(&m.wv[cbase + c]);
          const float4 w1 = *reinterpret_cast<const float4*>(&m.wv[cbase + c + 4]);
          const uint2 lo = pack4<T>(o[c + 0] * inv * w0.x * silu_fast(z0.x), o[c + 1] * inv * w0.y * silu_fast(z0.y),
                                    o[c + 2] * inv * w0.z * silu_fast(z0.z), o[c + 3] * inv * w0.w * silu_fast(z0.w));
          const uint2 hi = pack4<T>(o[c + 4] * inv * w1.x * silu_fast(z1.x), o[c + 5] * inv * w1.y * silu_fast(z1.y),
                                    o[c + 6] * inv * w1.z * silu_fast(z1.z), o[c + 7] * inv * w1.w * silu_fast(z1.w));
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }

    // ---- state: S <- e^{Gam} S + diag(e^{Gam - G_m}) k~^T V   (or + k^^T V), fp32
    {
      float ds[16];
      tmem_ld16x2(tm + lane_base + L::kColDS + half * 32, ds);
      tmem_ld_wait();
      const float rs = (tilde ? m.eK[row] : 1.0f) * pow2i(-ekt);
      const float a = m.aG[row];
#pragma unroll
      for (int c = 0; c < 16; ++c) S[c] = fmaf(a, S[c], ds[c] * rs * m.iev[cbase + c]);
      if (OUT) state_max();
    }
    if (!OUT && tid < kD) lsum += m.Gam[tid];
    tc_before_sync();
    if (__syncthreads_or(failed)) break;
    if (OUT && more) fetch_z(p, stg, m, ntok1, tid);     // z of this chunk is consumed
  }

  cp_async_wait(0);                       // no copy may land after the block exits
  if (failed) {
    if (tid == 0) gtr_flag(kStatusMbarTimeout);
  } else if (!OUT) {
    float4* dst = reinterpret_cast<float4*>(p.wsS + (((size_t)bh * p.nseg + seg) * kD + row) * kD + cbase);
#pragma unroll
    for (int c = 0; c < 4; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
    if (tid < kD) p.wsL[((size_t)bh * p.nseg + seg) * kD + tid] = lsum;
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  if (warp == 0) tmem_dealloc(tm, L::kTmemCols);
}

}  // namespace tc

inline bool tc_shape_supported(int dk, int dv, int chunk, int dtype) {
  return dk == tc::kD && dv == tc::kD && chunk == tc::kC && (dtype == kF16 || dtype == kBF16);
}
inline int tc_blocks_per_sm(int, int) { return tc::Layout<true>::kBlocksPerSM; }

template <typename T, bool OUT>
inline int launch_tc_kernel(const tc::Params& p, int BH, cudaStream_t st, int dev) {
  auto kern = tc::gla_tc<T, OUT>;
  static bool done[64];
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tc::Layout<OUT>::kSmem) != cudaSuccess)
      return -5;
    done[dev] = true;
  }
  kern<<<dim3(p.nseg, BH), tc::kThreads, tc::Layout<OUT>::kSmem, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

// stage 0: segment summaries (K2); stage 1: segment outputs (K4)
inline int launch_tc(int dtype, int stage, const void* q, const void* k, const void* v,
                     const float* g, const void* z, const float* w, void* out, float* wsS,
                     float* wsL, int B, int H, int T, int gh, int gw, int dk, int dv, int dir,
                     int chunk, int seg_chunks, int nseg, cudaStream_t st) {
  if (!tc_shape_supported(dk, dv, chunk, dtype)) return -2;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -5;
  tc::Params p{q, k, v, g, z, w, wsS, wsL, out, H, T, gh, gw, dir, seg_chunks, nseg};
  const int BH = B * H;
  if (dtype == kF16)
    return stage == 0 ? launch_tc_kernel<__half, false>(p, BH, st, dev)
                      : launch_tc_kernel<__half, true>(p, BH, st, dev);
  return stage == 0 ? launch_tc_kernel<__nv_bfloat16, false>(p, BH, st, dev)
                    : launch_tc_kernel<__nv_bfloat16, true>(p, BH, st, dev);
}

}  // namespace gtr

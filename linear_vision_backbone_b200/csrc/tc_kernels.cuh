// tc_kernels.cuh -- the tcgen05 / TMEM path of the Key-only GLA (sm_100a).
//
// Chunkwise evaluation (GTR article, 方法详解 §4 "硬件感知分块推理算子": chunk
// summaries on tensor cores, a light sequential pass over boundary states,
// chunk outputs with the scores kept on chip and the output gate fused into
// the epilogue), for 16-bit q/k/v/z, fp32 gates, dk = dv = 64, chunk C = 64.
//
// Operands.  In the output kernel every tensor-core operand is a pair of bf16
// tiles (hi, lo) of an fp32 value, hi = bf16(x), lo = bf16(x - hi),
// multiplied as hi*hi' + hi*lo' + lo*hi' (tcgen05.mma kind::f16 with bf16
// inputs, fp32 accumulators in tensor memory, M = 64, N = 64 or 128, K = 16
// per instruction).  A product carries about 16 significant bits, 32 times
// finer than a tf32 operand, and bf16 has fp32's exponent range, so no
// operand needs a scale and products of different operands add in one
// accumulator.  A bf16 V is used as it is (one term); an fp16 V is exactly
// hi + lo.  The summary kernel's key operand is bounded by |k| (its weights
// are at most one), so there it is a pair of fp16 tiles when the inputs are
// fp16 (22 significant bits), and v is the second operand as it is.
//
// Output kernel (gla_out_tc).  One CTA (256 threads) walks a segment of
// consecutive chunks of one (batch, head) sequence and carries the state in
// fp32 registers, transposed (S^T, rows dv).  For chunk c with in-chunk
// inclusive log-gate cumsum G_j (per key dim) and Gam = G at its last
// position, the factors are referenced to the chunk start:
//   q~_j = q_j e^{G_j},  k~_i = k_i e^{-G_i}
//   o_j  = q~_j S + sum_{i<=j} (q~_j . k~_i) v_i              -> RMSNorm x SiLU(z)
//   S^T <- (S^T + V^T k~) diag(e^{Gam})
// With every G_j in [-kSpanMax, 0] both factors stay within e^{kSpanMax} of
// one (bf16 has fp32's exponent range), and each product q~_jd k~_id equals
// q_jd k_id e^{G_jd - G_id} to the operands' precision, so the unmasked
// scores carry no cancellation.  A chunk with a gate cumsum outside that
// range evaluates its scores exactly on CUDA cores instead (key tile
// k^ = k e^{Gam - G}, P_ji = sum_d q_jd k_id e^{G_jd - G_id},
// S^T <- S^T diag(e^{Gam}) + V^T k^).  The cumsum, the exact-chunk test and
// the operand build run as one pass: each warp takes eight tokens, each lane
// two dims, so every shared-memory access of a warp is one whole 128-byte row.
// An MMA instruction costs about the same for N = 128 as for N = 64, so o and
// the scores come from one N = 128 product q~ [S^T; k~]^T (the state tile
// and the key tile adjacent in shared memory, K-major).
// Tensor memory (256 columns per chain): [0, 64) o = q~ S, then += P V;
// [64, 128) the scores q~ k~^T, then (once P has been read out) the
// increment (V^T k~)^T with rows dv, matching the transposed state;
// [128, 192) the masked two-term P, written back from registers as the
// tensor-memory A operand of P V (no shared-memory round trip; an exact
// chunk's CUDA-core P goes through the q~ tiles instead).
// Row phases (P, epilogue, state) run four threads per accumulator row: warp w
// reads the 16 TMEM lanes of quadrant w % 4 that an M = 64 accumulator uses
// (row r -> lane 32 (r / 16) + r % 16) with the 16x32bx2 shape, half w / 4 of
// the columns, 16 columns per thread.
//
// Summary kernel (gla_sum_tc).  The state a segment produces from zero is one
// contraction over all its tokens: dS = sum_s diag(e^{L - G_s}) k_s^T v_s, G_s
// the log-gate cumsum from the segment start and L its total.  The CTA walks
// its chunks last to first keeping R, the summed log-gate of the chunks
// already seen, so every weight e^{R + Gam_c - G_s} is known when its chunk is
// built (and is at most one for non-positive gates); all chunks accumulate
// into one TMEM accumulator and no state passes through registers.  Eight
// warps build the tiles; a ninth issues the products and the chunk loads, so
// the builders move on while the tensor pipe works.  Staging is double-
// buffered two chunks ahead.
//
// Data movement: every token's head vector is one contiguous 128-byte row (256
// bytes for the fp32 gate) of a [B, T, H, D] tensor, so one head's chunk is a
// tensor-map box: 64 consecutive tokens in scan order LR / RL, 64 consecutive
// grid rows of one column in TB / BT (when 64 divides the grid height).  A
// reversed scan loads the same box and walks its rows backwards.  Other
// shapes gather the chunk per token with 16-byte cp.async copies (the scan
// order in the source address).  No transpose kernel runs.  Rows past the end
// of a ragged last chunk are zero-filled (a zero gate repeats the last
// cumsum), so no later phase tests them.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace gtr {
namespace tc {

constexpr int kC = 64;                 // chunk length
constexpr int kD = 64;                 // head dim (dk = dv)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kSpanMax = 20.0f;      // nats of in-chunk decay the factorised scores take
constexpr unsigned long long kWaitNs = 500ull * 1000 * 1000;   // bounded waits: 0.5 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTile = kC * kD * 2;     // one 64 x 64 16-bit tile: 8 KB
constexpr int kGTile = kC * kD * 4;    // the fp32 gate tile: 16 KB
constexpr int kRowBytes = kD * 2;      // a token's 16-bit head vector

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
// One plain arrival.
__device__ __forceinline__ void mbar_arrive_one(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
// One arrival that also expects `bytes` of asynchronous copies on the barrier.
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes)
               : "memory");
}
// Tensor-map box loads (global -> shared), completing on an mbarrier.  The
// innermost coordinate is always 0 here (16-byte aligned); the others may be
// negative or past the end, which reads zeros.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5}], [%6];" ::"r"(saddr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(saddr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            int c4, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4, %5, %6}], [%7];" ::"r"(saddr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(saddr(bar))
      : "memory");
}
// Tiled tensor-map stores shared -> global (bulk-group completion).  The
// innermost coordinate must be 16-byte aligned and no coordinate negative.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                   map),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(saddr(src))
               : "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4, %5}], [%6];" ::"l"(map),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(saddr(src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N committed bulk stores still read shared memory / are in flight
template <int N> __device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N> __device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// 16-byte asynchronous global -> shared copy (L2 only), grouped by commit.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most N of this thread's committed groups are still in flight
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
// Wait for this thread's tcgen05.ld, tied to the 16 registers of the load so
// that no use of them can be scheduled before it (the compiler does not know
// the load is asynchronous).
__device__ __forceinline__ void tmem_ld_wait(float (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
                 "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]),
                 "+f"(v[14]), "+f"(v[15])
               :
               : "memory");
}
// 16 lanes x 32 bit in two halves, eight columns each (the store counterpart
// of tmem_ld16x2 at half the width): thread t of warp w writes lane
// 32(w%4) + t%16, columns [c, c+8) for t < 16 and [c+8, c+16) for t >= 16.
__device__ __forceinline__ void tmem_st8x2(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.16x32bx2.x8.b32 [%0], 8, {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// barrier over `count` threads (whole warps) on hardware barrier `id` (1..15)
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// The same barrier, also OR-ing a predicate across its threads.
__device__ __forceinline__ bool named_barrier_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %3, 0;\n\t"
      "barrier.cta.red.or.pred q, %1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(count), "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
// 2^x by the hardware approximation (ex2.approx, flush-to-zero)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Power-of-two operand scales: 2^e puts the magnitude m into [2^14, 2^15),
// inside fp16's range; exact, and undone on the fp32 accumulator.
__device__ __forceinline__ int scale_exp(float m) {
  if (!(m > 0.f) || !(m <= 3.0e38f)) return 0;
  const int ex = ((__float_as_int(m) >> 23) & 0xFF) - 127;
  return max(-60, min(60, 14 - ex));
}
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }
// logsigmoid(u) / tau = (min(u, 0) - ln(1 + e^{-|u|})) / tau, the exponential
// and the logarithm (as log2, scaled by ln2_tau = ln 2 / tau) by the hardware
// approximations.  1 + e^{-|u|} is formed in fp32, so the log term carries an
// absolute error below 1e-7 (it rounds to zero once e^{-|u|} is under fp32's
// resolution at one); both terms are <= 0, so the result is too.
__device__ __forceinline__ float logsigmoid_over_tau(float u, float inv_tau, float ln2_tau) {
  const float e = ex2(-fabsf(u) * 1.4426950408889634f);
  float l;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(l) : "f"(1.0f + e));
  return fmaf(-l, ln2_tau, fminf(u, 0.0f) * inv_tau);
}
// Two fp32 lanes per instruction (add / mul / fma .f32x2, sm_100): a pair of
// floats in one 64-bit register, the first in the low half.
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t r) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
  return make_float2(a, b);
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// q(t) = log2(1 + t) / t on [0, 1]: the degree-8 Chebyshev interpolant (nodes
// cos(pi (k + 1/2) / 9) mapped to [0, 1]) written in powers of t, from
// log2_1p_poly.py.  t q(t) is within 1.6e-7 of log2(1 + t) in fp32 Horner
// evaluation, exactly 0 at t = 0 and positive above.
__device__ constexpr float kL2q[9] = {1.442695022e+00f, -7.213395238e-01f, 4.806788862e-01f,
                                      -3.582990766e-01f, 2.752211988e-01f, -1.962389499e-01f,
                                      1.118320748e-01f, -4.194501042e-02f, 7.395402063e-03f};
// logsigmoid(u) / tau for two values, (min(u, 0) - ln(1 + e^{-|u|})) / tau:
// e^{-|u|} by the hardware ex2, the logarithm by the polynomial above on the
// FMA pipe (two lanes per instruction), so one MUFU operation per value
// instead of two.  Absolute error of the log term below 2e-7 (with ex2's
// relative error); both terms are <= 0, so the result is too.
__device__ __forceinline__ float2 logsigmoid_over_tau2(float ua, float ub, float inv_tau, float ln2_tau) {
  const uint64_t t = f2pack(ex2(-fabsf(ua) * 1.4426950408889634f), ex2(-fabsf(ub) * 1.4426950408889634f));
  uint64_t q = f2pack(kL2q[8], kL2q[8]);
#pragma unroll
  for (int k = 7; k >= 0; --k) q = ffma2(q, t, f2pack(kL2q[k], kL2q[k]));
  const uint64_t m = fmul2(f2pack(fminf(ua, 0.0f), fminf(ub, 0.0f)), f2pack(inv_tau, inv_tau));
  return f2unpack(ffma2(fmul2(q, t), f2pack(-ln2_tau, -ln2_tau), m));
}
// Two-term fp16 value pairs: x = hi + lo, hi = fp16(x), lo = fp16(x - hi),
// two consecutive elements per 32-bit word.
__device__ __forceinline__ void split2h(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
  memcpy(&hi, &h, 4);
  memcpy(&lo, &l, 4);
}
// Untiled bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing on `bar` (which must expect the bytes).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          saddr(dst)),
      "l"(src), "r"(bytes), "r"(saddr(bar))
      : "memory");
}

// ------------------------------------------------------- operand layouts
// 16-bit operand tiles of 64 rows x 64 elements (128 bytes per row), layout
// SWIZZLE_128B: atoms of 8 rows x 128 bytes, the 16-byte unit index XOR-ed
// with the row's position in its atom.  The same physical layout serves a
// K-major operand (rows = M or N, columns = K) and an MN-major one (rows = K,
// columns = M or N); only the descriptor differs.
__device__ __forceinline__ uint32_t sw_unit(int r, int u) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw16(int r, int c) { return sw_unit(r, c >> 3) + (c & 7) * 2; }
// tcgen05 shared-memory matrix descriptor (version 1): start address, leading
// and stride byte offsets, layout type 2 = SWIZZLE_128B.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// K-major tile: a K step of 16 elements is 32 bytes into every row.
__device__ __forceinline__ uint64_t desc_k(const void* tile) { return sdesc(saddr(tile), 16, 1024); }
// MN-major tile: a K step of 16 rows is two 8-row atoms, 2048 bytes.
__device__ __forceinline__ uint64_t desc_mn(const void* tile) { return sdesc(saddr(tile), 8192, 1024); }
constexpr uint32_t kStepK = 32 >> 4, kStepMN = 2048 >> 4;   // descriptor address units per K step
// Instruction descriptor: kind::f16 with bf16 A and B, fp32 accumulate, M = 64,
// N = n (64 unless given).
__host__ __device__ constexpr uint32_t idesc_bf16(int a_mn, int b_mn, int n = 64) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(64 >> 4) << 24);
}
// The same with fp16 A and B.
__host__ __device__ constexpr uint32_t idesc_f16(int a_mn, int b_mn, int n = 64) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(64 >> 4) << 24);
}
// One tcgen05.mma kind::f16 instruction; the instruction descriptor selects
// fp16 or bf16 operands.
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// One tcgen05.mma kind::f16 with A in tensor memory (M = 64: row r in lane
// 32 (r / 16) + r % 16, two 16-bit elements per 32-bit column, the even one
// in the low half; a K = 16 step is 8 columns).
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// d += (ah + al)(bh + bl) ~ ah bh + ah bl + al bh over K = 64, A in tensor memory
template <uint32_t SB>
__device__ __forceinline__ void mma_terms_ts(uint32_t d, uint32_t ah, uint32_t al, uint64_t bh, uint64_t bl,
                                             bool b_two, uint32_t id) {
#pragma unroll
  for (uint32_t s = 0; s < 4; ++s) mma_f16_ts(d, ah + 8 * s, bh + s * SB, id, 1u);
  if (b_two) {
#pragma unroll
    for (uint32_t s = 0; s < 4; ++s) mma_f16_ts(d, ah + 8 * s, bl + s * SB, id, 1u);
  }
#pragma unroll
  for (uint32_t s = 0; s < 4; ++s) mma_f16_ts(d, al + 8 * s, bh + s * SB, id, 1u);
}
// d (+)= A B over K = 64: four K = 16 instructions.
template <uint32_t SA, uint32_t SB>
__device__ __forceinline__ void mma_k64(uint32_t d, uint64_t a, uint64_t b, uint32_t id, bool acc) {
#pragma unroll
  for (uint32_t s = 0; s < 4; ++s) mma_f16(d, a + s * SA, b + s * SB, id, (acc || s) ? 1u : 0u);
}
// (ah + al)(bh + bl) ~ ah bh + ah bl + al bh, or ah b + al b for a one-term B.
template <uint32_t SA, uint32_t SB>
__device__ __forceinline__ void mma_terms(uint32_t d, uint64_t ah, uint64_t al, uint64_t bh,
                                          uint64_t bl, bool b_two, uint32_t id, bool acc) {
  mma_k64<SA, SB>(d, ah, bh, id, acc);
  if (b_two) mma_k64<SA, SB>(d, ah, bl, id, true);
  mma_k64<SA, SB>(d, al, bh, id, true);
}
// The same with the optional second term on A: a bh + a bl for a one-term A.
template <uint32_t SA, uint32_t SB>
__device__ __forceinline__ void mma_terms_a(uint32_t d, uint64_t ah, uint64_t al, uint64_t bh,
                                            uint64_t bl, bool a_two, uint32_t id, bool acc) {
  mma_k64<SA, SB>(d, ah, bh, id, acc);
  mma_k64<SA, SB>(d, ah, bl, id, true);
  if (a_two) mma_k64<SA, SB>(d, al, bh, id, true);
}

// --------------------------------------------------- two-term bf16 operands
__device__ __forceinline__ uint32_t bits2(__nv_bfloat162 h) {
  uint32_t u;
  memcpy(&u, &h, 4);
  return u;
}
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 f = __bfloat1622float2(h);
  hi = bits2(h);
  lo = bits2(__floats2bfloat162_rn(a - f.x, b - f.y));   // a - hi is exact in fp32
}
// four consecutive elements (8 bytes) at byte offset `off` of the (hi, lo) tiles
__device__ __forceinline__ void put4(uint8_t* H, uint8_t* L, uint32_t off, float a, float b, float c,
                                     float d) {
  uint32_t h0, l0, h1, l1;
  split2(a, b, h0, l0);
  split2(c, d, h1, l1);
  *reinterpret_cast<uint2*>(H + off) = make_uint2(h0, h1);
  *reinterpret_cast<uint2*>(L + off) = make_uint2(l0, l1);
}

// eight consecutive elements (16 bytes, one swizzle unit) at byte offset `off`
__device__ __forceinline__ void put8(uint8_t* H, uint8_t* L, uint32_t off, const float* x) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split2(x[2 * i], x[2 * i + 1], h[i], l[i]);
  *reinterpret_cast<uint4*>(H + off) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(L + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// two consecutive elements (4 bytes) at byte offset `off` of the (hi, lo) tiles
// the same in fp16 terms
__device__ __forceinline__ void put2h(uint8_t* H, uint8_t* L, uint32_t off, float a, float b) {
  uint32_t h, l;
  split2h(a, b, h, l);
  *reinterpret_cast<uint32_t*>(H + off) = h;
  *reinterpret_cast<uint32_t*>(L + off) = l;
}
__device__ __forceinline__ void put2x(uint8_t* H, uint8_t* L, uint32_t off, float a, float b) {
  uint32_t h, l;
  split2(a, b, h, l);
  *reinterpret_cast<uint32_t*>(H + off) = h;
  *reinterpret_cast<uint32_t*>(L + off) = l;
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
// two consecutive 16-bit elements as floats
__device__ __forceinline__ float2 ld2(const __half* p) { return __half22float2(*reinterpret_cast<const __half2*>(p)); }
__device__ __forceinline__ float2 ld2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

template <typename T> __device__ __forceinline__ uint2 pack4(float a, float b, float c, float d);
template <> __device__ __forceinline__ uint2 pack4<__half>(float a, float b, float c, float d) {
  const __half2 x = __floats2half2_rn(a, b), y = __floats2half2_rn(c, d);
  uint2 u;
  memcpy(&u.x, &x, 4);
  memcpy(&u.y, &y, 4);
  return u;
}
template <> __device__ __forceinline__ uint2 pack4<__nv_bfloat16>(float a, float b, float c, float d) {
  return make_uint2(bits2(__floats2bfloat162_rn(a, b)), bits2(__floats2bfloat162_rn(c, d)));
}

struct Params {
  const void* q; const void* k; const void* v; const float* g; const void* z; const float* w;
  float* wsS; float* wsA; void* out;
  int H, T, gh, gw, dir, nseg;
  int tma;                        // 1: chunks arrive by tensor-map loads (Maps valid)
  // Summary stage with the gate's second half in-kernel (gla_sum_tc<T, true>):
  // the rank-16 rows low = x W_down [B, T, 16] fp32, the packed W_up terms
  // (two fp16 tiles of 16 x H*dk, MN-major, `wu_term` bytes apart, head h's
  // 64 columns a 2 KB block at 2048 h), their inverse column scales, the bias
  // (or null) and 1/tau; the kernel writes g to `g_out`.
  const float* low; const uint8_t* wu; const float* wu_scale; const float* gbias; float* g_out;
  int wu_term;
  float inv_tau;
};
// Tensor maps of q, k, v, g ([B, T, H, D] row-major) for box loads of one
// chunk of one head: [0] the token order, dims (D, H, T, B), box (64, 1, 64,
// 1); [1] the grid columns, dims (D, H, gw, gh, B), box (64, 1, 1, 64, 1)
// (valid when 64 divides gh).  A reversed scan loads the same box and walks
// it backwards.  q, k, g are plain row-major boxes; v lands in the
// SWIZZLE_128B operand layout.
// [.][kMapL]: the rank-16 rows low [B, T, 16] fp32 as dims (16, 1, T, B) /
// (16, 1, gw, gh, B), box 16 x 64 tokens (head coordinate 0).  [.][kMapGS]:
// g_out for stores, box 32 x 64 (one 128-byte half of each row), SWIZZLE_128B.
enum { kMapQ = 0, kMapK = 1, kMapV = 2, kMapG = 3, kMapL = 4, kMapGS = 5 };
struct Maps {
  CUtensorMap t[2][6];
};

// ------------------------------------------------------------- fetching
// Scan order -> box: orientation (0 token order, 1 grid columns) and whether
// the chunk's box is walked backwards.
__device__ __forceinline__ int dir_orient(int d) { return d == kTB || d == kBT; }
__device__ __forceinline__ bool dir_reversed(int d) { return d == kRL || d == kBT; }
// Box loads of the chunk at scan position s0: q, k (row-major), v (operand
// layout, at vdst), g (row-major fp32), all completing on `bar`.  Box row j
// holds scan position s0 + j, or s0 + 63 - j for a reversed scan (whose
// last, ragged chunk then starts at a negative token and reads zeros there).
__device__ __forceinline__ void tma_box(const Params& p, const Maps& mp, int which, void* dst, uint64_t* bar,
                                        int d, int b, int h, int s0) {
  const int t0 = dir_reversed(d) ? p.T - s0 - kC : s0;   // first scan position of the box, in its order
  if (!dir_orient(d)) {
    tma_load_4d(dst, &mp.t[0][which], 0, h, t0, b, bar);
  } else {
    const int col = t0 / p.gh, r0 = t0 - col * p.gh;   // whole chunks: t0 >= 0, r0 + 64 <= gh
    tma_load_5d(dst, &mp.t[1][which], 0, h, col, r0, b, bar);
  }
}
// Store counterpart of tma_box (box rows in the same order), at column x of
// the rows; not for a reversed scan's ragged chunk (its box starts before
// token 0, and a store may not start at a negative coordinate).
__device__ __forceinline__ void tma_store_box(const Params& p, const Maps& mp, int which, const void* src, int d,
                                              int b, int h, int s0, int x) {
  const int t0 = dir_reversed(d) ? p.T - s0 - kC : s0;
  if (!dir_orient(d)) {
    tma_store_4d(&mp.t[0][which], src, x, h, t0, b);
  } else {
    const int col = t0 / p.gh, r0 = t0 - col * p.gh;
    tma_store_5d(&mp.t[1][which], src, x, h, col, r0, b);
  }
}
__device__ __forceinline__ void tma_chunk(const Params& p, const Maps& mp, uint8_t* kdst, uint8_t* qdst,
                                          uint8_t* vdst, uint8_t* gdst, uint64_t* bar, int d, int b, int h,
                                          int s0) {
  mbar_arrive_tx(bar, 3 * kTile + kGTile);
  tma_box(p, mp, kMapK, kdst, bar, d, b, h, s0);
  tma_box(p, mp, kMapQ, qdst, bar, d, b, h, s0);
  tma_box(p, mp, kMapV, vdst, bar, d, b, h, s0);
  tma_box(p, mp, kMapG, gdst, bar, d, b, h, s0);
}
// Token rows (b*T + t)*H + h of the chunk starting at scan position s0.
__device__ __forceinline__ void chunk_rows(const Params& p, long long* rows, int b, int h, int d,
                                           int s0, int ntok, int tid) {
  if (tid < ntok) rows[tid] = ((long long)b * p.T + scan_to_grid(d, s0 + tid, p.T, p.gh, p.gw)) * p.H + h;
}
// A 16-bit tensor's rows of the chunk into a 64 x 64 tile: row-major (row j
// at byte j * 128) or, with kSw, in the SWIZZLE_128B operand layout.  16-byte
// pieces, piece o = (row o / 8, unit o % 8); rows past ntok are zeroed.
template <bool kSw = false>
__device__ __forceinline__ void fetch16(uint8_t* dst, const void* src, const long long* rows, int ntok,
                                        int tid) {
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int o = tid + u * kThreads, j = o >> 3, part = (o & 7) * 16;
    uint8_t* to = dst + (kSw ? sw_unit(j, o & 7) : (uint32_t)(j * 128 + part));
    if (j < ntok) cp_async16(to, (const uint8_t*)src + rows[j] * kRowBytes + part);
    else *reinterpret_cast<uint4*>(to) = make_uint4(0u, 0u, 0u, 0u);
  }
}
// The fp32 gate rows (256 bytes each); rows past ntok get a zero gate.
__device__ __forceinline__ void fetch_g(uint8_t* dst, const float* g, const long long* rows, int ntok,
                                        int tid) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int o = tid + u * kThreads, j = o >> 4, part = (o & 15) * 16;
    if (j < ntok) cp_async16(dst + j * 256 + part, (const uint8_t*)g + rows[j] * (kD * 4) + part);
    else *reinterpret_cast<uint4*>(dst + j * 256 + part) = make_uint4(0u, 0u, 0u, 0u);
  }
}
// In-chunk inclusive cumsum of the gate tile, column dd, tokens 16 qt .. 16 qt
// + 15 of this thread, in registers; the four threads of a column exchange
// their partial sums once through `part` (one block barrier).  Returns the
// column total.
__device__ __forceinline__ float column_cumsum(const float* G, float (&gv)[16], float* part, int dd,
                                               int qt) {
#pragma unroll
  for (int i = 0; i < 16; ++i) gv[i] = G[(qt * 16 + i) * kD + dd];
#pragma unroll
  for (int i = 1; i < 16; ++i) gv[i] += gv[i - 1];
  part[qt * kD + dd] = gv[15];
  __syncthreads();
  const float p0 = part[dd], p1 = part[kD + dd], p2 = part[2 * kD + dd], p3 = part[3 * kD + dd];
  const float off = qt == 0 ? 0.f : qt == 1 ? p0 : qt == 2 ? p0 + p1 : (p0 + p1) + p2;
#pragma unroll
  for (int i = 0; i < 16; ++i) gv[i] += off;
  return ((p0 + p1) + p2) + p3;
}

// 32-byte store (st.global.v8, sm_100); `p` must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, uint4 a, uint4 b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// ===================================================================== K4
struct OutMisc {                  // per-chain scalars; arrays read as float4 are 16-byte aligned
  uint64_t mma[3];                // [0] q~ S and the scores, [1] + P V, [2] state increment
  uint64_t ld;                    // a chunk's box loads
  uint64_t built;                 // this chain has built a chunk's tiles (the other chain's turn)
  uint32_t tmem;
  int pad;
  alignas(16) float part[kWarps][kD];   // cumsum partials: tokens 8 w .. 8 w + 7, per dim
  alignas(16) float red[2][kD];   // epilogue row sums
  alignas(16) float Gam[kD];
  alignas(16) float aG[kD];       // e^{Gam}: state decay over the chunk
  alignas(16) float wv[kD];       // RMSNorm weight
  alignas(16) long long rows[2][kC];   // token rows of the current / next chunk
};
struct OutLayout {
  // Two chains per CTA (warps 0-7 and 8-15), each with the layout below at
  // offset kChain * chain.  Staging: k, q (row-major), v (operand layout),
  // gate (row-major fp32).
  static constexpr int kOffK = 0, kOffQ = kTile, kOffV = 2 * kTile, kOffG = 3 * kTile;
  // operand tiles (1024-aligned): VH VL QH QL SH KH SL KL.  The state tile
  // S^T and the key tile are adjacent, so that [S^T; k~] is one 128-row
  // K-major B operand.  A bf16 v read in scan order lands directly in VH / VL,
  // alternately by chunk parity.
  static constexpr int kTiles = 3 * kTile + kGTile;
  static constexpr int kMisc = kTiles + 8 * kTile;
  static constexpr int kChain = (kMisc + (int)sizeof(OutMisc) + 1023) & ~1023;
  static constexpr int kSmem = 2 * kChain + 1024;   // + alignment slack
  // per chain: o [0, 64), scores / increment [64, 128), P hi [128, 160), P lo [160, 192)
  static constexpr int kTmemCols = 512;             // 256 per chain
  static constexpr int kThreadsAll = 2 * kThreads;
  static constexpr int kChainsPerSM = 2;
};
static_assert(OutLayout::kTiles % 1024 == 0, "operand tiles must be 1024-byte aligned");

// The k, q, gate rows of a chunk into the output kernel's staging (cp.async),
// v into `vdst` in the operand layout.
__device__ __forceinline__ void fetch_chunk(uint8_t* sm, uint8_t* vdst, const Params& p, const long long* rows,
                                            int ntok, int tid) {
  fetch16(sm + OutLayout::kOffK, p.k, rows, ntok, tid);
  fetch16(sm + OutLayout::kOffQ, p.q, rows, ntok, tid);
  fetch16<true>(vdst, p.v, rows, ntok, tid);
  fetch_g(sm + OutLayout::kOffG, p.g, rows, ntok, tid);
}
static_assert(OutLayout::kSmem <= 227 * 1024, "the two-chain output CTA must fit one SM");

// Sum over the four threads that share an accumulator row: the other half of
// the warp (lane ^ 16) and the same lanes of the partner warp (warp ^ 4),
// through shared memory and a named barrier (`bar`) of those two warps.
__device__ __forceinline__ float row_combine_sum(float v, float (*red)[kD], int row, int half, int bar,
                                                 int lane) {
  v += __shfl_xor_sync(0xffffffffu, v, 16);
  if (lane < 16) red[half][row] = v;
  named_barrier(bar, 64);
  return v + red[half ^ 1][row];
}

// Two chains per CTA: warps 0-7 walk segment 2 blockIdx.x, warps 8-15 segment
// 2 blockIdx.x + 1, each with its own shared memory, TMEM columns and
// barriers (chain barrier 1 + 5 g over 256 threads, row-pair barriers
// 2 + 5 g + qd).  Their tile-build phases alternate (chain 0 builds chunk i
// after chain 1 has built chunk i - 1, chain 1 builds chunk i after chain 0
// has built chunk i), so each chain's build overlaps the other's MMAs, P and
// epilogue instead of contending with its build.
template <typename T>
__global__ void __launch_bounds__(OutLayout::kThreadsAll, 1)
gla_out_tc(const __grid_constant__ Params p, const __grid_constant__ Maps mp) {
  using L = OutLayout;
  constexpr bool kV2 = std::is_same<T, __half>::value;   // fp16 V: two bf16 terms
  extern __shared__ uint8_t smem_raw[];
  const int chain = threadIdx.x >> 8;
  uint8_t* const sm0 = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sm = sm0 + chain * L::kChain;
  OutMisc& m_other = *reinterpret_cast<OutMisc*>(sm0 + (chain ^ 1) * L::kChain + L::kMisc);
  const int bar_all = 1 + 5 * chain, bar_pair = 2 + 5 * chain;
  const T* kst = reinterpret_cast<const T*>(sm + L::kOffK);
  const T* qst = reinterpret_cast<const T*>(sm + L::kOffQ);
  float* G = reinterpret_cast<float*>(sm + L::kOffG);
  uint8_t* VH = sm + L::kTiles;
  uint8_t* VL = VH + kTile;
  uint8_t* QH = VH + 2 * kTile;       // q~, then P (K-major A)
  uint8_t* QL = VH + 3 * kTile;
  uint8_t* SH = VH + 4 * kTile;       // S^T, rows dv: rows 0-63 of the K-major B [S^T; k~]
  uint8_t* KH = VH + 5 * kTile;       // k~ or k^: rows 64-127 of that B; MN-major B of V^T k~
  uint8_t* SL = VH + 6 * kTile;
  uint8_t* KL = VH + 7 * kTile;
  OutMisc& m = *reinterpret_cast<OutMisc*>(sm + L::kMisc);

  const int tid = threadIdx.x & (kThreads - 1), warp = tid >> 5, lane = tid & 31;
  const int seg = 2 * blockIdx.x + chain, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = dir_of_batch(p.dir, b);
  const int nc = (p.T + kC - 1) / kC;
  // chunks of each chain (a chain past the last segment has none)
  auto chunks_of = [&](int sg) {
    return sg < p.nseg ? seg_first_chunk(sg + 1, nc, p.nseg) - seg_first_chunk(sg, nc, p.nseg) : 0;
  };
  const int c0 = seg < p.nseg ? seg_first_chunk(seg, nc, p.nseg) : 0;
  int nch = chunks_of(seg);
  const int nch_other = (d < 0 || d > 3) ? 0 : chunks_of(seg ^ 1);
  if (d < 0 || d > 3) {
    if (tid == 0) gtr_flag(kStatusBadDir);
    nch = 0;
  }
  const bool tma = p.tma != 0;
  const bool out32 = ((uintptr_t)p.out & 31) == 0;
  // staging row of scan offset i: box loads of a reversed scan hold the chunk backwards
  const int rmask = (tma && dir_reversed(d)) ? kC - 1 : 0;
  // a bf16 v in scan order is the operand tile itself (double-buffered by
  // chunk parity); otherwise it is staged and converted by the builder
  const bool vdirect = !kV2 && rmask == 0;
  auto vtile = [&](int it) -> uint8_t* { return vdirect ? ((it & 1) ? VL : VH) : sm + L::kOffV; };
  auto fetch = [&](int it, int s, int ntk, const long long* rws) {
    if (tma) {
      if (tid == 32) tma_chunk(p, mp, sm + L::kOffK, sm + L::kOffQ, vtile(it), sm + L::kOffG, &m.ld, d, b, h, s);
    } else {
      fetch_chunk(sm, vtile(it), p, rws, ntk, tid);
    }
  };
  // row phases: quadrant qd, column half, 16 columns from cbase of accumulator row `row`
  const int qd = warp & 3, half = warp >> 2;
  const int row = qd * 16 + (lane & 15);
  const int cbase = half * 32 + (lane >> 4) * 16;
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  // cumsum and tile build: dims 2 lane, 2 lane + 1 of scan offsets 8 warp ..
  // 8 warp + 7, so every shared-memory access of a warp covers one whole row
  const int dc = 2 * lane, tb = 8 * warp;

  if (tid == 0) {
    mbar_init(&m.mma[0], 1);
    mbar_init(&m.mma[1], 1);
    mbar_init(&m.mma[2], 1);
    mbar_init(&m.ld, 1);
    mbar_init(&m.built, 1);
    mbar_fence_init();
  }
  // chunk 0's copies go out first
  if (nch > 0) {
    const int ntok0 = min(kC, p.T - c0 * kC);
    chunk_rows(p, m.rows[0], b, h, d, c0 * kC, ntok0, tid);
    named_barrier(bar_all, kThreads);
    fetch(0, c0 * kC, ntok0, m.rows[0]);
    cp_async_commit();
  }
  if (tid < kD) m.wv[tid] = p.w ? p.w[tid] : 1.0f;
  // Launched programmatically after the boundary scan, this block may start
  // while the scan runs: q, k, v, g, z and w were complete before the summary
  // stage passed its own wait (the scan starts its dependents only after
  // that), so chunk 0 is fetched above; the boundary states need the wait.
  pdl_wait();
  pdl_trigger();
  // carried state, transposed: S[c] = S^T[row][cbase + c] = S[cbase + c][row]
  // (row a dv index), from the boundary scan's [dk][dv] states
  float S[16];
  if (nch > 0) {
    const float* src = p.wsS + ((size_t)bh * p.nseg + seg) * kD * kD + (size_t)cbase * kD + row;
#pragma unroll
    for (int c = 0; c < 16; ++c) S[c] = src[c * kD];
  }
  OutMisc& m0 = *reinterpret_cast<OutMisc*>(sm0 + L::kMisc);
  if (threadIdx.x < 32) {
    tmem_alloc(&m0.tmem, L::kTmemCols);
    tmem_relinquish();
  }
  cp_async_wait<0>();                     // chunk 0's k, q, v, g (copied by this thread)
  tc_before_sync();
  __syncthreads();                        // both chains: their barriers and the TMEM columns
  tc_after_sync();
  const uint32_t tm = m0.tmem + 256u * (uint32_t)chain;
  constexpr uint32_t kIdQSK = idesc_bf16(0, 0, 128);   // both K-major, N = 128: q~ [S^T; k~]^T
  constexpr uint32_t kIdQS = idesc_bf16(0, 0);          // both K-major: q~ S (an exact chunk)
  constexpr uint32_t kIdPV = idesc_bf16(0, 1);          // A K-major, B MN-major: P V
  constexpr uint32_t kIdVK = idesc_bf16(1, 1);          // both MN-major: V^T k~

  uint32_t ph0 = 0, ph1 = 0, ph2 = 0, phl = 0;
  bool failed = false, ld_pending = tma && nch > 0;   // chunk 0's boxes
  // The next chunk's k, q, v, g are requested once this chunk's tiles are
  // built (after P for an exact chunk, whose scores still read the staging);
  // z goes straight to registers, requested two phases before the epilogue.
  for (int it = 0; it < nch; ++it) {
    const int par = it & 1;
    const int s0 = (c0 + it) * kC;
    const int ntok = min(kC, p.T - s0);
    const bool more = it + 1 < nch;
    const int s1 = s0 + kC;
    const int ntok1 = more ? min(kC, p.T - s1) : 0;
    uint8_t* const Vh = vdirect ? vtile(it) : VH;
    uint8_t* const Vl = vdirect ? Vh : VL;      // VL is read only for a two-term (fp16) v
    // this chain's turn to build: chain 0 after the other's chunk it - 1, chain 1 after its chunk it
    {
      const int j = chain == 0 ? it - 1 : it;
      if (j >= 0 && j < nch_other) failed |= !mbar_wait(&m_other.built, (uint32_t)j & 1u);
    }
    if (tma) {
      failed |= !mbar_wait(&m.ld, phl);
      phl ^= 1;
      ld_pending = false;
    }

    // ---- in-chunk cumsum G: eight scan offsets in registers, then the
    // partial sums of the warps before this one (one block barrier)
    float2 gc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      gc[i] = *reinterpret_cast<const float2*>(G + ((tb + i) ^ rmask) * kD + dc);
      if (i) { gc[i].x += gc[i - 1].x; gc[i].y += gc[i - 1].y; }
    }
    *reinterpret_cast<float2*>(&m.part[warp][dc]) = gc[7];
    named_barrier(bar_all, kThreads);
    {
      float2 off = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kWarps - 1; ++w)
        if (w < warp) {
          const float2 pp = *reinterpret_cast<const float2*>(&m.part[w][dc]);
          off.x += pp.x; off.y += pp.y;
        }
#pragma unroll
      for (int i = 0; i < 8; ++i) { gc[i].x += off.x; gc[i].y += off.y; }
    }
    int bad = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      bad |= !(gc[i].x <= 0.f && gc[i].x >= -kSpanMax && gc[i].y <= 0.f && gc[i].y >= -kSpanMax);
    if (warp == kWarps - 1) {
      *reinterpret_cast<float2*>(&m.Gam[dc]) = gc[7];
      *reinterpret_cast<float2*>(&m.aG[dc]) = make_float2(expf(gc[7].x), expf(gc[7].y));
    }

    // ---- operand tiles, referenced to the chunk start: q~ = q e^{G}, k~ = k e^{-G}
    // (rows past ntok are zero: their q, k were zero-filled).  All eight rows
    // are loaded before any tile is written: the stores could alias the
    // staging as far as the compiler knows, so interleaving them with the
    // loads would serialise every row on the shared-memory latency.
    {
      uint32_t qr[8], kr[8], vr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rs = (tb + i) ^ rmask;
        qr[i] = *reinterpret_cast<const uint32_t*>(qst + rs * kD + dc);
        kr[i] = *reinterpret_cast<const uint32_t*>(kst + rs * kD + dc);
        vr[i] = vdirect ? 0u : *reinterpret_cast<const uint32_t*>(sm + L::kOffV + sw16(rs, dc));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t off = sw16(tb + i, dc);
        const float2 qq = ld2(reinterpret_cast<const T*>(&qr[i])), kk = ld2(reinterpret_cast<const T*>(&kr[i]));
        const float x0 = gc[i].x * kLog2e, x1 = gc[i].y * kLog2e;
        put2x(QH, QL, off, qq.x * ex2(x0), qq.y * ex2(x1));
        put2x(KH, KL, off, kk.x * ex2(-x0), kk.y * ex2(-x1));
        if (!vdirect) {
          if (kV2) {
            const float2 vv = ld2(reinterpret_cast<const T*>(&vr[i]));
            put2x(VH, VL, off, vv.x, vv.y);
          } else {
            *reinterpret_cast<uint32_t*>(VH + off) = vr[i];
          }
        }
      }
    }
    put8(SH, SL, sw16(row, cbase), S);
    put8(SH, SL, sw16(row, cbase + 8), S + 8);
    if (more) chunk_rows(p, m.rows[par ^ 1], b, h, d, s1, ntok1, tid);
    fence_async_smem();
    tc_before_sync();
    // with G in [-kSpanMax, 0] everywhere no factor leaves [e^{-kSpanMax}, e^{kSpanMax}]
    const bool exact = named_barrier_or(bar_all, kThreads, bad != 0);
    const bool tilde = !exact;
    tc_after_sync();
    if (tid == 0) mbar_arrive_one(&m.built);   // the other chain may build now

    // An MMA instruction costs about as much for N = 128 as for N = 64, so o
    // and the scores come from one N = 128 product q~ [S^T; k~]^T (o alone for
    // an exact chunk), issued by warp 0; later warp 0 adds P V onto o and warp
    // 4 forms the state increment, each thread's MMAs in issue order.
    if (tid == 0) {
      if (tilde)
        mma_terms<kStepK, kStepK>(tm + 0, desc_k(QH), desc_k(QL), desc_k(SH), desc_k(SL), true, kIdQSK,
                                  false);
      else
        mma_terms<kStepK, kStepK>(tm + 0, desc_k(QH), desc_k(QL), desc_k(SH), desc_k(SL), true, kIdQS,
                                  false);
      mma_commit(&m.mma[0]);
    }
    // the staging of k, q, v, g is consumed unless an exact chunk still reads it
    if (more && tilde) {
      fetch(it + 1, s1, ntok1, m.rows[par ^ 1]);
      ld_pending = tma;
    }
    cp_async_commit();
    if (exact) {
      // the CUDA-core scores read G (scan order) from the staging; the key
      // tile becomes k^ = k e^{Gam - G}, the state update S <- e^{Gam} S + k^^T V
      const float2 gam = *reinterpret_cast<const float2*>(&m.Gam[dc]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = tb + i;
        *reinterpret_cast<float2*>(G + r * kD + dc) = gc[i];
        const float2 kk = ld2(kst + (r ^ rmask) * kD + dc);
        put2x(KH, KL, sw16(r, dc), kk.x * expf(gam.x - gc[i].x), kk.y * expf(gam.y - gc[i].y));
      }
      named_barrier(bar_all, kThreads);
    }
    // this chunk's z for the epilogue: 16 elements of the thread's row
    uint4 zz0 = make_uint4(0u, 0u, 0u, 0u), zz1 = zz0;
    if (row < ntok) {
      const uint4* zp = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.z) + m.rows[par][row] * kD + cbase);
      zz0 = __ldg(zp);
      zz1 = __ldg(zp + 1);
    }

    failed |= !mbar_wait(&m.mma[0], ph0);
    ph0 ^= 1;
    tc_after_sync();
    if (tilde) {
      // ---- masked scores P (rows = queries j, columns = keys i) into the q~ tiles
      float sc[16];
      tmem_ld16x2(tm + lane_base + 64 + half * 32, sc);
      tmem_ld_wait(sc);
#pragma unroll
      for (int c = 0; c < 16; ++c) sc[c] = cbase + c <= row ? sc[c] : 0.f;
      // two-term P straight back into tensor memory: the A operand of P V
      uint32_t ph[8], pl[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split2(sc[2 * e], sc[2 * e + 1], ph[e], pl[e]);
      tmem_st8x2(tm + lane_base + 128 + half * 16, ph);
      tmem_st8x2(tm + lane_base + 160 + half * 16, pl);
      tmem_st_wait();
    } else {
      // exact scores on CUDA cores: P_ji = sum_d q_jd k_id e^{G_jd - G_id}; four threads per row
      if (tid == 0) atomicAdd(&g_gtr_exact_chunks, 1ull);
      const int j = tid >> 2, ib = (tid & 3) * 16;
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.f;
      if (j < ntok) {
        const T* qj_row = qst + (j ^ rmask) * kD;
        for (int x = 0; x < kD; ++x) {
          const float qj = Elem<T>::to_f(qj_row[x]);
          const float gj = G[j * kD + x];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i = ib + e;
            if (i <= j)
              acc[e] = fmaf(qj * Elem<T>::to_f(kst[(i ^ rmask) * kD + x]), expf(gj - G[i * kD + x]), acc[e]);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < 16; e += 4)
        put4(QH, QL, sw16(j, ib + e), acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    }
    fence_async_smem();
    tc_before_sync();
    if (named_barrier_or(bar_all, kThreads, failed)) { failed = true; break; }
    tc_after_sync();
    if (more && exact) {
      fetch(it + 1, s1, ntok1, m.rows[par ^ 1]);
      ld_pending = tma;
    }
    cp_async_commit();
    if (tid == 0) {
      if (tilde)
        mma_terms_ts<kStepMN>(tm + 0, tm + 128, tm + 160, desc_mn(Vh), desc_mn(Vl), kV2, kIdPV);
      else   // an exact chunk's P is in the q~ tiles
        mma_terms<kStepK, kStepMN>(tm + 0, desc_k(QH), desc_k(QL), desc_mn(Vh), desc_mn(Vl), kV2, kIdPV,
                                   true);
      mma_commit(&m.mma[1]);
    }
    if (tid == 128) {
      // (V^T k~)^T rows dv: A = V read MN-major, B = the key tile read MN-major
      mma_terms_a<kStepMN, kStepMN>(tm + 64, desc_mn(Vh), desc_mn(Vl), desc_mn(KH), desc_mn(KL), kV2,
                                    kIdVK, false);
      mma_commit(&m.mma[2]);
    }
    // the output gate w * SiLU(z) while P V and the increment run
    float wz[16];
#pragma unroll
    for (int c = 0; c < 16; c += 8) {
      const uint4 zz = c == 0 ? zz0 : zz1;
      const float4 z0 = Vec4<T>::from_bits(make_uint2(zz.x, zz.y));
      const float4 z1 = Vec4<T>::from_bits(make_uint2(zz.z, zz.w));
      const float4 w0 = *reinterpret_cast<const float4*>(&m.wv[cbase + c]);
      const float4 w1 = *reinterpret_cast<const float4*>(&m.wv[cbase + c + 4]);
      wz[c + 0] = w0.x * silu_fast(z0.x); wz[c + 1] = w0.y * silu_fast(z0.y);
      wz[c + 2] = w0.z * silu_fast(z0.z); wz[c + 3] = w0.w * silu_fast(z0.w);
      wz[c + 4] = w1.x * silu_fast(z1.x); wz[c + 5] = w1.y * silu_fast(z1.y);
      wz[c + 6] = w1.z * silu_fast(z1.z); wz[c + 7] = w1.w * silu_fast(z1.w);
    }

    // ---- epilogue: o_j / sqrt(mean o_j^2 + eps) * w * SiLU(z_j), stored at the token's grid row
    failed |= !mbar_wait(&m.mma[1], ph1);
    ph1 ^= 1;
    tc_after_sync();
    {
      float o[16];
      tmem_ld16x2(tm + lane_base + half * 32, o);
      tmem_ld_wait(o);
      float ss = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) ss = fmaf(o[c], o[c], ss);
      ss = row_combine_sum(ss, m.red, row, half, bar_pair + qd, lane);
      if (row < ntok) {
        const float inv = rsqrtf(ss * (1.0f / kD) + kRmsEps);
        T* dst = reinterpret_cast<T*>(p.out) + m.rows[par][row] * kD + cbase;
        uint4 y8[2];
#pragma unroll
        for (int c = 0; c < 16; c += 8) {
          const uint2 lo = pack4<T>(o[c + 0] * inv * wz[c + 0], o[c + 1] * inv * wz[c + 1],
                                    o[c + 2] * inv * wz[c + 2], o[c + 3] * inv * wz[c + 3]);
          const uint2 hi = pack4<T>(o[c + 4] * inv * wz[c + 4], o[c + 5] * inv * wz[c + 5],
                                    o[c + 6] * inv * wz[c + 6], o[c + 7] * inv * wz[c + 7]);
          y8[c >> 3] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        // the row's 32 bytes: one whole sector per thread when `out` is 32-byte aligned
        if (out32) {
          st_global_v8(dst, y8[0], y8[1]);
        } else {
          reinterpret_cast<uint4*>(dst)[0] = y8[0];
          reinterpret_cast<uint4*>(dst)[1] = y8[1];
        }
      }
    }

    // ---- state, transposed: S^T <- (S^T + V^T k~) diag(e^{Gam}), or
    // S^T diag(e^{Gam}) + V^T k^ for an exact chunk
    failed |= !mbar_wait(&m.mma[2], ph2);
    ph2 ^= 1;
    tc_after_sync();
    {
      float ds[16];
      tmem_ld16x2(tm + lane_base + 64 + half * 32, ds);
      tmem_ld_wait(ds);
#pragma unroll
      for (int c = 0; c < 16; c += 4) {
        const float4 a = *reinterpret_cast<const float4*>(&m.aG[cbase + c]);
        S[c + 0] = tilde ? a.x * (S[c + 0] + ds[c + 0]) : fmaf(a.x, S[c + 0], ds[c + 0]);
        S[c + 1] = tilde ? a.y * (S[c + 1] + ds[c + 1]) : fmaf(a.y, S[c + 1], ds[c + 1]);
        S[c + 2] = tilde ? a.z * (S[c + 2] + ds[c + 2]) : fmaf(a.z, S[c + 2], ds[c + 2]);
        S[c + 3] = tilde ? a.w * (S[c + 3] + ds[c + 3]) : fmaf(a.w, S[c + 3], ds[c + 3]);
      }
    }
    cp_async_wait<0>();                   // the next chunk's copies made by this thread
    tc_before_sync();
    if (named_barrier_or(bar_all, kThreads, failed)) { failed = true; break; }
    tc_after_sync();
  }
  // after an early exit the other chain may still wait for this one's turns
  if (failed && tid == 0)
    for (int j = 0; j < 2; ++j) mbar_arrive_one(&m.built);

  cp_async_wait<0>();                     // no copy may land after the block exits
  if (ld_pending && !mbar_wait(&m.ld, phl)) failed = true;
  if (failed && tid == 0) gtr_flag(kStatusMbarTimeout);
  tc_before_sync();
  __syncthreads();                        // both chains
  tc_after_sync();
  if (threadIdx.x < 32) tmem_dealloc(m0.tmem, L::kTmemCols);
}

// ===================================================================== K2
constexpr int kLowRank = 16;                   // rank of the gate projection
constexpr int kLowTile = kC * kLowRank * 4;    // a chunk's fp32 rank-16 rows: 4 KB
struct SumMisc {
  uint64_t mma[2];                // the k^T V products of even / odd steps
  uint64_t ld[2];                 // box loads into staging buffer 0 / 1
  uint64_t umma;                  // gate: the chunk's u = low W_up product
  uint64_t wl;                    // gate: W_up tiles, column scales, bias
  uint64_t gready;                // gate: the chunk's g tile is staged (one arrival per builder warp)
  uint32_t tmem;
  int waited, fetched, issued;    // steps whose loads were consumed / issued, products issued
  alignas(16) float part[kWarps][kD];   // cumsum partials: tokens 8 w .. 8 w + 7, per dim
  alignas(16) long long rows[2][kC];    // token rows (cp.async gathers only)
  alignas(16) float ri[kC];       // gate: inverse row scales of the staged low rows
  alignas(16) float ci[kD];       // gate: inverse W_up column scales of this head
  alignas(16) float gb[kD];       // gate: bias of this head
};
template <bool kGate>
struct SumLayoutT {
  // two staging buffers of k (8 KB, row-major), v (8 KB, operand layout) and
  // the gate: g (16 KB, fp32 rows) or, with the gate in-kernel, the rank-16
  // rows low (4 KB)
  static constexpr int kOffK = 0, kOffV = kTile, kOffG = 2 * kTile;
  static constexpr int kStage = 2 * kTile + (kGate ? kLowTile : kGTile);
  // gate in-kernel: the chunk's g (fp32 rows, 16-byte units XOR-ed with
  // row % 16), single-buffered
  static constexpr int kOffGT = 2 * kStage;
  // operand tiles (1024-aligned): the two-term key tile k^ (hi, lo) of even
  // and odd steps; then, gate in-kernel, the A tile of low (fp16 hi in K
  // columns 0-15, lo in 16-31) and the two B tiles of W_up (16 x 64,
  // MN-major, 2 KB each)
  static constexpr int kTiles = kOffGT + (kGate ? kGTile : 0);
  static constexpr int kOffAU = kTiles + 4 * kTile;
  static constexpr int kOffBU = kOffAU + (kGate ? kTile : 0);
  static constexpr int kMisc = kOffBU + (kGate ? 2 * 2048 : 0);
  static constexpr int kSmem = kMisc + (int)sizeof(SumMisc) + 1024;
  // [0, 128) two accumulators, summed at the end; gate: [128, 192) u
  static constexpr int kTmemCols = kGate ? 256 : 128;
  static constexpr int kBlocksPerSM = 2;
  // eight warps build the tiles; a ninth issues the MMAs and the box loads, so
  // the builders go on to the next chunk while the tensor pipe works
  static constexpr int kThreadsAll = kThreads + 32;
  static_assert(kTiles % 1024 == 0 && kStage % 1024 == 0 && kOffAU % 1024 == 0 && kOffBU % 1024 == 0,
                "operand tiles and swizzled boxes must be 1024-byte aligned");
  static_assert(2 * (kSmem + 1024) <= 228 * 1024, "two summary CTAs must share an SM");
};
using SumLayout = SumLayoutT<false>;

// The staged low rows of a chunk (64 bytes each), gathered with cp.async;
// rows past ntok are zeroed.  `rows` are token rows (b T + t) H + h.
__device__ __forceinline__ void fetch_low(uint8_t* dst, const float* low, const long long* rows, int ntok,
                                          int H, int tid) {
  const int j = tid >> 2, part = (tid & 3) * 16;
  if (j < ntok) cp_async16(dst + j * 64 + part, (const uint8_t*)low + (rows[j] / H) * 64 + part);
  else *reinterpret_cast<uint4*>(dst + j * 64 + part) = make_uint4(0u, 0u, 0u, 0u);
}
// Byte offset of fp32 element (row, col) of a 64 x 64 tile kept as two
// SWIZZLE_128B halves (columns 0-31, 32-63; 128-byte rows, 16-byte units
// XOR-ed with row % 8): the layout a tensor-map store of 32-column boxes
// reads, and conflict-free for a row per thread and for a row per warp.
__device__ __forceinline__ uint32_t gt_off(int row, int col) {
  return (uint32_t)((col >> 5) * 8192 + row * 128 + (((((col & 31) >> 2) ^ (row & 7))) << 4) + (col & 3) * 4);
}

// kGate: the gate's second half runs here (GTR article, 方法详解 §1, the
// low-rank gate): per chunk the rank-16 rows low of its tokens become a
// scaled two-term fp16 A tile, u = low W_up comes from three MMAs (hi*hi +
// hi*lo + lo*hi, as in the gate kernel), and g = logsigmoid(u + b)/tau is
// formed from TMEM (thread = token row, 16 dims), written to g_out for the
// output stage and staged for the cumsum.  Scan positions past the sequence
// get g = 0.
template <typename T, bool kGate>
__global__ void __launch_bounds__(SumLayoutT<kGate>::kThreadsAll, SumLayoutT<kGate>::kBlocksPerSM)
gla_sum_tc(const __grid_constant__ Params p, const __grid_constant__ Maps mp) {
  using L = SumLayoutT<kGate>;
  constexpr bool kV2 = std::is_same<T, __half>::value;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // k^ (MN-major A) of step it: hi at ktile(it), lo kTile after it
  auto ktile = [&](int it) -> uint8_t* { return sm + L::kTiles + (it & 1) * 2 * kTile; };
  uint8_t* GT = sm + L::kOffGT;       // gate: the chunk's g
  uint8_t* AU = sm + L::kOffAU;       // gate: low (A)
  uint8_t* BU = sm + L::kOffBU;       // gate: W_up hi, lo (B)
  SumMisc& m = *reinterpret_cast<SumMisc*>(sm + L::kMisc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = dir_of_batch(p.dir, b);
  const int nc = (p.T + kC - 1) / kC;
  const int c0 = seg_first_chunk(seg, nc, p.nseg);
  const int nch = seg_first_chunk(seg + 1, nc, p.nseg) - c0;
  if (d < 0 || d > 3 || nch <= 0) {
    if (tid == 0) gtr_flag(d < 0 || d > 3 ? kStatusBadDir : kStatusBadShape);
    return;
  }
  const bool tma = p.tma != 0;
  const int rmask = (tma && dir_reversed(d)) ? kC - 1 : 0;   // staging row of scan offset i: i ^ rmask
  // The contraction over the chunk's tokens does not depend on their order,
  // so the key tile keeps the staging's row order and the staged v (operand
  // layout) is the B operand as it is, in its own type: an fp16 v with fp16
  // key terms, a bf16 v with bf16 ones.  Every weight e^{R + Gam - G_s} is at
  // most one, so the fp16 terms of k^ never overflow.
  // final accumulator read (and, gate, the u read): quadrant qd, column half,
  // 16 columns from cbase of row `row`
  const int qd = warp & 3, half = warp >> 2;
  const int row = qd * 16 + (lane & 15);
  const int cbase = half * 32 + (lane >> 4) * 16;
  const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
  // cumsum and tile build: dims 2 lane, 2 lane + 1 of scan offsets 8 warp .. 8 warp + 7
  const int dc = 2 * lane, tb = 8 * warp;
  // step `it` handles chunk c0 + nch - 1 - it (last to first); only the first can be ragged
  const int clast = c0 + nch - 1;
  auto stage = [&](int it) -> uint8_t* { return sm + (it & 1) * L::kStage; };
  // step it's k, v (v in the operand layout), gate rows into stage(it)
  // (the box loads of k and v may be issued apart from the gate's: `parts`
  // 1 = k, v; 2 = g or low; 3 = all; the barrier expects all three from the
  // first part)
  auto fetch = [&](int it, int parts = 3) {
    const int s0 = (clast - it) * kC;
    uint8_t* st = stage(it);
    if (tma) {
      if (tid == kThreads) {
        uint64_t* bar = &m.ld[it & 1];
        if (parts & 1) {
          mbar_arrive_tx(bar, 2 * kTile + (kGate ? kLowTile : kGTile));
          tma_box(p, mp, kMapK, st + L::kOffK, bar, d, b, h, s0);
          tma_box(p, mp, kMapV, st + L::kOffV, bar, d, b, h, s0);
        }
        if (parts & 2) {
          if (kGate) tma_box(p, mp, kMapL, st + L::kOffG, bar, d, b, 0, s0);
          else tma_box(p, mp, kMapG, st + L::kOffG, bar, d, b, h, s0);
        }
      }
    } else {
      const int ntok = min(kC, p.T - s0);
      fetch16(st + L::kOffK, p.k, m.rows[it & 1], ntok, tid);
      fetch16<true>(st + L::kOffV, p.v, m.rows[it & 1], ntok, tid);
      if (kGate) fetch_low(st + L::kOffG, p.low, m.rows[it & 1], ntok, p.H, tid);
      else fetch_g(st + L::kOffG, p.g, m.rows[it & 1], ntok, tid);
      cp_async_commit();
    }
  };

  const bool control = tid >= kThreads;   // warp 8
  if (tid == 0) {
    mbar_init(&m.mma[0], 1);
    mbar_init(&m.mma[1], 1);
    mbar_init(&m.ld[0], 1);
    mbar_init(&m.ld[1], 1);
    mbar_init(&m.umma, 1);
    mbar_init(&m.wl, 1);
    mbar_init(&m.gready, kWarps);
    mbar_fence_init();
  }
  if (!tma) {
    chunk_rows(p, m.rows[0], b, h, d, clast * kC, min(kC, p.T - clast * kC), tid);
    if (nch > 1) chunk_rows(p, m.rows[1], b, h, d, (clast - 1) * kC, kC, tid);
  }
  __syncthreads();
  // k and v are inputs: their first boxes go out before the wait; the gate
  // rows come from the previous kernel
  if (tma) {
    fetch(0, 1);
    if (nch > 1) fetch(1, 1);
  }
  pdl_wait();
  pdl_trigger();
  if (tma) {
    fetch(0, 2);
    if (nch > 1) fetch(1, 2);
  } else if (!control) {
    fetch(0);
    if (nch > 1) fetch(1);
  }
  if (kGate && tid == kThreads) {
    // this head's W_up terms (2 KB each), column scales and bias
    mbar_arrive_tx(&m.wl, 2 * 2048 + 256 + (p.gbias ? 256 : 0));
    bulk_g2s(BU, p.wu + 2048 * h, 2048, &m.wl);
    bulk_g2s(BU + 2048, p.wu + p.wu_term + 2048 * h, 2048, &m.wl);
    bulk_g2s(m.ci, p.wu_scale + kD * h, 256, &m.wl);
    if (p.gbias) bulk_g2s(m.gb, p.gbias + kD * h, 256, &m.wl);
  }
  if (kGate && !p.gbias && tid < kD) m.gb[tid] = 0.f;
  int fetched = nch > 1 ? 1 : 0, waited = -1;   // box loads issued / consumed, by step
  if (warp == 0) {
    tmem_alloc(&m.tmem, L::kTmemCols);
    tmem_relinquish();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = m.tmem;
  constexpr uint32_t kIdKV = kV2 ? idesc_f16(1, 1) : idesc_bf16(1, 1);   // both MN-major
  constexpr uint32_t kIdU = idesc_f16(0, 1);     // A K-major, B MN-major
  // gate: u = low W_up into columns [128, 192), hi*hi + hi*lo + lo*hi
  auto issue_u = [&]() {
    const uint64_t ah = desc_k(AU), bhi = desc_mn(BU), blo = desc_mn(BU + 2048);
    mma_f16(tm + 128, ah, bhi, kIdU, 0u);
    mma_f16(tm + 128, ah, blo, kIdU, 1u);
    mma_f16(tm + 128, ah + kStepK, bhi, kIdU, 1u);
    mma_commit(&m.umma);
  };

  bool failed = false;
  int issued = -1;
  if (control) {
    // ---- control warp: products of each chunk once the builders have its
    // tiles, then (box loads) the chunk after next into the buffer they read
    for (int it = 0; it < nch; ++it) {
      if (kGate) {
        // the chunk's g tile out by two tensor-map stores (not for gathered
        // loads or a reversed scan's ragged chunk: the builders store those),
        // read out of shared memory before barrier B frees the tile
        const int s0 = (clast - it) * kC;
        if (!mbar_wait(&m.gready, (uint32_t)it & 1u)) failed = true;
        if (tid == kThreads && !failed && tma && !(rmask && s0 + kC > p.T)) {
          tma_store_box(p, mp, kMapGS, GT, d, b, h, s0, 0);
          tma_store_box(p, mp, kMapGS, GT + 8192, d, b, h, s0, 32);
          bulk_commit();
          bulk_wait_read<0>();
        }
      }
      tc_before_sync();
      if (__syncthreads_or(failed)) {                 // the builders' barrier B
        failed = true;
        break;
      }
      tc_after_sync();
      uint8_t* const Vb = stage(it) + L::kOffV;
      if (tid == kThreads) {
        if (kGate && it + 1 < nch) issue_u();   // chunk it + 1's gate product (its A tile is built)
        // k^hi V into columns [0, 64), k^lo V into [64, 128)
        mma_k64<kStepMN, kStepMN>(tm, desc_mn(ktile(it)), desc_mn(Vb), kIdKV, it > 0);
        mma_k64<kStepMN, kStepMN>(tm + 64, desc_mn(ktile(it) + kTile), desc_mn(Vb), kIdKV, it > 0);
        mma_commit(&m.mma[it & 1]);
      }
      issued = it;
      if (tma && it + 2 < nch) {
        if (!mbar_wait(&m.mma[it & 1], (uint32_t)(it >> 1) & 1u)) failed = true;
        tc_after_sync();
        fetch(it + 2);
        fetched = it + 2;
      }
      __syncwarp();
    }
  } else {
    // gate: the A tile of chunk `it`'s low rows (row tid / 4, ranks 4 (tid %
    // 4) .. + 3; a power-of-two scale per row over the four threads of the
    // row).  Chunk it + 1's tile is built before barrier B of chunk it and
    // the control warp issues its product ahead of chunk it's k^T V products,
    // so u is ready when chunk it + 1 starts.
    int u_issued = 0, u_waited = 0;
    auto gate_tile = [&](int it) {
      const float* lw = reinterpret_cast<const float*>(stage(it) + L::kOffG);
      const int r = tid >> 2, k0 = (tid & 3) * 4;
      const float4 l = *reinterpret_cast<const float4*>(lw + r * kLowRank + k0);
      float mx = fmaxf(fmaxf(fabsf(l.x), fabsf(l.y)), fmaxf(fabsf(l.z), fabsf(l.w)));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const int e = scale_exp(mx);
      const float sc = pow2i(e);
      if ((tid & 3) == 0) m.ri[r] = pow2i(-e);
      uint32_t h0, h1, l0, l1;
      split2h(l.x * sc, l.y * sc, h0, l0);
      split2h(l.z * sc, l.w * sc, h1, l1);
      *reinterpret_cast<uint2*>(AU + sw16(r, k0)) = make_uint2(h0, h1);
      *reinterpret_cast<uint2*>(AU + sw16(r, kLowRank + k0)) = make_uint2(l0, l1);
      fence_async_smem();
    };
    // the loads of chunk `it` have landed (box loads: its barrier; gathers:
    // every cp.async group of this thread, then the builders' barrier)
    auto wait_loads = [&](int it) {
      if (tma) {
        failed |= !mbar_wait(&m.ld[it & 1], (uint32_t)(it >> 1) & 1u);
        waited = it > waited ? it : waited;
      } else {
        if (it == 0 && nch > 1) cp_async_wait<1>();
        else cp_async_wait<0>();
        named_barrier(1, kThreads);
      }
    };
    if (kGate) {
      failed |= !mbar_wait(&m.wl, 0);
      wait_loads(0);
      gate_tile(0);
      tc_before_sync();
      named_barrier(1, kThreads);
      if (tid == 0) {
        tc_after_sync();
        issue_u();
      }
      u_issued = 1;
    }
    // gate: chunk it's g goes out by two tensor-map stores of the staged
    // tile, except with gathered loads or where the box would start before
    // token 0 (a reversed scan's ragged chunk): then each warp stores its rows
    const bool gt_tma = tma;
    // R: summed log-gate, per dim, of the chunks already seen (the segment's tail)
    float2 R = make_float2(0.f, 0.f);
    for (int it = 0; it < nch; ++it) {
      uint8_t* st = stage(it);
      const T* kst = reinterpret_cast<const T*>(st + L::kOffK);
      const float* G = reinterpret_cast<const float*>(kGate ? GT : st + L::kOffG);
      const int s0 = (clast - it) * kC;   // first scan position of the chunk
      wait_loads(it);
      // rows of the next chunk (cp.async gathers; that buffer's gather is long done)
      if (!tma && it >= 1 && it + 1 < nch) chunk_rows(p, m.rows[(it + 1) & 1], b, h, d, (clast - it - 1) * kC, kC, tid);

      if (kGate) {
        // ---- g of this chunk from u (thread = token row `row`, dims cbase ..
        // cbase + 15), staged for the cumsum; scan positions past the
        // sequence get g = 0
        if (!mbar_wait(&m.umma, (uint32_t)u_waited & 1u)) failed = true;
        ++u_waited;
        tc_after_sync();
        float u[16];
        tmem_ld16x2(tm + lane_base + 128 + half * 32, u);
        tmem_ld_wait(u);
        const bool valid = s0 + (row ^ rmask) < p.T;
        const float ri = m.ri[row];
        const float inv_tau = p.inv_tau, ln2_tau = 0.6931471805599453f * p.inv_tau;
        float gv[16];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const float2 gg = logsigmoid_over_tau2(fmaf(u[c] * ri, m.ci[cbase + c], m.gb[cbase + c]),
                                                 fmaf(u[c + 1] * ri, m.ci[cbase + c + 1], m.gb[cbase + c + 1]),
                                                 inv_tau, ln2_tau);
          gv[c] = valid ? gg.x : 0.f;
          gv[c + 1] = valid ? gg.y : 0.f;
        }
#pragma unroll
        for (int c = 0; c < 16; c += 4)
          *reinterpret_cast<float4*>(GT + gt_off(row, cbase + c)) = make_float4(gv[c], gv[c + 1], gv[c + 2], gv[c + 3]);
        fence_async_smem();               // the tile, then the tensor-map stores' reads
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&m.gready);   // the control warp stores it
        tc_before_sync();
        named_barrier(1, kThreads);
      }

      // ---- in-chunk cumsum G (eight scan offsets in registers), the partial
      // sums of the other warps, and the chunk total Gam
      float2 gc[8];
      // gate: each warp writes g of its eight scan positions to g_out, one
      // whole 256-byte row per position (box loads: consecutive positions of
      // a chunk are `gstep` grid indices apart)
      const bool gst = kGate && !(gt_tma && !(rmask && s0 + kC > p.T));   // this chunk's g by the warps
      long long grow = 0, gstep = 0;
      if (gst && tma) {
        grow = (long long)b * p.T + scan_to_grid(d, min(s0 + tb, p.T - 1), p.T, p.gh, p.gw);
        gstep = d == kLR ? 1 : d == kRL ? -1 : d == kTB ? p.gw : -p.gw;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rg = (tb + i) ^ rmask;
        gc[i] = kGate ? *reinterpret_cast<const float2*>(GT + gt_off(rg, dc))
                      : *reinterpret_cast<const float2*>(G + rg * kD + dc);
        if (gst && s0 + tb + i < p.T) {
          const long long tr = tma ? (grow + gstep * i) * p.H + h : m.rows[it & 1][tb + i];
          *reinterpret_cast<float2*>(p.g_out + tr * kD + dc) = gc[i];
        }
        if (i) { gc[i].x += gc[i - 1].x; gc[i].y += gc[i - 1].y; }
      }
      *reinterpret_cast<float2*>(&m.part[warp][dc]) = gc[7];
      named_barrier(1, kThreads);
      float2 off = make_float2(0.f, 0.f), tot = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float2 pp = *reinterpret_cast<const float2*>(&m.part[w][dc]);
        if (w < warp) { off.x += pp.x; off.y += pp.y; }
        tot.x += pp.x; tot.y += pp.y;
      }
      // weights e^{R + Gam - G_s}: the decay from token s to the segment end
      const float2 base = make_float2(R.x + tot.x - off.x, R.y + tot.y - off.y);
      R.x += tot.x; R.y += tot.y;
      uint32_t kr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        kr[i] = *reinterpret_cast<const uint32_t*>(kst + ((tb + i) ^ rmask) * kD + dc);
      if (it >= 2) {                      // step it - 2's products have read this key tile
        failed |= !mbar_wait(&m.mma[it & 1], (uint32_t)((it - 2) >> 1) & 1u);
      }
      tc_after_sync();
      if (!tma && it >= 1 && it + 1 < nch) {   // into the buffer step it - 1's products read
        failed |= !mbar_wait(&m.mma[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u);
        fetch(it + 1);
      }

      // ---- key tile k^ = k * weight (two terms), rows in the staging's order
      uint8_t* const KH = ktile(it);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t o = sw16((tb + i) ^ rmask, dc);
        const float2 kk = ld2(reinterpret_cast<const T*>(&kr[i]));
        const float wa = ex2((base.x - gc[i].x) * kLog2e), wb = ex2((base.y - gc[i].y) * kLog2e);
        if (kV2) put2h(KH, KH + kTile, o, kk.x * wa, kk.y * wb);
        else put2x(KH, KH + kTile, o, kk.x * wa, kk.y * wb);
      }
      if (kGate && it + 1 < nch) {        // the next chunk's gate tile
        wait_loads(it + 1);
        gate_tile(it + 1);
      }
      fence_async_smem();
      tc_before_sync();
      if (__syncthreads_or(failed)) {                 // barrier B: the control warp issues
        failed = true;
        break;
      }
      tc_after_sync();
      if (kGate && it + 1 < nch) ++u_issued;
    }
    if (warp == 0)
      *reinterpret_cast<float2*>(&m.part[0][dc]) = R;  // the segment's summed log-gate
    // a gate product not waited for (early exit) completes before tensor
    // memory is released
    if (kGate && tid == 0 && u_issued > u_waited) (void)mbar_wait(&m.umma, (uint32_t)(u_issued - 1) & 1u);

  }
  // Drain: the last issued products, then box loads issued but not consumed
  // (only after an early exit), before TMEM and shared memory are released.
  if (tid == kThreads) {
    m.issued = issued;
    m.fetched = fetched;
  }
  if (tid == 0) m.waited = waited;
  failed = __syncthreads_or(failed) != 0;
  const int last = m.issued;
  if (last >= 0 && !mbar_wait(&m.mma[last & 1], (uint32_t)(last >> 1) & 1u)) failed = true;
  tc_after_sync();
  cp_async_wait<0>();
  if (tma && tid == 0)
    for (int x = m.waited + 1; x <= m.fetched; ++x)
      if (!mbar_wait(&m.ld[x & 1], (uint32_t)(x >> 1) & 1u)) failed = true;
  if (kGate && tid == kThreads) {
    (void)mbar_wait(&m.wl, 0);                    // the weight copies have landed
    bulk_wait<0>();                               // every g store is complete
  }
  failed = __syncthreads_or(failed) != 0;
  if (!failed && !control) {
    float ds[16], dl[16];
    tmem_ld16x2(tm + lane_base + half * 32, ds);
    tmem_ld16x2(tm + lane_base + 64 + half * 32, dl);
    tmem_ld_wait(ds);
    tmem_ld_wait(dl);
#pragma unroll
    for (int c = 0; c < 16; ++c) ds[c] += dl[c];
    float* dst = p.wsS + (((size_t)bh * p.nseg + seg) * kD + row) * kD + cbase;
    uint4 w4[4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
      w4[c] = make_uint4(__float_as_uint(ds[4 * c]), __float_as_uint(ds[4 * c + 1]), __float_as_uint(ds[4 * c + 2]),
                         __float_as_uint(ds[4 * c + 3]));
    if (((uintptr_t)p.wsS & 31) == 0) {           // whole 32-byte sectors (the row's 64 bytes)
      st_global_v8(dst, w4[0], w4[1]);
      st_global_v8(dst + 8, w4[2], w4[3]);
    } else {                                      // a caller's states buffer: 16-byte alignment only
#pragma unroll
      for (int c = 0; c < 4; ++c) reinterpret_cast<uint4*>(dst)[c] = w4[c];
    }
    if (warp == 0) {
      const float2 R = *reinterpret_cast<const float2*>(&m.part[0][dc]);
      *reinterpret_cast<float2*>(p.wsA + ((size_t)bh * p.nseg + seg) * kD + dc) = make_float2(expf(R.x), expf(R.y));
    }
  } else if (failed && tid == 0) {
    gtr_flag(kStatusMbarTimeout);
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
// segments resident per SM (the output kernel's chains; the summary kernel's blocks)
inline int tc_blocks_per_sm(int, int) { return tc::OutLayout::kChainsPerSM; }

template <typename K, typename... Args>
inline int launch_tc_kernel(K kern, int smem, int threads, int nseg, int BH, cudaStream_t st, bool* done,
                            int dev, const Args&... args) {
  if (!done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return -5;
    done[dev] = true;
  }
  return launch_pdl(kern, dim3(nseg, BH), dim3(threads), smem, st, args...);
}

// stage 0: segment summaries (K2); stage 1: segment outputs (K4)
template <typename T>
inline int launch_tc_typed(int stage, const tc::Params& p, const tc::Maps& mp, int BH, cudaStream_t st,
                           int dev) {
  static bool done_sum[64], done_out[64], done_gsum[64];
  if (stage == 0)
    return launch_tc_kernel(tc::gla_sum_tc<T, false>, tc::SumLayout::kSmem, tc::SumLayout::kThreadsAll, p.nseg,
                            BH, st, done_sum, dev, p, mp);
  if (stage == 2)   // summary with the gate's second half in-kernel
    return launch_tc_kernel(tc::gla_sum_tc<T, true>, tc::SumLayoutT<true>::kSmem,
                            tc::SumLayoutT<true>::kThreadsAll, p.nseg, BH, st, done_gsum, dev, p, mp);
  return launch_tc_kernel(tc::gla_out_tc<T>, tc::OutLayout::kSmem, tc::OutLayout::kThreadsAll, (p.nseg + 1) / 2,
                          BH, st, done_out, dev, p, mp);
}

// `maps`: tensor maps of q, k, v, g for the output stage's box loads, or
// null (the chunks are then gathered with cp.async).
inline int launch_tc(int dtype, int stage, const void* q, const void* k, const void* v,
                     const float* g, const void* z, const float* w, void* out, float* wsS,
                     float* wsA, int B, int H, int T, int gh, int gw, int dk, int dv, int dir,
                     int chunk, int nseg, const tc::Maps* maps, cudaStream_t st) {
  if (!tc_shape_supported(dk, dv, chunk, dtype)) return -2;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -5;
  const tc::Params p{q, k, v, g, z, w, wsS, wsA, out, H, T, gh, gw, dir, nseg, maps ? 1 : 0};
  static const tc::Maps kNoMaps{};
  const tc::Maps& mp = maps ? *maps : kNoMaps;
  const int BH = B * H;
  return dtype == kF16 ? launch_tc_typed<__half>(stage, p, mp, BH, st, dev)
                       : launch_tc_typed<__nv_bfloat16>(stage, p, mp, BH, st, dev);
}

// The summary stage with the gate's second half in-kernel (stage 2 of
// launch_tc_typed): low [B, T, 16] fp32, the packed W_up terms (`wu`,
// `wu_term` bytes apart), their inverse column scales, bias (or null), 1/tau;
// writes g_out [B, T, H, 64] fp32 and the segment states.  `maps` must hold
// the k, v and low maps when not null.
inline int launch_tc_gated_sum(int dtype, const void* k, const void* v, const float* low, const uint8_t* wu,
                               int wu_term, const float* wu_scale, const float* gbias, float inv_tau,
                               float* g_out, float* wsS, float* wsA, int B, int H, int T, int gh, int gw,
                               int dir, int nseg, const tc::Maps* maps, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -5;
  tc::Params p{nullptr, k, v, nullptr, nullptr, nullptr, wsS, wsA, nullptr, H, T, gh, gw, dir, nseg,
               maps ? 1 : 0};
  p.low = low;
  p.wu = wu;
  p.wu_scale = wu_scale;
  p.gbias = gbias;
  p.g_out = g_out;
  p.wu_term = wu_term;
  p.inv_tau = inv_tau;
  static const tc::Maps kNoMaps{};
  const tc::Maps& mp = maps ? *maps : kNoMaps;
  const int BH = B * H;
  return dtype == kF16 ? launch_tc_typed<__half>(2, p, mp, BH, st, dev)
                       : launch_tc_typed<__nv_bfloat16>(2, p, mp, BH, st, dev);
}

}  // namespace gtr

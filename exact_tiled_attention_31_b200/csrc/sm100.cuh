// sm100.cuh - thin inline-PTX layer for Blackwell (sm_100a): mbarriers with
// bounded waits, TMA tile loads, Tensor Memory allocation, tcgen05 MMA issue,
// commit, and TMEM <-> register moves.  Every helper is one or two PTX
// instructions; the kernels decide all scheduling.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fa {

// ---------------------------------------------------------------------------
// Device error word.  A wait that gives up, or a check that fails, records
// why and where; the host reads it with fa_check_device_error().
// DEV_ERR_ARG: calls that had to agree did not (see bwd_post).
// ---------------------------------------------------------------------------
enum : uint32_t { DEV_ERR_NONE = 0, DEV_ERR_TIMEOUT = 1, DEV_ERR_ARG = 2 };

// Defined here: each shared library is built from a single translation unit.
__device__ uint32_t g_dev_error = 0;   // first error code (0 = none)
__device__ uint32_t g_dev_where = 0;   // site id of the first error

// Upper bound on any single barrier wait.  Every wait in a healthy launch
// lasts microseconds; this bound only turns a logic error into a clean exit.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(uint32_t code, uint32_t where) {
  if (atomicCAS(&g_dev_error, 0u, code) == 0u) atomicExch(&g_dev_where, where);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Returns false
// (after recording DEV_ERR_TIMEOUT at `where`) if it takes longer than
// kWaitLimitNs, so no wait in this library is unbounded.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t where) {
  const uint32_t a = smem_addr(bar);
  if (mbar_test(a, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_test(a, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      record_error(DEV_ERR_TIMEOUT, where);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (no cluster multicast anywhere in this library)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load into shared memory, completion counted in bytes on `bar`.
// c0 (the innermost coordinate) is always a multiple of 64 elements here.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// Generic-proxy writes to shared memory made visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Tensor Memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05.mma (kind::f16: bf16 or fp16 operands, fp32 accumulate)
// ---------------------------------------------------------------------------
// Instruction descriptor: D format f32 (bits 4-5 = 1), A/B format (bits 7-9,
// 10-12: 0 = f16, 1 = bf16), A/B major (bits 15/16: 0 = K-major, 1 = MN-major),
// N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool bf16, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand: start
// address (bits 0-13, >> 4), leading byte offset (16-29, >> 4), stride byte
// offset (32-45, >> 4), descriptor version 1 (bits 46-47), base offset 0,
// layout type 2 = SWIZZLE_128B (bits 61-63).
//  K-major:  rows of 128 B (64 16-bit elements of K), 8-row atoms; SBO = 1024
//            (next 8 rows), LBO unused.  K advances inside the 128-B row by
//            moving the start address 32 B per 16 elements.
//  MN-major: rows of 128 B hold 64 consecutive M/N elements for one k;
//            SBO = 1024 (next 8 k), LBO = byte distance to the next 64 M/N.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Descriptor of a K-major operand whose rows are 32 bytes (16 16-bit values,
// one K step) in the 32-byte swizzle: 8-row groups 256 bytes apart.
__device__ __forceinline__ uint64_t make_sdesc_sw32(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(256 >> 4) << 32) | (1ull << 46) |
         (6ull << 61);
}

// D(tmem) = A(smem) * B(smem) (+ D if accumulate)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) = A(tmem) * B(smem) (+ D if accumulate); A is K-major in TMEM:
// lane = row, two 16-bit elements per 32-bit column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---- issue from a converged warp: every lane runs the same straight-line
// code with the same (warp-uniform) operands and one elected lane executes
// the instruction.  Keeping the issuing loop converged and branch-free
// between products lets the tensor core run back to back.
__device__ __forceinline__ uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred;
}

__device__ __forceinline__ void mma_ss_e(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate, uint32_t elected) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(elected)
      : "memory");
}

__device__ __forceinline__ void mma_ts_e(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate, uint32_t elected) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(elected)
      : "memory");
}

__device__ __forceinline__ void mma_commit_e(uint64_t* bar, uint32_t elected) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_addr(bar)),
      "r"(elected)
      : "memory");
}

// Descriptor of the same operand moved by `bytes` (a multiple of 16) inside
// its buffer: only the 14-bit start-address field changes, and buffers here
// are below 256 KB so it never carries.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

// ---------------------------------------------------------------------------
// TMEM <-> registers, 32x32b shape: thread t of the warp moves lane
// (32 * (warp % 4) + t); xN moves N consecutive 32-bit columns.
// ---------------------------------------------------------------------------
#define FA_R8(b) "=r"(r[b + 0]), "=r"(r[b + 1]), "=r"(r[b + 2]), "=r"(r[b + 3]), "=r"(r[b + 4]), \
                 "=r"(r[b + 5]), "=r"(r[b + 6]), "=r"(r[b + 7])
#define FA_W8(b) "r"(r[b + 0]), "r"(r[b + 1]), "r"(r[b + 2]), "r"(r[b + 3]), "r"(r[b + 4]), \
                 "r"(r[b + 5]), "r"(r[b + 6]), "r"(r[b + 7])
#define FA_M8(b) "+r"(r[b + 0]), "+r"(r[b + 1]), "+r"(r[b + 2]), "+r"(r[b + 3]), "+r"(r[b + 4]), \
                 "+r"(r[b + 5]), "+r"(r[b + 6]), "+r"(r[b + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FA_R8(0), FA_R8(8), FA_R8(16), FA_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : FA_R8(0), FA_R8(8)
      : "r"(taddr));
}

// Wait for this thread's outstanding tcgen05.ld; the registers are tied to
// the wait so the compiler cannot read them before it.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_M8(0), FA_M8(8), FA_M8(16), FA_M8(24)::"memory");
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_M8(0), FA_M8(8)::"memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FA_W8(0), FA_W8(8), FA_W8(16), FA_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      FA_W8(0), FA_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#undef FA_R8
#undef FA_W8
#undef FA_M8

// ---------------------------------------------------------------------------
// Scalar helpers
// ---------------------------------------------------------------------------
// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 arithmetic (sm_100 f32x2 instructions): a 64-bit register
// holds {lo, hi}.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// A packed 16-bit pair widened exactly to a paired fp32 value.
template <bool BF16>
__device__ __forceinline__ uint64_t widen2(uint32_t v) {
  if constexpr (BF16) {
    return f2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    const float2 f = __half22float2(h);
    return f2(f.x, f.y);
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 values rounded to nearest into one packed 16-bit pair: `lo` in
// bits 0-15 (the lower column / element index), `hi` in bits 16-31.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  if constexpr (BF16) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  }
  return r;
}

// Add the two 16-bit values of a packed pair, widened exactly to fp32, to
// two running sums.
template <bool BF16>
__device__ __forceinline__ void accum2(uint32_t v, float& s0, float& s1) {
  if constexpr (BF16) {
    s0 += __uint_as_float(v << 16);
    s1 += __uint_as_float(v & 0xffff0000u);
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    const float2 f = __half22float2(h);
    s0 += f.x;
    s1 += f.y;
  }
}

template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t v) {
  if constexpr (BF16) {
    // bf16 -> fp32 is exact: the 16 bits become the top of the fp32 word
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    return __half22float2(h);
  }
}

__device__ __forceinline__ uint32_t lane_id() {
  uint32_t l;
  asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
  return l;
}

// Per-warpgroup register budget (all four warps of a warpgroup execute the
// same call).  `inc` may only raise and `dec` only lower the count the warps
// hold (the launch's per-thread count at first), and the new counts summed
// over the block must stay within the registers the block was launched with.
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers:
// as easy as 1, 2, 3", SC 2011): ten rounds, each multiplying counter words
// 0 and 2 by the round constants and mixing the products' high halves with
// words 1 and 3 and the round key; the key advances by the Weyl increments
// between rounds.  Counter-based, so the dropout mask of any (head, query,
// key) can be regenerated anywhere from its indices.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    // one 32 x 32 -> 64-bit product per multiplier gives both halves
    uint64_t p0, p1;
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(p0) : "r"(c.x), "r"(0xD2511F53u));
    asm("mul.wide.u32 %0, %1, %2;" : "=l"(p1) : "r"(c.z), "r"(0xCD9E8D57u));
    c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ k0, (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ k1, (uint32_t)p0);
  }
  return c;
}

// Four byte-wise keep decisions at once: the top bit of byte n of the result
// is set when byte n of u is below t (1 <= t <= 255); the other bits carry
// nothing.  t4 = t * 0x01010101, t4lo = t4 & 0x7f7f7f7f.  Per byte,
// (u | 0x80) - (t & 0x7f) cannot borrow from the next byte, and its top bit
// is set exactly when the low seven bits of u are at least those of t; so
// u < t when u's top bit is clear and t's set, or the top bits agree and that
// difference's top bit is clear.
__device__ __forceinline__ uint32_t bytes_below(uint32_t u, uint32_t t4, uint32_t t4lo) {
  const uint32_t x = (u | 0x80808080u) - t4lo;
  return (~u & t4) | (~(u ^ t4) & ~x);
}
// The byte decisions of bytes_below packed for pairs: byte 0's at bit 0,
// byte 2's at bit 1, byte 1's at bit 8 and byte 3's at bit 9.
__device__ __forceinline__ uint32_t pair_bits(uint32_t w) {
  const uint32_t y = (w & 0x80808080u) >> 7;
  return (y | (y >> 15)) & 0x0303u;
}
// Bit of pair slot i (0..15) of a pair-packed word: the first element of
// pair i at bit pair_slot(i), the second at pair_slot(i) + 8.
__device__ __forceinline__ constexpr int pair_slot(int i) { return (i & 7) + 16 * (i >> 3); }
// Halfword keep masks of pair slot i of a pair-packed word x: the low
// halfword is 0xFFFF when the first element is kept, the high one when the
// second is (prmt with sign replication from bits 7 and 15).  i is a
// compile-time constant at every call (unrolled loops), so the shift folds.
__device__ __forceinline__ uint32_t pair_keep_halves(uint32_t x, int i) {
  const int b = pair_slot(i);
  const uint32_t y = b <= 7 ? x << (7 - b) : x >> (b - 7);
  uint32_t m;
  asm("prmt.b32 %0, %1, %1, 0x9988;" : "=r"(m) : "r"(y));
  return m;
}

// Dropout parameters shared by the forward and backward kernels.  Element
// (head bh, query i, key j) is kept when byte (j & 3) of word
// 2 (i & 1) + ((j >> 2) & 1) of Philox4x32-10 at counter (j >> 3, i >> 1,
// bh, offset), key (seed_lo, seed_hi), is below `thresh` =
// max(1, floor((1 - p) 2^8)); kept values are scaled by `scale` =
// 2^8 / thresh, the inverse of the exact keep probability.
struct Dropout {
  uint32_t thresh, seed_lo, seed_hi, offset;
  float scale;
};

// 128-byte swizzle of a byte offset inside a 1024-byte-aligned block of 8
// rows x 128 B: the 16-byte chunk index is XORed with the row index (the
// layout TMA writes for CU_TENSOR_MAP_SWIZZLE_128B).
__device__ __forceinline__ uint32_t swz128(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }
// 32-byte swizzle: 16-byte chunk index (bit 4) XOR bit 7.
__device__ __forceinline__ uint32_t swz32(uint32_t off) { return off ^ (((off >> 7) & 1u) << 4); }
// x rounded to the nearest bf16 value, returned as fp32.
__device__ __forceinline__ float bf16_round(float x) {
  uint16_t h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
  return __uint_as_float((uint32_t)h << 16);
}

}  // namespace fa

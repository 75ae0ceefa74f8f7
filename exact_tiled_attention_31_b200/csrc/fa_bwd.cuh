// fa_bwd.cuh - backward kernels of exact tiled attention on sm_100a.
//
// The pages only say that the training backward keeps a few statistics from
// the forward and recomputes the local attention blocks instead of storing
// P ("Flash Attention 的算法设计原理", "核心机制", third item; "ops-transformer里的
// FlashAttention", "意外收获" notes that the backward exists and is harder).
// The gradients of L = sum(dO * O) are the textbook ones:
//     P_ij  = exp(s_ij - LSE_i)                (rebuilt from the saved LSE)
//     dV_j  = sum_i P_ij dO_i
//     dP_ij = dO_i . v_j,   D_i = dO_i . O_i
//     dS_ij = P_ij (dP_ij - D_i)
//     dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
//
// Three launches on the caller's stream:
//   bwd_pre   D_i = dO_i . O_i (fp32, warp-shuffle reduction); per query row a
//             16-column bf16 row holding -LSE_i*log2(e) and -D_i, each split
//             into three bf16 parts (128-row padded); zero the fp32 dQ
//             accumulator and the ordering counters.
//   bwd_main  a persistent grid (at most one CTA per SM, 512 threads): each
//             CTA claims work units (key/value tile j of one head, and of one
//             sequence in a packed batch) one after another from a counter
//             in the workspace, in increasing unit order, and broadcasts each
//             claim to its roles through a two-slot ring in shared memory:
//               warp 0     TMA producer: claims the next unit, then K_j, V_j
//                          (once the previous unit's products are done with
//                          the old ones), Q_i (+ the per-query rows of tile i)
//                          into a 2-slot ring and dO_i into its own slot.
//               warp 1     tcgen05 issuer and TMEM owner.  Two 128-column
//                          regions swap roles every step g: X(g) takes S^T(g),
//                          which the P warps turn into P^T (16-bit, columns
//                          [64h, 64h + 32) for query half h) and then dS^T
//                          (columns [64h + 32, 64h + 64)); Y(g) takes dP^T(g).
//                          Per step:
//                            dV  += P^T dO_i               (A = P^T in X)
//                            S^T(g+1) = K_j Q_{i+1}^T -> Y (as soon as the dS
//                                       warps have read dP^T(g) out of Y), plus
//                                       one K step that adds -LSE / scale
//                            dK  += dS^T Q_i               (A = dS^T in X)
//                            dQ_i = dS K_j -> X            (A = dS in smem)
//                            dP^T(g+1) = V_j dO_{i+1}^T -> X (after dQ_i has
//                                       been drained), plus one K step that
//                                       adds -D
//                          so the next step's exponentials start while dK,
//                          dQ and the next dP^T are on the tensor core.
//                          dV [256,256+D), dK [256+D,256+2D).
//               warp 2     deterministic mode only: adds the dQ warps'
//                          counts to the ordering counters (one gpu-scope
//                          release per step, off the dQ warps' path).
//               warps 4-11 one thread per key row and half of the query
//                          columns (warps 4-7 queries 0-63, 8-11 queries
//                          64-127).  P phase: P^T = exp2(S'^T*scale*log2e)
//                          (S' already holds -LSE/scale), kept as 16-bit
//                          pairs in registers and written to X.  dS phase:
//                          read dP'^T (it already holds -D) out of Y, then
//                          dS^T = P^T dP'^T to X and, as the MN-major A
//                          operand of dQ = dS K, to shared memory.  After a
//                          unit's last step: its dV and scale*dK rows to global
//                          memory.
//               warps 12-15 one thread per query row: move dQ_i from TMEM to
//                          a per-warp 128-byte-swizzled staging buffer and add
//                          it to the fp32 accumulator with TMA bulk reductions
//                          (cp.reduce.async.bulk.tensor .add); under
//                          deterministic mode even and odd key tiles add into
//                          two accumulators, and in each the key tiles take
//                          turns for tile i, from the highest j down (the
//                          order in which they reach tile i); the units are
//                          numbered so that every key tile is claimed after
//                          the one whose turn precedes it: that one is always
//                          held by a running CTA, whatever order the hardware
//                          starts CTAs in.
//   bwd_post  dQ = scale * accumulator (+ the second one after a deterministic
//             bwd_main), rounded to the input dtype.
// Causal: key tile j only meets query tiles i >= j; only the diagonal tile
// is masked element-wise.  Packed batches ([H, T, D], cu_seqlens): every
// sequence is its own problem with tiles counted from its first token; keys
// past its end get P = 0 and query rows past its end carry a -1e30 score
// offset (so P = 0) and D = 0, so their dS rows are exactly 0 and nothing leaks into the next
// sequence's rows (the fp32 reductions of those zero rows add 0).
#pragma once

#include "sm100.cuh"

// Timeline hooks: BWD_TRACE(condition, slot) records a clock at a point of
// the pipeline in builds that define it; it compiles to nothing otherwise.
#ifndef BWD_TRACE
#define BWD_TRACE(cond, slot) ((void)sizeof((cond) ? 1 : 0))
#endif

namespace fa {

struct BwdParams {
  void* dk;                // [heads, rows, D]
  void* dv;                // [heads, rows, D]
  float* dq_acc;           // [2, heads, rows, D] fp32: the accumulator, then the second one of
                           //   deterministic mode (odd key tiles)
  uint16_t* cols;          // [heads, nseq, S_pad, 16] bf16 per-query rows (written by bwd_pre):
                           //   0-8: -LSE*log2(e) in three parts (part k % 3 in column k),
                           //   9-11: -D_i in three parts, 12-15: 0; padding rows -1e30 and 0
  uint32_t* sem;           // [heads, nseq, n_q, 2] ordering counters (deterministic mode, per chain)
  uint32_t* ticket;        // next unit to claim (zeroed by bwd_pre); ticket[1]: nonzero once a
                           //   deterministic bwd_main has filled the second accumulator
  const int* cu_seqlens;   // packed batch only: device int32 [nseq + 1]
  int heads;               // dense: B*H, packed: H
  int S;                   // dense: S, packed: max_seqlen
  int rows;                // rows of one head slice in memory: S or total
  int nseq;                // dense: 1
  int S_pad, n_q;          // ceil(S / 128) * 128, ceil(S / 128)
  int units;               // unit numbers: groups of kBwdGroup slices x n_q key tiles (some empty)
  float scale, scale_log2;
  int deterministic;
  Dropout drop;            // DROPOUT instances only
};

template <int D>
struct BwdCfg {
  static constexpr int CH = D / 64;
  static constexpr uint32_t CHUNK = 128u * 128u;                // 128 rows x 128 bytes
  static constexpr uint32_t TILE = CH * CHUNK;                   // one 128 x D 16-bit tile
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = TILE;
  static constexpr uint32_t Q_OFF = 2 * TILE;                    // 2 slots
  static constexpr uint32_t DO_OFF = 4 * TILE;                   // 1 slot
  static constexpr uint32_t DS_OFF = 5 * TILE;                   // 128 x 128 16-bit, 2 chunks
  static constexpr uint32_t STG_OFF = DS_OFF + 2 * CHUNK;        // 4 warps x (32 rows x 128 B) fp32 staging
  static constexpr uint32_t CT_OFF = STG_OFF + 4 * 4096;         // 2 slots x per-query rows (128 x 32 B)
  static constexpr uint32_t ONES_OFF = CT_OFF + 2 * 4096;         // the two constant key-side rows (128 x 32 B)
  static constexpr uint32_t BAR_OFF = ONES_OFF + 2 * 4096;
  // kv_full kv_empty q_full[2] q_empty[2] do_full do_empty s_full dp_full
  // p_full dp_taken ds_full dq_full dq_empty dkv_full drain (one unused)
  // unit_full[2] unit_empty[2] rel_full[2] rel_empty[2]
  static constexpr int NBAR = 26;
  // then the TMEM address, the two-slot unit ring, and the two-slot ring of
  // counters the release warp adds to
  static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 32 + 1024;
  static constexpr uint32_t TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
};

// (sequence, head) slices per group of the backward's block order
constexpr int kBwdGroup = 4;

enum : uint32_t {
  BWD_SITE_PROD = 0x200, BWD_SITE_KV = 0x201, BWD_SITE_Q = 0x202, BWD_SITE_DO = 0x203, BWD_SITE_P = 0x204,
  BWD_SITE_DS = 0x205, BWD_SITE_DQE = 0x206, BWD_SITE_S = 0x207, BWD_SITE_DP = 0x208, BWD_SITE_DQF = 0x209,
  BWD_SITE_DKV = 0x20a, BWD_SITE_SEM = 0x20b, BWD_SITE_DRAIN = 0x20c, BWD_SITE_STAT = 0x20d, BWD_SITE_UNIT = 0x20e,
  BWD_SITE_TAKEN = 0x20f, BWD_SITE_POST = 0x210, BWD_SITE_REL = 0x211
};

// One work unit: key/value tile j of one (sequence, head) slice, which meets
// query tiles i_begin .. n_q - 1 of its sequence.
struct BwdUnit {
  int j, seq, head, row_base, seq_len, n_q, i_begin, n_steps;
};

// Unit u as its key tile and slice.  Unit numbers walk the (sequence, head)
// slices in groups of kBwdGroup and, inside a group, ascending j (longest
// causal work first), so only a few slices are live at a time and their fp32
// dQ accumulators and Q/K/V/dO tiles stay in L2, where the dQ reductions run
// about twice as fast as against device memory.  False for a number past the
// end of a shorter last group or of its sequence; those are skipped.
template <bool CAUSAL, bool VARLEN>
__device__ __forceinline__ bool bwd_decode(const BwdParams& p, int u, BwdUnit& x) {
  const int slices = p.nseq * p.heads;
  const int group = u / (kBwdGroup * p.n_q);
  const int rg = u - group * (kBwdGroup * p.n_q);
  const int gsize = min(kBwdGroup, slices - group * kBwdGroup);
  const int jr = rg / gsize;
  if (jr >= p.n_q) return false;
  // deterministic mode takes a slice's key tiles from the last one down: its
  // query tiles receive their dQ parts in that order, which is the order in
  // which the key tiles reach them
  x.j = p.deterministic ? p.n_q - 1 - jr : jr;
  const int slice = group * kBwdGroup + (rg - jr * gsize);
  x.seq = slice / p.heads;
  x.head = slice - x.seq * p.heads;
  x.row_base = 0;
  x.seq_len = p.S;
  if constexpr (VARLEN) {
    x.row_base = p.cu_seqlens[x.seq];
    x.seq_len = p.cu_seqlens[x.seq + 1] - x.row_base;
  }
  if (128 * x.j >= x.seq_len) return false;
  x.n_q = (x.seq_len + 127) / 128;
  x.i_begin = CAUSAL ? x.j : 0;
  x.n_steps = x.n_q - x.i_begin;
  return true;
}

// ---------------------------------------------------------------------------
// bwd_pre: one group of D/8 lanes per row, 16-byte loads, shuffle reduction.
// blockIdx.y walks the (head, sequence) slices and blockIdx.x the rows of a
// slice, so a row's indices need no division by a runtime size.
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool VARLEN>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      const float* __restrict__ lse, BwdParams p) {
  constexpr int G = D / 8;  // lanes per row (divides 32)
  const int slices = p.heads * p.nseq;
  const int work = p.S_pad * G;
  const int bound = (work + 31) / 32 * 32;  // whole warps take the same trips
  for (int slice = blockIdx.y; slice < slices; slice += gridDim.y) {
    const int h = slice / p.nseq, seq = slice - h * p.nseq;
    int base = 0, len = p.S;
    if constexpr (VARLEN) {
      base = p.cu_seqlens[seq];
      len = p.cu_seqlens[seq + 1] - base;
    }
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < bound; idx += gridDim.x * blockDim.x) {
      const bool in = idx < work;
      const int s = in ? idx / G : len;  // padded row of the slice
      const int part = idx % G;
      const bool valid = s < len;
      const size_t tok = (size_t)h * p.rows + base + s;  // token row in memory (valid rows only)
      float acc = 0.f;
      if (valid) {
        const size_t off = tok * D + part * 8;
        const uint4 a = *reinterpret_cast<const uint4*>(o + off);
        const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 x = unpack2<BF16>(av[i]), y = unpack2<BF16>(bv[i]);
          acc = fmaf(x.x, y.x, acc);
          acc = fmaf(x.y, y.y, acc);
        }
      }
      // the G lanes of one row are consecutive lanes of one warp
#pragma unroll
      for (int w = G / 2; w > 0; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w);
      if (in && part == 0) {
        // per-query row of the extra K step: the tensor core adds
        // (1/(scale log2 e)) * (-LSE log2 e) to S^T and -D to dP^T
        const float nl = valid ? lse[tok] * -1.4426950408889634f : -1e30f;
        const float nd = valid ? -acc : 0.f;
        float a[3], b[3];
        a[0] = bf16_round(nl);
        a[1] = valid ? bf16_round(nl - a[0]) : 0.f;
        a[2] = valid ? bf16_round(nl - a[0] - a[1]) : 0.f;
        b[0] = bf16_round(nd);
        b[1] = bf16_round(nd - b[0]);
        b[2] = bf16_round(nd - b[0] - b[1]);
        float v[16];
#pragma unroll
        for (int k = 0; k < 9; ++k) v[k] = a[k % 3];
#pragma unroll
        for (int k = 0; k < 3; ++k) v[9 + k] = b[k];
#pragma unroll
        for (int k = 12; k < 16; ++k) v[k] = 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.cols + ((size_t)slice * p.S_pad + s) * 16);
        dst[0] = make_uint4(pack2<true>(v[0], v[1]), pack2<true>(v[2], v[3]), pack2<true>(v[4], v[5]),
                            pack2<true>(v[6], v[7]));
        dst[1] = make_uint4(pack2<true>(v[8], v[9]), pack2<true>(v[10], v[11]), pack2<true>(v[12], v[13]),
                            pack2<true>(v[14], v[15]));
      }
    }
  }
  // zero the dQ accumulator (16-byte stores) and the ordering counters
  const long long nthreads = (long long)gridDim.x * gridDim.y * blockDim.x;
  const long long gtid = ((long long)blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
  const long long n4 = (long long)p.heads * p.rows * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long i = gtid; i < n4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long ns = (long long)p.heads * p.nseq * p.n_q * 2;
  for (long long i = gtid; i < ns; i += nthreads) p.sem[i] = 0u;
  if (gtid == 0) {
    p.ticket[0] = 0u;
    p.ticket[1] = 0u;
  }
}

// ---------------------------------------------------------------------------
// bwd_post: dQ = scale * accumulator, rounded to nearest in the input dtype.
// TWO (deterministic bwd_main): the odd key tiles' sums sit in a second
// accumulator n8 * 8 floats further on, added to the first in this order.
// Separate instances, each held to the 32 registers that let the launch's 8
// CTAs per SM all be resident at once.
// bwd_main left its own word in *det (nonzero: deterministic); one thread
// compares it with TWO, with the load issued before the loop so that it
// costs no time, and records DEV_ERR_ARG when they disagree (the result then
// misses the odd key tiles, or adds a stale second accumulator).
// ---------------------------------------------------------------------------
template <bool BF16, bool TWO>
__global__ void __launch_bounds__(256, 8) bwd_post_kernel(const float* __restrict__ acc, const uint32_t* __restrict__ det,
                                                       uint16_t* __restrict__ dq, long long n8, float scale) {
  const bool checker = blockIdx.x == 0 && threadIdx.x == 0;
  uint32_t left = 0;
  if (checker) left = __ldcg(det);
  const float* acc2 = acc + n8 * 8;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += nthreads) {
    float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    if constexpr (TWO) {
      const float4 a2 = reinterpret_cast<const float4*>(acc2)[2 * i];
      const float4 b2 = reinterpret_cast<const float4*>(acc2)[2 * i + 1];
      a = make_float4(a.x + a2.x, a.y + a2.y, a.z + a2.z, a.w + a2.w);
      b = make_float4(b.x + b2.x, b.y + b2.y, b.z + b2.z, b.w + b2.w);
    }
    uint4 r;
    r.x = pack2<BF16>(a.x * scale, a.y * scale);
    r.y = pack2<BF16>(a.z * scale, a.w * scale);
    r.z = pack2<BF16>(b.x * scale, b.y * scale);
    r.w = pack2<BF16>(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = r;
  }
  if (checker && (left != 0u) != TWO) record_error(DEV_ERR_ARG, BWD_SITE_POST);
}

// fp32 tile in shared memory added element-wise into global memory by the
// TMA unit (bulk-group completion).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, const void* src, int c0, int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(src))
      : "memory");
}
// Orders this thread's global accesses of the generic proxy with its bulk
// (async-proxy) operations on global memory.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// bwd_main
// ---------------------------------------------------------------------------
// DET: deterministic mode (p.deterministic), a separate instance so that the
// atomic mode's dQ warps carry none of its ordering state.
template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT = false, bool DET = false>
__global__ void __launch_bounds__(512, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_cols,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;        // K_j, V_j loaded
  uint64_t* kv_empty = bars + 1;   // the unit's last products are done with K_j, V_j
  uint64_t* q_full = bars + 2;     // [2]
  uint64_t* q_empty = bars + 4;    // [2]
  uint64_t* do_full = bars + 6;
  uint64_t* do_empty = bars + 7;
  uint64_t* s_full = bars + 8;     // S^T(g) in X(g)
  uint64_t* dp_full = bars + 9;    // dP^T(g) in Y(g)
  uint64_t* p_full = bars + 10;    // P^T(g) written (256 P/dS threads)
  uint64_t* dp_taken = bars + 11;  // dP^T(g) read out of Y(g) (256 P/dS threads)
  uint64_t* ds_full = bars + 12;   // dS(g) in X(g) and in shared memory (256 P/dS threads)
  uint64_t* dq_full = bars + 13;   // dQ(g) in X(g)
  uint64_t* dq_empty = bars + 14;  // dQ(g) read out of X(g) (128 dQ threads)
  uint64_t* dkv_full = bars + 15;  // the unit's dV and dK are final
  uint64_t* drain = bars + 16;
  uint64_t* unit_full = bars + 18;   // [2] a claimed unit number is in the ring
  uint64_t* unit_empty = bars + 20;  // [2] every role has read it (one lane of each of 13 warps)
  uint64_t* rel_full = bars + 22;    // [2] deterministic mode: the four dQ warps' reductions of a
                                     //   step are performed and its counter is in rel_sem
  uint64_t* rel_empty = bars + 24;   // [2] the release warp has taken the counter
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(tmem_holder + 1);  // [2]
  uint32_t* volatile* rel_sem = reinterpret_cast<uint32_t* volatile*>(tmem_holder + 4);  // [2]

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  BWD_TRACE(threadIdx.x == 0, 4000);
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&unit_full[i], 1);
      mbar_init(&unit_empty[i], 13);
      mbar_init(&rel_full[i], 4);
      mbar_init(&rel_empty[i], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(dp_taken, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (threadIdx.x < 256) {
    // The two constant key-side rows of the extra K step (bf16, 32-byte
    // swizzle): row set 0 holds 1/(scale log2 e) in three parts (part k / 3 in
    // column k, k < 9), so against the per-query rows it adds -LSE / scale to
    // every score; row set 1 holds 1 in columns 9-11, which adds -D to dP.
    const int set = threadIdx.x >> 7, r = threadIdx.x & 127;
    const float inv = 1.f / p.scale_log2;
    const float i0 = bf16_round(inv), i1 = bf16_round(inv - i0), i2 = bf16_round(inv - i0 - i1);
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = set == 0 ? (k < 9 ? (k < 3 ? i0 : k < 6 ? i1 : i2) : 0.f)
                                                 : ((k >= 9 && k < 12) ? 1.f : 0.f);
    uint8_t* row = smem + C::ONES_OFF + set * 4096;
    *reinterpret_cast<uint4*>(row + swz32(r * 32)) =
        make_uint4(pack2<true>(v[0], v[1]), pack2<true>(v[2], v[3]), pack2<true>(v[4], v[5]), pack2<true>(v[6], v[7]));
    *reinterpret_cast<uint4*>(row + swz32(r * 32 + 16)) =
        make_uint4(pack2<true>(v[8], v[9]), pack2<true>(v[10], v[11]), pack2<true>(v[12], v[13]),
                   pack2<true>(v[14], v[15]));
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Every role but the producer takes the k-th claimed unit from the ring
  // (-1 ends the list); one lane per warp reports that it has read it.
  auto next_unit = [&](int k, int& u) -> bool {
    const int slot = k & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&unit_full[slot], (k >> 1) & 1, BWD_SITE_UNIT))) return false;
    u = unit_ring[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(&unit_empty[slot]);
    return true;
  };
  // TMEM region that holds S^T / P^T / dS^T at step g (the other one holds
  // dP^T and then dQ)
  auto region_x = [](uint32_t g) -> uint32_t { return (g & 1) ? C::TM_B : C::TM_A; };

  // register split over 512 threads launched with 128 each (65536):
  // 128 x 56 (warps 0-3) + 256 x RP (P/dS) + 128 x RQ (dQ), with (RP, RQ) =
  // (136, 176) = 64512, and (144, 168) = 65536 for dropout, whose dS phase
  // keeps the keep bits and D_i live as well.
  // Each warpgroup changes its budget inside its own branch.
  constexpr int RP = DROPOUT ? 144 : 136, RQ = DROPOUT ? 168 : 176;
  static_assert(128 * 56 + 256 * RP + 128 * RQ <= 65536, "register split");
  if (warp < 4) {
  regs_dec<56>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_cols);
      uint32_t g = 0, kc = 0;  // query steps and units loaded so far
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // claim the next non-empty unit (numbers past the end claim nothing)
        int u;
        BwdUnit x;
        do {
          u = (int)atomicAdd(p.ticket, 1u);
        } while (u < p.units && !bwd_decode<CAUSAL, VARLEN>(p, u, x));
        const int slot = k & 1;
        BWD_TRACE(k < 16, 3100 + k);
        if (k >= 2 && !(ok = mbar_wait(&unit_empty[slot], ((k >> 1) - 1) & 1, BWD_SITE_PROD))) break;
        unit_ring[slot] = u < p.units ? u : -1;
        mbar_arrive(&unit_full[slot]);
        if (u >= p.units) break;
        // K_j, V_j once the previous unit's products are done with the old ones
        if (kc > 0 && !(ok = mbar_wait(kv_empty, (kc - 1) & 1, BWD_SITE_PROD))) break;
        mbar_expect_tx(kv_full, 2 * C::TILE);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_3d(smem + C::K_OFF + c * C::CHUNK, &tm_k, kv_full, c * 64, x.row_base + 128 * x.j, x.head);
          tma_load_3d(smem + C::V_OFF + c * C::CHUNK, &tm_v, kv_full, c * 64, x.row_base + 128 * x.j, x.head);
        }
        ++kc;
        const size_t stat_row0 = ((size_t)x.head * p.nseq + x.seq) * p.S_pad;  // padded statistics of this sequence
        for (int st = 0; st < x.n_steps && ok; ++st, ++g) {
          const int i = x.i_begin + st;
          // Q_i and its LSE / D rows into Q slot g % 2
          const int qs = g & 1;
          if (g >= 2 && !(ok = mbar_wait(&q_empty[qs], ((g >> 1) - 1) & 1, BWD_SITE_PROD))) break;
          mbar_expect_tx(&q_full[qs], C::TILE + 4096u);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::Q_OFF + qs * C::TILE + c * C::CHUNK, &tm_q, &q_full[qs], c * 64,
                        x.row_base + 128 * i, x.head);
          tma_load_3d(smem + C::CT_OFF + qs * 4096, &tm_cols, &q_full[qs], 0, (int)(stat_row0 + 128 * i), 0);
          // dO_i into the dO slot
          if (g >= 1 && !(ok = mbar_wait(do_empty, (g - 1) & 1, BWD_SITE_PROD))) break;
          mbar_expect_tx(do_full, C::TILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::DO_OFF + c * C::CHUNK, &tm_do, do_full, c * 64, x.row_base + 128 * i, x.head);
        }
      }
      // no tile copy may still be landing in shared memory at exit
      if (kc > 0) mbar_wait(kv_full, (kc - 1) & 1, BWD_SITE_PROD);
      for (uint32_t v = (g > 2 ? g - 2 : 0); v < g; ++v) mbar_wait(&q_full[v & 1], (v >> 1) & 1, BWD_SITE_PROD);
      if (g > 0) mbar_wait(do_full, (g - 1) & 1, BWD_SITE_PROD);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Converged warp, one elected lane issues; descriptors formed once and
    // offset by constants inside fully unrolled groups of 8 products.
    const uint32_t e = elect_one();
    constexpr uint32_t ID_KK = make_idesc(128, 128, BF16, false, false);  // dP^T, S^T
    constexpr uint32_t ID_TS = make_idesc(128, D, BF16, false, true);     // dV, dK
    constexpr uint32_t ID_DQ = make_idesc(128, D, BF16, true, true);      // dQ
    const uint64_t kK = make_sdesc(smem_addr(smem + C::K_OFF), 16, 1024);       // K as A (K-major)
    const uint64_t kMN = make_sdesc(smem_addr(smem + C::K_OFF), C::CHUNK, 1024);  // K as B of dQ (MN-major)
    const uint64_t vK = make_sdesc(smem_addr(smem + C::V_OFF), 16, 1024);
    const uint64_t qK = make_sdesc(smem_addr(smem + C::Q_OFF), 16, 1024);       // Q slot 0 as B of S^T
    const uint64_t qMN = make_sdesc(smem_addr(smem + C::Q_OFF), C::CHUNK, 1024);  // Q slot 0 as B of dK
    const uint64_t doK = make_sdesc(smem_addr(smem + C::DO_OFF), 16, 1024);
    const uint64_t doMN = make_sdesc(smem_addr(smem + C::DO_OFF), C::CHUNK, 1024);
    const uint64_t dsMN = make_sdesc(smem_addr(smem + C::DS_OFF), C::CHUNK, 1024);  // dS as A of dQ (MN-major)
    const uint64_t onesL = make_sdesc_sw32(smem_addr(smem + C::ONES_OFF));         // adds -LSE / scale
    const uint64_t onesD = make_sdesc_sw32(smem_addr(smem + C::ONES_OFF + 4096));  // adds -D
    const uint64_t ctK = make_sdesc_sw32(smem_addr(smem + C::CT_OFF));              // per-query rows, slot 0
    constexpr uint32_t ID_AUG = make_idesc(128, 128, true, false, false);           // bf16 x bf16
    // X^T = A_kv B_q^T with both operands K-major (X = S or dP)
    auto kk_product = [&](uint32_t d_col, uint64_t a, uint64_t b) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
        mma_ss_e(tmem + d_col, desc_add(a, off), desc_add(b, off), ID_KK, kk > 0 ? 1u : 0u, e);
      }
    };
    // acc += A(TMEM, 16-bit pairs) * B (MN-major), K = 128 queries.  Queries
    // 0-63 sit in columns a_col .. a_col + 31, queries 64-127 in columns
    // a_col + 64 .. a_col + 95 (each half is written by the warpgroup that
    // read those score columns).
    auto ts_product = [&](uint32_t d_col, uint32_t a_col, uint64_t b, uint32_t acc) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_e(tmem + d_col, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), desc_add(b, kk * 2048), ID_TS,
                 kk > 0 ? 1u : acc, e);
    };
    uint32_t g = 0, kc = 0;  // query steps and units so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u;
      if (!(ok = next_unit(k, u)) || u < 0) break;
      BwdUnit x;
      bwd_decode<CAUSAL, VARLEN>(p, u, x);
      BWD_TRACE(lane == 0 && k < 16, 3000 + 2 * k);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(kv_full, kc & 1, BWD_SITE_KV)))) break;
      BWD_TRACE(lane == 0 && k < 16, 3000 + 2 * k + 1);
      ++kc;
      // first step of the unit: S^T(g) into X(g), dP^T(g) into Y(g) = X(g - 1),
      // which still holds dQ(g - 1) until the dQ warps have drained it
      {
        const int qs = g & 1;
        const uint32_t X = region_x(g), Y = X ^ (C::TM_A ^ C::TM_B);
        ok = mbar_wait(&q_full[qs], (g >> 1) & 1, BWD_SITE_Q) && mbar_wait(do_full, g & 1, BWD_SITE_DO);
        if (ok && g > 0) ok = mbar_wait(dq_empty, (g - 1) & 1, BWD_SITE_DQE);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        kk_product(X, kK, desc_add(qK, qs * C::TILE));  // S^T(g), then - LSE / scale
        mma_ss_e(tmem + X, onesL, desc_add(ctK, qs * 4096), ID_AUG, 1u, e);
        mma_commit_e(s_full, e);
        kk_product(Y, vK, doK);  // dP^T(g), then - D
        mma_ss_e(tmem + Y, onesD, desc_add(ctK, qs * 4096), ID_AUG, 1u, e);
        mma_commit_e(dp_full, e);
      }
      for (int st = 0; st < x.n_steps && ok; ++st, ++g) {
        const int qs = g & 1;
        const uint32_t X = region_x(g), Y = X ^ (C::TM_A ^ C::TM_B);
        const uint32_t acc = st > 0 ? 1u : 0u;
        const bool more = st + 1 < x.n_steps;
        // dV += P^T dO_i (dO_i is not read again: dP^T(g) came before)
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_full, g & 1, BWD_SITE_P)))) break;
        BWD_TRACE(lane == 0 && g < 200, g * 8);
        tc_fence_after();
        ts_product(C::TM_DV, X, doMN, acc);
        mma_commit_e(do_empty, e);
        // S^T(g+1) into Y as soon as the dS warps have read dP^T(g) out of it
        if (more) {
          ok = mbar_wait(dp_taken, g & 1, BWD_SITE_TAKEN) && mbar_wait(&q_full[qs ^ 1], ((g + 1) >> 1) & 1, BWD_SITE_Q);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          tc_fence_after();
          BWD_TRACE(lane == 0 && g < 200, g * 8 + 1);
          kk_product(Y, kK, desc_add(qK, (qs ^ 1) * C::TILE));
          mma_ss_e(tmem + Y, onesL, desc_add(ctK, (qs ^ 1) * 4096), ID_AUG, 1u, e);
          mma_commit_e(s_full, e);
        }
        // dK += dS^T Q_i (A = dS^T in X; Q_i is not read again)
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_full, g & 1, BWD_SITE_DS)))) break;
        BWD_TRACE(lane == 0 && g < 200, g * 8 + 2);
        tc_fence_after();
        ts_product(C::TM_DK, X + 32, desc_add(qMN, qs * C::TILE), acc);
        mma_commit_e(&q_empty[qs], e);
        // dQ_i = dS K_j into X  (A = dS MN-major in smem, B = K MN-major),
        // after dK has read dS^T out of X
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_e(tmem + X, desc_add(dsMN, kk * 2048), desc_add(kMN, kk * 2048), ID_DQ, kk > 0 ? 1u : 0u, e);
        mma_commit_e(dq_full, e);
        BWD_TRACE(lane == 0 && g < 200, g * 8 + 3);
        // dP^T(g+1) into X once dQ_i has been drained
        if (more) {
          ok = mbar_wait(dq_empty, g & 1, BWD_SITE_DQE) && mbar_wait(do_full, (g + 1) & 1, BWD_SITE_DO);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          BWD_TRACE(lane == 0 && g < 200, g * 8 + 4);
          tc_fence_after();
          kk_product(X, vK, doK);
          mma_ss_e(tmem + X, onesD, desc_add(ctK, (qs ^ 1) * 4096), ID_AUG, 1u, e);
          mma_commit_e(dp_full, e);
        }
      }
      if (!ok) break;
      mma_commit_e(kv_empty, e);  // K_j, V_j may be replaced
      mma_commit_e(dkv_full, e);  // this unit's dV, dK are final
    }
    mma_commit_e(drain, e);
    mbar_wait(drain, 0, BWD_SITE_DRAIN);
    __syncwarp();
  } else if (DET && warp == 2) {
    // ------------------------------------------------------------ release
    // Deterministic mode: adds each step's four dQ-warp counts to its chain
    // counter with one gpu-scope release, which takes ~1100 clk that the dQ
    // warps would otherwise wait out every step.  Each dQ warp's lane 0 has
    // waited for its reductions and fenced them against the generic proxy
    // before arriving on rel_full (a CTA-scope release); the wait here
    // acquires that, and the release below passes it on to the next key
    // tile's acquire.  A null counter ends the loop.
    if (lane == 0) {
      for (uint32_t h = 0;; ++h) {
        const int slot = h & 1;
        if (!mbar_wait(&rel_full[slot], (h >> 1) & 1, BWD_SITE_REL)) break;
        uint32_t* sem = rel_sem[slot];
        mbar_arrive(&rel_empty[slot]);
        if (!sem) break;
        red_release_gpu_add(sem, 4u);
      }
    }
    __syncwarp();
  }
  } else if (warp < 12) {
    regs_inc<RP>();
    // ------------------------------------------------------------ P / dS
    // One thread per key row and half of the 128 query columns: warps 4-7
    // take queries 0-63, warps 8-11 queries 64-127.  P and dS are
    // elementwise given LSE and D_i, so the halves never exchange data.
    const int half = (warp - 4) >> 2;
    const int r = (threadIdx.x - 128) & 127;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float sl2 = p.scale_log2;
    uint8_t* ds_smem = smem + C::DS_OFF;
    uint32_t g = 0, ucnt = 0;  // query steps and units so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int u;
      if (!(ok = next_unit(k, u)) || u < 0) break;
      BwdUnit x;
      bwd_decode<CAUSAL, VARLEN>(p, u, x);
      const int kv = 128 * x.j + r;  // key row inside the sequence
      const bool kv_valid = kv < x.seq_len;
      // Dropout keep decisions of this key row against the half's 64 query
      // columns of tile iq, pair-packed: queries 2e, 2e + 1 at bits
      // pair_slot(e & 15), pair_slot(e & 15) + 8 of keep[e >> 4].  One Philox
      // call covers query pair e x key octet (8m .. 8m + 7), one byte per
      // element, and a key octet sits in eight consecutive lanes: lane 8m + c
      // draws query pairs 4c .. 4c + 3, and each lane hands every other lane
      // of its octet that lane's bytes of two calls at a time (XOR shuffles
      // over the octet).  Drawn for the next step while this step's products
      // run, so the generator stays off the critical path of P and dS.
      uint32_t keep[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
      auto make_keep = [&](int iq) {
        const uint32_t c8 = lane & 7u;
        const uint32_t t4 = p.drop.thresh * 0x01010101u, t4lo = t4 & 0x7f7f7f7fu;
        const uint32_t keyoct = (uint32_t)kv >> 3, qp0 = (uint32_t)(128 * iq + 64 * half) >> 1;
        // head word of the counter: b * H + h, a packed batch's sequence as b
        const uint32_t mask_head = (uint32_t)(x.seq * p.heads + x.head);
        uint32_t k0 = 0u, k1 = 0u;
#pragma unroll
        for (int q = 0; q < 4; q += 2) {
          const uint4 w0 = philox4x32_10(make_uint4(keyoct, qp0 + 4 * c8 + q, mask_head, p.drop.offset),
                                         p.drop.seed_lo, p.drop.seed_hi);
          const uint4 w1 = philox4x32_10(make_uint4(keyoct, qp0 + 4 * c8 + q + 1, mask_head, p.drop.offset),
                                         p.drop.seed_lo, p.drop.seed_hi);
          // key 8m + t: byte t & 3 of word (t >> 2) for the even query and of
          // word 2 + (t >> 2) for the odd one; the bytes of both calls packed
          // as (even q, odd q, even q + 1, odd q + 1)
          auto vals_for = [&w0, &w1](uint32_t t) -> uint32_t {
            const uint32_t e0 = (t & 4u) ? w0.y : w0.x, o0 = (t & 4u) ? w0.w : w0.z;
            const uint32_t e1 = (t & 4u) ? w1.y : w1.x, o1 = (t & 4u) ? w1.w : w1.z;
            // byte t & 3 of e and of o, side by side, for each call; then both
            const uint32_t sel = (t & 3u) | ((4u | (t & 3u)) << 4);
            uint32_t a, b, r;
            asm("prmt.b32 %0, %1, %2, %3;" : "=r"(a) : "r"(e0), "r"(o0), "r"(sel));
            asm("prmt.b32 %0, %1, %2, %3;" : "=r"(b) : "r"(e1), "r"(o1), "r"(sel));
            asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(a), "r"(b));
            return r;
          };
#pragma unroll
          for (uint32_t d = 0; d < 8; ++d) {
            const uint32_t v = d == 0 ? vals_for(c8) : __shfl_xor_sync(0xffffffffu, vals_for(c8 ^ d), (int)d);
            const uint32_t e = 4u * (c8 ^ d) + (uint32_t)q;  // query pairs e, e + 1 drawn by lane c8 ^ d
            const uint32_t bits = pair_bits(bytes_below(v, t4, t4lo)) << ((e & 7u) + 16u * ((e >> 3) & 1u));
            k0 |= (e & 16u) ? 0u : bits;
            k1 |= (e & 16u) ? bits : 0u;
          }
        }
        keep[0] = k0;
        keep[1] = k1;
      };
      if constexpr (DROPOUT) make_keep(x.i_begin);
      for (int st = 0; st < x.n_steps; ++st, ++g) {
        const int i = x.i_begin + st;
        const int qs = g & 1;
        const uint32_t X = region_x(g), Y = X ^ (C::TM_A ^ C::TM_B);
        const uint32_t tX = tmem + lane_off + X, tY = tmem + lane_off + Y;
        ok = mbar_wait(s_full, g & 1, BWD_SITE_S) && mbar_wait(&q_full[qs], (g >> 1) & 1, BWD_SITE_STAT);
        ok = __all_sync(0xffffffffu, ok);
        const bool tw = warp == 4 && lane == 0 && g < 200;
        BWD_TRACE(tw, 1600 + 4 * g);
        if (!ok) break;
        tc_fence_after();
        // visible queries of this key row in tile i: q >= kv under the causal mask
        const int qlo = (CAUSAL && i == x.j) ? r : 0;
        const bool masked = qlo > 64 * half || !kv_valid;  // some column of this half is invisible
        // ---- P phase (score columns 64*half .. +63): the scores already hold
        // -LSE / scale (extra K step), so P^T = 2^(S'^T scale log2 e)
        uint32_t sv[2][32];
        tmem_ld32(tX + 64 * half, sv[0]);
        tmem_ld32(tX + 64 * half + 32, sv[1]);
        tmem_ld_wait(sv[0]);
        tmem_ld_wait(sv[1]);
        const uint64_t sl2x2 = f2(sl2, sl2);
        uint32_t pk[32];  // P pairs rounded to 16 bits (the products' and dS's P)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = 64 * half + 2 * e;
          const uint32_t* src = sv[e >> 4] + 2 * (e & 15);
          float p0, p1;
          f2split(fmul2(f2(__uint_as_float(src[0]), __uint_as_float(src[1])), sl2x2), p0, p1);
          p0 = ex2(p0);
          p1 = ex2(p1);
          if (masked) {
            if (c < qlo || !kv_valid) p0 = 0.f;
            if (c + 1 < qlo || !kv_valid) p1 = 0.f;
          }
          pk[e] = pack2<BF16>(p0, p1);
        }
        // P^T pairs go to columns [64*half, 64*half + 32) of X (inside this
        // half's own score columns, already read); with dropout the dV operand
        // is P * M (dV is scaled by s = 1 / keep probability at the end)
        if constexpr (DROPOUT) {
          uint32_t pd[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pd[e] = pk[e] & pair_keep_halves(keep[e >> 4], e & 15);
          tmem_st32(tX + 64 * half, pd);
        } else {
          tmem_st32(tX + 64 * half, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        BWD_TRACE(tw, 1600 + 4 * g + 1);
        // ---- dS phase: dS^T = P^T (dP^T - D), P as rounded for the products;
        // dP^T already holds -D (extra K step).  Once it is in registers Y
        // is free for the next step's scores.
        ok = __all_sync(0xffffffffu, mbar_wait(dp_full, g & 1, BWD_SITE_DP));
        BWD_TRACE(tw, 1600 + 4 * g + 2);
        if (!ok) break;
        tc_fence_after();
        uint32_t dv[2][32];
        tmem_ld32(tY + 64 * half, dv[0]);
        tmem_ld32(tY + 64 * half + 32, dv[1]);
        tmem_ld_wait(dv[0]);
        tmem_ld_wait(dv[1]);
        tc_fence_before();
        mbar_arrive(dp_taken);
        BWD_TRACE(tw, 3700 + g);
        uint32_t dd[32];
        if constexpr (DROPOUT) {
          // dP'^T = dPd^T - D (extra K step).  dS = P (M s dPd - D) with
          // M s = m (s = 1 / keep probability for a kept element, 0 for a
          // dropped one): dS = P (m (dP' + D) - D).  D_i of the half's 64
          // query columns comes from their per-query rows (-D in three bf16
          // parts, columns 9-11) in shared memory: lane l reads those of
          // columns l and 32 + l, and hands them round.
          const uint8_t* ct = smem + C::CT_OFF + qs * 4096;
          const float rp = p.drop.scale;
          float d_l[2];
#pragma unroll
          for (int w2 = 0; w2 < 2; ++w2) {
            const uint32_t qrow = (uint32_t)(64 * half + 32 * w2) + lane;
            const uint2 c = *reinterpret_cast<const uint2*>(ct + swz32(qrow * 32u + 16u));
            d_l[w2] = -(__uint_as_float(c.x & 0xFFFF0000u) + __uint_as_float(c.y << 16) +
                        __uint_as_float(c.y & 0xFFFF0000u));
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t* src = dv[e >> 4] + 2 * (e & 15);
            // query columns 2e, 2e + 1 of the half
            const float d0 = __shfl_sync(0xffffffffu, d_l[e >> 4], (2 * e) & 31);
            const float d1 = __shfl_sync(0xffffffffu, d_l[e >> 4], (2 * e + 1) & 31);
            const uint32_t kb = keep[e >> 4] >> pair_slot(e & 15);
            const float m0 = (kb & 1u) ? rp : 0.f, m1 = (kb & 0x100u) ? rp : 0.f;
            const float2 pw = unpack2<BF16>(pk[e]);
            const float a = pw.x * fmaf(m0, __uint_as_float(src[0]) + d0, -d0);
            const float b = pw.y * fmaf(m1, __uint_as_float(src[1]) + d1, -d1);
            dd[e] = pack2<BF16>(a, b);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t* src = dv[e >> 4] + 2 * (e & 15);
            float a, b;
            f2split(fmul2(widen2<BF16>(pk[e]), f2(__uint_as_float(src[0]), __uint_as_float(src[1]))), a, b);
            dd[e] = pack2<BF16>(a, b);
          }
        }
        BWD_TRACE(tw, 3500 + g);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          // dS row r (key), 32 query columns: MN-major A operand of dQ = dS K,
          // [key][query] with queries contiguous, 64-query chunk = half, 128-B swizzled
          const uint32_t base = half * C::CHUNK + r * 128 + ch * 64;
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            *reinterpret_cast<uint4*>(ds_smem + swz128(base + v4 * 16)) =
                make_uint4(dd[16 * ch + 4 * v4], dd[16 * ch + 4 * v4 + 1], dd[16 * ch + 4 * v4 + 2],
                           dd[16 * ch + 4 * v4 + 3]);
        }
        // dS^T pairs to columns [64*half + 32, 64*half + 64) of X (score
        // columns this half has read)
        tmem_st32(tX + 64 * half + 32, dd);
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_full);
        BWD_TRACE(tw, 1600 + 4 * g + 3);
        if constexpr (DROPOUT)
          if (st + 1 < x.n_steps) make_keep(i + 1);
        BWD_TRACE(tw, 3300 + g);
      }
      if (!ok) break;
      // ---- epilogue: dV and scale * dK rows of this key tile
      ok = __all_sync(0xffffffffu, mbar_wait(dkv_full, ucnt & 1, BWD_SITE_DKV));
      BWD_TRACE(warp == 4 && lane == 0 && ucnt < 16, 3200 + ucnt);
      ++ucnt;
      if (!ok) break;
      tc_fence_after();
      const size_t grow = ((size_t)x.head * p.rows + x.row_base + kv) * D;
      const int which = half;  // half 0 writes dV, half 1 writes scale * dK
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(which ? p.dk : p.dv) + grow);
      const float mul = which ? p.scale : (DROPOUT ? p.drop.scale : 1.f);
      const uint32_t col = which ? C::TM_DK : C::TM_DV;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_off + col + 32 * cc, ov);
        tmem_ld_wait(ov);
        uint32_t pkk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pkk[e] = pack2<BF16>(__uint_as_float(ov[2 * e]) * mul, __uint_as_float(ov[2 * e + 1]) * mul);
        if (kv_valid) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[cc * 4 + e] = make_uint4(pkk[4 * e], pkk[4 * e + 1], pkk[4 * e + 2], pkk[4 * e + 3]);
        }
      }
      // the next unit's first dV / dK products overwrite the accumulators only
      // after this warpgroup has published that unit's first P / dS
      tc_fence_before();
    }
  } else {
    regs_inc<RQ>();
    // ------------------------------------------------------------ dQ (one thread per query row)
    const int wq = warp - 12;                        // this warp's 32 rows: 32*wq ..
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* stg = smem + C::STG_OFF + wq * 4096;    // 32 rows x 128 B, 128-B swizzled
    if (lane == 0) tma_prefetch_desc(&tm_dq);
    uint32_t g = 0;  // query steps so far
    bool ok = true;
    // deterministic mode: the chain counter this warp still owes its count
    // to (the last step's), and the posts made to the release warp
    uint32_t* pend_new = nullptr;
    uint32_t posts = 0;
    // lane 0, once this warp's reductions of that step have been performed:
    // hand the counter to the release warp (null: no more steps)
    auto count_in = [&](uint32_t* sem) {
      const int slot = posts & 1;
      if (posts >= 2 && !mbar_wait(&rel_empty[slot], ((posts >> 1) - 1) & 1, BWD_SITE_REL)) return;
      if (warp == 12) rel_sem[slot] = sem;
      fence_proxy_async_global();
      mbar_arrive(&rel_full[slot]);
      ++posts;
    };
    for (int k = 0; ok; ++k) {
      int u;
      if (!(ok = next_unit(k, u)) || u < 0) break;
      BwdUnit x;
      bwd_decode<CAUSAL, VARLEN>(p, u, x);
      for (int st = 0; st < x.n_steps; ++st, ++g) {
        const int i = x.i_begin + st;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(dq_full, g & 1, BWD_SITE_DQF)))) break;
        const bool qw = warp == 12 && lane == 0 && g < 200;
        BWD_TRACE(qw, 2400 + 3 * g);
        tc_fence_after();
        const uint32_t X = region_x(g);
        uint32_t a[D / 32][32];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_off + X + 32 * cc, a[cc]);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld_wait(a[cc]);
        tc_fence_before();
        mbar_arrive(dq_empty);
        BWD_TRACE(qw, 2400 + 3 * g + 1);
        // This tile's fp32 partial: TMEM -> per-warp swizzled staging -> TMA bulk
        // reduce-add into the accumulator, 32 columns at a time.
        auto reduce_partial = [&](int hc) {  // hc: the head coordinate in the accumulator map
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            if (lane == 0) bulk_wait_read0();  // the previous reduction has read the buffer
            __syncwarp();
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              *reinterpret_cast<uint4*>(stg + swz128(lane * 128 + v4 * 16)) =
                  make_uint4(a[cc][4 * v4], a[cc][4 * v4 + 1], a[cc][4 * v4 + 2], a[cc][4 * v4 + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&tm_dq, stg, 32 * cc, x.row_base + 128 * i + 32 * wq, hc);
              bulk_commit();
            }
          }
        };
        if constexpr (!DET) {
          reduce_partial(x.head);
          BWD_TRACE(qw, 2400 + 3 * g + 2);
        } else {
          // Key tiles add into query tile i in a fixed order, in two chains:
          // even j into the first accumulator, odd j into the second, each
          // from its highest j down (j = i or i - 1 first under the causal
          // mask, j = n_q - 1 or n_q - 2 without it).  A chain's counter for
          // tile i counts the dQ warps (four per key tile) whose reductions
          // into it have been performed: a warp waits until all four warps of
          // every earlier key tile of the chain are in, adds its partial with
          // the same bulk reductions, and is counted only once those have
          // been performed (the release warp adds the four warps' counts), so
          // every element sees its additions in one fixed order.  The count
          // is posted one step later, after the next partial has been
          // drained, when the reductions have mostly completed, or at once
          // after a unit's last tile; the predecessor in the chain, key tile
          // j + 2, reached tile i two steps before us under the causal mask,
          // which leaves that hand-over a step of time.  (Three chains with
          // the count two steps later measured slower.)
          if (pend_new && lane == 0) {
            bulk_wait0();
            count_in(pend_new);
          }
          pend_new = nullptr;
          const int chain = x.j & 1;
          const int top = CAUSAL ? i : x.n_q - 1;
          const uint32_t turn = (uint32_t)((top - ((top - chain) & 1) - x.j) >> 1);
          uint32_t* sem = p.sem + (((size_t)x.head * p.nseq + x.seq) * p.n_q + i) * 2 + chain;
          if (lane == 0) {
            if (ld_acquire_gpu(sem) < 4u * turn) {
              const uint64_t t0 = global_ns();
              while (ld_acquire_gpu(sem) < 4u * turn) {
                if (global_ns() - t0 > kWaitLimitNs) {
                  // reported; go on so that the later key tiles are not held up too
                  record_error(DEV_ERR_TIMEOUT, BWD_SITE_SEM);
                  break;
                }
              }
            }
            fence_proxy_async_global();  // our reductions come after the acquire
          }
          __syncwarp();
          BWD_TRACE(qw, 2400 + 3 * g + 2);
          reduce_partial(x.head + chain * p.heads);
          pend_new = sem;
          if (st == x.n_steps - 1) {  // a unit's last tile: count it in now
            if (lane == 0) {
              bulk_wait0();
              count_in(pend_new);
            }
            pend_new = nullptr;
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) {
      bulk_wait0();  // every reduction issued by this warp has completed
      if constexpr (DET) count_in(nullptr);  // the release warp may stop
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  BWD_TRACE(threadIdx.x == 0, 4001);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa

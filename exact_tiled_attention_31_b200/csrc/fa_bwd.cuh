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
//   bwd_main  one CTA per 128-row key/value tile j of one head (and, for a
//             packed batch, one sequence; 512 threads):
//               warp 0     TMA producer: K_j, V_j once; then Q_i (+ the
//                          per-query rows of tile i) into a 2-slot ring and
//                          dO_i into its own slot.
//               warp 1     tcgen05 issuer and TMEM owner.  TMEM columns:
//                          A = [0,128): S^T, then P^T (16-bit) in [0,64)
//                          B = [128,256): dP^T, then dS^T in [0,64), then dQ_i
//                          dV [256,256+D), dK [256+D,256+2D).
//                          Issue order for query tile i (one step):
//                            dV  += P^T dO_i          (A = P^T in TMEM)
//                            S^T(i+1) = K_j Q_{i+1}^T  -> A, plus one K step
//                                       that adds -LSE / scale per query
//                            dK  += dS^T Q_i          (A = dS^T in TMEM)
//                            dQ_i = dS K_j            (A = dS in smem) -> B
//                            dP^T(i+1) = V_j dO_{i+1}^T -> B (after dQ_i left
//                                       TMEM), plus one K step that adds -D
//                          so the exponentials of tile i+1 run while the
//                          tensor core does dK_i, dQ_i and dP^T(i+1).
//               warps 4-11 one thread per key row and half of the query
//                          columns (warps 4-7 queries 0-63, 8-11 queries
//                          64-127).  P phase: P^T = exp2(S'^T*scale*log2e)
//                          (S' already holds -LSE/scale), kept as 16-bit
//                          pairs in registers and written to TMEM A.  dS
//                          phase: dS^T = P^T dP'^T (dP' already holds -D) to
//                          TMEM B and, as the MN-major A operand of
//                          dQ = dS K, to shared memory.  At the end: dV and
//                          scale*dK rows to global memory.
//               warps 12-15 one thread per query row: move dQ_i from TMEM to
//                          a per-warp 128-byte-swizzled staging buffer and add
//                          it to the fp32 accumulator with TMA bulk reductions
//                          (cp.reduce.async.bulk.tensor .add); under
//                          deterministic mode the key tiles take turns (in
//                          increasing j) to issue those reductions for tile i.
//   bwd_post  dQ = scale * accumulator, rounded to the input dtype.
// Causal: key tile j only meets query tiles i >= j; only the diagonal tile
// is masked element-wise.  Packed batches ([H, T, D], cu_seqlens): every
// sequence is its own problem with tiles counted from its first token; keys
// past its end get P = 0 and query rows past its end carry a -1e30 score
// offset (so P = 0) and D = 0, so their dS rows are exactly 0 and nothing leaks into the next
// sequence's rows (the fp32 reductions of those zero rows add 0).
#pragma once

#include "sm100.cuh"

namespace fa {

struct BwdParams {
  void* dk;                // [heads, rows, D]
  void* dv;                // [heads, rows, D]
  float* dq_acc;           // [heads, rows, D] fp32
  uint16_t* cols;          // [heads, nseq, S_pad, 16] bf16 per-query rows (written by bwd_pre):
                           //   0-8: -LSE*log2(e) in three parts (part k % 3 in column k),
                           //   9-11: -D_i in three parts, 12-15: 0; padding rows -1e30 and 0
  uint32_t* sem;           // [heads, nseq, n_q] ordering counters (deterministic mode)
  const int* cu_seqlens;   // packed batch only: device int32 [nseq + 1]
  int heads;               // dense: B*H, packed: H
  int S;                   // dense: S, packed: max_seqlen
  int rows;                // rows of one head slice in memory: S or total
  int nseq;                // dense: 1
  int S_pad, n_q;          // ceil(S / 128) * 128, ceil(S / 128)
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
  // kv_full q_full[2] q_empty[2] do_full do_empty s_full dp_full p_full ds_full
  // dq_full dq_empty dkv_full drain dq_done
  static constexpr int NBAR = 17;
  static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TM_A = 0, TM_B = 128, TM_DV = 256, TM_DK = 256 + D;
};

// (sequence, head) slices per group of the backward's block order
constexpr int kBwdGroup = 4;

enum : uint32_t {
  BWD_SITE_PROD = 0x200, BWD_SITE_KV = 0x201, BWD_SITE_Q = 0x202, BWD_SITE_DO = 0x203, BWD_SITE_P = 0x204,
  BWD_SITE_DS = 0x205, BWD_SITE_DQE = 0x206, BWD_SITE_S = 0x207, BWD_SITE_DP = 0x208, BWD_SITE_DQF = 0x209,
  BWD_SITE_DKV = 0x20a, BWD_SITE_SEM = 0x20b, BWD_SITE_DRAIN = 0x20c, BWD_SITE_STAT = 0x20d
};

// ---------------------------------------------------------------------------
// bwd_pre: one group of D/8 lanes per row, 16-byte loads, shuffle reduction.
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool VARLEN>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      const float* __restrict__ lse, BwdParams p) {
  constexpr int G = D / 8;  // lanes per row
  const long long work = (long long)p.heads * p.nseq * p.S_pad * G;
  const long long bound = (work + 31) / 32 * 32;  // whole warps take the same trips
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long idx = gtid; idx < bound; idx += nthreads) {
    const bool in = idx < work;
    const long long row = idx / G;  // padded row: (head * nseq + seq) * S_pad + s
    const int part = (int)(idx % G);
    const long long hs = in ? row / p.S_pad : 0;
    const int h = (int)(hs / p.nseq);
    const int seq = (int)(hs - (long long)h * p.nseq);
    int base = 0, len = p.S;
    if constexpr (VARLEN) {
      base = p.cu_seqlens[seq];
      len = p.cu_seqlens[seq + 1] - base;
    }
    const int s = in ? (int)(row - hs * p.S_pad) : len;
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
    // the G lanes of one row are consecutive lanes of one warp (G divides 32)
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
      uint4* dst = reinterpret_cast<uint4*>(p.cols + (size_t)row * 16);
      dst[0] = make_uint4(pack2<true>(v[0], v[1]), pack2<true>(v[2], v[3]), pack2<true>(v[4], v[5]),
                          pack2<true>(v[6], v[7]));
      dst[1] = make_uint4(pack2<true>(v[8], v[9]), pack2<true>(v[10], v[11]), pack2<true>(v[12], v[13]),
                          pack2<true>(v[14], v[15]));
    }
  }
  // zero the dQ accumulator (16-byte stores) and the ordering counters
  const long long n4 = (long long)p.heads * p.rows * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long i = gtid; i < n4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long ns = (long long)p.heads * p.nseq * p.n_q;
  for (long long i = gtid; i < ns; i += nthreads) p.sem[i] = 0u;
}

// ---------------------------------------------------------------------------
// bwd_post: dQ = scale * accumulator, rounded to nearest in the input dtype.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq,
                                                       long long n8, float scale) {
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += nthreads) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    uint4 r;
    r.x = pack2<BF16>(a.x * scale, a.y * scale);
    r.y = pack2<BF16>(a.z * scale, a.w * scale);
    r.z = pack2<BF16>(b.x * scale, b.y * scale);
    r.w = pack2<BF16>(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = r;
  }
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
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// bwd_main
// ---------------------------------------------------------------------------
template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT = false>
__global__ void __launch_bounds__(512, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_cols,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  // work unit: (key/value tile j, sequence, head).  Blocks walk groups of
  // kBwdGroup (sequence, head) slices; inside a group, ascending j (longest
  // causal work first).  Only a few slices are live at a time, so their fp32
  // dQ accumulators and Q/K/V/dO tiles stay in L2, where the dQ reductions
  // run about twice as fast as against device memory.
  const int units = p.nseq * p.heads;
  const int group = blockIdx.x / (kBwdGroup * p.n_q);
  const int rg = blockIdx.x - group * (kBwdGroup * p.n_q);
  const int gsize = min(kBwdGroup, units - group * kBwdGroup);
  const int j = rg / gsize;
  if (j >= p.n_q) return;  // the last group may be smaller than kBwdGroup
  const int unit = group * kBwdGroup + (rg - j * gsize);
  const int seq = unit / p.heads;
  const int head = unit - seq * p.heads;
  int row_base = 0, seq_len = p.S;  // first token row and length of this sequence
  if constexpr (VARLEN) {
    row_base = p.cu_seqlens[seq];
    seq_len = p.cu_seqlens[seq + 1] - row_base;
  }
  if (128 * j >= seq_len) return;  // uniform over the CTA, before any set-up
  const int n_q = (seq_len + 127) / 128;
  const int i_begin = CAUSAL ? j : 0;
  const int n_steps = n_q - i_begin;
  const int kv_row0 = 128 * j;  // inside the sequence
  const size_t stat_row0 = ((size_t)head * p.nseq + seq) * p.S_pad;  // padded statistics of this sequence

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;    // [2]
  uint64_t* q_empty = bars + 3;   // [2]
  uint64_t* do_full = bars + 5;
  uint64_t* do_empty = bars + 6;
  uint64_t* s_full = bars + 7;
  uint64_t* dp_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* ds_full = bars + 10;
  uint64_t* dq_full = bars + 11;
  uint64_t* dq_empty = bars + 12;
  uint64_t* dkv_full = bars + 13;
  uint64_t* drain = bars + 14;
  uint64_t* dq_done = bars + 15;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_full, 1);
    mbar_init(drain, 1);
    mbar_init(dq_done, 128);
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

  // register split over 512 threads launched with 128 each (65536):
  // 128 x 56 (warps 0-3) + 256 x 136 (P/dS) + 128 x 176 (dQ) = 64512.
  // Each warpgroup changes its budget inside its own branch.
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
      mbar_expect_tx(kv_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(smem + C::K_OFF + c * C::CHUNK, &tm_k, kv_full, c * 64, row_base + kv_row0, head);
        tma_load_3d(smem + C::V_OFF + c * C::CHUNK, &tm_v, kv_full, c * 64, row_base + kv_row0, head);
      }
      bool ok = true;
      int q_issued = 0, do_issued = 0;
      for (int st = 0; st < n_steps && ok; ++st) {
        const int i = i_begin + st;
        // Q_i and its LSE / D rows into Q slot st % 2
        const int qs = st & 1;
        if (st >= 2 && !(ok = mbar_wait(&q_empty[qs], ((st >> 1) - 1) & 1, BWD_SITE_PROD))) break;
        mbar_expect_tx(&q_full[qs], C::TILE + 4096u);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(smem + C::Q_OFF + qs * C::TILE + c * C::CHUNK, &tm_q, &q_full[qs], c * 64,
                      row_base + 128 * i, head);
        tma_load_3d(smem + C::CT_OFF + qs * 4096, &tm_cols, &q_full[qs], 0, (int)(stat_row0 + 128 * i), 0);
        ++q_issued;
        // dO_i into the dO slot
        if (st >= 1 && !(ok = mbar_wait(do_empty, (st - 1) & 1, BWD_SITE_PROD))) break;
        mbar_expect_tx(do_full, C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(smem + C::DO_OFF + c * C::CHUNK, &tm_do, do_full, c * 64, row_base + 128 * i, head);
        ++do_issued;
      }
      // no tile copy may still be landing in shared memory at exit
      mbar_wait(kv_full, 0, BWD_SITE_PROD);
      for (int u = (q_issued > 2 ? q_issued - 2 : 0); u < q_issued; ++u)
        mbar_wait(&q_full[u & 1], (u >> 1) & 1, BWD_SITE_PROD);
      if (do_issued > 0) mbar_wait(do_full, (do_issued - 1) & 1, BWD_SITE_PROD);
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
    const uint64_t dsMN = make_sdesc(smem_addr(smem + C::DS_OFF), C::CHUNK, 1024);
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
    // 0-63 sit in the first 32 columns of the A region, queries 64-127 in
    // columns 64-95 (each half is written by the warpgroup that read those
    // score columns).
    auto ts_product = [&](uint32_t d_col, uint32_t a_col, uint64_t b, uint32_t acc) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_e(tmem + d_col, tmem + a_col + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8), desc_add(b, kk * 2048), ID_TS,
                 kk > 0 ? 1u : acc, e);
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(kv_full, 0, BWD_SITE_KV) && mbar_wait(&q_full[0], 0, BWD_SITE_Q) &&
                                          mbar_wait(do_full, 0, BWD_SITE_DO));
    if (ok) {
      tc_fence_after();
      kk_product(C::TM_A, kK, qK);  // S^T(0), then - LSE / scale
      mma_ss_e(tmem + C::TM_A, onesL, ctK, ID_AUG, 1u, e);
      mma_commit_e(s_full, e);
      kk_product(C::TM_B, vK, doK);  // dP^T(0), then - D
      mma_ss_e(tmem + C::TM_B, onesD, ctK, ID_AUG, 1u, e);
      mma_commit_e(dp_full, e);
    }
    for (int st = 0; st < n_steps && ok; ++st) {
      const int qs = st & 1;
      const uint32_t acc = st > 0 ? 1u : 0u;
      // dV += P^T dO_i
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_full, st & 1, BWD_SITE_P)))) break;
      tc_fence_after();
      ts_product(C::TM_DV, C::TM_A, doMN, acc);
      mma_commit_e(do_empty, e);
      // S^T(i+1) into A (P^T(i) has been read by the products above)
      const bool more = st + 1 < n_steps;
      if (more) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qs ^ 1], ((st + 1) >> 1) & 1, BWD_SITE_Q)))) break;
        tc_fence_after();
        kk_product(C::TM_A, kK, desc_add(qK, (qs ^ 1) * C::TILE));
        mma_ss_e(tmem + C::TM_A, onesL, desc_add(ctK, (qs ^ 1) * 4096), ID_AUG, 1u, e);
        mma_commit_e(s_full, e);
      }
      // dK += dS^T Q_i
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(ds_full, st & 1, BWD_SITE_DS)))) break;
      tc_fence_after();
      ts_product(C::TM_DK, C::TM_B, desc_add(qMN, qs * C::TILE), acc);
      mma_commit_e(&q_empty[qs], e);
      // dQ_i = dS K_j into B  (A = dS MN-major in smem, B = K MN-major)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_e(tmem + C::TM_B, desc_add(dsMN, kk * 2048), desc_add(kMN, kk * 2048), ID_DQ, kk > 0 ? 1u : 0u, e);
      mma_commit_e(dq_full, e);
      // dP^T(i+1) into B once dQ_i has been drained
      if (more) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(dq_empty, st & 1, BWD_SITE_DQE)))) break;
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(do_full, (st + 1) & 1, BWD_SITE_DO)))) break;
        tc_fence_after();
        kk_product(C::TM_B, vK, doK);
        mma_ss_e(tmem + C::TM_B, onesD, desc_add(ctK, (qs ^ 1) * 4096), ID_AUG, 1u, e);
        mma_commit_e(dp_full, e);
      }
    }
    mma_commit_e(dkv_full, e);
    mma_commit_e(drain, e);
    mbar_wait(drain, 0, BWD_SITE_DRAIN);
    __syncwarp();
  }
  } else if (warp < 12) {
    regs_inc<136>();
    // ------------------------------------------------------------ P / dS
    // One thread per key row and half of the 128 query columns: warps 4-7
    // take queries 0-63, warps 8-11 queries 64-127.  P and dS are
    // elementwise given LSE and D_i, so the halves never exchange data.
    const int half = (warp - 4) >> 2;
    const int r = (threadIdx.x - 128) & 127;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tA = tmem + lane_off + C::TM_A, tB = tmem + lane_off + C::TM_B;
    const int kv = kv_row0 + r;
    const bool kv_valid = kv < seq_len;
    const float sl2 = p.scale_log2;
    uint8_t* ds_smem = smem + C::DS_OFF;
    bool ok = true;
    for (int st = 0; st < n_steps; ++st) {
      const int i = i_begin + st;
      const int qs = st & 1;
      ok = mbar_wait(s_full, st & 1, BWD_SITE_S) && mbar_wait(&q_full[qs], (st >> 1) & 1, BWD_SITE_STAT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // visible queries of this key row in tile i: q >= kv under the causal mask
      const int qlo = (CAUSAL && i == j) ? r : 0;
      const bool masked = qlo > 64 * half || !kv_valid;  // some column of this half is invisible
      // ---- P phase (score columns 64*half .. +63): the scores already hold
      // -LSE / scale (extra K step), so P^T = 2^(S'^T scale log2 e)
      uint32_t sv[2][32];
      tmem_ld32(tA + 64 * half, sv[0]);
      tmem_ld32(tA + 64 * half + 32, sv[1]);
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
      // dropout keep masks of the 64 query columns: bit e of keep_lo / keep_hi
      // for queries 2e and 2e + 1 of this half.  One Philox call covers query
      // pair e x key quad (4m .. 4m + 3), 16 bits per element, and a key quad
      // sits in four consecutive lanes: lane 4m + c draws query pairs
      // 8c .. 8c + 7, and each lane hands every other lane of its quad that
      // lane's two 16-bit values (XOR shuffles over the quad).
      uint32_t keep_lo = 0xFFFFFFFFu, keep_hi = 0xFFFFFFFFu;
      if constexpr (DROPOUT) {
        const uint32_t c4 = lane & 3u, th = p.drop.thresh;
        const uint32_t keyquad = (uint32_t)kv >> 2, qp0 = (uint32_t)(128 * i + 64 * half) >> 1;
        keep_lo = keep_hi = 0u;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 w = philox4x32_10(make_uint4(keyquad, qp0 + 8 * c4 + k, (uint32_t)head, p.drop.offset),
                                        p.drop.seed_lo, p.drop.seed_hi);
          // key 4m + t: word (t >> 1) for the even query, 2 + (t >> 1) for
          // the odd one; half t & 1 of each; packed (even, odd) as 2 x 16 bits
          auto vals_for = [&w](uint32_t t) -> uint32_t {
            const uint32_t we = (t & 2u) ? w.y : w.x, wo = (t & 2u) ? w.w : w.z;
            return (t & 1u) ? ((we >> 16) | (wo & 0xFFFF0000u)) : ((we & 0xFFFFu) | (wo << 16));
          };
#pragma unroll
          for (uint32_t d = 0; d < 4; ++d) {
            const uint32_t v = d == 0 ? vals_for(c4) : __shfl_xor_sync(0xffffffffu, vals_for(c4 ^ d), (int)d);
            const uint32_t e = 8u * (c4 ^ d) + (uint32_t)k;  // query pair drawn by lane c4 ^ d
            keep_lo |= ((v & 0xFFFFu) < th ? 1u : 0u) << e;
            keep_hi |= ((v >> 16) < th ? 1u : 0u) << e;
          }
        }
      }
      // P^T pairs go to columns [64*half, 64*half + 32) of A (inside this
      // half's own score columns, already read); with dropout the dV operand
      // is P * M (dV is scaled by s = 1 / keep probability at the end)
      if constexpr (DROPOUT) {
        uint32_t pd[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          pd[e] = pk[e] & (((keep_lo >> e) & 1u ? 0x0000FFFFu : 0u) | ((keep_hi >> e) & 1u ? 0xFFFF0000u : 0u));
        tmem_st32(tA + 64 * half, pd);
      } else {
        tmem_st32(tA + 64 * half, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      // ---- dS phase: dS^T = P^T (dP^T - D), P as rounded for the products;
      // dP^T already holds -D (extra K step)
      ok = __all_sync(0xffffffffu, mbar_wait(dp_full, st & 1, BWD_SITE_DP));
      if (!ok) break;
      tc_fence_after();
      uint32_t dv[2][32];
      tmem_ld32(tB + 64 * half, dv[0]);
      tmem_ld32(tB + 64 * half + 32, dv[1]);
      tmem_ld_wait(dv[0]);
      tmem_ld_wait(dv[1]);
      uint32_t dd[32];
      if constexpr (DROPOUT) {
        // dP'^T = dPd^T - D (extra K step).  Kept: dS = P (dPd s - D)
        // = P (dP' s + D (s - 1)); dropped: dS = -P D  (s = 1 / keep probability).
        // D_i of the query rows comes from their per-query row (-D in three
        // bf16 parts, columns 9-11) in shared memory.
        const uint8_t* ct = smem + C::CT_OFF + qs * 4096;
        const float rp = p.drop.scale, rp1 = p.drop.scale - 1.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const uint32_t* src = dv[e >> 4] + 2 * (e & 15);
          float dq[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const uint32_t qrow = (uint32_t)(64 * half + 2 * e + u);
            const uint2 c = *reinterpret_cast<const uint2*>(ct + swz32(qrow * 32u + 16u));
            dq[u] = -(__uint_as_float(c.x & 0xFFFF0000u) + __uint_as_float(c.y << 16) +
                      __uint_as_float(c.y & 0xFFFF0000u));
          }
          const float2 pw = unpack2<BF16>(pk[e]);
          const float a = pw.x * (((keep_lo >> e) & 1u) ? fmaf(__uint_as_float(src[0]), rp, dq[0] * rp1) : -dq[0]);
          const float b = pw.y * (((keep_hi >> e) & 1u) ? fmaf(__uint_as_float(src[1]), rp, dq[1] * rp1) : -dq[1]);
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
      // dS^T pairs to columns [64*half, 64*half + 32) of B (dP columns already read)
      tmem_st32(tB + 64 * half, dd);
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ---- epilogue: dV and scale * dK rows of this key tile
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dkv_full, 0, BWD_SITE_DKV));
    if (ok) {
      tc_fence_after();
      const size_t grow = ((size_t)head * p.rows + row_base + kv) * D;
      {
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
      }
    }
  } else {
    regs_inc<176>();
    // ------------------------------------------------------------ dQ (one thread per query row)
    const int c = threadIdx.x - 384;                 // query row within the tile = TMEM lane
    const int wq = warp - 12;                        // this warp's 32 rows: 32*wq ..
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    uint8_t* stg = smem + C::STG_OFF + wq * 4096;    // 32 rows x 128 B, 128-B swizzled
    if (lane == 0) tma_prefetch_desc(&tm_dq);
    for (int st = 0; st < n_steps; ++st) {
      const int i = i_begin + st;
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, st & 1, BWD_SITE_DQF))) break;
      tc_fence_after();
      uint32_t a[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_off + C::TM_B + 32 * cc, a[cc]);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld_wait(a[cc]);
      tc_fence_before();
      mbar_arrive(dq_empty);
      // This tile's fp32 partial: TMEM -> per-warp swizzled staging -> TMA bulk
      // reduce-add into the accumulator, 32 columns at a time.
      auto reduce_partial = [&]() {
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
            tma_reduce_add_3d(&tm_dq, stg, 32 * cc, row_base + 128 * i + 32 * wq, head);
            bulk_commit();
          }
        }
      };
      if (!p.deterministic) {
        reduce_partial();
      } else {
        // Key tiles add into query tile i in increasing j: one poller per warp
        // waits for our turn, the partial goes in with the same bulk
        // reductions, and the turn passes on only once they have been
        // performed, so every element sees its additions in one fixed order.
        uint32_t* sem = p.sem + ((size_t)head * p.nseq + seq) * p.n_q + i;
        bool ok = true;
        if (lane == 0) {
          if (ld_acquire_gpu(sem) != (uint32_t)j) {
            const uint64_t t0 = global_ns();
            while (ld_acquire_gpu(sem) != (uint32_t)j) {
              if (global_ns() - t0 > kWaitLimitNs) {
                record_error(DEV_ERR_TIMEOUT, BWD_SITE_SEM);
                ok = false;
                break;
              }
            }
          }
          fence_proxy_async_global();  // our reductions come after the acquire
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
          reduce_partial();
          if (lane == 0) {
            bulk_wait0();  // this warp's reductions have been performed
            fence_proxy_async_global();
          }
        }
        __syncwarp();
        mbar_arrive(dq_done);
        if (c == 0) {
          if (mbar_wait(dq_done, st & 1, BWD_SITE_SEM) && ok) {
            __threadfence();
            st_release_gpu(sem, (uint32_t)j + 1);
          }
        }
      }
    }
    if (lane == 0) bulk_wait0();  // every reduction issued by this warp has completed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa

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
//   bwd_pre   D_i = dO_i . O_i (fp32, warp-shuffle reduction), LSE_i*log2(e)
//             into a 128-row-padded copy, zero the fp32 dQ accumulator and
//             the ordering counters.
//   bwd_main  one CTA per 128-row key/value tile j of one head (384 threads):
//               warp 0     TMA producer: K_j, V_j once; then dO_i and Q_i
//                          (plus the padded LSE/D rows of tile i) through a
//                          ring of three shared-memory slots.
//               warp 1     tcgen05 issuer and TMEM owner.  Per query tile i:
//                            dP^T = V_j dO_i^T        -> TMEM [128,256)
//                            S^T  = K_j Q_i^T         -> TMEM [0,128)
//                            dV  += P^T dO_i   (P^T from TMEM)  -> [256,256+D)
//                            dK  += dS^T Q_i   (dS^T from TMEM) -> [256+D,256+2D)
//                            dQ_i = dS K_j     (dS from smem)   -> TMEM [0,D)
//               warps 4-7  one thread per key row: P^T = exp2(S^T*scale*log2e
//                          - LSE*log2e), dS^T = P^T (dP^T - D) in one pass over
//                          32-column chunks; P^T and dS^T go back to TMEM as
//                          16-bit pairs, dS also to shared memory (the A operand
//                          of the dQ product); at the end dV and scale*dK.
//               warps 8-11 one thread per query row: drain dQ_i from TMEM and
//                          add it to the fp32 accumulator (fp32 atomics, or in
//                          key-tile order under deterministic mode).
//   bwd_post  dQ = scale * accumulator, rounded to the input dtype.
// Causal: key tile j only meets query tiles i >= j; only the diagonal tile
// is masked element-wise.
#pragma once

#include "sm100.cuh"

namespace fa {

struct BwdParams {
  void* dk;                // [heads, S, D]
  void* dv;                // [heads, S, D]
  float* dq_acc;           // [heads, S, D] fp32
  const float* lse2;       // [heads, S_pad]  LSE * log2(e), +inf in padding rows
  const float* delta;      // [heads, S_pad]  D_i, 0 in padding rows
  float* lse2_w;           // the same two buffers, written by bwd_pre
  float* delta_w;
  uint32_t* sem;           // [heads, n_q] ordering counters (deterministic mode)
  int heads, S, S_pad, n_q;
  float scale, scale_log2;
  int deterministic;
};

template <int D>
struct BwdCfg {
  static constexpr int CH = D / 64;
  static constexpr uint32_t CHUNK = 128u * 128u;
  static constexpr uint32_t TILE = CH * CHUNK;
  static constexpr int NSLOT = 3;                        // ring for dO_i / Q_i
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = TILE;
  static constexpr uint32_t RING_OFF = 2 * TILE;
  static constexpr uint32_t DS_OFF = RING_OFF + NSLOT * TILE;   // 128 x 128 16-bit, 2 chunks
  static constexpr uint32_t STAT_OFF = DS_OFF + 2 * CHUNK;      // NSLOT x (128 lse2 + 128 delta) fp32
  static constexpr uint32_t BAR_OFF = STAT_OFF + NSLOT * 1024;
  // kv_full ring_full[3] ring_empty[3] s_full dp_full pds_full dq_full dq_empty dkv_full drain dq_done
  static constexpr int NBAR = 1 + 2 * NSLOT + 8;
  static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D, TM_DQ = 0;
};

enum : uint32_t {
  BWD_SITE_PROD = 0x200, BWD_SITE_KV = 0x201, BWD_SITE_RING = 0x202, BWD_SITE_PDS = 0x203,
  BWD_SITE_DQE = 0x204, BWD_SITE_S = 0x205, BWD_SITE_DQF = 0x206, BWD_SITE_DKV = 0x207,
  BWD_SITE_SEM = 0x208, BWD_SITE_DRAIN = 0x209, BWD_SITE_STAT = 0x20a
};

// ---------------------------------------------------------------------------
// bwd_pre: one group of D/8 lanes per row, 16-byte loads, shuffle reduction.
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      const float* __restrict__ lse, BwdParams p) {
  constexpr int G = D / 8;  // lanes per row
  const long long work = (long long)p.heads * p.S_pad * G;
  const long long bound = (work + 31) / 32 * 32;  // whole warps take the same trips
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * blockDim.x;
  for (long long idx = gtid; idx < bound; idx += nthreads) {
    const bool in = idx < work;
    const long long row = idx / G;
    const int part = (int)(idx % G);
    const int h = in ? (int)(row / p.S_pad) : 0;
    const int s = in ? (int)(row % p.S_pad) : p.S;
    float acc = 0.f;
    if (s < p.S) {
      const size_t off = ((size_t)h * p.S + s) * D + part * 8;
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
      p.delta_w[row] = s < p.S ? acc : 0.f;
      p.lse2_w[row] = s < p.S ? lse[(size_t)h * p.S + s] * 1.4426950408889634f : INFINITY;
    }
  }
  // zero the dQ accumulator (16-byte stores) and the ordering counters
  const long long n4 = (long long)p.heads * p.S * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long i = gtid; i < n4; i += nthreads) acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  const long long ns = (long long)p.heads * p.n_q;
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

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

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
template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  const int j = blockIdx.x / p.heads;       // key/value tile (ascending: longest causal work first)
  const int head = blockIdx.x - j * p.heads;
  const int i_begin = CAUSAL ? j : 0;
  const int n_steps = p.n_q - i_begin;
  const int kv_row0 = 128 * j;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* ring_full = bars + 1;
  uint64_t* ring_empty = ring_full + C::NSLOT;
  uint64_t* s_full = ring_empty + C::NSLOT;
  uint64_t* dp_full = s_full + 1;
  uint64_t* pds_full = dp_full + 1;
  uint64_t* dq_full = pds_full + 1;
  uint64_t* dq_empty = dq_full + 1;
  uint64_t* dkv_full = dq_empty + 1;
  uint64_t* drain = dkv_full + 1;
  uint64_t* dq_done = drain + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  float* stats = reinterpret_cast<float*>(smem + C::STAT_OFF);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(pds_full, 128);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(kv_full, 2 * C::TILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(smem + C::K_OFF + c * C::CHUNK, &tm_k, kv_full, c * 64, kv_row0, head);
        tma_load_3d(smem + C::V_OFF + c * C::CHUNK, &tm_v, kv_full, c * 64, kv_row0, head);
      }
      uint32_t fill = 0;
      bool ok = true;
      for (int st = 0; st < n_steps && ok; ++st) {
        const int i = i_begin + st;
        for (int which = 0; which < 2; ++which) {  // 0: dO_i, 1: Q_i (+ its LSE/D rows)
          const uint32_t slot = fill % C::NSLOT, round = fill / C::NSLOT;
          if (round > 0 && !mbar_wait(&ring_empty[slot], (round - 1) & 1, BWD_SITE_PROD)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&ring_full[slot], C::TILE + (which ? 1024u : 0u));
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::RING_OFF + slot * C::TILE + c * C::CHUNK, which ? &tm_q : &tm_do, &ring_full[slot],
                        c * 64, 128 * i, head);
          if (which) {
            const size_t srow = (size_t)head * p.S_pad + 128 * i;
            bulk_load(stats + slot * 256, p.lse2 + srow, 512, &ring_full[slot]);
            bulk_load(stats + slot * 256 + 128, p.delta + srow, 512, &ring_full[slot]);
          }
          ++fill;
        }
      }
      for (uint32_t f = (fill > (uint32_t)C::NSLOT ? fill - C::NSLOT : 0); f < fill; ++f)
        mbar_wait(&ring_full[f % C::NSLOT], (f / C::NSLOT) & 1, BWD_SITE_PROD);
      mbar_wait(kv_full, 0, BWD_SITE_PROD);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_KK = make_idesc(128, 128, BF16, false, false);  // dP^T, S^T
      constexpr uint32_t ID_TS = make_idesc(128, D, BF16, false, true);     // dV, dK
      constexpr uint32_t ID_DQ = make_idesc(128, D, BF16, true, true);      // dQ
      const uint32_t sk = smem_addr(smem + C::K_OFF), sv = smem_addr(smem + C::V_OFF);
      const uint32_t sring = smem_addr(smem + C::RING_OFF), sds = smem_addr(smem + C::DS_OFF);
      bool ok = mbar_wait(kv_full, 0, BWD_SITE_KV);
      uint32_t use = 0;
      for (int st = 0; st < n_steps && ok; ++st) {
        const uint32_t so = use % C::NSLOT;
        if (!(ok = mbar_wait(&ring_full[so], (use / C::NSLOT) & 1, BWD_SITE_RING))) break;
        ++use;
        const uint32_t sqs = use % C::NSLOT;
        // dP^T = V dO^T  (M = keys, N = queries, K = D; both K-major)
        {
          const uint32_t da = sring + so * C::TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
            mma_ss(tmem + C::TM_DP, make_sdesc(sv + off, 16, 1024), make_sdesc(da + off, 16, 1024), ID_KK, kk > 0);
          }
          mma_commit(dp_full);
        }
        if (!(ok = mbar_wait(&ring_full[sqs], (use / C::NSLOT) & 1, BWD_SITE_RING))) break;
        ++use;
        // the previous dQ_i has left TMEM [0, D)
        if (st > 0 && !(ok = mbar_wait(dq_empty, (st - 1) & 1, BWD_SITE_DQE))) break;
        tc_fence_after();
        // S^T = K Q^T
        {
          const uint32_t qa = sring + sqs * C::TILE;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
            mma_ss(tmem + C::TM_S, make_sdesc(sk + off, 16, 1024), make_sdesc(qa + off, 16, 1024), ID_KK, kk > 0);
          }
          mma_commit(s_full);
        }
        if (!(ok = mbar_wait(pds_full, st & 1, BWD_SITE_PDS))) break;
        tc_fence_after();
        // dV += P^T dO  (A = P^T in TMEM [0,64), B = dO MN-major)
        {
          const uint32_t da = sring + so * C::TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + C::TM_DV, tmem + C::TM_S + kk * 8, make_sdesc(da + kk * 2048, C::CHUNK, 1024), ID_TS,
                   (st > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&ring_empty[so]);
        }
        // dK += dS^T Q  (A = dS^T in TMEM [128,192), B = Q MN-major)
        {
          const uint32_t qa = sring + sqs * C::TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + C::TM_DK, tmem + C::TM_DP + kk * 8, make_sdesc(qa + kk * 2048, C::CHUNK, 1024), ID_TS,
                   (st > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&ring_empty[sqs]);
        }
        // dQ_i = dS K  (M = queries: A = dS MN-major in smem; B = K MN-major)
        {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + C::TM_DQ, make_sdesc(sds + kk * 2048, C::CHUNK, 1024),
                   make_sdesc(sk + kk * 2048, C::CHUNK, 1024), ID_DQ, kk > 0);
          mma_commit(dq_full);
        }
      }
      mma_commit(dkv_full);
      mma_commit(drain);
      mbar_wait(drain, 0, BWD_SITE_DRAIN);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ P / dS (one thread per key row)
    const int r = threadIdx.x - 128;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int kv = kv_row0 + r;
    const bool kv_valid = kv < p.S;
    const float sl2 = p.scale_log2;
    uint8_t* ds_smem = smem + C::DS_OFF;
    bool ok = true;
    for (int st = 0; st < n_steps; ++st) {
      const int i = i_begin + st;
      const uint32_t use_q = 2 * st + 1;
      ok = mbar_wait(s_full, st & 1, BWD_SITE_S);
      ok = ok && mbar_wait(dp_full, st & 1, BWD_SITE_S);
      ok = ok && mbar_wait(&ring_full[use_q % C::NSLOT], (use_q / C::NSLOT) & 1, BWD_SITE_STAT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = stats + (use_q % C::NSLOT) * 256;
      const float* dlt = lse2 + 128;
      // visible queries of this key row in tile i: q >= kv under the causal mask
      const int qlo = (CAUSAL && i == j) ? r : 0;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tmem + lane_off + C::TM_S + 32 * ch, sv);
        tmem_ld32(tmem + lane_off + C::TM_DP + 32 * ch, dv);
        tmem_ld_wait(sv);
        tmem_ld_wait(dv);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float pr[2], dsr[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = 32 * ch + 2 * e + u;
            float pe = ex2(fmaf(__uint_as_float(sv[2 * e + u]), sl2, -lse2[c]));
            if (c < qlo || !kv_valid) pe = 0.f;
            pr[u] = pe;
            dsr[u] = pe * (__uint_as_float(dv[2 * e + u]) - dlt[c]);
          }
          pp[e] = pack2<BF16>(pr[0], pr[1]);
          dd[e] = pack2<BF16>(dsr[0], dsr[1]);
        }
        tmem_st16(tmem + lane_off + C::TM_S + 16 * ch, pp);
        tmem_st16(tmem + lane_off + C::TM_DP + 16 * ch, dd);
        // dS row r (key) holds 32 query columns of chunk ch: MN-major A operand
        // of dQ = dS K, i.e. [key][query] with queries contiguous, 128-B swizzled.
        const uint32_t colbyte = (ch & 1) * 64;               // 32 queries = 64 B inside the 128-B row
        const uint32_t base = (ch >> 1) * C::CHUNK + r * 128;  // 64-query chunk, key row
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint32_t off = swz128(base + colbyte + v4 * 16);
          *reinterpret_cast<uint4*>(ds_smem + off) = make_uint4(dd[4 * v4], dd[4 * v4 + 1], dd[4 * v4 + 2], dd[4 * v4 + 3]);
        }
      }
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(pds_full);
    }
    // ---- epilogue: dV and scale * dK rows of this key tile
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(dkv_full, 0, BWD_SITE_DKV));
    if (ok) {
      tc_fence_after();
      const size_t grow = ((size_t)head * p.S + kv) * D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(which ? p.dk : p.dv) + grow);
        const float mul = which ? p.scale : 1.f;
        const uint32_t col = which ? C::TM_DK : C::TM_DV;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + col + 32 * cc, ov);
          tmem_ld_wait(ov);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack2<BF16>(__uint_as_float(ov[2 * e]) * mul, __uint_as_float(ov[2 * e + 1]) * mul);
          if (kv_valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[cc * 4 + e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dQ drain (one thread per query row)
    const int c = threadIdx.x - 256;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    for (int st = 0; st < n_steps; ++st) {
      const int i = i_begin + st;
      if (!__all_sync(0xffffffffu, mbar_wait(dq_full, st & 1, BWD_SITE_DQF))) break;
      tc_fence_after();
      uint32_t a[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tmem + lane_off + C::TM_DQ + 32 * cc, a[cc]);
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld_wait(a[cc]);
      tc_fence_before();
      mbar_arrive(dq_empty);
      const int q = 128 * i + c;
      uint32_t* sem = p.sem + (size_t)head * p.n_q + i;
      if (p.deterministic) {
        // key tiles add into query tile i in increasing j: wait for our turn
        bool ok = true;
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
        if (ok && q < p.S) {
          float4* dst = reinterpret_cast<float4*>(p.dq_acc + ((size_t)head * p.S + q) * D);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 v = dst[cc * 8 + e];
              v.x += __uint_as_float(a[cc][4 * e]);
              v.y += __uint_as_float(a[cc][4 * e + 1]);
              v.z += __uint_as_float(a[cc][4 * e + 2]);
              v.w += __uint_as_float(a[cc][4 * e + 3]);
              dst[cc * 8 + e] = v;
            }
        }
        // every thread's adds are visible device-wide before the counter
        // moves on (bounded wait on an arrival barrier, no bar.sync)
        __threadfence();
        mbar_arrive(dq_done);
        if (c == 0) {
          if (mbar_wait(dq_done, st & 1, BWD_SITE_SEM) && ok) {
            __threadfence();
            st_release_gpu(sem, (uint32_t)j + 1);
          }
        }
      } else if (q < p.S) {
        float4* dst = reinterpret_cast<float4*>(p.dq_acc + ((size_t)head * p.S + q) * D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicAdd(&dst[cc * 8 + e], make_float4(__uint_as_float(a[cc][4 * e]), __uint_as_float(a[cc][4 * e + 1]),
                                                     __uint_as_float(a[cc][4 * e + 2]),
                                                     __uint_as_float(a[cc][4 * e + 3])));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa

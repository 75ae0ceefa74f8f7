// fa_fwd.cuh - forward kernel of exact tiled attention on sm_100a.
//
// What it computes (per head, per query row i):
//     m_i = max_j s_ij,  l_i = sum_j exp(s_ij - m_i),  O_i = sum_j exp(s_ij - m_i) v_j / l_i,
//     LSE_i = m_i + ln l_i,        s_ij = scale * q_i . k_j  over the visible keys j,
// visiting the keys one 128-row K/V tile at a time with the running-max /
// running-sum update of "From Self-Attention to FlashAttention", §二 (the
// running sum and the unnormalised output are rescaled by exp(m_old - m_new)
// whenever the row maximum grows, and O is divided by the running sum once at
// the end).  Each Q tile stays on chip while the K/V tiles stream past, and
// only O and the per-row LSE are written back ("ops-transformer里的FlashAttention",
// "核心计算流程" and "在线softmax" for the structure; its printed per-block
// update divides inside the loop and is not followed).
//
// B200 mapping (one CTA = two 128-row query tiles of one head, 384 threads):
//   warp 0      TMA producer: Q tiles once, then K_j, V_j into a ring of
//               NSLOT shared-memory slots (128-byte swizzled 64-column chunks).
//   warp 1      tcgen05 issuer (one lane): S_t = Q_t K_j^T (SS form) into
//               TMEM, then O_t += P_t V_j with P_t read from TMEM (TS form).
//               Also owns the 512-column TMEM allocation.
//   warps 4-7   softmax for query tile 0, warps 8-11 for tile 1: one thread
//               per row (TMEM lane); scores are taken to the log2 domain
//               (scale * log2 e) and exponentiated with ex2; P is written
//               back into the first 64 columns of the S_t it came from, as
//               packed 16-bit pairs; O_t and the running sums are rescaled
//               when the row max grows (the TMEM loads of O_t are issued
//               ahead of the exponentials that hide them); the sum that
//               normalises O adds the P values as rounded for the P V
//               product; at the end O_t / l and LSE go to global memory.
//   The two query tiles ping-pong: while one softmax group works, the
//   tensor core runs the other tile's products.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Fully masked causal tiles are never loaded or multiplied.
#pragma once

#include "sm100.cuh"

namespace fa {

struct FwdParams {
  void* o;                // [heads, rows, D]
  float* lse;             // [heads, rows]
  const int* cu_seqlens;  // packed batch only: device int32 [nseq + 1]
  int heads;              // dense: B*H, packed: H
  int seqlen;             // dense: S, packed: max_seqlen
  int rows;               // rows of one head slice in memory: S or total
  int nseq;               // dense: 1
  int n_pairs;            // ceil(seqlen / 256)
  float scale_log2;       // scale * log2(e)
};

template <int D>
struct FwdCfg {
  static constexpr int CH = D / 64;                      // 64-column chunks of a tile
  static constexpr uint32_t CHUNK = 128u * 128u;         // 128 rows x 128 bytes
  static constexpr uint32_t TILE = CH * CHUNK;           // one 128 x D tile
  static constexpr int NSLOT = (D == 128) ? 4 : 8;       // K/V ring depth
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = 2 * TILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NSLOT * TILE;
  // q_full[2] kv_full[NSLOT] kv_empty[NSLOT] s_full[2] p_half[4] o_full[2] drain
  static constexpr int NBAR = 2 + 2 * NSLOT + 9;
  static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TM_S = 0, TM_O = 256;
  static constexpr int THREADS = 384;
};

// Row-max growth (log2 units) tolerated before O and l are rescaled.  Zero
// keeps the exact running max, so the dominant P of every row is exactly 1
// and only the smaller weights carry 16-bit rounding into P V.
constexpr float kRescaleLog2 = 0.f;

// wait-site ids reported through the error word
enum : uint32_t {
  FWD_SITE_PROD = 0x100, FWD_SITE_Q = 0x101, FWD_SITE_KV = 0x102, FWD_SITE_P = 0x103,
  FWD_SITE_S = 0x104, FWD_SITE_O = 0x105, FWD_SITE_DRAIN = 0x106
};

template <int D, bool BF16, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using C = FwdCfg<D>;

  // ---- work unit: (query pair w, sequence, head), longest causal rows first
  const int per_w = p.nseq * p.heads;
  const int wi = blockIdx.x / per_w;
  const int rem = blockIdx.x - wi * per_w;
  const int w = CAUSAL ? (p.n_pairs - 1 - wi) : wi;
  const int seq = rem / p.heads;
  const int head = rem - seq * p.heads;
  int row_base = 0, seq_len = p.seqlen;
  if constexpr (VARLEN) {
    row_base = p.cu_seqlens[seq];
    seq_len = p.cu_seqlens[seq + 1] - row_base;
  }
  const int q_start = w * 256;
  if (q_start >= seq_len) return;  // uniform over the CTA, before any set-up

  const bool has_t1 = q_start + 128 < seq_len;
  const int n_kv_all = (seq_len + 127) / 128;
  int n0, n1;
  if constexpr (CAUSAL) {
    n0 = min(2 * w + 1, n_kv_all);
    n1 = has_t1 ? min(2 * w + 2, n_kv_all) : 0;
  } else {
    n0 = n_kv_all;
    n1 = has_t1 ? n_kv_all : 0;
  }
  const int n_kv = max(n0, n1);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + C::NSLOT;
  uint64_t* s_full = kv_empty + C::NSLOT;
  uint64_t* p_half = s_full + 2;  // [2 * tile + half]: P keys 0-63 / 64-127 written
  uint64_t* o_full = p_half + 4;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_half[2 * i], 128);
      mbar_init(&p_half[2 * i + 1], 128);
      mbar_init(&o_full[i], 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(drain, 1);
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
  const uint32_t sq = smem_addr(smem + C::Q_OFF);
  const uint32_t skv = smem_addr(smem + C::KV_OFF);

  // register split: 128 x 56 (warps 0-3) + 256 x 208 (softmax) = 60416 <= 384 x 168.
  // Each warpgroup changes its budget inside its own branch so the compiler
  // allocates every role with the budget it runs under.
  if (warp < 4) {
  regs_dec<56>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      for (int t = 0; t < 2; ++t) {
        if (t == 1 && !has_t1) break;
        mbar_expect_tx(&q_full[t], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(smem + C::Q_OFF + t * C::TILE + c * C::CHUNK, &tm_q, &q_full[t], c * 64,
                      row_base + q_start + 128 * t, head);
      }
      uint32_t fill = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int which = 0; which < 2; ++which) {
          const uint32_t slot = fill % C::NSLOT, round = fill / C::NSLOT;
          if (round > 0 && !mbar_wait(&kv_empty[slot], (round - 1) & 1, FWD_SITE_PROD)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&kv_full[slot], C::TILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::KV_OFF + slot * C::TILE + c * C::CHUNK, which ? &tm_v : &tm_k, &kv_full[slot],
                        c * 64, row_base + 128 * j, head);
          ++fill;
        }
      }
      // Never leave a tile copy in flight into shared memory we are about to
      // give back: wait for the newest fill of every slot (already complete
      // on the normal path).
      for (uint32_t f = (fill > (uint32_t)C::NSLOT ? fill - C::NSLOT : 0); f < fill; ++f)
        mbar_wait(&kv_full[f % C::NSLOT], (f / C::NSLOT) & 1, FWD_SITE_PROD);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this converged; one elected lane issues.  Operand
    // descriptors are formed once and offset by constants inside each fully
    // unrolled group of products.
    const uint32_t e = elect_one();
    constexpr uint32_t IDESC_QK = make_idesc(128, 128, BF16, false, false);
    constexpr uint32_t IDESC_PV = make_idesc(128, D, BF16, false, true);
    const uint64_t dq_base = make_sdesc(sq, 16, 1024);         // Q tile 0, K-major
    const uint64_t dk_base = make_sdesc(skv, 16, 1024);        // K/V slot 0 as K (K-major)
    const uint64_t dv_base = make_sdesc(skv, C::CHUNK, 1024);  // K/V slot 0 as V (MN-major)
    uint32_t use = 0;
    bool ok = __all_sync(0xffffffffu, mbar_wait(&q_full[0], 0, FWD_SITE_Q));
    auto next_slot = [&](uint32_t& slot) {
      slot = use % C::NSLOT;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[slot], (use / C::NSLOT) & 1, FWD_SITE_KV));
      ++use;
    };
    // S_t = Q_t K^T: M = 128 query rows, N = 128 keys, K = D (both K-major)
    auto qk = [&](int t, uint32_t kslot) {
      const uint64_t a = desc_add(dq_base, t * C::TILE), b = desc_add(dk_base, kslot * C::TILE);
      const uint32_t d = tmem + C::TM_S + 128 * t;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
        mma_ss_e(d, desc_add(a, off), desc_add(b, off), IDESC_QK, kk > 0 ? 1u : 0u, e);
      }
    };
    // O_t += P_t V: M = 128, N = D, K = 128 keys; P from TMEM, V MN-major.
    // Keys 0-63 (k-steps 0-3) once the first half of P is published, keys
    // 64-127 once the second is.
    auto pv = [&](int t, uint32_t vslot, uint32_t acc, int j) -> bool {
      const uint64_t b = desc_add(dv_base, vslot * C::TILE);
      const uint32_t d = tmem + C::TM_O + D * t, pa = tmem + C::TM_S + 128 * t;
      if (!__all_sync(0xffffffffu, mbar_wait(&p_half[2 * t], j & 1, FWD_SITE_P))) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts_e(d, pa + kk * 8, desc_add(b, kk * 2048), IDESC_PV, kk > 0 ? 1u : acc, e);
      if (!__all_sync(0xffffffffu, mbar_wait(&p_half[2 * t + 1], j & 1, FWD_SITE_P))) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 4; kk < 8; ++kk) mma_ts_e(d, pa + kk * 8, desc_add(b, kk * 2048), IDESC_PV, 1u, e);
      return true;
    };

    uint32_t ks = 0;
    next_slot(ks);
    if (ok) {
      tc_fence_after();
      qk(0, ks);
      mma_commit_e(&s_full[0], e);
      if (has_t1) {
        ok = __all_sync(0xffffffffu, mbar_wait(&q_full[1], 0, FWD_SITE_Q));
        if (ok) {
          qk(1, ks);
          mma_commit_e(&s_full[1], e);
        }
      }
      mma_commit_e(&kv_empty[ks], e);
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      uint32_t vs = 0;
      next_slot(vs);
      if (!ok) break;
      if (j < n0) {
        if (!(ok = pv(0, vs, j > 0 ? 1u : 0u, j))) break;
        if (j == n0 - 1) mma_commit_e(&o_full[0], e);
      }
      const bool more = j + 1 < n_kv;
      uint32_t ks2 = 0;
      if (more) {
        next_slot(ks2);
        if (!ok) break;
        if (j + 1 < n0) {
          qk(0, ks2);
          mma_commit_e(&s_full[0], e);
        }
      }
      if (j < n1) {
        if (!(ok = pv(1, vs, j > 0 ? 1u : 0u, j))) break;
        if (j == n1 - 1) mma_commit_e(&o_full[1], e);
      }
      mma_commit_e(&kv_empty[vs], e);
      if (more) {
        if (j + 1 < n1) {
          qk(1, ks2);
          mma_commit_e(&s_full[1], e);
        }
        mma_commit_e(&kv_empty[ks2], e);
      }
    }
    // every product issued above has finished before TMEM is released
    mma_commit_e(drain, e);
    mbar_wait(drain, 0, FWD_SITE_DRAIN);
    __syncwarp();
  }
  } else {
    regs_inc<208>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int n_t = t == 0 ? n0 : n1;
    const int r = threadIdx.x - 128 * (1 + t);
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 128 * t;
    const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
    const int row = q_start + 128 * t + r;  // row inside the sequence
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, FWD_SITE_S));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32], s2[32], s3[32];
      tmem_ld32(tS + 0, s0);
      tmem_ld32(tS + 32, s1);
      tmem_ld32(tS + 64, s2);
      tmem_ld32(tS + 96, s3);
      tmem_ld_wait(s0);
      tmem_ld_wait(s1);
      tmem_ld_wait(s2);
      tmem_ld_wait(s3);
      float* x0 = reinterpret_cast<float*>(s0);
      float* x1 = reinterpret_cast<float*>(s1);
      float* x2 = reinterpret_cast<float*>(s2);
      float* x3 = reinterpret_cast<float*>(s3);
      // keys this row may see in this tile: [0, limit)
      const int kv0 = 128 * j;
      int limit = min(128, seq_len - kv0);
      if constexpr (CAUSAL) limit = min(limit, row - kv0 + 1);
      if (limit < 128) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c >= limit) x0[c] = -INFINITY;
          if (c + 32 >= limit) x1[c] = -INFINITY;
          if (c + 64 >= limit) x2[c] = -INFINITY;
          if (c + 96 >= limit) x3[c] = -INFINITY;
        }
      }
      // row max as a tree of independent 3-input maxima
      float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        mxa = fmax3(mxa, x0[c], x0[c + 1]);
        mxb = fmax3(mxb, x1[c], x1[c + 1]);
        mxc = fmax3(mxc, x2[c], x2[c + 1]);
        mxd = fmax3(mxd, x3[c], x3[c + 1]);
      }
      const float mx = fmax3(mxa, mxb, fmaxf(mxc, mxd));
      // Rescale O and the running sums only when the row max actually grew
      // (by more than kRescaleLog2): every P is then <= 2^kRescaleLog2, and
      // with kRescaleLog2 = 0 the largest P of the row is exactly 1.
      const float m_max = fmaxf(m, mx * sl2);
      const bool rescale = m_max > m + kRescaleLog2;  // false while the row has no visible key
      const float m_new = rescale ? m_max : m;
      const float alpha = rescale ? ex2(m - m_new) : 1.f;  // ex2(-inf) = 0 on the first tile
      const float neg = (m_new == -INFINITY) ? 0.f : -m_new;
      const uint64_t scale2 = f2(sl2, sl2), neg2 = f2(neg, neg);
      // fsum: fp32 sum of P (for LSE); rsum: sum of P as rounded to 16 bits
      // (the weights the P V product uses, for normalising O).
      uint64_t fsum0 = f2(0.f, 0.f), fsum1 = f2(0.f, 0.f), rsum0 = f2(0.f, 0.f), rsum1 = f2(0.f, 0.f);
      auto finish_pair = [&](float a, float b, uint64_t& fs, uint64_t& rs) -> uint32_t {
        fs = fadd2(fs, f2(a, b));
        const uint32_t pk = pack2<BF16>(a, b);
        rs = fadd2(rs, widen2<BF16>(pk));
        return pk;
      };
      // P from the special-function unit
      auto exp_sfu = [&](float x, float y, uint64_t& fs, uint64_t& rs) -> uint32_t {
        float a, b;
        f2split(ffma2(f2(x, y), scale2, neg2), a, b);
        return finish_pair(ex2(a), ex2(b), fs, rs);
      };
      // P from the FMA pipe (exp2_poly2): used for the last 32 columns of
      // tiles every row of this warp sees in full, to share the exponentials
      // between the two pipes.
      const bool full_tile = __all_sync(0xffffffffu, limit == 128);
      auto exp_fma = [&](float x, float y, uint64_t& fs, uint64_t& rs) -> uint32_t {
        float a, b;
        f2split(exp2_poly2(ffma2(f2(x, y), scale2, neg2)), a, b);
        return finish_pair(a, b, fs, rs);
      };
      // O_t (written by the previous P V product, complete once S_t arrived)
      // is rescaled 32 columns at a time while the first half of P is made;
      // each load is issued one step ahead so its latency hides behind the
      // exponentials.  The first half of P (keys 0-63) is published before the
      // second is computed, so the P V product can start on it.
      const bool do_rs = j > 0 && __any_sync(0xffffffffu, rescale);
      const uint64_t alpha2 = f2(alpha, alpha);
      uint32_t ov[32];
      auto rescale_chunk = [&](int cc) {
        if (!do_rs || cc >= D / 32) return;
        tmem_ld_wait(ov);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a, b;
          f2split(fmul2(f2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1])), alpha2), a, b);
          ov[2 * i] = __float_as_uint(a);
          ov[2 * i + 1] = __float_as_uint(b);
        }
        tmem_st32(tO + 32 * cc, ov);
        if (cc + 1 < D / 32) tmem_ld32(tO + 32 * (cc + 1), ov);
      };
      if (do_rs) tmem_ld32(tO, ov);
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = exp_sfu(x0[2 * i], x0[2 * i + 1], fsum0, rsum0);
        rescale_chunk(0);
#pragma unroll
        for (int i = 8; i < 16; ++i) pk[i] = exp_sfu(x0[2 * i], x0[2 * i + 1], fsum1, rsum1);
        rescale_chunk(1);
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[16 + i] = exp_sfu(x1[2 * i], x1[2 * i + 1], fsum0, rsum0);
        rescale_chunk(2);
#pragma unroll
        for (int i = 8; i < 16; ++i) pk[16 + i] = exp_sfu(x1[2 * i], x1[2 * i + 1], fsum1, rsum1);
        rescale_chunk(3);
        tmem_st32(tS + 0, pk);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_half[2 * t]);
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = exp_sfu(x2[2 * i], x2[2 * i + 1], fsum0, rsum0);
        if (full_tile) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[16 + i] = exp_fma(x3[2 * i], x3[2 * i + 1], fsum1, rsum1);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[16 + i] = exp_sfu(x3[2 * i], x3[2 * i + 1], fsum1, rsum1);
        }
        tmem_st32(tS + 32, pk);
      }
      // l (fp32 sum) gives LSE; lr (sum of the rounded P) normalises O, so
      // O / lr is a convex combination of the V rows with exactly the weights
      // the P V product used.
      float f0, f1, f2_, f3, r0, r1, r2, r3;
      f2split(fsum0, f0, f1);
      f2split(fsum1, f2_, f3);
      f2split(rsum0, r0, r1);
      f2split(rsum1, r2, r3);
      l = l * alpha + ((f0 + f1) + (f2_ + f3));
      lr = lr * alpha + ((r0 + r1) + (r2 + r3));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_half[2 * t + 1]);
      m = m_new;
    }
    // ---- epilogue: O / l and LSE for the rows inside the sequence
    if (ok && n_t > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[t], 0, FWD_SITE_O));
      if (ok) {
        tc_fence_after();
        const float inv = lr > 0.f ? 1.f / lr : 0.f;
        const bool valid = row < seq_len;
        const size_t grow = (size_t)head * p.rows + row_base + row;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + grow * D);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tO + 32 * cc, ov);
          tmem_ld_wait(ov);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
          if (valid) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[cc * 4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        if (valid) p.lse[grow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }

  // ---- teardown: every TMEM access above has completed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa

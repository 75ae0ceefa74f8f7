// fa_fwd.cuh - forward kernel of exact tiled attention on sm_100a.
//
// What it computes (per head, per query row i):
//     m_i = max_j s_ij,  l_i = sum_j exp(s_ij - m_i),  O_i = sum_j exp(s_ij - m_i) v_j / l_i,
//     LSE_i = m_i + ln l_i,        s_ij = scale * q_i . k_j  over the visible keys j,
// visiting the keys one K/V tile at a time with the running-max / running-sum
// update of "From Self-Attention to FlashAttention", §二 (the running sum and
// the unnormalised output are rescaled by exp(m_old - m_new) whenever the row
// maximum grows, and O is divided by the running sum once at the end).  Each
// Q tile stays on chip while the K/V tiles stream past, and only O and the
// per-row LSE are written back ("ops-transformer里的FlashAttention",
// "核心计算流程" and "在线softmax" for the structure; its printed per-block
// update divides inside the loop and is not followed).
//
// B200 mapping: one CTA = two 128-row query tiles of one head, K/V tiles of
// 64 keys, 512 threads in four warpgroups:
//   warp 0      TMA producer: the Q tiles once, then K_0, K_1, and (V_j,
//               K_{j+2}) for j = 0, 1, ... into a ring of shared-memory
//               slots, which is the order the tensor core consumes them in.
//   warp 1      tcgen05 issuer (converged warp, one elected lane) and TMEM
//               owner.  Each query tile t has two S buffers, so the product
//               S_t(j+2) = Q_t K_{j+2}^T goes in right behind
//               O_t += P_t(j) V_j and is ready before the softmax needs it.
//   warps 4-7   softmax of query tile 0, warps 8-11 of tile 1: one thread per
//               row (TMEM lane): row max of the 64 scores, exponentials in
//               the log2 domain (scale * log2 e folded into one FFMA), P as
//               16-bit pairs written back over the scores it came from, the
//               fp32 running sum (for LSE) and the running sum of P as
//               rounded for the P V product (to normalise O).
//   warps 12-15 correction: when a row max grows, rescale that tile's O
//               accumulator in TMEM by exp(m_old - m_new) while the softmax is
//               still exponentiating; at the end, O / l and LSE to global.
// TMEM columns: S0a [0,64) S0b [64,128) S1a [128,192) S1b [192,256),
//               O0 [256,256+D), O1 [256+D,256+2D).
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
  static constexpr int CH = D / 64;                  // 64-column chunks of a tile
  static constexpr uint32_t QCHUNK = 128u * 128u;    // 128 rows x 128 bytes
  static constexpr uint32_t KCHUNK = 64u * 128u;     // 64 rows x 128 bytes
  static constexpr uint32_t QTILE = CH * QCHUNK;     // one 128 x D query tile
  static constexpr uint32_t KTILE = CH * KCHUNK;     // one 64 x D key or value tile
  static constexpr int NSLOT = (D == 128) ? 8 : 16;  // K/V ring depth (128 KB)
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = 2 * QTILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NSLOT * KTILE;
  // q_full[2] kv_full[N] kv_empty[N] s_full[4] p_full[4] a_ready[2] o_ready[2]
  // pv_done[2] stats_ready[2] o_full[2] drain
  static constexpr int NBAR = 2 + 2 * NSLOT + 4 + 4 + 2 + 2 + 2 + 2 + 2 + 1;
  // alpha[tile][parity][128] and the final (m, l, lr)[tile][3][128], fp32
  static constexpr uint32_t XCH_OFF = (BAR_OFF + NBAR * 8 + 16 + 15) & ~15u;
  static constexpr uint32_t XCH_BYTES = (2 * 2 * 128 + 2 * 3 * 128) * 4;
  static constexpr uint32_t SMEM = XCH_OFF + XCH_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TM_S = 0, TM_O = 256;
  static constexpr int THREADS = 512;
};

// Row-max growth (log2 units) tolerated before O and l are rescaled.  Zero
// keeps the exact running max, so the dominant P of every row is exactly 1
// and only the smaller weights carry 16-bit rounding into P V.
constexpr float kRescaleLog2 = 0.f;

// wait-site ids reported through the error word
enum : uint32_t {
  FWD_SITE_PROD = 0x100, FWD_SITE_Q = 0x101, FWD_SITE_KV = 0x102, FWD_SITE_P = 0x103, FWD_SITE_S = 0x104,
  FWD_SITE_O = 0x105, FWD_SITE_DRAIN = 0x106, FWD_SITE_A = 0x107, FWD_SITE_OR = 0x108, FWD_SITE_PV = 0x109,
  FWD_SITE_ST = 0x10a
};

template <int D, bool BF16, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(512, 1)
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

  // number of 64-key steps each query tile takes
  const bool has_t1 = q_start + 128 < seq_len;
  const int n_kv_all = (seq_len + 63) / 64;
  int n0, n1;
  if constexpr (CAUSAL) {
    n0 = min(4 * w + 2, n_kv_all);
    n1 = has_t1 ? min(4 * w + 4, n_kv_all) : 0;
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
  uint64_t* s_full = kv_empty + C::NSLOT;  // [tile * 2 + buffer]: S ready (tensor core)
  uint64_t* p_full = s_full + 4;           // [tile * 2 + buffer]: P written (softmax)
  uint64_t* a_ready = p_full + 4;          // [tile]: this step's rescale factors published (softmax)
  uint64_t* o_ready = a_ready + 2;         // [tile]: O rescaled for this step (correction)
  uint64_t* pv_done = o_ready + 2;         // [tile]: one more P V product finished (tensor core)
  uint64_t* stats_ready = pv_done + 2;     // [tile]: final m, l, lr published (softmax)
  uint64_t* o_full = stats_ready + 2;      // [tile]: every P V product finished (tensor core)
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  float* alpha_buf = reinterpret_cast<float*>(smem + C::XCH_OFF);  // [tile][parity][128]
  float* stat_buf = alpha_buf + 2 * 2 * 128;                       // [tile][m, l, lr][128]

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&a_ready[i], 128);
      mbar_init(&o_ready[i], 128);
      mbar_init(&pv_done[i], 1);
      mbar_init(&stats_ready[i], 128);
      mbar_init(&o_full[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
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

  // register split over 512 threads launched with 128 each (65536):
  // 128 x 40 (warps 0-3) + 256 x 152 (softmax) + 128 x 152 (correction) = 63488.
  // Each warpgroup changes its budget inside its own branch.
  if (warp < 4) {
    regs_dec<40>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        for (int t = 0; t < 2; ++t) {
          if (t == 1 && !has_t1) break;
          mbar_expect_tx(&q_full[t], C::QTILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::Q_OFF + t * C::QTILE + c * C::QCHUNK, &tm_q, &q_full[t], c * 64,
                        row_base + q_start + 128 * t, head);
        }
        // K_0, K_1, then (V_j, K_{j+2}) for j = 0, 1, ...: the tensor core's order
        int fill = 0;
        bool ok = true;
        auto load = [&](bool is_v, int jj) {
          const uint32_t slot = fill % C::NSLOT, round = fill / C::NSLOT;
          if (round > 0 && !(ok = mbar_wait(&kv_empty[slot], (round - 1) & 1, FWD_SITE_PROD))) return;
          mbar_expect_tx(&kv_full[slot], C::KTILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::KV_OFF + slot * C::KTILE + c * C::KCHUNK, is_v ? &tm_v : &tm_k, &kv_full[slot],
                        c * 64, row_base + 64 * jj, head);
          ++fill;
        };
        for (int jj = 0; jj < 2 && jj < n_kv && ok; ++jj) load(false, jj);
        for (int jj = 0; jj < n_kv && ok; ++jj) {
          load(true, jj);
          if (ok && jj + 2 < n_kv) load(false, jj + 2);
        }
        // Never leave a tile copy in flight into shared memory we are about
        // to give back: wait for the newest fill of every slot.
        for (int f = (fill > C::NSLOT ? fill - C::NSLOT : 0); f < fill; ++f)
          mbar_wait(&kv_full[f % C::NSLOT], (f / C::NSLOT) & 1, FWD_SITE_PROD);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t e = elect_one();
      constexpr uint32_t IDESC_QK = make_idesc(128, 64, BF16, false, false);
      constexpr uint32_t IDESC_PV = make_idesc(128, D, BF16, false, true);
      const uint64_t dq_base = make_sdesc(sq, 16, 1024);          // Q tile 0, K-major
      const uint64_t dk_base = make_sdesc(skv, 16, 1024);         // slot 0 as K (K-major)
      const uint64_t dv_base = make_sdesc(skv, C::KCHUNK, 1024);  // slot 0 as V (MN-major)
      bool ok = __all_sync(0xffffffffu, mbar_wait(&q_full[0], 0, FWD_SITE_Q));
      if (ok && has_t1) ok = __all_sync(0xffffffffu, mbar_wait(&q_full[1], 0, FWD_SITE_Q));
      int fill = 0;  // same sequence as the producer's fills
      auto take = [&](uint32_t& slot) {
        slot = fill % C::NSLOT;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[slot], (fill / C::NSLOT) & 1, FWD_SITE_KV));
        ++fill;
      };
      // S_t[b] = Q_t K^T: M = 128 query rows, N = 64 keys, K = D (both K-major)
      auto qk = [&](int t, int b, uint32_t kslot) {
        const uint64_t a = desc_add(dq_base, t * C::QTILE), bb = desc_add(dk_base, kslot * C::KTILE);
        const uint32_t d = tmem + C::TM_S + 64 * (2 * t + b);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_e(d, desc_add(a, (kk >> 2) * C::QCHUNK + (kk & 3) * 32),
                   desc_add(bb, (kk >> 2) * C::KCHUNK + (kk & 3) * 32), IDESC_QK, kk > 0 ? 1u : 0u, e);
      };
      // O_t += P_t[b] V: M = 128, N = D, K = 64 keys; P from TMEM, V MN-major
      auto pv = [&](int t, int b, uint32_t vslot, uint32_t acc) {
        const uint64_t bb = desc_add(dv_base, vslot * C::KTILE);
        const uint32_t d = tmem + C::TM_O + D * t, pa = tmem + C::TM_S + 64 * (2 * t + b);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_e(d, pa + kk * 8, desc_add(bb, kk * 2048), IDESC_PV, kk > 0 ? 1u : acc, e);
      };
      const int nt0 = n0, nt1 = n1;
      // prologue: S of steps 0 and 1 for both tiles
      for (int j = 0; j < 2 && j < n_kv && ok; ++j) {
        uint32_t ks;
        take(ks);
        if (!ok) break;
        tc_fence_after();
        if (j < nt0) {
          qk(0, j, ks);
          mma_commit_e(&s_full[j], e);
        }
        if (j < nt1) {
          qk(1, j, ks);
          mma_commit_e(&s_full[2 + j], e);
        }
        mma_commit_e(&kv_empty[ks], e);
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int b = j & 1;
        uint32_t vs;
        take(vs);
        if (!ok) break;
        for (int t = 0; t < 2; ++t) {
          if (j >= (t ? nt1 : nt0)) continue;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&p_full[2 * t + b], (j >> 1) & 1, FWD_SITE_P)))) break;
          if (j > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], (j - 1) & 1, FWD_SITE_OR)))) break;
          tc_fence_after();
          pv(t, b, vs, j > 0 ? 1u : 0u);
          mma_commit_e(&pv_done[t], e);
          if (j == (t ? nt1 : nt0) - 1) mma_commit_e(&o_full[t], e);
        }
        if (!ok) break;
        mma_commit_e(&kv_empty[vs], e);
        if (j + 2 < n_kv) {
          uint32_t ks;
          take(ks);
          if (!ok) break;
          // into buffer b: the P_t(j) held there has been read by the products above
          if (j + 2 < nt0) {
            qk(0, b, ks);
            mma_commit_e(&s_full[b], e);
          }
          if (j + 2 < nt1) {
            qk(1, b, ks);
            mma_commit_e(&s_full[2 + b], e);
          }
          mma_commit_e(&kv_empty[ks], e);
        }
      }
      // every product issued above has finished before TMEM is released
      mma_commit_e(drain, e);
      mbar_wait(drain, 0, FWD_SITE_DRAIN);
      __syncwarp();
    }
  } else if (warp < 12) {
    regs_inc<152>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;
    const int n_t = t == 0 ? n0 : n1;
    const int r = 32 * (warp & 3) + (int)lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int row = q_start + 128 * t + r;  // row inside the sequence
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      const int b = j & 1;
      const uint32_t tS = tmem + lane_off + C::TM_S + 64 * (2 * t + b);
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[2 * t + b], (j >> 1) & 1, FWD_SITE_S));
      if (!ok) break;
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(tS, s0);
      tmem_ld32(tS + 32, s1);
      tmem_ld_wait(s0);
      tmem_ld_wait(s1);
      float* x0 = reinterpret_cast<float*>(s0);
      float* x1 = reinterpret_cast<float*>(s1);
      // keys this row may see in this 64-key tile: [0, limit)
      const int kv0 = 64 * j;
      int limit = min(64, seq_len - kv0);
      if constexpr (CAUSAL) limit = min(limit, row - kv0 + 1);
      if (limit < 64) {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c >= limit) x0[c] = -INFINITY;
          if (c + 32 >= limit) x1[c] = -INFINITY;
        }
      }
      float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        mxa = fmax3(mxa, x0[c], x0[c + 1]);
        mxb = fmax3(mxb, x0[c + 16], x0[c + 17]);
        mxc = fmax3(mxc, x1[c], x1[c + 1]);
        mxd = fmax3(mxd, x1[c + 16], x1[c + 17]);
      }
      const float mx = fmax3(mxa, mxb, fmaxf(mxc, mxd));
      // Rescale only when the row max actually grew (by more than
      // kRescaleLog2): every P is then <= 2^kRescaleLog2, and with
      // kRescaleLog2 = 0 the largest P of the row is exactly 1.
      const float m_max = fmaxf(m, mx * sl2);
      const bool rescale = m_max > m + kRescaleLog2;  // false while the row has no visible key
      const float m_new = rescale ? m_max : m;
      const float alpha = rescale ? ex2(m - m_new) : 1.f;  // ex2(-inf) = 0 on the first tile
      if (j > 0) {
        // the correction warpgroup rescales O_t while we exponentiate
        alpha_buf[(2 * t + b) * 128 + r] = alpha;
        mbar_arrive(&a_ready[t]);
      }
      const float neg = (m_new == -INFINITY) ? 0.f : -m_new;
      const uint64_t scale2 = f2(sl2, sl2), neg2 = f2(neg, neg);
      // fsum: fp32 sum of P (for LSE); rsum: sum of P as rounded to 16 bits
      // (the weights the P V product uses, for normalising O).
      uint64_t fsum0 = f2(0.f, 0.f), fsum1 = f2(0.f, 0.f), rsum0 = f2(0.f, 0.f), rsum1 = f2(0.f, 0.f);
      auto exp_pair = [&](float x, float y, uint64_t& fs, uint64_t& rs) -> uint32_t {
        float a, bb;
        f2split(ffma2(f2(x, y), scale2, neg2), a, bb);
        a = ex2(a);
        bb = ex2(bb);
        fs = fadd2(fs, f2(a, bb));
        const uint32_t pk = pack2<BF16>(a, bb);
        rs = fadd2(rs, widen2<BF16>(pk));
        return pk;
      };
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = exp_pair(x0[2 * i], x0[2 * i + 1], fsum0, rsum0);
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[16 + i] = exp_pair(x1[2 * i], x1[2 * i + 1], fsum1, rsum1);
      // P pairs go over the first 32 score columns of this buffer (already read)
      tmem_st32(tS, pk);
      float f0, f1, f2_, f3, r0, r1, r2, r3;
      f2split(fsum0, f0, f1);
      f2split(fsum1, f2_, f3);
      f2split(rsum0, r0, r1);
      f2split(rsum1, r2, r3);
      // l (fp32 sum) gives LSE; lr (sum of the rounded P) normalises O, so
      // O / lr is a convex combination of the V rows with exactly the weights
      // the P V product used.
      l = l * alpha + ((f0 + f1) + (f2_ + f3));
      lr = lr * alpha + ((r0 + r1) + (r2 + r3));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[2 * t + b]);
      m = m_new;
    }
    if (ok && n_t > 0) {
      stat_buf[(3 * t + 0) * 128 + r] = m;
      stat_buf[(3 * t + 1) * 128 + r] = l;
      stat_buf[(3 * t + 2) * 128 + r] = lr;
      mbar_arrive(&stats_ready[t]);
    }
  } else {
    regs_inc<152>();
    // ------------------------------------------------------------ correction + epilogue
    const int r = 32 * (warp & 3) + (int)lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    bool ok = true;
    for (int j = 1; j < n_kv && ok; ++j) {
      for (int t = 0; t < 2; ++t) {
        if (j >= (t ? n1 : n0)) continue;
        // this step's rescale factors, then (if any differs from 1) the
        // previous P V product of tile t
        ok = __all_sync(0xffffffffu, mbar_wait(&a_ready[t], (j - 1) & 1, FWD_SITE_A));
        if (!ok) break;
        const float alpha = alpha_buf[(2 * t + (j & 1)) * 128 + r];
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[t], (j - 1) & 1, FWD_SITE_PV));
          if (!ok) break;
          tc_fence_after();
          const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
          const uint64_t alpha2 = f2(alpha, alpha);
          // all of the row's O columns in flight at once: one load latency
          uint32_t ov[D / 32][32];
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tO + 32 * cc, ov[cc]);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_ld_wait(ov[cc]);
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a, b;
              f2split(fmul2(f2(__uint_as_float(ov[cc][2 * i]), __uint_as_float(ov[cc][2 * i + 1])), alpha2), a, b);
              ov[cc][2 * i] = __float_as_uint(a);
              ov[cc][2 * i + 1] = __float_as_uint(b);
            }
            tmem_st32(tO + 32 * cc, ov[cc]);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&o_ready[t]);
      }
    }
    // ---- epilogue: O / lr and LSE for the rows inside the sequence
    for (int t = 0; t < 2 && ok; ++t) {
      if ((t ? n1 : n0) == 0) continue;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&stats_ready[t], 0, FWD_SITE_ST) && mbar_wait(&o_full[t], 0, FWD_SITE_O));
      if (!ok) break;
      tc_fence_after();
      const float m = stat_buf[(3 * t + 0) * 128 + r];
      const float l = stat_buf[(3 * t + 1) * 128 + r];
      const float lr = stat_buf[(3 * t + 2) * 128 + r];
      const float inv = lr > 0.f ? 1.f / lr : 0.f;
      const int row = q_start + 128 * t + r;
      const bool valid = row < seq_len;
      const size_t grow = (size_t)head * p.rows + row_base + row;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + grow * D);
      const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(tO + 32 * cc, ov);
        tmem_ld_wait(ov);
        uint32_t pko[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pko[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[cc * 4 + i] = make_uint4(pko[4 * i], pko[4 * i + 1], pko[4 * i + 2], pko[4 * i + 3]);
        }
      }
      if (valid) p.lse[grow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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

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
// 128 keys, 768 threads in six warpgroups:
//   warp 0      TMA producer: the Q tiles once, then K_0 and (V_j, K_{j+1})
//               for j = 0, 1, ... into a ring of shared-memory slots, the
//               order the tensor core consumes them in.
//   warp 1      tcgen05 issuer (converged warp, one elected lane) and TMEM
//               owner.  The two query tiles ping-pong: O_t += P_t(j) V_j
//               (first the 64 keys whose P is already published, then the
//               rest) and S_t(j+1) = Q_t K_{j+1}^T for one tile run on the
//               tensor core while the other tile's softmax exponentiates.
//               Products issued by one thread execute in order, so S_t(j+1)
//               overwrites P_t(j) only after O_t has consumed it.
//   warps 4-19  softmax, two threads per row: warps 4-11 take query tile 0,
//               12-19 tile 1; within a tile, warps 4k..4k+3 take keys 0-63
//               and the next four keys 64-127 of the same 128 rows (TMEM
//               lanes).  The two halves of a row swap their partial maxima
//               through shared memory (one barrier per 32 rows: the two
//               warps of those rows and the correction warp that rescales
//               them), then exponentiate in the log2 domain
//               (scale * log2 e folded into one FFMA), write P as 16-bit
//               pairs over the first 64 score columns (half h -> columns
//               [32h, 32h + 32)) and keep fp32 partial sums (for LSE) and
//               partial sums of P as rounded for the P V product (to
//               normalise O).
//   warps 20-23 correction: from the same partial maxima it tracks each row
//               max and, when it grows, rescales that tile's O accumulator in
//               TMEM by exp(m_old - m_new) while the softmax exponentiates;
//               at the end, O / l and LSE to global.
// TMEM columns: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// Fully masked causal tiles are never loaded or multiplied.
// DROPOUT instances (dense or packed batches) zero the dropped P values before they
// are published for the P V product, from a Philox4x32-10 mask regenerated
// from (head, query, key) indices, and scale O by 1 / (keep probability) at
// the end; the sums that normalise O and give LSE stay those of the
// undropped P.
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
  Dropout drop;           // DROPOUT instances only
};

template <int D>
struct FwdCfg {
  static constexpr int CH = D / 64;                  // 64-column chunks of a tile
  static constexpr int KROWS = 128;                  // keys per K/V tile
  static constexpr uint32_t CHUNK = 128u * 128u;     // 128 rows x 128 bytes
  static constexpr uint32_t TILE = CH * CHUNK;       // one 128 x D tile (Q, K or V)
  static constexpr int NSLOT = (D == 128) ? 4 : 8;   // K/V ring depth (128 KB)
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t KV_OFF = 2 * TILE;
  static constexpr uint32_t BAR_OFF = KV_OFF + NSLOT * TILE;
  // q_full[2] kv_full[N] kv_empty[N] s_full[2] p_full[4] mx_full[8] o_ready[2]
  // pv_done[2] stats_ready[2] o_full[2] drain
  static constexpr int NBAR = 2 + 2 * NSLOT + 2 + 4 + 8 + 2 + 2 + 2 + 2 + 1;
  // partial row maxima [tile][half][128] and the final partial sums
  // (l, lr)[tile][half][2][128], fp32
  static constexpr uint32_t XCH_OFF = (BAR_OFF + NBAR * 8 + 16 + 15) & ~15u;
  static constexpr uint32_t XCH_BYTES = (2 * 2 * 128 + 2 * 2 * 2 * 128) * 4;
  static constexpr uint32_t SMEM = XCH_OFF + XCH_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TM_S = 0, TM_O = 256;
  static constexpr int THREADS = 768;
};

// wait-site ids reported through the error word
enum : uint32_t {
  FWD_SITE_PROD = 0x100, FWD_SITE_Q = 0x101, FWD_SITE_KV = 0x102, FWD_SITE_P = 0x103, FWD_SITE_S = 0x104,
  FWD_SITE_O = 0x105, FWD_SITE_DRAIN = 0x106, FWD_SITE_A = 0x107, FWD_SITE_OR = 0x108, FWD_SITE_PV = 0x109,
  FWD_SITE_ST = 0x10a, FWD_SITE_MX = 0x10b
};

template <int D, bool BF16, bool CAUSAL, bool VARLEN, bool DROPOUT = false>
__global__ void __launch_bounds__(768, 1)
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

  // number of 128-key steps each query tile takes
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
  uint64_t* s_full = kv_empty + C::NSLOT;  // [tile]: S ready (tensor core)
  uint64_t* p_full = s_full + 2;           // [tile * 2 + half]: P of 64 keys written (softmax)
  uint64_t* mx_full = p_full + 4;          // [tile * 4 + quarter]: both partial maxima of the
                                           //   quarter's 32 rows published (its two softmax warps)
  uint64_t* o_ready = mx_full + 8;         // [tile]: O ready for this step's P V (correction)
  uint64_t* pv_done = o_ready + 2;         // [tile]: one more P V product finished (tensor core)
  uint64_t* stats_ready = pv_done + 2;     // [tile]: final partial sums published (softmax)
  uint64_t* o_full = stats_ready + 2;      // [tile]: every P V product finished (tensor core)
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBAR);
  float* pmax_buf = reinterpret_cast<float*>(smem + C::XCH_OFF);  // [tile][half][128]
  float* sum_buf = pmax_buf + 2 * 2 * 128;                        // [tile][half][l, lr][128]

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&o_ready[i], 128);
      for (int q = 0; q < 4; ++q) mbar_init(&mx_full[4 * i + q], 64);
      mbar_init(&pv_done[i], 1);
      mbar_init(&stats_ready[i], 256);
      mbar_init(&o_full[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&p_full[i], 128);
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

  // register split over 768 threads launched with 80 each (61440):
  // 128 x R0 (warps 0-3) + 512 x 96 (softmax) + 128 x RC (correction) = 61440,
  // with (R0, RC) = (40, 56) for dense heads and (48, 48) for packed batches
  // (whose producer and issuer keep the sequence offsets live).
  // Each warpgroup changes its budget inside its own branch.
  constexpr int R0 = VARLEN ? 48 : 40, RC = VARLEN ? 48 : 56;
  static_assert(128 * R0 + 512 * 96 + 128 * RC == 768 * 80, "register split");
  if (warp < 4) {
    regs_dec<R0>();
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
        // K_0, then (V_j, K_{j+1}) for j = 0, 1, ...: the tensor core's order
        int fill = 0;
        bool ok = true;
        auto load = [&](bool is_v, int jj) {
          const uint32_t slot = fill % C::NSLOT, round = fill / C::NSLOT;
          if (round > 0 && !(ok = mbar_wait(&kv_empty[slot], (round - 1) & 1, FWD_SITE_PROD))) return;
          mbar_expect_tx(&kv_full[slot], C::TILE);
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(smem + C::KV_OFF + slot * C::TILE + c * C::CHUNK, is_v ? &tm_v : &tm_k, &kv_full[slot],
                        c * 64, row_base + 128 * jj, head);
          ++fill;
        };
        load(false, 0);
        for (int jj = 0; jj < n_kv && ok; ++jj) {
          load(true, jj);
          if (ok && jj + 1 < n_kv) load(false, jj + 1);
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
      constexpr uint32_t IDESC_QK = make_idesc(128, 128, BF16, false, false);
      constexpr uint32_t IDESC_PV = make_idesc(128, D, BF16, false, true);
      const uint64_t dq_base = make_sdesc(sq, 16, 1024);        // Q tile 0, K-major
      const uint64_t dk_base = make_sdesc(skv, 16, 1024);       // slot 0 as K (K-major)
      const uint64_t dv_base = make_sdesc(skv, C::CHUNK, 1024);  // slot 0 as V (MN-major)
      bool ok = true;
      int fill = 0;  // same sequence as the producer's fills
      auto take = [&](uint32_t& slot) {
        slot = fill % C::NSLOT;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[slot], (fill / C::NSLOT) & 1, FWD_SITE_KV));
        ++fill;
      };
      // S_t = Q_t K^T: M = 128 query rows, N = 128 keys, K = D (both K-major)
      auto qk = [&](int t, uint32_t kslot) {
        const uint64_t a = desc_add(dq_base, t * C::TILE), bb = desc_add(dk_base, kslot * C::TILE);
        const uint32_t d = tmem + C::TM_S + 128 * t;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss_e(d, desc_add(a, (kk >> 2) * C::CHUNK + (kk & 3) * 32),
                   desc_add(bb, (kk >> 2) * C::CHUNK + (kk & 3) * 32), IDESC_QK, kk > 0 ? 1u : 0u, e);
      };
      // O_t += P_t V for keys [64h, 64h + 64): M = 128, N = D, K = 64 keys;
      // P from TMEM (8 columns per 16 keys), V MN-major (2048 bytes per 16 keys)
      auto pv = [&](int t, int h, uint32_t vslot, uint32_t acc) {
        const uint64_t bb = desc_add(dv_base, vslot * C::TILE + h * 8192);
        const uint32_t d = tmem + C::TM_O + D * t, pa = tmem + C::TM_S + 128 * t + 32 * h;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts_e(d, pa + kk * 8, desc_add(bb, kk * 2048), IDESC_PV, kk > 0 ? 1u : acc, e);
      };
      // prologue: S of step 0 for both tiles
      uint32_t ks;
      take(ks);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&q_full[0], 0, FWD_SITE_Q));
      if (ok) {
        tc_fence_after();
        qk(0, ks);
        mma_commit_e(&s_full[0], e);
      }
      if (ok && n1 > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&q_full[1], 0, FWD_SITE_Q));
        if (ok) {
          tc_fence_after();
          qk(1, ks);
          mma_commit_e(&s_full[1], e);
        }
      }
      if (ok) mma_commit_e(&kv_empty[ks], e);
      for (int j = 0; j < n_kv && ok; ++j) {
        uint32_t vs;
        take(vs);
        if (!ok) break;
        bool have_k = false;
        for (int t = 0; t < 2; ++t) {
          const int n_t = t ? n1 : n0;
          if (j >= n_t) continue;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&p_full[2 * t], j & 1, FWD_SITE_P)))) break;
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&o_ready[t], j & 1, FWD_SITE_OR)))) break;
          tc_fence_after();
          pv(t, 0, vs, j > 0 ? 1u : 0u);
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&p_full[2 * t + 1], j & 1, FWD_SITE_P)))) break;
          tc_fence_after();
          pv(t, 1, vs, 1u);
          mma_commit_e(&pv_done[t], e);
          if (j == n_t - 1) {
            mma_commit_e(&o_full[t], e);
          } else {
            if (!have_k) {
              take(ks);
              if (!ok) break;
              have_k = true;
            }
            // into S_t: behind the P V product above, which reads P_t(j) there
            qk(t, ks);
            mma_commit_e(&s_full[t], e);
          }
        }
        if (!ok) break;
        mma_commit_e(&kv_empty[vs], e);
        if (have_k) mma_commit_e(&kv_empty[ks], e);
      }
      // every product issued above has finished before TMEM is released
      mma_commit_e(drain, e);
      mbar_wait(drain, 0, FWD_SITE_DRAIN);
      __syncwarp();
    }
  } else if (warp < 20) {
    regs_inc<96>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 3;        // query tile
    const int h = ((warp - 4) >> 2) & 1;  // key half: keys [64h, 64h + 64) of each tile
    const int n_t = t == 0 ? n0 : n1;
    const int r = 32 * (warp & 3) + (int)lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + 128 * t;
    const int row = q_start + 128 * t + r;  // row inside the sequence
    const float sl2 = p.scale_log2;
    float* my_max = pmax_buf + (2 * t + h) * 128 + r;
    const float* other_max = pmax_buf + (2 * t + (h ^ 1)) * 128 + r;
    float m = -INFINITY, l = 0.f, lr = 0.f;
    // Dropout keep decisions of this row's 64 keys of one step, pair-packed:
    // keys 2i, 2i + 1 of the half's first 32 at bits pair_slot(i),
    // pair_slot(i) + 8 of keep[0], the next 32 in keep[1].  One Philox call
    // covers rows (2m, 2m + 1) x key octet o (one byte per element: byte
    // key & 3 of word 2 (row & 1) + ((key >> 2) & 1)), and rows 2m, 2m + 1
    // sit in the two lanes of a pair: the even lane draws the half's octets
    // 0-3, the odd lane 4-7, and each hands the other row's two words
    // across.  Drawn for step j + 1 while step j's products run, so the
    // generator stays off the softmax's critical path.
    uint32_t keep[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};
    auto make_keep = [&](int jj) {
      const bool odd = (lane & 1u) != 0;
      const uint32_t t4 = p.drop.thresh * 0x01010101u, t4lo = t4 & 0x7f7f7f7fu;
      const uint32_t rowpair = (uint32_t)row >> 1, ko0 = (uint32_t)(128 * jj + 64 * h) >> 3;
      // head word of the counter: b * H + h, with a packed batch's sequence
      // as its b (row and key indices count from the sequence's start)
      const uint32_t mask_head = (uint32_t)(seq * p.heads + head);
      uint32_t k0 = 0u, k1 = 0u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint4 w = philox4x32_10(make_uint4(ko0 + k + (odd ? 4u : 0u), rowpair, mask_head, p.drop.offset),
                                      p.drop.seed_lo, p.drop.seed_hi);
        const uint32_t own0 = odd ? w.z : w.x, own1 = odd ? w.w : w.y;  // this row
        const uint32_t oth0 = odd ? w.x : w.z, oth1 = odd ? w.y : w.w;  // the partner row
        const uint32_t got0 = __shfl_xor_sync(0xffffffffu, oth0, 1), got1 = __shfl_xor_sync(0xffffffffu, oth1, 1);
        // keys 8k .. 8k + 3 are pairs 4k, 4k + 1; keys 8k + 4 .. are 4k + 2, 4k + 3
        k0 |= (pair_bits(bytes_below(odd ? got0 : own0, t4, t4lo)) << pair_slot(4 * k)) |
              (pair_bits(bytes_below(odd ? got1 : own1, t4, t4lo)) << pair_slot(4 * k + 2));  // octet k
        k1 |= (pair_bits(bytes_below(odd ? own0 : got0, t4, t4lo)) << pair_slot(4 * k)) |
              (pair_bits(bytes_below(odd ? own1 : got1, t4, t4lo)) << pair_slot(4 * k + 2));  // octet 4 + k
      }
      keep[0] = k0;
      keep[1] = k1;
    };
    if constexpr (DROPOUT)
      if (n_t > 0) make_keep(0);
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, FWD_SITE_S));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][32];
      tmem_ld32(tS + 64 * h, sv[0]);
      tmem_ld32(tS + 64 * h + 32, sv[1]);
      tmem_ld_wait(sv[0]);
      tmem_ld_wait(sv[1]);
      // keys this row may see in this half tile: [0, limit)
      const int kv0 = 128 * j + 64 * h;
      int limit = min(64, seq_len - kv0);
      if constexpr (CAUSAL) limit = min(limit, row - kv0 + 1);
      if (limit < 64) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= limit) sv[c][i] = __float_as_uint(-INFINITY);
      }
      float mx2[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float a = fmax3(__uint_as_float(sv[c][0]), __uint_as_float(sv[c][1]), __uint_as_float(sv[c][2]));
        float b = fmax3(__uint_as_float(sv[c][3]), __uint_as_float(sv[c][4]), __uint_as_float(sv[c][5]));
#pragma unroll
        for (int i = 6; i < 30; i += 4) {
          a = fmax3(a, __uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1]));
          b = fmax3(b, __uint_as_float(sv[c][i + 2]), __uint_as_float(sv[c][i + 3]));
        }
        mx2[c] = fmax3(a, b, fmaxf(__uint_as_float(sv[c][30]), __uint_as_float(sv[c][31])));
      }
      // swap partial maxima with the other half of the row: only the two
      // warps of these 32 rows arrive (and the correction warp of the same
      // rows reads them too), so no warp waits for the tile's slowest one
      const float pm = fmaxf(mx2[0], mx2[1]);
      *my_max = pm;
      mbar_arrive(&mx_full[4 * t + (warp & 3)]);
      ok = __all_sync(0xffffffffu, mbar_wait(&mx_full[4 * t + (warp & 3)], j & 1, FWD_SITE_MX));
      if (!ok) break;
      const float mx = fmaxf(pm, *other_max);
      // Exact running max: rescale whenever the row max grows, so the
      // largest P of the row is exactly 1 and only the smaller weights carry
      // 16-bit rounding into P V.  The correction warpgroup makes the same
      // decision from the same values.
      const float m_new = fmaxf(m, mx * sl2);
      const float alpha = m_new > m ? ex2(m - m_new) : 1.f;  // ex2(-inf) = 0 on the first tile
      const float neg = (m_new == -INFINITY) ? 0.f : -m_new;
      const uint64_t scale2 = f2(sl2, sl2), neg2 = f2(neg, neg);
      // fsum: fp32 sum of P (for LSE); rsum: sum of P as rounded to 16 bits
      // (the weights the P V product uses, for normalising O).
      uint64_t fsum0 = f2(0.f, 0.f), fsum1 = f2(0.f, 0.f), rsum0 = f2(0.f, 0.f), rsum1 = f2(0.f, 0.f);
      auto exp_pair = [&](uint32_t x, uint32_t y, uint64_t& fs, uint64_t& rs) -> uint32_t {
        const uint64_t arg = ffma2(f2(__uint_as_float(x), __uint_as_float(y)), scale2, neg2);
        float a, bb;
        f2split(arg, a, bb);
        a = ex2(a);
        bb = ex2(bb);
        fs = fadd2(fs, f2(a, bb));
        const uint32_t pk = pack2<BF16>(a, bb);
        rs = fadd2(rs, widen2<BF16>(pk));
        return pk;
      };
      // keys [64h, 64h + 64) -> 32 packed pairs -> TMEM columns [32h, 32h + 32)
      // of this tile's S region (every score of the tile has been read: both
      // halves passed the max exchange), then publish
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pk[i] = exp_pair(sv[0][2 * i], sv[0][2 * i + 1], fsum0, rsum0);
        pk[16 + i] = exp_pair(sv[1][2 * i], sv[1][2 * i + 1], fsum1, rsum1);
      }
      if constexpr (DROPOUT) {
        // drop: pk[i] holds keys 2i, 2i + 1 of the half (pair slot i & 15 of
        // keep[i >> 4])
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          pk[i] &= pair_keep_halves(keep[0], i);
          pk[16 + i] &= pair_keep_halves(keep[1], i);
        }
      }
      tmem_st32(tS + 32 * h, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[2 * t + h]);
      float f0, f1, f2_, f3, r0, r1, r2, r3;
      f2split(fsum0, f0, f1);
      f2split(fsum1, f2_, f3);
      f2split(rsum0, r0, r1);
      f2split(rsum1, r2, r3);
      // l (fp32 sum) gives LSE; lr (sum of the rounded P) normalises O, so
      // O / lr is a convex combination of the V rows with exactly the weights
      // the P V product used.  Each half keeps its own partial sums.
      l = l * alpha + ((f0 + f1) + (f2_ + f3));
      lr = lr * alpha + ((r0 + r1) + (r2 + r3));
      m = m_new;
      // the next step's keep bits, while the tensor core works on this step
      if constexpr (DROPOUT)
        if (j + 1 < n_t) make_keep(j + 1);
    }
    if (ok && n_t > 0) {
      sum_buf[((2 * t + h) * 2 + 0) * 128 + r] = l;
      sum_buf[((2 * t + h) * 2 + 1) * 128 + r] = lr;
      mbar_arrive(&stats_ready[t]);
    }
  } else {
    regs_dec<RC>();
    // ------------------------------------------------------------ correction + epilogue
    const int r = 32 * (warp & 3) + (int)lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float sl2 = p.scale_log2;
    float m_row0 = -INFINITY, m_row1 = -INFINITY;  // running max of row r of each tile (log2 units)
    bool ok = true;
    for (int j = 0; j < n_kv && ok; ++j) {
      for (int t = 0; t < 2; ++t) {
        if (j >= (t ? n1 : n0)) continue;
        // this step's partial maxima -> the same running max the softmax keeps
        ok = __all_sync(0xffffffffu, mbar_wait(&mx_full[4 * t + (warp & 3)], j & 1, FWD_SITE_MX));
        if (!ok) break;
        const float mx = fmaxf(pmax_buf[(2 * t) * 128 + r], pmax_buf[(2 * t + 1) * 128 + r]);
        const float m = t ? m_row1 : m_row0;
        const float m_new = fmaxf(m, mx * sl2);
        const float alpha = m_new > m ? ex2(m - m_new) : 1.f;
        if (t) m_row1 = m_new; else m_row0 = m_new;
        // O_t is written fresh by the first P V product; later, if any factor
        // differs from 1, wait for the previous P V product of tile t, then
        // O_t *= alpha, 16 columns at a time.  o_ready is released every step,
        // so the tile's next scores (and the next partial maxima) cannot come
        // before this step's maxima have been read here.
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[t], (j - 1) & 1, FWD_SITE_PV));
          if (!ok) break;
          tc_fence_after();
          const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
          const uint64_t alpha2 = f2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t ov[16];
            tmem_ld16(tO + 16 * c, ov);
            tmem_ld_wait(ov);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float x, y;
              f2split(fmul2(f2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1])), alpha2), x, y);
              ov[2 * i] = __float_as_uint(x);
              ov[2 * i + 1] = __float_as_uint(y);
            }
            tmem_st16(tO + 16 * c, ov);
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
      const float m = t ? m_row1 : m_row0;
      const float l = sum_buf[((2 * t + 0) * 2 + 0) * 128 + r] + sum_buf[((2 * t + 1) * 2 + 0) * 128 + r];
      const float lr = sum_buf[((2 * t + 0) * 2 + 1) * 128 + r] + sum_buf[((2 * t + 1) * 2 + 1) * 128 + r];
      // dropout: O = (P * M) V * s (s = 1 / keep probability), P normalised
      // by the undropped sum
      const float inv = lr > 0.f ? (DROPOUT ? p.drop.scale : 1.f) / lr : 0.f;
      const int row = q_start + 128 * t + r;
      const bool valid = row < seq_len;
      const size_t grow = (size_t)head * p.rows + row_base + row;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + grow * D);
      const uint32_t tO = tmem + lane_off + C::TM_O + D * t;
#pragma unroll 1
      for (int c = 0; c < D / 16; ++c) {
        uint32_t ov[16];
        tmem_ld16(tO + 16 * c, ov);
        tmem_ld_wait(ov);
        uint32_t pko[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          pko[i] = pack2<BF16>(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
        if (valid) {
          dst[c * 2] = make_uint4(pko[0], pko[1], pko[2], pko[3]);
          dst[c * 2 + 1] = make_uint4(pko[4], pko[5], pko[6], pko[7]);
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

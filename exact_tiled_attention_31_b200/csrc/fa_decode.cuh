// fa_decode.cuh - one decode step of exact attention over a KV cache.
//
// Each sequence b brings one new query token per query head; it attends to
// the seq_lens[b] keys of its cache (the new token is the last position, so
// every cached key is visible).  Query head h reads KV head h / G with
// G = Hq / Hkv (grouped-query attention; G = 1 multi-head, Hkv = 1
// multi-query).  Per token step the cost is reading the cache once, which
// is what decode is about ("Flash Attention 的算法设计原理", "训练与推理价值" and
// "练习口述回答": decode reads an ever longer KV cache for one new token, and
// GQA/MQA change the balance).  The arithmetic is the same online softmax as
// the forward ("From Self-Attention to FlashAttention", §二): running row
// maximum (exact), rescaled running sums and output, one division at the end.
//
// B200 mapping.  The work is a stream of the cache through the SMs, bounded by
// HBM bandwidth, so the cache is split along its length: one CTA per
// (split, KV head, sequence) covers a contiguous key range, and the ranges
// are combined by the merge of disjoint key subsets (LSE = log sum
// exp(LSE_s), O = sum exp(LSE_s - LSE) O_s).  When the launch runs the
// splits of one (sequence, KV head) as one thread-block cluster (the host
// does so for 2 to 4 splits that fit in one wave), rank 0 merges the others'
// parts through distributed shared memory at the end; with one split the CTA
// writes O and LSE itself; otherwise each CTA writes a normalised partial O
// and its LSE and decode_merge_kernel combines them.
// Inside a CTA, 4 warps take alternate 32-key tiles, each warp with its own
// ring of stages that its lane 0 fills by TMA (K and V tiles of 32 rows x
// 64 columns, 128-byte swizzle, completion counted on the stage's mbarrier).
// A tile that runs past the sequence's last key is copied row by row with
// cp.async instead, zero-filling the rows past the end, so no cache row at
// or past the length is ever read.  The G query rows of the group
// (padded to 16) are the M dimension of m16n8k16 tensor-core products
// (S = Q K^T, then O += P V with P in registers), which are far from the
// bound here: 32 KB of K/V per 32-key tile per warp against two products of
// 16 x 32 x D.  The four warps merge through shared memory at the end.
#pragma once

#include "sm100.cuh"

namespace fa {

struct DecParams {
  const uint16_t* q;     // [B, Hq, D]
  const uint16_t* k;     // [B, Hkv, L, D]
  const uint16_t* v;     // [B, Hkv, L, D]
  const int* seq_lens;   // [B] valid cached keys per sequence
  float* o_part;         // [B, Hq, n_splits, D] fp32, normalised over the split's keys
  float* lse_part;       // [B, Hq, n_splits] natural log, -inf for an empty split
  void* o;               // [B, Hq, D] 16-bit output
  float* lse;            // [B, Hq]
  int B, Hq, Hkv, L, n_splits, group;
  float scale_log2;      // scale * log2(e)
};

template <int D>
struct DecCfg {
  static constexpr int KT = 32;                          // keys per warp tile
  static constexpr int HALF = KT * 128;                  // 32 rows x 64 columns, 128-byte swizzled
  static constexpr int TILE = KT * D * 2;                // one K or V tile (D / 64 halves)
  static constexpr int WARPS = 4;
  static constexpr int STAGES = D == 128 ? 3 : 6;        // K+V tiles in flight per warp: STAGES - 1
  static constexpr int WARP_BYTES = 2 * STAGES * TILE;
  static constexpr int SMEM = WARPS * WARP_BYTES + 1024; // + alignment slack; D = 128: 197632 bytes
  static constexpr int CHUNKS = KT * D * 2 / 16;         // 16-byte pieces per tile
  static constexpr int SCRATCH = 3 * 16 + 16 * D;        // floats per warp for the final merge
  static_assert(SMEM <= 227 * 1024 - WARPS * STAGES * 8, "shared memory per block");
  static_assert((WARPS + 1) * SCRATCH * 4 <= WARPS * WARP_BYTES, "merge scratch fits in the tile buffers");
};

enum : uint32_t { DEC_SITE_KV = 0x300, DEC_SITE_DRAIN = 0x301 };

// byte offset of (row, 8-column chunk c8 of D / 8) in a K or V tile
template <int D>
__device__ __forceinline__ uint32_t dec_off(int row, int c8) {
  return (c8 >> 3) * DecCfg<D>::HALF + row * 128 + (((c8 & 7) ^ (row & 7)) << 4);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// thread-block cluster: rank, size, barrier, and loads from a peer CTA's
// shared memory (distributed shared memory)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_addr(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ float ld_dsmem(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_dsmem4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

// c[4] += a[4] (16 x 16, row) * b[2] (16 x 8, col), fp32 accumulate
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(128, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const DecParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t dsm_raw[];
  __shared__ uint64_t bars[C::WARPS][C::STAGES];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int len = min(max(p.seq_lens[b], 0), p.L);
  // this split's keys: [start, end), a multiple of KT long except at the end
  const int per = ((len + p.n_splits - 1) / p.n_splits + C::KT - 1) / C::KT * C::KT;
  const int start = split * per, end = min(len, start + per);
  const int n_tiles = end > start ? (end - start + C::KT - 1) / C::KT : 0;
  const int bh = b * p.Hkv + kvh;  // cache head index (third tensor-map coordinate)
  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&bars[warp][s], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  // the merge launch may start once every block has got here; it still waits
  // for this grid's completion before reading the partial results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncwarp();

  // Q as the A operand (rows = the group's query heads, padded to 16 with zeros)
  const int r0 = lane >> 2, r1 = r0 + 8, cq = 2 * (lane & 3);
  const uint32_t* q0 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)b * p.Hq + kvh * p.group + r0) * D);
  const uint32_t* q1 = reinterpret_cast<const uint32_t*>(p.q + ((size_t)b * p.Hq + kvh * p.group + r1) * D);
  const bool v0 = r0 < p.group, v1 = r1 < p.group;
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    qa[kk][0] = v0 ? q0[(16 * kk + cq) / 2] : 0u;
    qa[kk][1] = v1 ? q1[(16 * kk + cq) / 2] : 0u;
    qa[kk][2] = v0 ? q0[(16 * kk + 8 + cq) / 2] : 0u;
    qa[kk][3] = v1 ? q1[(16 * kk + 8 + cq) / 2] : 0u;
  }

  uint8_t* kbuf = dsm + warp * C::WARP_BYTES;  // K tiles [STAGES], then V tiles [STAGES]
  uint8_t* vbuf = kbuf + C::STAGES * C::TILE;
  const uint16_t* kh = p.k + (size_t)bh * p.L * D;
  const uint16_t* vh = p.v + (size_t)bh * p.L * D;
  // The warp's i-th tile is tile warp + WARPS * i of the split, in stage
  // i % STAGES.  A whole tile comes by TMA; the one tile that runs past
  // `end` (always the split's last, so the warp's last) by cp.async with
  // the rows past `end` zero-filled.
  auto full_tile = [&](int i) { return start + C::KT * (warp + C::WARPS * i) + C::KT <= end; };
  auto issue = [&](int i) {
    const int t = warp + C::WARPS * i;
    if (t >= n_tiles) return;
    const int key0 = start + C::KT * t, s = i % C::STAGES;
    uint8_t* kd = kbuf + s * C::TILE;
    uint8_t* vd = vbuf + s * C::TILE;
    if (key0 + C::KT <= end) {
      if (lane == 0) {
        mbar_expect_tx(&bars[warp][s], 2 * C::TILE);
#pragma unroll
        for (int h = 0; h < D / 64; ++h) {
          tma_load_3d(kd + h * C::HALF, &tm_k, &bars[warp][s], 64 * h, key0, bh);
          tma_load_3d(vd + h * C::HALF, &tm_v, &bars[warp][s], 64 * h, key0, bh);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < C::CHUNKS / 32; ++j) {
        const int c = lane + 32 * j;
        const int row = c / (D / 8), c8 = c % (D / 8);
        const int key = key0 + row;
        const bool in = key < end;
        const size_t off = (size_t)(in ? key : 0) * D + c8 * 8;
        cp_async16(kd + dec_off<D>(row, c8), kh + off, in ? 16u : 0u);
        cp_async16(vd + dec_off<D>(row, c8), vh + off, in ? 16u : 0u);
      }
      cp_async_commit();
    }
  };

  float oacc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, lr[2] = {0.f, 0.f};  // rows r0, r1 (lane's share of l, lr)
  const float sl2 = p.scale_log2;

  const int my_tiles = n_tiles > warp ? (n_tiles - warp + C::WARPS - 1) / C::WARPS : 0;
#pragma unroll
  for (int i = 0; i < C::STAGES - 1; ++i) issue(i);
  for (int i = 0; i < my_tiles; ++i) {
    issue(i + C::STAGES - 1);
    const int t = warp + C::WARPS * i, st = i % C::STAGES;
    if (full_tile(i)) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[warp][st], (i / C::STAGES) & 1, DEC_SITE_KV));
      if (!ok) {  // error recorded: let the warp's copies in flight, this tile's included, land
                  // (bounded waits again), then stop
        for (int j = i; j < min(i + C::STAGES, my_tiles); ++j)
          if (full_tile(j)) mbar_wait(&bars[warp][j % C::STAGES], (j / C::STAGES) & 1, DEC_SITE_DRAIN);
        break;
      }
    } else {
      cp_async_wait<0>();
      __syncwarp();
    }
    const uint32_t ks = smem_addr(kbuf + st * C::TILE), vs = smem_addr(vbuf + st * C::TILE);
    // S = Q K^T: 16 rows x 32 keys (4 tiles of 8)
    float sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        uint32_t b0, b1;
        ldsm_x2(ks + dec_off<D>(8 * nt + (lane & 7), 2 * kk + ((lane >> 3) & 1)), b0, b1);
        mma16816<BF16>(sacc[nt], qa[kk], b0, b1);
      }
    }
    // log2 domain, keys past the end masked
    const int kbase = start + C::KT * t;
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kbase + 8 * nt + cq + (e & 1);
        const float sv = key < end ? sacc[nt][e] * sl2 : -INFINITY;
        sacc[nt][e] = sv;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], sv);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
      const float m_new = fmaxf(m[r], tmax[r]);  // exact running maximum
      alpha[r] = ex2(m[r] - m_new);              // ex2(-inf) = 0 on the first tile
      m[r] = m_new;
      l[r] *= alpha[r];
      lr[r] *= alpha[r];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      oacc[n][0] *= alpha[0];
      oacc[n][1] *= alpha[0];
      oacc[n][2] *= alpha[1];
      oacc[n][3] *= alpha[1];
    }
    // P = 2^(s - m), rounded to 16 bits as the A operand of P V; l sums the
    // fp32 values (for LSE), lr the rounded ones (to normalise O)
    uint32_t pa[2][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = ex2(sacc[nt][0] - m[0]), p1 = ex2(sacc[nt][1] - m[0]);
      const float p2 = ex2(sacc[nt][2] - m[1]), p3 = ex2(sacc[nt][3] - m[1]);
      l[0] += p0 + p1;
      l[1] += p2 + p3;
      const uint32_t k01 = pack2<BF16>(p0, p1), k23 = pack2<BF16>(p2, p3);
      const float2 w01 = unpack2<BF16>(k01), w23 = unpack2<BF16>(k23);
      lr[0] += w01.x + w01.y;
      lr[1] += w23.x + w23.y;
      // m16n8k16 A layout: regs 0/1 = keys 0-7 of the k step (rows r0/r1), 2/3 = keys 8-15
      pa[nt >> 1][(nt & 1) * 2 + 0] = k01;
      pa[nt >> 1][(nt & 1) * 2 + 1] = k23;
    }
    // O += P V: 16 rows x D, K = 32 keys in two steps of 16
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
#pragma unroll
      for (int n = 0; n < D / 8; ++n) {
        uint32_t b0, b1;
        ldsm_x2_trans(vs + dec_off<D>(16 * k2 + (lane & 15), n), b0, b1);
        mma16816<BF16>(oacc[n], pa[k2], b0, b1);
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();

  // the lane's shares of the row sums -> the row's (4 lanes of a quad)
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 1);
    lr[r] += __shfl_xor_sync(0xffffffffu, lr[r], 2);
  }
  // merge the four warps through shared memory (the tile buffers are free now)
  __syncthreads();
  float* ws = reinterpret_cast<float*>(dsm) + warp * C::SCRATCH;  // m[16] l[16] lr[16] O[16][D]
  if ((lane & 3) == 0) {
    ws[r0] = m[0];
    ws[r1] = m[1];
    ws[16 + r0] = l[0];
    ws[16 + r1] = l[1];
    ws[32 + r0] = lr[0];
    ws[32 + r1] = lr[1];
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    ws[48 + r0 * D + 8 * n + cq] = oacc[n][0];
    ws[48 + r0 * D + 8 * n + cq + 1] = oacc[n][1];
    ws[48 + r1 * D + 8 * n + cq] = oacc[n][2];
    ws[48 + r1 * D + 8 * n + cq + 1] = oacc[n][3];
  }
  __syncthreads();
  // thread -> (row, 16 of the D columns): this CTA's (max, sums, unnormalised O)
  constexpr int PARTS = D / 16;
  const int row = threadIdx.x / PARTS, part = threadIdx.x % PARTS;
  const bool active = row < p.group && threadIdx.x < 16 * PARTS;
  float mm = -INFINITY, lt = 0.f, lrt = 0.f, acc[16];
#pragma unroll
  for (int d = 0; d < 16; ++d) acc[d] = 0.f;
  if (active) {
    const float* w0 = reinterpret_cast<const float*>(dsm);
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) mm = fmaxf(mm, w0[w * C::SCRATCH + row]);
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) {
      const float* wp = w0 + w * C::SCRATCH;
      const float sc = mm == -INFINITY ? 0.f : ex2(wp[row] - mm);  // empty warp ranges weigh 0
      lt += wp[16 + row] * sc;
      lrt += wp[32 + row] * sc;
#pragma unroll
      for (int d = 0; d < 16; ++d) acc[d] += wp[48 + row * D + 16 * part + d] * sc;
    }
  }
  const size_t qrow = (size_t)b * p.Hq + kvh * p.group + row;

  if (cluster_nctarank() > 1) {
    // The splits of this (sequence, KV head) form one cluster: each CTA
    // publishes its part in its own shared memory and rank 0 merges them
    // through distributed shared memory, the same rescaling as between warps.
    float* pub = reinterpret_cast<float*>(dsm) + C::WARPS * C::SCRATCH;  // m[16] l[16] lr[16] O[16][D]
    if (active) {
      if (part == 0) {
        pub[row] = mm;
        pub[16 + row] = lt;
        pub[32 + row] = lrt;
      }
#pragma unroll
      for (int d = 0; d < 16; ++d) pub[48 + row * D + 16 * part + d] = acc[d];
    }
    cluster_sync();  // every part is published
    if (cluster_ctarank() == 0 && active) {
      const uint32_t nct = cluster_nctarank();
      float M = -INFINITY;
      for (uint32_t r = 0; r < nct; ++r) M = fmaxf(M, ld_dsmem(dsmem_addr(pub + row, r)));
      float L = 0.f, LR = 0.f, O[16];
#pragma unroll
      for (int d = 0; d < 16; ++d) O[d] = 0.f;
      for (uint32_t r = 0; r < nct; ++r) {
        const float mr = ld_dsmem(dsmem_addr(pub + row, r));
        const float w = M == -INFINITY ? 0.f : ex2(mr - M);
        L += w * ld_dsmem(dsmem_addr(pub + 16 + row, r));
        LR += w * ld_dsmem(dsmem_addr(pub + 32 + row, r));
        const uint32_t oa = dsmem_addr(pub + 48 + row * D + 16 * part, r);
#pragma unroll
        for (int d = 0; d < 4; ++d) {
          const float4 v = ld_dsmem4(oa + 16 * d);
          O[4 * d] += w * v.x;
          O[4 * d + 1] += w * v.y;
          O[4 * d + 2] += w * v.z;
          O[4 * d + 3] += w * v.w;
        }
      }
      const float inv = LR > 0.f ? 1.f / LR : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + qrow * D + 16 * part);
#pragma unroll
      for (int d = 0; d < 2; ++d)
        dst[d] = make_uint4(pack2<BF16>(O[8 * d] * inv, O[8 * d + 1] * inv),
                            pack2<BF16>(O[8 * d + 2] * inv, O[8 * d + 3] * inv),
                            pack2<BF16>(O[8 * d + 4] * inv, O[8 * d + 5] * inv),
                            pack2<BF16>(O[8 * d + 6] * inv, O[8 * d + 7] * inv));
      if (part == 0) p.lse[qrow] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    cluster_sync();  // rank 0 has read every peer before any CTA exits
    return;
  }

  if (active) {
    const float inv = lrt > 0.f ? 1.f / lrt : 0.f;
    const float lse = lt > 0.f ? (mm + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
    if (p.n_splits == 1) {  // the split is the whole cache: final O and LSE
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + qrow * D + 16 * part);
#pragma unroll
      for (int d = 0; d < 2; ++d)
        dst[d] = make_uint4(pack2<BF16>(acc[8 * d] * inv, acc[8 * d + 1] * inv),
                            pack2<BF16>(acc[8 * d + 2] * inv, acc[8 * d + 3] * inv),
                            pack2<BF16>(acc[8 * d + 4] * inv, acc[8 * d + 5] * inv),
                            pack2<BF16>(acc[8 * d + 6] * inv, acc[8 * d + 7] * inv));
      if (part == 0) p.lse[qrow] = lse;
    } else {  // partial result for decode_merge_kernel
      const size_t orow = qrow * p.n_splits + split;
      float4* dst = reinterpret_cast<float4*>(p.o_part + orow * D + 16 * part);
#pragma unroll
      for (int d = 0; d < 4; ++d)
        dst[d] = make_float4(acc[4 * d] * inv, acc[4 * d + 1] * inv, acc[4 * d + 2] * inv, acc[4 * d + 3] * inv);
      if (part == 0) p.lse_part[orow] = lse;
    }
  }
}

// O and LSE of each (sequence, query head) from its splits: LSE = log sum
// exp(LSE_s), O = sum exp(LSE_s - LSE) O_s.  One block of D threads per row.
// Launched as a programmatic dependent of decode_split_kernel: its blocks may
// be resident before the split kernel ends and wait here for its results.
template <int D, bool BF16>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t row = blockIdx.x;  // b * Hq + h
  const float* lp = p.lse_part + row * p.n_splits;
  float mx = -INFINITY;
  for (int s = 0; s < p.n_splits; ++s) mx = fmaxf(mx, lp[s]);
  float tot = 0.f, acc = 0.f;
  for (int s = 0; s < p.n_splits; ++s) {
    const float w = mx == -INFINITY ? 0.f : __expf(lp[s] - mx);
    tot += w;
    acc += w * p.o_part[(row * p.n_splits + s) * D + threadIdx.x];
  }
  const float o = tot > 0.f ? acc / tot : 0.f;
  uint16_t* dst = static_cast<uint16_t*>(p.o) + row * D + threadIdx.x;
  const uint32_t pk = pack2<BF16>(o, 0.f);
  *dst = (uint16_t)(pk & 0xffffu);
  if (threadIdx.x == 0) p.lse[row] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
}

}  // namespace fa

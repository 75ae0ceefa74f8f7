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
  float* o_part;         // fp32 partial O, normalised over its keys: [B, Hq, n_splits, D]
                         // (balanced mode: [B * Hkv + grid, group, D], see decode_balanced_kernel)
  float* lse_part;       // natural log, -inf for an empty key range: [B, Hq, n_splits]
                         // (balanced mode: [B * Hkv + grid, group])
  void* o;               // [B, Hq, D] 16-bit output
  float* lse;            // [B, Hq]
  int B, Hq, Hkv, L, n_splits, group;
  float scale_log2;      // scale * log2(e)
  // balanced mode (n_splits = 0): the B * Hkv caches' 32-key tiles, tpp per
  // cache, are dealt out evenly over `grid` CTAs
  long long tiles;
  int tpp, grid;
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

enum : uint32_t { DEC_SITE_KV = 0x300, DEC_SITE_DRAIN = 0x301, DEC_SITE_MERGE = 0x302 };

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

// This thread's share of one CTA's result over a key range: the (max, sum
// of exponentials, sum of rounded exponentials, 16 columns of unnormalised O)
// of query row `row` (a query head of the group) and columns [16 part, +16).
struct DecPart {
  float mm, lt, lrt, acc[16];
  int row, part;
  bool active;
};

// The CTA's four warps over keys [start, end) of cache (b, kvh), then merged
// across the warps through shared memory.  `it` counts the tiles this warp
// has taken from its ring so far (it carries the barrier phases from one
// range to the next); every thread of the CTA calls this with the same range.
template <int D, bool BF16>
__device__ __forceinline__ void dec_range(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const DecParams& p,
                                          uint8_t* dsm, uint64_t (*bars)[DecCfg<D>::STAGES], int b, int kvh,
                                          int start, int end, uint32_t& it, DecPart& out) {
  using C = DecCfg<D>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = end > start ? (end - start + C::KT - 1) / C::KT : 0;
  const int bh = b * p.Hkv + kvh;  // cache head index (third tensor-map coordinate)

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
  // The warp's i-th tile of the range is tile warp + WARPS * i, in stage
  // (it + i) % STAGES.  A whole tile comes by TMA; the one tile that runs past
  // `end` (always the range's last, so the warp's last) by cp.async with the
  // rows past `end` zero-filled.
  auto full_tile = [&](int i) { return start + C::KT * (warp + C::WARPS * i) + C::KT <= end; };
  auto issue = [&](int i) {
    const int t = warp + C::WARPS * i;
    if (t >= n_tiles) return;
    const int key0 = start + C::KT * t, s = (it + i) % C::STAGES;
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
    const int t = warp + C::WARPS * i, st = (it + i) % C::STAGES;
    if (full_tile(i)) {
      const bool ok =
          __all_sync(0xffffffffu, mbar_wait(&bars[warp][st], ((it + i) / C::STAGES) & 1, DEC_SITE_KV));
      if (!ok) {  // error recorded: let the warp's copies in flight, this tile's included, land
                  // (bounded waits again), then stop
        for (int j = i; j < min(i + C::STAGES, my_tiles); ++j)
          if (full_tile(j))
            mbar_wait(&bars[warp][(it + j) % C::STAGES], ((it + j) / C::STAGES) & 1, DEC_SITE_DRAIN);
        break;
      }
    } else {
      cp_async_wait<0>();
      __syncwarp();
      // a copied tile completes its stage's barrier phase too, so that every
      // tile, however it came, moves its stage on by exactly one phase (the
      // next range of a balanced-mode CTA relies on the parities)
      if (lane == 0) mbar_arrive(&bars[warp][st]);
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
  it += (uint32_t)my_tiles;

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
  out.row = threadIdx.x / PARTS;
  out.part = threadIdx.x % PARTS;
  out.active = out.row < p.group && threadIdx.x < 16 * PARTS;
  out.mm = -INFINITY;
  out.lt = out.lrt = 0.f;
#pragma unroll
  for (int d = 0; d < 16; ++d) out.acc[d] = 0.f;
  if (out.active) {
    const float* w0 = reinterpret_cast<const float*>(dsm);
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) out.mm = fmaxf(out.mm, w0[w * C::SCRATCH + out.row]);
#pragma unroll
    for (int w = 0; w < C::WARPS; ++w) {
      const float* wp = w0 + w * C::SCRATCH;
      const float sc = out.mm == -INFINITY ? 0.f : ex2(wp[out.row] - out.mm);  // empty warp ranges weigh 0
      out.lt += wp[16 + out.row] * sc;
      out.lrt += wp[32 + out.row] * sc;
#pragma unroll
      for (int d = 0; d < 16; ++d) out.acc[d] += wp[48 + out.row * D + 16 * out.part + d] * sc;
    }
  }
}

// A CTA's normalised partial O (fp32) and its LSE for one key range.
template <int D>
__device__ __forceinline__ void dec_store_part(const DecPart& r, float* o_part_row, float* lse_part_row) {
  const float inv = r.lrt > 0.f ? 1.f / r.lrt : 0.f;
  float4* dst = reinterpret_cast<float4*>(o_part_row + 16 * r.part);
#pragma unroll
  for (int d = 0; d < 4; ++d)
    dst[d] = make_float4(r.acc[4 * d] * inv, r.acc[4 * d + 1] * inv, r.acc[4 * d + 2] * inv, r.acc[4 * d + 3] * inv);
  if (r.part == 0) *lse_part_row = r.lt > 0.f ? (r.mm + __log2f(r.lt)) * 0.69314718055994531f : -INFINITY;
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

  uint32_t it = 0;
  DecPart r;
  dec_range<D, BF16>(tm_k, tm_v, p, dsm, bars, b, kvh, start, end, it, r);
  const int row = r.row, part = r.part;
  const bool active = r.active;
  const float mm = r.mm, lt = r.lt, lrt = r.lrt;
  const float* acc = r.acc;
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
      for (uint32_t q = 0; q < nct; ++q) M = fmaxf(M, ld_dsmem(dsmem_addr(pub + row, q)));
      float L = 0.f, LR = 0.f, O[16];
#pragma unroll
      for (int d = 0; d < 16; ++d) O[d] = 0.f;
      for (uint32_t q = 0; q < nct; ++q) {
        const float mr = ld_dsmem(dsmem_addr(pub + row, q));
        const float w = M == -INFINITY ? 0.f : ex2(mr - M);
        L += w * ld_dsmem(dsmem_addr(pub + 16 + row, q));
        LR += w * ld_dsmem(dsmem_addr(pub + 32 + row, q));
        const uint32_t oa = dsmem_addr(pub + 48 + row * D + 16 * part, q);
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
    if (p.n_splits == 1) {  // the split is the whole cache: final O and LSE
      const float inv = lrt > 0.f ? 1.f / lrt : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + qrow * D + 16 * part);
#pragma unroll
      for (int d = 0; d < 2; ++d)
        dst[d] = make_uint4(pack2<BF16>(acc[8 * d] * inv, acc[8 * d + 1] * inv),
                            pack2<BF16>(acc[8 * d + 2] * inv, acc[8 * d + 3] * inv),
                            pack2<BF16>(acc[8 * d + 4] * inv, acc[8 * d + 5] * inv),
                            pack2<BF16>(acc[8 * d + 6] * inv, acc[8 * d + 7] * inv));
      if (part == 0) p.lse[qrow] = lt > 0.f ? (mm + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
    } else {  // partial result for decode_merge_kernel
      const size_t orow = qrow * p.n_splits + split;
      dec_store_part<D>(r, p.o_part + orow * D, p.lse_part + orow);
    }
  }
}

// Balanced mode: the caches' 32-key tiles, in (sequence, KV head) order,
// are dealt out in equal contiguous runs to `grid` CTAs (one per SM), so every
// SM streams the same number of cache bytes whatever the batch and lengths.
// A run can cover the end of one cache and the start of the next: the CTA
// writes one partial result per cache it meets.  Cache pr's part from CTA c
// goes to slot pr + c: along the tile list both only grow, and every new
// part moves to a new cache, a new CTA or both, so slots never collide and
// B * Hkv + grid of them are enough.
template <int D, bool BF16>
__global__ void __launch_bounds__(128, 1)
    decode_balanced_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const DecParams p) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t dsm_raw[];
  __shared__ uint64_t bars[C::WARPS][C::STAGES];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&bars[warp][s], 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __syncwarp();
  const long long c = blockIdx.x;
  const long long t0 = c * p.tiles / p.grid, t1 = (c + 1) * p.tiles / p.grid;  // this CTA's tiles [t0, t1)
  uint32_t it = 0;
  if (t1 <= t0) return;
  const long long first_pair = t0 / p.tpp, last_pair = (t1 - 1) / p.tpp;  // the caches this run meets
  for (long long pr = first_pair; pr <= last_pair; ++pr) {
    const int b = (int)(pr / p.Hkv), kvh = (int)(pr - (long long)b * p.Hkv);
    const int len = min(max(p.seq_lens[b], 0), p.L);
    const long long a0 = max(t0, pr * p.tpp) - pr * p.tpp, a1 = min(t1, (pr + 1) * p.tpp) - pr * p.tpp;
    const int start = min((int)a0 * C::KT, len), end = min((int)a1 * C::KT, len);
    DecPart r;
    dec_range<D, BF16>(tm_k, tm_v, p, dsm, bars, b, kvh, start, end, it, r);
    if (r.active) {
      const size_t slot = (size_t)(pr + c) * p.group + r.row;
      dec_store_part<D>(r, p.o_part + slot * D, p.lse_part + slot);
    }
    __syncthreads();  // the scratch in the tile buffers is read before the next range refills them
  }
}

// O and LSE of each (sequence, query head) from its parts: LSE = log sum
// exp(LSE_s), O = sum exp(LSE_s - LSE) O_s.  One block of D threads per row.
// Launched as a programmatic dependent of the split or balanced kernel: its
// blocks may be resident before that kernel ends and wait here for its
// results.  Every load whose address is known is issued before the first
// result is needed: thread d's column of the first kPrefetch parts, and the
// parts' LSEs spread over the threads, so a row costs about one memory
// latency instead of one per part.  A row has at most kMergeMax parts (the
// host allows at most 1024 splits and 1024 balanced-mode CTAs).
constexpr int kMergeMax = 1024, kPrefetch = 16;

template <int D, bool BF16>
__global__ void __launch_bounds__(D) decode_merge_kernel(const DecParams p) {
  __shared__ float w_s[kMergeMax];  // the parts' LSEs, then their weights exp(LSE_s - max)
  __shared__ float red[D / 32];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t row = blockIdx.x;  // b * Hq + h
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  // the row's parts: n of them, part s at index part_at(s) of lse_part (and
  // of o_part in rows of D)
  int n;
  size_t first, rest0, rest_stride;  // part 0 at `first`, part s >= 1 at rest0 + (s - 1) * rest_stride
  if (p.n_splits > 0) {
    n = p.n_splits;
    first = row * p.n_splits;
    rest0 = first + 1;
    rest_stride = 1;
  } else {
    // balanced mode: the cache's tiles [pr tpp, (pr + 1) tpp) were run by CTAs
    // c0 .. c1, whose parts sit in slots pr + c0 .. pr + c1
    const long long b = (long long)(row / p.Hq), h = (long long)(row % p.Hq);
    const long long pr = b * p.Hkv + h / p.group;
    const size_t gi = (size_t)(h % p.group);
    // CTA whose run holds tile x: the largest c with floor(c tiles / grid) <= x
    auto cta_of = [&](long long x) { return ((x + 1) * p.grid - 1) / p.tiles; };
    const long long c0 = cta_of(pr * p.tpp), c1 = cta_of((pr + 1) * p.tpp - 1);
    n = (int)(c1 - c0 + 1);
    first = (size_t)(pr + c0) * p.group + gi;
    rest0 = first + p.group;
    rest_stride = p.group;
  }
  if (n > kMergeMax) {  // excluded by the host's limits
    if (t == 0) record_error(DEV_ERR_ARG, DEC_SITE_MERGE);
    return;
  }
  auto part_at = [&](int s) { return s == 0 ? first : rest0 + (size_t)(s - 1) * rest_stride; };
  float ov[kPrefetch];
#pragma unroll
  for (int s = 0; s < kPrefetch; ++s) ov[s] = s < n ? p.o_part[part_at(s) * D + t] : 0.f;
  float mx = -INFINITY;
  for (int s = t; s < n; s += D) {
    const float l = p.lse_part[part_at(s)];
    w_s[s] = l;
    mx = fmaxf(mx, l);
  }
  // block maximum
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();  // red is reused below
  // weights (all zero when every part is empty) and their sum
  float tot = 0.f;
  for (int s = t; s < n; s += D) {
    const float w = mx == -INFINITY ? 0.f : __expf(w_s[s] - mx);
    w_s[s] = w;
    tot += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) red[warp] = tot;
  __syncthreads();  // w_s and red are complete
  tot = red[0];
#pragma unroll
  for (int w = 1; w < D / 32; ++w) tot += red[w];
  // O column t, parts added in order
  float acc = 0.f;
#pragma unroll
  for (int s = 0; s < kPrefetch; ++s)
    if (s < n) acc += w_s[s] * ov[s];
#pragma unroll 8
  for (int s = kPrefetch; s < n; ++s) acc += w_s[s] * p.o_part[part_at(s) * D + t];
  const float o = tot > 0.f ? acc / tot : 0.f;
  uint16_t* dst = static_cast<uint16_t*>(p.o) + row * D + t;
  const uint32_t pk = pack2<BF16>(o, 0.f);
  *dst = (uint16_t)(pk & 0xffffu);
  if (t == 0) p.lse[row] = tot > 0.f ? mx + __logf(tot) : -INFINITY;
}

}  // namespace fa
